"""Thin Python binding of libsvga.so (C ABI in include/svga.h).

Argument marshalling only: every step runs in the library's CUDA kernels.  torch
provides device memory and streams.  The library must be built (``build.py``); if it
is missing, the first call raises ``SvgaError`` -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvga.so")

SVGA_OK = 0
STATUS_NAMES = {0: "SVGA_OK", 1: "SVGA_ERR_INVALID_ARG", 2: "SVGA_ERR_SHAPE",
                3: "SVGA_ERR_ALIGNMENT", 4: "SVGA_ERR_UNSUPPORTED", 5: "SVGA_ERR_WORKSPACE",
                6: "SVGA_ERR_CUDA", 7: "SVGA_ERR_TIMEOUT"}
HEAD_SPATIAL, HEAD_TEMPORAL = 0, 1
ORDER_FRAME_MAJOR, ORDER_TEMPORAL_MAJOR, ORDER_TEMPORAL_MAJOR_STRICT = 0, 1, 2
FLAG_NAIVE_B1 = 1
FLAG_TILE_ALIGNED = 2
FLAG_QO_FRAME_MAJOR = 4
FLAG_KV_FRAME_MAJOR = 8
FLAG_CTA_PAIR = 16
FLAG_TEST_STALL = 1 << 16

EXPORTED = ["svga_problem_rows", "svga_block_map_size", "svga_build_block_map",
            "svga_build_block_map_static",
            "svga_permute_tokens",
            "svga_unpermute_tokens", "svga_sparse_attention_fwd", "svga_sparse_attention_fwd_part",
            "svga_validate_block_map", "svga_classify_heads_async", "svga_build_block_map_routed",
            "svga_permute_tokens_mapped", "svga_unpermute_tokens_mapped",
            "svga_dense_attention_fwd",
            "svga_classify_size", "svga_classify_heads", "svga_kept_fraction",
            "svga_autotune_size", "svga_autotune_heads", "svga_last_error",
            "svga_status_string", "svga_version"]


class SvgaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Problem(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int), ("num_frames", ctypes.c_int),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("head_dim", ctypes.c_int),
                ("head_type", ctypes.POINTER(ctypes.c_int32)),
                ("band", ctypes.POINTER(ctypes.c_int32)),
                ("order", ctypes.POINTER(ctypes.c_int32)),
                ("anchor_frame0", ctypes.c_int), ("tile_q", ctypes.c_int),
                ("tile_k", ctypes.c_int), ("frame_pad", ctypes.c_int)]


class BlockMapC(ctypes.Structure):
    _fields_ = [("cls", ctypes.c_void_p), ("full_ptr", ctypes.c_void_p),
                ("full_idx", ctypes.c_void_p), ("bnd_ptr", ctypes.c_void_p),
                ("bnd_idx", ctypes.c_void_p), ("full_cap", ctypes.c_int64),
                ("bnd_cap", ctypes.c_int64), ("plan", ctypes.c_void_p),
                ("plan_bytes", ctypes.c_size_t), ("status", ctypes.c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libsvga.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise SvgaError(6, f"{LIB_PATH} not built; run python -m "
                               "block_sparse_spatio_attn_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        PP = ctypes.POINTER(Problem)
        lib.svga_problem_rows.argtypes = [PP, ctypes.POINTER(ctypes.c_int64)]
        lib.svga_block_map_size.argtypes = [PP, ctypes.POINTER(SZ), ctypes.POINTER(SZ),
                                            ctypes.POINTER(ctypes.c_int64),
                                            ctypes.POINTER(ctypes.c_int64),
                                            ctypes.POINTER(SZ), ctypes.POINTER(SZ)]
        lib.svga_build_block_map.argtypes = [PP, ctypes.POINTER(BlockMapC), P, SZ, P]
        lib.svga_build_block_map_static.argtypes = [PP, ctypes.POINTER(BlockMapC), P]
        lib.svga_permute_tokens.argtypes = [P, P, PP, P]
        lib.svga_unpermute_tokens.argtypes = [P, P, PP, P]
        lib.svga_sparse_attention_fwd.argtypes = [P, P, P, P, P, PP, ctypes.POINTER(BlockMapC),
                                                  F, I, P]
        lib.svga_sparse_attention_fwd_part.argtypes = [P, P, P, P, P, PP,
                                                      ctypes.POINTER(BlockMapC), F, I, I, I, P]
        lib.svga_dense_attention_fwd.argtypes = [P, P, P, P, P, I, I, I, F, P, P]
        lib.svga_classify_size.argtypes = [PP, I, ctypes.POINTER(SZ)]
        lib.svga_classify_heads.argtypes = [P, P, P, PP, P, P, P, I, F, P, P, P, SZ, P]
        lib.svga_classify_heads_async.argtypes = [P, P, P, PP, P, P, P, I, F, P, P, P, P, SZ, P]
        lib.svga_kept_fraction.argtypes = [PP, I, I, ctypes.POINTER(ctypes.c_double)]
        lib.svga_autotune_size.argtypes = [PP, I, I, ctypes.POINTER(SZ)]
        lib.svga_autotune_heads.argtypes = [P, P, P, PP, P, P, I, ctypes.c_double, P, I, F, P,
                                            P, P, P, SZ, P]
        lib.svga_build_block_map_routed.argtypes = [PP, P, P, P, ctypes.POINTER(BlockMapC), P,
                                                   SZ, P]
        lib.svga_permute_tokens_mapped.argtypes = [P, P, PP, ctypes.POINTER(BlockMapC), P]
        lib.svga_validate_block_map.argtypes = [PP, ctypes.POINTER(BlockMapC), P]
        lib.svga_unpermute_tokens_mapped.argtypes = [P, P, PP, ctypes.POINTER(BlockMapC), P]
        lib.svga_last_error.restype = ctypes.c_char_p
        lib.svga_last_error.argtypes = []
        lib.svga_status_string.restype = ctypes.c_char_p
        lib.svga_status_string.argtypes = [I]
        lib.svga_version.restype = I
        lib.svga_version.argtypes = []
        for name in EXPORTED:
            if name not in ("svga_last_error", "svga_status_string", "svga_version"):
                getattr(lib, name).restype = I
        _lib = lib
    return _lib


def _check(rc: int):
    if rc != SVGA_OK:
        raise SvgaError(rc, load().svga_last_error().decode())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class _Args:
    """The tensor arguments of one call, checked for what the C ABI cannot see from a
    pointer: the library reads and writes exactly the elements the problem implies, so
    each tensor must have that dtype and shape (or element count) and be contiguous;
    once all are checked, all must live on a CUDA device.  Raises SvgaError before
    anything is launched."""

    def __init__(self):
        self.seen = []

    def t(self, t, name: str, dtype, shape=None, numel=None, optional=False):
        if t is None:
            if optional:
                return None
            raise SvgaError(1, f"{name} is None")
        if not isinstance(t, torch.Tensor):
            raise SvgaError(1, f"{name} must be a torch.Tensor, got {type(t).__name__}")
        if t.dtype != dtype:
            raise SvgaError(1, f"{name} must be {dtype}, got {t.dtype}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise SvgaError(2, f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if numel is not None and t.numel() != numel:
            raise SvgaError(2, f"{name} has {t.numel()} elements, expected {numel}")
        if not t.is_contiguous():
            raise SvgaError(1, f"{name} must be contiguous")
        self.seen.append((name, t))
        return _ptr(t)

    def tokens(self, problem, **named):
        """bf16 [heads, tokens, head_dim] frame-major tensors, in argument order."""
        shape = (problem.heads, problem.tokens, problem.head_dim)
        return [self.t(t, n, torch.bfloat16, shape) for n, t in named.items()]

    def positions(self, problem, **named):
        """bf16 [heads, rows, head_dim] tensors in token order (rows = problem.rows:
        the tokens, or the padded layout's positions), in argument order."""
        shape = (problem.heads, problem.rows, problem.head_dim)
        return [self.t(t, n, torch.bfloat16, shape) for n, t in named.items()]

    def attention(self, problem, flags, q, k, v, o, lse):
        """q, k, v, o and lse of an attention call: in token order, or frame-major
        where the flags say so."""
        qo = self.tokens if flags & FLAG_QO_FRAME_MAJOR else self.positions
        kv = self.tokens if flags & FLAG_KV_FRAME_MAJOR else self.positions
        pq, po = qo(problem, q=q, o=o)
        pk, pv = kv(problem, k=k, v=v)
        n = problem.tokens if flags & FLAG_QO_FRAME_MAJOR else problem.rows
        pl = self.t(lse, "lse", torch.float32, (problem.heads, n), optional=True)
        return pq, pk, pv, po, pl

    def done(self):
        for name, t in self.seen:
            if not t.is_cuda:
                raise SvgaError(1, f"{name} must be on a CUDA device")


@dataclass
class ProblemSpec:
    """A problem with its host arrays kept alive for the C struct."""
    heads: int
    num_frames: int
    grid_h: int
    grid_w: int
    head_dim: int
    head_type: Sequence[int]
    band: Sequence[int]
    order: Sequence[int]
    anchor_frame0: int = 1
    tile_q: int = 128
    tile_k: int = 128
    frame_pad: int = 0

    def __post_init__(self):
        H = self.heads
        self._ht = (ctypes.c_int32 * H)(*self.head_type)
        self._bd = (ctypes.c_int32 * H)(*self.band)
        self._od = (ctypes.c_int32 * H)(*self.order)
        self.c = Problem(H, self.num_frames, self.grid_h, self.grid_w, self.head_dim,
                         self._ht, self._bd, self._od, self.anchor_frame0, self.tile_q,
                         self.tile_k, self.frame_pad)

    @property
    def tokens(self) -> int:
        return self.num_frames * self.grid_h * self.grid_w

    @property
    def rows(self) -> int:
        """Rows per head of a tensor in token order (svga_problem_rows)."""
        r = ctypes.c_int64()
        _check(load().svga_problem_rows(ctypes.byref(self.c), ctypes.byref(r)))
        return r.value

    @classmethod
    def from_workload(cls, wl, head_type=None, order=None, tile_q=None, tile_k=None,
                      frame_pad=0):
        return cls(wl.heads, wl.frames, wl.grid_h, wl.grid_w, wl.head_dim,
                   list(wl.head_type if head_type is None else head_type), list(wl.band),
                   list(wl.order if order is None else order), wl.anchor_frame0,
                   wl.tile_q if tile_q is None else tile_q,
                   wl.tile_k if tile_k is None else tile_k, frame_pad)


def svga_block_map_size(problem: ProblemSpec) -> dict:
    sz = [ctypes.c_size_t() for _ in range(2)]
    caps = [ctypes.c_int64() for _ in range(2)]
    plan, ws = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().svga_block_map_size(ctypes.byref(problem.c), ctypes.byref(sz[0]),
                                      ctypes.byref(sz[1]), ctypes.byref(caps[0]),
                                      ctypes.byref(caps[1]), ctypes.byref(plan),
                                      ctypes.byref(ws)))
    return {"cls_bytes": sz[0].value, "ptr_bytes": sz[1].value, "full_cap": caps[0].value,
            "bnd_cap": caps[1].value, "plan_bytes": plan.value, "workspace_bytes": ws.value}


class BlockMap:
    """Device buffers of a block map, allocated with torch (caller-owned memory)."""

    def __init__(self, problem: ProblemSpec, device="cuda"):
        s = svga_block_map_size(problem)
        self.problem = problem
        self.sizes = s
        u8 = torch.uint8
        self.cls = torch.empty(max(1, s["cls_bytes"]), dtype=u8, device=device)
        self.full_ptr = torch.empty(s["ptr_bytes"] // 4, dtype=torch.int32, device=device)
        self.bnd_ptr = torch.empty(s["ptr_bytes"] // 4, dtype=torch.int32, device=device)
        self.full_idx = torch.empty(max(1, s["full_cap"]), dtype=torch.int32, device=device)
        self.bnd_idx = torch.empty(max(1, s["bnd_cap"]), dtype=torch.int32, device=device)
        self.plan = torch.empty(s["plan_bytes"], dtype=u8, device=device)
        self.workspace = torch.empty(max(256, s["workspace_bytes"]), dtype=u8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.c = BlockMapC(self.cls.data_ptr(), self.full_ptr.data_ptr(),
                           self.full_idx.data_ptr(), self.bnd_ptr.data_ptr(),
                           self.bnd_idx.data_ptr(), s["full_cap"], s["bnd_cap"],
                           self.plan.data_ptr(), s["plan_bytes"], self.status.data_ptr())

    def device_status(self) -> int:
        return int(self.status.item())


def svga_build_block_map(problem: ProblemSpec, bmap: BlockMap, stream=None) -> BlockMap:
    _check(load().svga_build_block_map(ctypes.byref(problem.c), ctypes.byref(bmap.c),
                                       _ptr(bmap.workspace), bmap.workspace.numel(),
                                       _stream(stream)))
    return bmap


def build_block_map(problem: ProblemSpec, stream=None) -> BlockMap:
    return svga_build_block_map(problem, BlockMap(problem), stream)


def svga_validate_block_map(problem: ProblemSpec, bmap: BlockMap, stream=None) -> None:
    """Host-side consistency check of a built map; raises SvgaError naming the violation."""
    _check(load().svga_validate_block_map(ctypes.byref(problem.c), ctypes.byref(bmap.c),
                                          _stream(stream)))


def svga_permute_tokens(src: torch.Tensor, dst: torch.Tensor, problem: ProblemSpec,
                        stream=None) -> torch.Tensor:
    a = _Args()
    ps, = a.tokens(problem, src=src)
    pd, = a.positions(problem, dst=dst)
    a.done()
    _check(load().svga_permute_tokens(ps, pd, ctypes.byref(problem.c), _stream(stream)))
    return dst


def svga_unpermute_tokens(src: torch.Tensor, dst: torch.Tensor, problem: ProblemSpec,
                          stream=None) -> torch.Tensor:
    a = _Args()
    ps, = a.positions(problem, src=src)
    pd, = a.tokens(problem, dst=dst)
    a.done()
    _check(load().svga_unpermute_tokens(ps, pd, ctypes.byref(problem.c), _stream(stream)))
    return dst


def svga_sparse_attention_fwd(q, k, v, o, lse, problem: ProblemSpec, bmap: BlockMap,
                              scale: float, flags: int = 0, stream=None) -> torch.Tensor:
    a = _Args()
    pq, pk, pv, po, pl = a.attention(problem, flags, q, k, v, o, lse)
    a.done()
    _check(load().svga_sparse_attention_fwd(pq, pk, pv, po, pl,
                                            ctypes.byref(problem.c), ctypes.byref(bmap.c),
                                            float(scale), int(flags), _stream(stream)))
    return o


def svga_sparse_attention_fwd_part(q, k, v, o, lse, problem: ProblemSpec, bmap: BlockMap,
                                   scale: float, flags: int, part: int, num_parts: int,
                                   stream=None) -> torch.Tensor:
    a = _Args()
    pq, pk, pv, po, pl = a.attention(problem, flags, q, k, v, o, lse)
    a.done()
    _check(load().svga_sparse_attention_fwd_part(
        pq, pk, pv, po, pl, ctypes.byref(problem.c), ctypes.byref(bmap.c),
        float(scale), int(flags), int(part), int(num_parts), _stream(stream)))
    return o


def svga_dense_attention_fwd(q, k, v, o, lse, scale: float, status=None,
                             stream=None) -> torch.Tensor:
    if not isinstance(q, torch.Tensor) or q.dim() != 3:
        raise SvgaError(2, "q must be a [heads, tokens, head_dim] tensor")
    H, N, d = q.shape
    a = _Args()
    pq, pk, pv, po = (a.t(t, n, torch.bfloat16, (H, N, d))
                      for n, t in (("q", q), ("k", k), ("v", v), ("o", o)))
    pl = a.t(lse, "lse", torch.float32, (H, N), optional=True)
    pst = a.t(status, "status", torch.int32, numel=1, optional=True)
    a.done()
    _check(load().svga_dense_attention_fwd(pq, pk, pv, po, pl, H, N, d, float(scale), pst,
                                           _stream(stream)))
    return o


def svga_classify_size(problem: ProblemSpec, n_rows: int) -> int:
    ws = ctypes.c_size_t()
    _check(load().svga_classify_size(ctypes.byref(problem.c), int(n_rows), ctypes.byref(ws)))
    return ws.value


def svga_classify_heads(q, k, v, problem: ProblemSpec, w_spatial, w_temporal, rows, n_rows,
                        scale: float, workspace: Optional[torch.Tensor] = None, stream=None):
    """Returns (head_type list, mse [heads, 2] list).  Synchronises the stream."""
    H = problem.heads
    a = _Args()
    pq, pk, pv = a.tokens(problem, q=q, k=k, v=v)
    pr = a.t(rows, "rows", torch.int32, numel=int(n_rows), optional=True)
    a.done()
    ws_bytes = svga_classify_size(problem, n_rows)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    a.t(workspace, "workspace", torch.uint8)
    a.done()
    types = (ctypes.c_int32 * H)()
    mse = (ctypes.c_float * (2 * H))()
    wsp = (ctypes.c_int32 * H)(*w_spatial)
    wtp = (ctypes.c_int32 * H)(*w_temporal)
    _check(load().svga_classify_heads(pq, pk, pv, ctypes.byref(problem.c),
                                      wsp, wtp, pr, int(n_rows), float(scale),
                                      types, mse, _ptr(workspace), workspace.numel(),
                                      _stream(stream)))
    return list(types), [[mse[2 * h], mse[2 * h + 1]] for h in range(H)]


def svga_classify_heads_async(q, k, v, problem: ProblemSpec, w_spatial, w_temporal, rows,
                              n_rows, scale: float, head_type_dev: torch.Tensor,
                              mse_dev: Optional[torch.Tensor] = None,
                              status_dev: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Head types (and deviations, status) written to device tensors; no synchronisation."""
    H = problem.heads
    a = _Args()
    pq, pk, pv = a.tokens(problem, q=q, k=k, v=v)
    pr = a.t(rows, "rows", torch.int32, numel=int(n_rows), optional=True)
    pt = a.t(head_type_dev, "head_type_dev", torch.int32, numel=H)
    pm = a.t(mse_dev, "mse_dev", torch.float32, numel=2 * H, optional=True)
    ps = a.t(status_dev, "status_dev", torch.int32, numel=1, optional=True)
    a.done()
    if workspace is None:
        workspace = torch.empty(svga_classify_size(problem, n_rows), dtype=torch.uint8,
                                device=q.device)
    a.t(workspace, "workspace", torch.uint8)
    a.done()
    wsp = (ctypes.c_int32 * H)(*w_spatial)
    wtp = (ctypes.c_int32 * H)(*w_temporal)
    _check(load().svga_classify_heads_async(
        pq, pk, pv, ctypes.byref(problem.c), wsp, wtp, pr, int(n_rows), float(scale), pt, pm,
        ps, _ptr(workspace), workspace.numel(), _stream(stream)))


def svga_kept_fraction(problem: ProblemSpec, head_type: int, band: int) -> float:
    f = ctypes.c_double()
    _check(load().svga_kept_fraction(ctypes.byref(problem.c), int(head_type), int(band),
                                     ctypes.byref(f)))
    return f.value


def svga_autotune_size(problem: ProblemSpec, n_rows: int, n_cand: int) -> int:
    sz = ctypes.c_size_t()
    _check(load().svga_autotune_size(ctypes.byref(problem.c), int(n_rows), int(n_cand),
                                     ctypes.byref(sz)))
    return sz.value


def svga_autotune_heads(q, k, v, problem: ProblemSpec, candidates, max_kept_fraction: float,
                        rows, n_rows: int, scale: float, workspace=None, stream=None):
    """candidates: [(type, band), ...].  Returns (types [heads], bands [heads],
    mse [heads][n_cand])."""
    a = _Args()
    pq, pk, pv = a.tokens(problem, q=q, k=k, v=v)
    pr = a.t(rows, "rows", torch.int32, numel=n_rows, optional=True)
    n_cand = len(candidates)
    need = svga_autotune_size(problem, n_rows, n_cand)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    pw = a.t(workspace, "workspace", torch.uint8)
    a.done()
    H = problem.heads
    ct = (ctypes.c_int32 * n_cand)(*[int(c[0]) for c in candidates])
    cb = (ctypes.c_int32 * n_cand)(*[int(c[1]) for c in candidates])
    types = (ctypes.c_int32 * H)()
    bands = (ctypes.c_int32 * H)()
    mse = (ctypes.c_float * (H * n_cand))()
    _check(load().svga_autotune_heads(pq, pk, pv, ctypes.byref(problem.c), ct, cb, n_cand,
                                      float(max_kept_fraction), pr, int(n_rows), float(scale),
                                      types, bands, mse, pw, workspace.numel(), _stream(stream)))
    return (list(types), list(bands),
            [list(mse[h * n_cand:(h + 1) * n_cand]) for h in range(H)])


def svga_build_block_map_routed(problem: ProblemSpec, head_type_dev: torch.Tensor, w_spatial,
                                w_temporal, bmap: BlockMap, stream=None) -> BlockMap:
    H = problem.heads
    a = _Args()
    pt = a.t(head_type_dev, "head_type_dev", torch.int32, numel=H)
    a.done()
    wsp = (ctypes.c_int32 * H)(*w_spatial)
    wtp = (ctypes.c_int32 * H)(*w_temporal)
    _check(load().svga_build_block_map_routed(ctypes.byref(problem.c), pt, wsp,
                                              wtp, ctypes.byref(bmap.c), _ptr(bmap.workspace),
                                              bmap.workspace.numel(), _stream(stream)))
    return bmap


def svga_permute_tokens_mapped(src: torch.Tensor, dst: torch.Tensor, problem: ProblemSpec,
                               bmap: BlockMap, stream=None) -> torch.Tensor:
    a = _Args()
    ps, = a.tokens(problem, src=src)
    pd, = a.positions(problem, dst=dst)
    a.done()
    _check(load().svga_permute_tokens_mapped(ps, pd, ctypes.byref(problem.c),
                                             ctypes.byref(bmap.c), _stream(stream)))
    return dst


def svga_unpermute_tokens_mapped(src: torch.Tensor, dst: torch.Tensor, problem: ProblemSpec,
                                 bmap: BlockMap, stream=None) -> torch.Tensor:
    a = _Args()
    ps, = a.positions(problem, src=src)
    pd, = a.tokens(problem, dst=dst)
    a.done()
    _check(load().svga_unpermute_tokens_mapped(ps, pd, ctypes.byref(problem.c),
                                               ctypes.byref(bmap.c), _stream(stream)))
    return dst


def version() -> int:
    return load().svga_version()


def status_string(status: int) -> str:
    return load().svga_status_string(int(status)).decode()
