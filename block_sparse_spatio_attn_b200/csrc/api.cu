// api.cu -- the C entry points of svga.h: validation, sizes and launches.
#include <cuda_runtime.h>

#include <climits>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "svga_internal.h"

namespace svga {

namespace {
thread_local char g_last_error[512] = "";

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

void set_error(const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

static bool valid_tile(int t) { return t == 64 || t == 128 || t == 256; }

// Shape checks shared by every call that takes a problem.  Per-head arrays: kHeadsSkip
// does not look at them, kHeadsRequired needs and checks them, kHeadsIfGiven checks them
// unless all three are NULL (a problem routed by the classifier on the device).
enum { kHeadsSkip = 0, kHeadsRequired = 1, kHeadsIfGiven = 2 };

static svga_status validate_shape(const svga_problem *p, Geometry *g, int heads_mode)
{
    if (!p) {
        set_error("problem is NULL");
        return SVGA_ERR_INVALID_ARG;
    }
    if (p->heads < 1 || p->heads > kMaxHeads) {
        set_error("heads = %d outside 1..%d", p->heads, kMaxHeads);
        return SVGA_ERR_SHAPE;
    }
    if (p->num_frames < 1 || p->grid_h < 1 || p->grid_w < 1 || p->num_frames > 65535) {
        set_error("frames %d and grid %dx%d must be positive (frames <= 65535)", p->num_frames,
                  p->grid_h, p->grid_w);
        return SVGA_ERR_SHAPE;
    }
    const long long S = (long long)p->grid_h * p->grid_w;
    const long long N = S * p->num_frames;
    if (S > 65535 || N > kMaxTokens) {
        set_error("tokens per frame %lld (max 65535) or tokens %lld (max %d) too large", S, N,
                  kMaxTokens);
        return SVGA_ERR_SHAPE;
    }
    if (p->head_dim != 64 && p->head_dim != 128) {
        set_error("head_dim %d unsupported (64 or 128)", p->head_dim);
        return SVGA_ERR_UNSUPPORTED;
    }
    if (p->anchor_frame0 != 0 && p->anchor_frame0 != 1) {
        set_error("anchor_frame0 must be 0 or 1");
        return SVGA_ERR_INVALID_ARG;
    }
    if (!valid_tile(p->tile_q) || !valid_tile(p->tile_k)) {
        set_error("tile %dx%d unsupported (64, 128 or 256)", p->tile_q, p->tile_k);
        return SVGA_ERR_UNSUPPORTED;
    }
    const int tmax = p->tile_q > p->tile_k ? p->tile_q : p->tile_k;
    if (p->frame_pad < 0 || p->frame_pad > 65536 || (p->frame_pad % tmax) != 0) {
        set_error("frame_pad %d must be 0 or a multiple of max(tile_q, tile_k) = %d up to 65536",
                  p->frame_pad, tmax);
        return SVGA_ERR_INVALID_ARG;
    }
    const long long Sp = p->frame_pad ? (S + p->frame_pad - 1) / p->frame_pad * p->frame_pad : S;
    const long long NP = Sp * p->num_frames;  // positions per head
    if (NP > kMaxTokens) {
        set_error("padded positions %lld (frames x %lld) above %d", NP, Sp, kMaxTokens);
        return SVGA_ERR_SHAPE;
    }
    {
        // the CSR offsets and the plan's entry offsets are int32: the tile count (the
        // lists' capacity) and the plan's entry capacity must fit
        const long long tiles = (long long)p->heads * ((NP + p->tile_q - 1) / p->tile_q) *
                                ((NP + p->tile_k - 1) / p->tile_k);
        const long long kn = p->tile_k < 128 ? p->tile_k : 128;
        const long long entries =
            (long long)p->heads * (((NP + kBlockM - 1) / kBlockM + 1) / 2) * ((NP + kn - 1) / kn);
        if (tiles > INT32_MAX || entries > INT32_MAX) {
            set_error("problem too large: %lld tiles and %lld plan entries, int32 offsets "
                      "hold at most %d",
                      tiles, entries, INT32_MAX);
            return SVGA_ERR_SHAPE;
        }
    }
    const bool none_given = p->head_type == nullptr && p->band == nullptr && p->order == nullptr;
    if (heads_mode == kHeadsRequired || (heads_mode == kHeadsIfGiven && !none_given)) {
        if (!p->head_type || !p->band || !p->order) {
            set_error("head_type, band and order must be host arrays of `heads` entries");
            return SVGA_ERR_INVALID_ARG;
        }
        for (int h = 0; h < p->heads; ++h) {
            if (p->head_type[h] != SVGA_HEAD_SPATIAL && p->head_type[h] != SVGA_HEAD_TEMPORAL) {
                set_error("head %d: head_type %d invalid", h, p->head_type[h]);
                return SVGA_ERR_INVALID_ARG;
            }
            if (p->band[h] < 0 || p->band[h] > 65535) {
                set_error("head %d: band %d outside 0..65535", h, p->band[h]);
                return SVGA_ERR_INVALID_ARG;
            }
            if (p->order[h] < SVGA_ORDER_FRAME_MAJOR || p->order[h] > SVGA_ORDER_TEMPORAL_MAJOR_STRICT) {
                set_error("head %d: order %d invalid", h, p->order[h]);
                return SVGA_ERR_INVALID_ARG;
            }
        }
    }
    g->heads = p->heads;
    g->F = p->num_frames;
    g->S = (int)S;
    g->N = (int)N;
    g->Sp = (int)Sp;
    g->NP = (int)NP;
    g->d = p->head_dim;
    g->tile_q = p->tile_q;
    g->tile_k = p->tile_k;
    g->n_q = ceil_div(NP, p->tile_q);
    g->n_k = ceil_div(NP, p->tile_k);
    g->kn = p->tile_k < 128 ? p->tile_k : 128;
    g->n_qblk = ceil_div(NP, kBlockM);
    g->n_pairs = ceil_div(g->n_qblk, 2);
    g->n_kc = ceil_div(NP, g->kn);
    g->n_items = g->heads * g->n_pairs;
    return SVGA_OK;
}

svga_status validate_problem(const svga_problem *p, Geometry *g)
{
    return validate_shape(p, g, kHeadsRequired);
}

svga_status validate_geometry(const svga_problem *p, Geometry *g)
{
    return validate_shape(p, g, kHeadsSkip);
}

size_t plan_header_bytes(const Geometry &g)
{
    return align_up(sizeof(PlanHeader) + sizeof(int4) * ((size_t)g.heads + g.n_items), 256);
}

int64_t plan_entry_cap(const Geometry &g) { return (int64_t)g.n_items * g.n_kc; }

size_t plan_bytes_needed(const Geometry &g)
{
    return plan_header_bytes(g) + sizeof(uint32_t) * (size_t)plan_entry_cap(g);
}

static svga_status check_tensor(const void *p, const char *name)
{
    if (!p) {
        set_error("%s is NULL", name);
        return SVGA_ERR_INVALID_ARG;
    }
    if (!aligned(p, 16)) {
        set_error("%s is not 16-byte aligned", name);
        return SVGA_ERR_ALIGNMENT;
    }
    return SVGA_OK;
}

static svga_status check_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("%s: %s", what, cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    return SVGA_OK;
}

svga_status check_map_outputs(const Geometry &g, const svga_block_map *map)
{
    if (!map || !map->cls || !map->full_ptr || !map->full_idx || !map->bnd_ptr || !map->bnd_idx ||
        !map->plan) {
        set_error("block map buffers must be non-NULL device pointers");
        return SVGA_ERR_INVALID_ARG;
    }
    if (!aligned(map->plan, 256) || !aligned(map->full_ptr, 4) || !aligned(map->bnd_ptr, 4) ||
        !aligned(map->full_idx, 4) || !aligned(map->bnd_idx, 4)) {
        set_error("plan must be 256-byte aligned, CSR arrays 4-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    // The plan's worst case is required: a build into a smaller plan would have to drop
    // entries while its items still count them.
    if (map->plan_bytes < plan_bytes_needed(g) || map->full_cap < 0 || map->bnd_cap < 0) {
        set_error("plan (%zu bytes, needs %zu) smaller than svga_block_map_size, or a negative "
                  "list capacity",
                  map->plan_bytes, plan_bytes_needed(g));
        return SVGA_ERR_WORKSPACE;
    }
    return SVGA_OK;
}

svga_status check_map_plan(const Geometry &g, const svga_block_map *map)
{
    if (!map || !map->plan) {
        set_error("block map or its plan is NULL");
        return SVGA_ERR_INVALID_ARG;
    }
    if (!aligned(map->plan, 256)) {
        set_error("the block map's plan must be 256-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    if (map->plan_bytes < plan_bytes_needed(g)) {
        set_error("block map plan (%zu bytes) smaller than svga_block_map_size (%zu) for this "
                  "problem",
                  map->plan_bytes, plan_bytes_needed(g));
        return SVGA_ERR_INVALID_ARG;
    }
    return SVGA_OK;
}

static svga_status check_map_buffers(const Geometry &g, const svga_block_map *map,
                                     const void *workspace, size_t workspace_bytes)
{
    svga_status rc = check_map_outputs(g, map);
    if (rc != SVGA_OK) return rc;
    if (!workspace) {
        set_error("the build workspace must be a non-NULL device pointer");
        return SVGA_ERR_INVALID_ARG;
    }
    if (!aligned(workspace, 256)) {
        set_error("the build workspace must be 256-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    if (workspace_bytes < block_map_workspace_bytes(g)) {
        set_error("workspace (%zu < %zu) smaller than svga_block_map_size", workspace_bytes,
                  block_map_workspace_bytes(g));
        return SVGA_ERR_WORKSPACE;
    }
    return SVGA_OK;
}

}  // namespace svga

using namespace svga;

extern "C" {

svga_status svga_problem_rows(const svga_problem *problem, int64_t *rows)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if (!rows) {
        set_error("rows is NULL");
        return SVGA_ERR_INVALID_ARG;
    }
    *rows = g.NP;
    return SVGA_OK;
}

svga_status svga_block_map_size(const svga_problem *problem, size_t *cls_bytes, size_t *ptr_bytes,
                                int64_t *full_cap, int64_t *bnd_cap, size_t *plan_bytes,
                                size_t *workspace_bytes)
{
    Geometry g;  // sizes depend on the geometry only, not on the heads' types
    svga_status rc = validate_shape(problem, &g, kHeadsIfGiven);
    if (rc != SVGA_OK) return rc;
    const int64_t tiles = (int64_t)g.heads * g.n_q * g.n_k;
    if (cls_bytes) *cls_bytes = (size_t)tiles;
    if (ptr_bytes) *ptr_bytes = sizeof(int32_t) * ((size_t)g.heads * g.n_q + 1);
    if (full_cap) *full_cap = tiles;
    if (bnd_cap) *bnd_cap = tiles;
    if (plan_bytes) *plan_bytes = plan_bytes_needed(g);
    if (workspace_bytes) *workspace_bytes = block_map_workspace_bytes(g);
    return SVGA_OK;
}

static svga_status check_bands(int heads, const int32_t *w_spatial, const int32_t *w_temporal)
{
    if (!w_spatial || !w_temporal) {
        set_error("w_spatial and w_temporal must be host arrays of `heads` entries");
        return SVGA_ERR_INVALID_ARG;
    }
    for (int h = 0; h < heads; ++h)
        if (w_spatial[h] < 0 || w_spatial[h] > 65535 || w_temporal[h] < 0 || w_temporal[h] > 65535) {
            set_error("head %d: candidate bands must be in 0..65535", h);
            return SVGA_ERR_INVALID_ARG;
        }
    return SVGA_OK;
}

svga_status svga_build_block_map(const svga_problem *problem, svga_block_map *map, void *workspace,
                                 size_t workspace_bytes, svga_stream_t stream)
{
    Geometry g;
    svga_status rc = validate_problem(problem, &g);
    if (rc != SVGA_OK) return rc;
    if ((rc = check_map_buffers(g, map, workspace, workspace_bytes)) != SVGA_OK) return rc;
    return launch_build_block_map(problem, g, map, workspace, workspace_bytes, stream);
}

svga_status svga_build_block_map_routed(const svga_problem *problem, const int32_t *head_type_dev,
                                        const int32_t *w_spatial, const int32_t *w_temporal,
                                        svga_block_map *map, void *workspace,
                                        size_t workspace_bytes, svga_stream_t stream)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if ((rc = check_bands(g.heads, w_spatial, w_temporal)) != SVGA_OK) return rc;
    if (!head_type_dev || !aligned(head_type_dev, 4)) {
        set_error("head_type_dev must be a 4-byte aligned device array of `heads` int32");
        return SVGA_ERR_INVALID_ARG;
    }
    if ((rc = check_map_buffers(g, map, workspace, workspace_bytes)) != SVGA_OK) return rc;
    return launch_build_block_map(problem, g, map, workspace, workspace_bytes, stream,
                                  head_type_dev, w_spatial, w_temporal);
}

// src and dst of a permutation must not overlap: the frame-major side has N rows per
// head, the token-order side NP.
static svga_status check_no_overlap(const Geometry &g, const void *src, const void *dst,
                                   int inverse)
{
    const size_t fm = (size_t)g.heads * g.N * g.d * 2, pos = (size_t)g.heads * g.NP * g.d * 2;
    const size_t sb = inverse ? pos : fm, db = inverse ? fm : pos;
    const char *s = static_cast<const char *>(src), *d = static_cast<const char *>(dst);
    if (s < d + db && d < s + sb) {
        set_error("src and dst overlap");
        return SVGA_ERR_INVALID_ARG;
    }
    return SVGA_OK;
}

static svga_status permute_common(const void *src, void *dst, const svga_problem *problem,
                                  svga_stream_t stream, int inverse)
{
    Geometry g;
    svga_status rc = validate_problem(problem, &g);
    if (rc != SVGA_OK) return rc;
    if ((rc = check_tensor(src, "src")) != SVGA_OK || (rc = check_tensor(dst, "dst")) != SVGA_OK)
        return rc;
    if ((rc = check_no_overlap(g, src, dst, inverse)) != SVGA_OK) return rc;
    return launch_permute(src, dst, problem, g, inverse, stream);
}

static svga_status permute_mapped_common(const void *src, void *dst, const svga_problem *problem,
                                         const svga_block_map *map, svga_stream_t stream,
                                         int inverse)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if ((rc = check_map_plan(g, map)) != SVGA_OK) return rc;
    if ((rc = check_tensor(src, "src")) != SVGA_OK || (rc = check_tensor(dst, "dst")) != SVGA_OK)
        return rc;
    if ((rc = check_no_overlap(g, src, dst, inverse)) != SVGA_OK) return rc;
    return launch_permute(src, dst, problem, g, inverse, stream, map->plan, map->status);
}

svga_status svga_permute_tokens_mapped(const void *src, void *dst, const svga_problem *problem,
                                       const svga_block_map *map, svga_stream_t stream)
{
    return permute_mapped_common(src, dst, problem, map, stream, 0);
}

svga_status svga_unpermute_tokens_mapped(const void *src, void *dst, const svga_problem *problem,
                                         const svga_block_map *map, svga_stream_t stream)
{
    return permute_mapped_common(src, dst, problem, map, stream, 1);
}

svga_status svga_permute_tokens(const void *src, void *dst, const svga_problem *problem,
                                svga_stream_t stream)
{
    return permute_common(src, dst, problem, stream, 0);
}

svga_status svga_unpermute_tokens(const void *src, void *dst, const svga_problem *problem,
                                  svga_stream_t stream)
{
    return permute_common(src, dst, problem, stream, 1);
}

namespace {

svga_status sparse_fwd_common(const void *q, const void *k, const void *v, void *o, float *lse,
                              const svga_problem *problem, const svga_block_map *map,
                              float scale, int flags, int part, int num_parts,
                              svga_stream_t stream)
{
    if (num_parts < 1 || num_parts > kMaxParts || part < 0 || part >= num_parts) {
        set_error("part %d of %d: need 1 <= num_parts <= %d and 0 <= part < num_parts", part,
                  num_parts, kMaxParts);
        return SVGA_ERR_INVALID_ARG;
    }
    Geometry g;  // per-head type, band and order are read from the plan on the device
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if ((rc = check_tensor(q, "q")) != SVGA_OK || (rc = check_tensor(k, "k")) != SVGA_OK ||
        (rc = check_tensor(v, "v")) != SVGA_OK || (rc = check_tensor(o, "o")) != SVGA_OK)
        return rc;
    if (lse && !aligned(lse, 4)) {
        set_error("lse is not 4-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    if ((rc = check_map_plan(g, map)) != SVGA_OK) return rc;
    if (flags & ~(SVGA_FLAG_NAIVE_B1 | SVGA_FLAG_TILE_ALIGNED | SVGA_FLAG_TEST_STALL |
                  SVGA_FLAG_QO_FRAME_MAJOR | SVGA_FLAG_KV_FRAME_MAJOR | SVGA_FLAG_CTA_PAIR)) {
        set_error("unknown flags 0x%x", flags);
        return SVGA_ERR_INVALID_ARG;
    }
    if ((flags & SVGA_FLAG_NAIVE_B1) && (flags & SVGA_FLAG_TILE_ALIGNED)) {
        set_error("SVGA_FLAG_NAIVE_B1 and SVGA_FLAG_TILE_ALIGNED exclude each other");
        return SVGA_ERR_INVALID_ARG;
    }
    if ((flags & (SVGA_FLAG_QO_FRAME_MAJOR | SVGA_FLAG_KV_FRAME_MAJOR |
                  SVGA_FLAG_TILE_ALIGNED)) &&
        g.Sp != g.S) {
        // the padded layout is the other reading of the tile-aligned traversal
        set_error("frame-major q / o or k / v and the snapped tile-aligned mask need "
                  "frame_pad = 0 (got %d)",
                  problem->frame_pad);
        return SVGA_ERR_UNSUPPORTED;
    }
    if ((flags & SVGA_FLAG_TILE_ALIGNED) && problem->tile_q < kBlockM) {
        // a 128-row query block would hold two query tiles with different key sets
        set_error("SVGA_FLAG_TILE_ALIGNED needs tile_q >= %d (got %d)", kBlockM, problem->tile_q);
        return SVGA_ERR_UNSUPPORTED;
    }
    if (!(scale > 0.f) || !(scale < 1e30f)) {
        set_error("scale must be a positive finite number");
        return SVGA_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (map->status && cudaMemsetAsync(map->status, 0, sizeof(int32_t), st) != cudaSuccess)
        return check_launch("cudaMemsetAsync(status)");
    AttnLaunch a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.lse = lse;
    a.heads = g.heads;
    a.nq_rows = g.NP;
    a.nk_rows = g.NP;
    a.d = g.d;
    a.F = g.F;
    a.S = g.S;
    a.N = g.N;
    a.Sp = g.Sp;
    a.anchor = problem->anchor_frame0;
    a.scale = scale;
    a.mode = 0;
    a.naive = (flags & SVGA_FLAG_NAIVE_B1) ? 1 : 0;
    a.aligned = (flags & SVGA_FLAG_TILE_ALIGNED) ? 1 : 0;
    a.test_stall = (flags & SVGA_FLAG_TEST_STALL) ? 1 : 0;
    a.qo_fm = (flags & SVGA_FLAG_QO_FRAME_MAJOR) ? 1 : 0;
    a.kv_fm = (flags & SVGA_FLAG_KV_FRAME_MAJOR) ? 1 : 0;
    a.cta_pair = (flags & SVGA_FLAG_CTA_PAIR) ? 1 : 0;
    a.kn = g.kn;
    a.tile_q = g.tile_q;
    a.tile_k = g.tile_k;
    a.check_plan = 1;  // the map is the caller's: its header must describe this problem
    a.plan = map->plan;
    a.n_items = g.n_items;
    a.part = part;
    a.num_parts = num_parts;
    a.status = map->status;
    return launch_attention(a, stream);
}

}  // namespace

svga_status svga_sparse_attention_fwd(const void *q, const void *k, const void *v, void *o,
                                      float *lse, const svga_problem *problem,
                                      const svga_block_map *map, float scale, int flags,
                                      svga_stream_t stream)
{
    return sparse_fwd_common(q, k, v, o, lse, problem, map, scale, flags, 0, 1, stream);
}

svga_status svga_sparse_attention_fwd_part(const void *q, const void *k, const void *v, void *o,
                                           float *lse, const svga_problem *problem,
                                           const svga_block_map *map, float scale, int flags,
                                           int part, int num_parts, svga_stream_t stream)
{
    return sparse_fwd_common(q, k, v, o, lse, problem, map, scale, flags, part, num_parts,
                             stream);
}

svga_status svga_dense_attention_fwd(const void *q, const void *k, const void *v, void *o,
                                     float *lse, int heads, int tokens, int head_dim, float scale,
                                     int32_t *status, svga_stream_t stream)
{
    if (heads < 1 || heads > kMaxHeads || tokens < 1 || tokens > kMaxTokens) {
        set_error("heads %d / tokens %d outside 1..%d / 1..%d", heads, tokens, kMaxHeads,
                  kMaxTokens);
        return SVGA_ERR_SHAPE;
    }
    if (head_dim != 64 && head_dim != 128) {
        set_error("head_dim %d unsupported (64 or 128)", head_dim);
        return SVGA_ERR_UNSUPPORTED;
    }
    svga_status rc;
    if ((rc = check_tensor(q, "q")) != SVGA_OK || (rc = check_tensor(k, "k")) != SVGA_OK ||
        (rc = check_tensor(v, "v")) != SVGA_OK || (rc = check_tensor(o, "o")) != SVGA_OK)
        return rc;
    if (lse && !aligned(lse, 4)) {
        set_error("lse is not 4-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    if (!(scale > 0.f) || !(scale < 1e30f)) {
        set_error("scale must be a positive finite number");
        return SVGA_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (status && cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess)
        return check_launch("cudaMemsetAsync(status)");
    AttnLaunch a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.lse = lse;
    a.heads = heads;
    a.nq_rows = tokens;
    a.nk_rows = tokens;
    a.d = head_dim;
    a.F = 1;
    a.S = tokens;
    a.scale = scale;
    a.mode = 1;
    a.kn = 128;
    const int n_qblk = (tokens + kBlockM - 1) / kBlockM;
    a.n_items = heads * ((n_qblk + 1) / 2);
    a.status = status;
    return launch_attention(a, stream);
}

svga_status svga_classify_size(const svga_problem *problem, int n_rows, size_t *workspace_bytes)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if (n_rows < 1 || n_rows > g.N) {
        set_error("n_rows %d outside 1..%d", n_rows, g.N);
        return SVGA_ERR_SHAPE;
    }
    if (workspace_bytes) *workspace_bytes = classify_workspace_bytes(problem, n_rows, 2);
    return SVGA_OK;
}

static svga_status check_classify(const void *q, const void *k, const void *v,
                                  const svga_problem *problem, const int32_t *w_spatial,
                                  const int32_t *w_temporal, const int32_t *rows, int n_rows,
                                  float scale, const int32_t *head_type_out, const void *workspace,
                                  size_t workspace_bytes)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if ((rc = check_tensor(q, "q")) != SVGA_OK || (rc = check_tensor(k, "k")) != SVGA_OK ||
        (rc = check_tensor(v, "v")) != SVGA_OK)
        return rc;
    if (n_rows < 1 || n_rows > g.N) {
        set_error("n_rows %d outside 1..%d", n_rows, g.N);
        return SVGA_ERR_SHAPE;
    }
    if ((rc = check_bands(g.heads, w_spatial, w_temporal)) != SVGA_OK) return rc;
    if (!head_type_out || !aligned(head_type_out, 4)) {
        set_error("head_type_out missing or not 4-byte aligned");
        return SVGA_ERR_INVALID_ARG;
    }
    if (rows && !aligned(rows, 4)) {
        set_error("rows is not 4-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    if (!(scale > 0.f) || !(scale < 1e30f)) {
        set_error("scale must be a positive finite number");
        return SVGA_ERR_INVALID_ARG;
    }
    if (!workspace || !aligned(workspace, 256) ||
        workspace_bytes < classify_workspace_bytes(problem, n_rows, 2)) {
        set_error("workspace missing, not 256-byte aligned or smaller than svga_classify_size");
        return SVGA_ERR_WORKSPACE;
    }
    return SVGA_OK;
}

svga_status svga_classify_heads(const void *q, const void *k, const void *v,
                                const svga_problem *problem, const int32_t *w_spatial,
                                const int32_t *w_temporal, const int32_t *rows, int n_rows,
                                float scale, int32_t *head_type_out, float *mse_out,
                                void *workspace, size_t workspace_bytes, svga_stream_t stream)
{
    svga_status rc = check_classify(q, k, v, problem, w_spatial, w_temporal, rows, n_rows, scale,
                                    head_type_out, workspace, workspace_bytes);
    if (rc != SVGA_OK) return rc;
    return run_classify(q, k, v, problem, w_spatial, w_temporal, rows, n_rows, scale,
                        head_type_out, mse_out, nullptr, 0, workspace, workspace_bytes, stream);
}

svga_status svga_classify_heads_async(const void *q, const void *k, const void *v,
                                      const svga_problem *problem, const int32_t *w_spatial,
                                      const int32_t *w_temporal, const int32_t *rows, int n_rows,
                                      float scale, int32_t *head_type_dev, float *mse_dev,
                                      int32_t *status_dev, void *workspace,
                                      size_t workspace_bytes, svga_stream_t stream)
{
    svga_status rc = check_classify(q, k, v, problem, w_spatial, w_temporal, rows, n_rows, scale,
                                    head_type_dev, workspace, workspace_bytes);
    if (rc != SVGA_OK) return rc;
    if ((mse_dev && !aligned(mse_dev, 4)) || (status_dev && !aligned(status_dev, 4))) {
        set_error("mse_dev and status_dev must be 4-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    return run_classify(q, k, v, problem, w_spatial, w_temporal, rows, n_rows, scale,
                        head_type_dev, mse_dev, status_dev, 1, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

// Kept (query, key) pairs of one head over the whole problem, counted in closed form
// from the masks' definitions (every query keeps the keys of frames within `band` of its
// own, or of in-frame indices within `band` of its own, plus frame 0 with the anchor).
long long kept_pairs(int type, int band, int anchor, long long F, long long S)
{
    if (type == SVGA_HEAD_SPATIAL) {
        long long frames = 0;  // kept key frames, summed over the query frames
        for (long long fq = 0; fq < F; ++fq) {
            const long long lo = fq - band > 0 ? fq - band : 0;
            const long long hi = fq + band < F - 1 ? fq + band : F - 1;
            frames += hi - lo + 1 + ((anchor && lo > 0) ? 1 : 0);
        }
        return frames * S * S;
    }
    long long c = 0;  // kept in-frame pairs (|s_q - s_k| <= band), summed over s_q
    for (long long sq = 0; sq < S; ++sq) {
        const long long lo = sq - band > 0 ? sq - band : 0;
        const long long hi = sq + band < S - 1 ? sq + band : S - 1;
        c += hi - lo + 1;
    }
    return F * (F * c + (anchor ? S * S - c : 0));
}

}  // namespace

extern "C" {

svga_status svga_kept_fraction(const svga_problem *problem, int head_type, int band,
                               double *fraction)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if ((head_type != SVGA_HEAD_SPATIAL && head_type != SVGA_HEAD_TEMPORAL) || band < 0 ||
        band > 65535 || !fraction) {
        set_error("head_type must be 0 / 1, band 0..65535 and fraction non-NULL");
        return SVGA_ERR_INVALID_ARG;
    }
    const double n = (double)g.N;
    *fraction = (double)kept_pairs(head_type, band, problem->anchor_frame0, g.F, g.S) / (n * n);
    return SVGA_OK;
}

svga_status svga_autotune_size(const svga_problem *problem, int n_rows, int n_cand,
                               size_t *workspace_bytes)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if (n_rows < 1 || n_rows > g.N || n_cand < 1 || n_cand > max_candidates()) {
        set_error("n_rows %d outside 1..%d or n_cand %d outside 1..%d", n_rows, g.N, n_cand,
                  max_candidates());
        return SVGA_ERR_SHAPE;
    }
    if (workspace_bytes) *workspace_bytes = classify_workspace_bytes(problem, n_rows, n_cand);
    return SVGA_OK;
}

svga_status svga_autotune_heads(const void *q, const void *k, const void *v,
                                const svga_problem *problem, const int32_t *cand_type,
                                const int32_t *cand_band, int n_cand, double max_kept_fraction,
                                const int32_t *rows, int n_rows, float scale,
                                int32_t *head_type_out, int32_t *band_out, float *mse_out,
                                void *workspace, size_t workspace_bytes, svga_stream_t stream)
{
    Geometry g;
    svga_status rc = validate_shape(problem, &g, kHeadsSkip);
    if (rc != SVGA_OK) return rc;
    if ((rc = check_tensor(q, "q")) != SVGA_OK || (rc = check_tensor(k, "k")) != SVGA_OK ||
        (rc = check_tensor(v, "v")) != SVGA_OK)
        return rc;
    if (n_rows < 1 || n_rows > g.N || n_cand < 1 || n_cand > max_candidates()) {
        set_error("n_rows %d outside 1..%d or n_cand %d outside 1..%d", n_rows, g.N, n_cand,
                  max_candidates());
        return SVGA_ERR_SHAPE;
    }
    if (!cand_type || !cand_band || !head_type_out || !band_out) {
        set_error("cand_type, cand_band, head_type_out and band_out must be host arrays");
        return SVGA_ERR_INVALID_ARG;
    }
    if (!(max_kept_fraction > 0.0) || !(max_kept_fraction <= 1.0)) {
        set_error("max_kept_fraction must lie in (0, 1]");
        return SVGA_ERR_INVALID_ARG;
    }
    uint32_t eligible = 0;
    for (int c = 0; c < n_cand; ++c) {
        double f = 0.0;
        if ((rc = svga_kept_fraction(problem, cand_type[c], cand_band[c], &f)) != SVGA_OK)
            return rc;
        if (f <= max_kept_fraction) eligible |= 1u << c;
    }
    if (!eligible) {
        set_error("no candidate keeps at most %.6f of the pairs", max_kept_fraction);
        return SVGA_ERR_INVALID_ARG;
    }
    if (rows && !aligned(rows, 4)) {
        set_error("rows is not 4-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    if (!(scale > 0.f) || !(scale < 1e30f)) {
        set_error("scale must be a positive finite number");
        return SVGA_ERR_INVALID_ARG;
    }
    if (!workspace || !aligned(workspace, 256) ||
        workspace_bytes < classify_workspace_bytes(problem, n_rows, n_cand)) {
        set_error("workspace missing, not 256-byte aligned or smaller than svga_autotune_size");
        return SVGA_ERR_WORKSPACE;
    }
    return run_select(q, k, v, problem, n_cand, cand_type, cand_band, eligible, nullptr,
                      nullptr, rows, n_rows, scale, head_type_out, band_out, mse_out, nullptr, 0,
                      workspace, workspace_bytes, stream);
}

const char *svga_last_error(void) { return g_last_error; }

const char *svga_status_string(svga_status s)
{
    switch (s) {
    case SVGA_OK: return "SVGA_OK";
    case SVGA_ERR_INVALID_ARG: return "SVGA_ERR_INVALID_ARG";
    case SVGA_ERR_SHAPE: return "SVGA_ERR_SHAPE";
    case SVGA_ERR_ALIGNMENT: return "SVGA_ERR_ALIGNMENT";
    case SVGA_ERR_UNSUPPORTED: return "SVGA_ERR_UNSUPPORTED";
    case SVGA_ERR_WORKSPACE: return "SVGA_ERR_WORKSPACE";
    case SVGA_ERR_CUDA: return "SVGA_ERR_CUDA";
    case SVGA_ERR_TIMEOUT: return "SVGA_ERR_TIMEOUT";
    }
    return "unknown svga_status";
}

int svga_version(void) { return SVGA_VERSION; }

}  // extern "C"
