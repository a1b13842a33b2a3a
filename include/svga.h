/*
 * svga.h -- C ABI of the block-sparse spatio-temporal attention library (B200, sm_100a).
 *
 * The library computes the forward pass of Sparse-VideoGen-style block-sparse
 * self-attention for video diffusion, as described in "Accelerating Spatio-Temporal
 * Attention for Video Diffusion on TPUs" (Google for Developers), of which three
 * summaries exist: ainews.tenesys.com (Polish), aihirek.info (Hungarian) and
 * oossa.com (German).  Citations below name the page and its section.
 *
 * Conventions for every call:
 *   - Tensors are DEVICE pointers to contiguous [heads, tokens, head_dim] bf16
 *     (row-major, head_dim fastest), 16-byte aligned.  tokens = F * H * W.
 *   - The caller owns all memory.  The library never allocates device memory;
 *     sizes of the caller-provided buffers come from the *_size queries.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) unless stated otherwise.
 *   - Arguments are validated on the host before any launch.  A failed check
 *     returns a status other than SVGA_OK and launches nothing; the message is
 *     available from svga_last_error() (thread-local).
 *   - Kernels that wait on the GPU (mbarrier waits) give up after about one
 *     second, write SVGA_ERR_TIMEOUT into the caller's status word (when one is
 *     given) and return; the CUDA context stays usable.
 *   - Launch errors are reported as SVGA_ERR_CUDA.
 */
#ifndef SVGA_H
#define SVGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SVGA_VERSION 1

#if defined(__GNUC__)
#define SVGA_API __attribute__((visibility("default")))
#else
#define SVGA_API
#endif

typedef void *svga_stream_t; /* a cudaStream_t */

typedef enum {
    SVGA_OK = 0,
    SVGA_ERR_INVALID_ARG = 1, /* null pointer, bad enum value, negative band ... */
    SVGA_ERR_SHAPE = 2,       /* sizes outside the supported range */
    SVGA_ERR_ALIGNMENT = 3,   /* a pointer not aligned as required */
    SVGA_ERR_UNSUPPORTED = 4, /* a valid request this build does not implement */
    SVGA_ERR_WORKSPACE = 5,   /* a caller buffer smaller than the size query says */
    SVGA_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
    SVGA_ERR_TIMEOUT = 7      /* written by a kernel that gave up waiting */
} svga_status;

/* Head types.  Spatial heads attend to patches of the same or nearby frames;
 * temporal heads follow a small in-frame region across many frames (aihirek.info,
 * section "A Sparse VideoGen a figyelmi fejeket osztalyozza"). */
enum { SVGA_HEAD_SPATIAL = 0, SVGA_HEAD_TEMPORAL = 1 };

/* Token orders.  Tokens arrive frame-major (position f*S + s).  The pages move the
 * tokens of temporal heads to temporal-major order (ainews.tenesys.com, "Co sie
 * zmienilo?" item 5) without giving the exact map.  This library's reading:
 *   SVGA_ORDER_TEMPORAL_MAJOR: frame-0 tokens first (position s), then the other
 *       frames s-major: position S + s*(F-1) + (f-1)  ("anchor-first");
 *   SVGA_ORDER_TEMPORAL_MAJOR_STRICT: the literal transpose, position s*F + f. */
enum {
    SVGA_ORDER_FRAME_MAJOR = 0,
    SVGA_ORDER_TEMPORAL_MAJOR = 1,
    SVGA_ORDER_TEMPORAL_MAJOR_STRICT = 2
};

/* Flags of svga_sparse_attention_fwd. */
enum {
    /* Naive traversal: every visited tile goes through the masked (boundary) path,
     * the first sparse kernel of the pages, which masked exactly inside every
     * visited tile (aihirek.info, section "A TPU-kernel kialakitasa dontonek
     * bizonyult"; ainews.tenesys.com, "Co sie zmienilo?" item 1). */
    SVGA_FLAG_NAIVE_B1 = 1,
    /* Tile-aligned traversal (B3): the mask is snapped to the tiles of the block map,
     * so a query keeps every key of every visited tile, and no visited tile is masked
     * element by element (ainews.tenesys.com, "Co sie zmienilo?" item 4: the final
     * "tile-aligned" sparse traversal; oossa.com, opening paragraph: the kernel aligns
     * the attention mask with the tiles it computes).  The kept set then depends on
     * order[h] and the tile size and is a superset of the exact one; the result is the
     * plain masked softmax over that set.  Needs tile_q >= 128 (SVGA_ERR_UNSUPPORTED
     * otherwise); cannot be combined with SVGA_FLAG_NAIVE_B1 (SVGA_ERR_INVALID_ARG). */
    SVGA_FLAG_TILE_ALIGNED = 2,
    /* q, o and lse are FRAME-MAJOR for every head (k and v stay in order[h]): the
     * kernel gathers each query row from its frame-major token and writes O and LSE
     * back to it, so the permutation of Q and the inverse permutation of O are not
     * needed (the pages move the tokens of temporal heads to temporal-major order,
     * ainews.tenesys.com, "Co sie zmienilo?" item 5; here only K and V move).
     * Results are identical bit for bit to permute -> attention -> unpermute. */
    SVGA_FLAG_QO_FRAME_MAJOR = 4,
    /* k and v are FRAME-MAJOR for every head: the kernel reads the key rows of a head
     * kept in a temporal-major order from their frame-major tokens (a gather of the
     * chunk's rows into the same shared-memory layout the tile load gives), so the
     * permutation of K and V is not needed either.  With SVGA_FLAG_QO_FRAME_MAJOR no
     * tensor moves at all.  Results are identical bit for bit to the permuted call. */
    SVGA_FLAG_KV_FRAME_MAJOR = 8,
    /* Run the work items on CTA pairs (two SMs, one tcgen05.mma over both blocks of an
     * item, each SM holding half of every K and V chunk and two S tiles) instead of
     * one CTA per item.  Same result within the tolerance, not bit for bit: the
     * softmax takes its reference maximum per tile pair of visits differently.  Slower
     * than the default on B200 at d = 128 (about 10 % at 75,600 tokens); kept for
     * study.  Applies to head_dim 128 with 128-key chunks, bf16 K / V in each head's
     * order (not with SVGA_FLAG_KV_FRAME_MAJOR); elsewhere the flag is ignored. */
    SVGA_FLAG_CTA_PAIR = 16,
    /* Test hook for the failure path: the first K chunk of every CTA is never loaded,
     * so the kernel's bounded waits run out (about one second per CTA wave), every role
     * stops, copies in flight are drained, TMEM is released and map->status reads
     * SVGA_ERR_TIMEOUT.  O is left unwritten.  The CUDA context stays usable. */
    SVGA_FLAG_TEST_STALL = 1 << 16
};

/* The problem.  Host struct; the arrays it points to are HOST arrays of `heads`
 * entries and are read during the call only.
 *   heads          number of attention heads (1 .. 4096)
 *   num_frames     F >= 1;  grid_h, grid_w: patch grid, S = grid_h * grid_w
 *                  tokens N = F * S, 1 <= N <= 2^24, S <= 65535, F <= 65535
 *   head_dim       64 or 128
 *   head_type      SVGA_HEAD_SPATIAL or SVGA_HEAD_TEMPORAL per head
 *   band           per head: spatial keeps |f_q - f_k| <= band (frames); temporal
 *                  keeps |s_q - s_k| <= band on the flattened in-frame index
 *                  s = row * grid_w + col.  Inclusive, >= 0.
 *   order          per head: the token order Q, K, V (and O) of that head are in
 *   anchor_frame0  1: every query also keeps all keys of frame 0, the anchor
 *                  (aihirek.info, section "A Sparse VideoGen ..."); 0: no anchor
 *   tile_q, tile_k tile size of the block map: 64, 128 or 256 each
 *   frame_pad      0, or a multiple of max(tile_q, tile_k) up to 65536: the padded
 *                  layout, the exact reading of the pages' tile-aligned traversal (B3:
 *                  ainews.tenesys.com, "Co sie zmienilo?" item 4; oossa.com, opening
 *                  paragraph: the mask aligned with the tiles the kernel computes).
 *                  Frame-major heads lay frame f out at positions f*Sp + s with the
 *                  frame stride Sp = S rounded up to a multiple of frame_pad, so no
 *                  tile holds two frames; positions f*Sp + s with s >= S hold no token.
 *                  Temporal-major heads keep their order; positions N and up hold no
 *                  token.  Every tensor in token order then has NP = F * Sp rows per
 *                  head (svga_problem_rows), frame-major tensors keep N.  The kept
 *                  pairs do not change: results equal the unpadded layout's up to the
 *                  order of the fp32 sums.  A row without a token reads O = 0 and
 *                  lse = -inf.  SVGA_FLAG_QO_FRAME_MAJOR and SVGA_FLAG_KV_FRAME_MAJOR
 *                  need frame_pad = 0 (SVGA_ERR_UNSUPPORTED otherwise).
 * Lists and plan are indexed with int32: heads * ceil(NP/tile_q) * ceil(NP/tile_k) and
 * heads * ceil(NP/256) * ceil(NP/min(tile_k, 128)) must each stay below 2^31, and
 * NP <= 2^24 (SVGA_ERR_SHAPE otherwise).  NP = N without padding. */
typedef struct {
    int heads;
    int num_frames;
    int grid_h;
    int grid_w;
    int head_dim;
    const int32_t *head_type;
    const int32_t *band;
    const int32_t *order;
    int anchor_frame0;
    int tile_q;
    int tile_k;
    int frame_pad;
} svga_problem;

/* Rows per head of a tensor in token order (the permuted Q, K, V, O and lse): NP =
 * num_frames * Sp with frame_pad, N without.  Host-only; per-head arrays not read. */
SVGA_API svga_status svga_problem_rows(const svga_problem *problem, int64_t *rows);

/* The block map.  DEVICE buffers owned by the caller, sized by svga_block_map_size.
 *   cls       uint8 [heads][n_q][n_k]: 0 = no kept pair (skipped), 1 = every pair
 *             kept (full: unmasked fast path), 2 = some kept (boundary: masked).
 *             Classes are taken on the grid padded to whole tiles, where padded
 *             pairs count as not kept, so a tile holding padding is never full.
 *   full_ptr  int32 [heads * n_q + 1]: CSR row pointers over rows r = h * n_q + i
 *   full_idx  int32 [full_cap]: ascending k-tile indices of the full tiles of row r
 *             in full_idx[full_ptr[r] .. full_ptr[r+1])
 *   bnd_ptr, bnd_idx: the same for the boundary tiles
 *   plan      execution plan of the attention kernel (work items in longest-first
 *             order and their merged tile lists), plan_bytes long; its layout is
 *             internal to the library
 *   status    int32 device word or NULL; cleared by each call that takes the map,
 *             set to an svga_status by a kernel that fails on the device.
 * Every call that builds or reads a map requires plan_bytes to be at least
 * svga_block_map_size's plan_bytes for the call's problem (the worst case, so a build
 * never drops entries); a smaller plan is rejected on the host.
 * Full/boundary specialisation: full tiles take an unmasked fast path, only
 * boundary tiles are masked by coordinates (aihirek.info, section "A TPU-kernel
 * kialakitasa ..."; ainews.tenesys.com, "Co sie zmienilo?" item 2). */
typedef struct {
    uint8_t *cls;
    int32_t *full_ptr;
    int32_t *full_idx;
    int32_t *bnd_ptr;
    int32_t *bnd_idx;
    int64_t full_cap;
    int64_t bnd_cap;
    void *plan;
    size_t plan_bytes;
    int32_t *status;
} svga_block_map;

/* Sizes of the block map buffers and of the build workspace (host-only, no GPU).
 * Any output pointer may be NULL.  Capacities are worst-case (every tile in a list),
 * so a map built with them never overflows. */
SVGA_API svga_status svga_block_map_size(const svga_problem *problem, size_t *cls_bytes,
                                size_t *ptr_bytes, int64_t *full_cap, int64_t *bnd_cap,
                                size_t *plan_bytes, size_t *workspace_bytes);

/* Classify every (q-tile, k-tile) pair of every head as empty / full / boundary for
 * the tokens in order[h], and build the per-q-tile ascending CSR lists of full and
 * boundary tiles plus the execution plan.  Tile skipping over such lists is the core
 * of the method (aihirek.info, section "A TPU-kernel kialakitasa ..."; ainews.tenesys.com,
 * "Co sie zmienilo?" items 1-2).  The map depends on the problem only, not on Q/K/V,
 * so one map serves every layer and denoising step with the same problem.
 * workspace: DEVICE buffer of at least the queried size, caller-owned, scratch. */
SVGA_API svga_status svga_build_block_map(const svga_problem *problem, svga_block_map *map,
                                 void *workspace, size_t workspace_bytes,
                                 svga_stream_t stream);

/* Size of the library's static build scratch used by svga_build_block_map_static. */
#define SVGA_MAP_STATIC_SCRATCH_BYTES (1u << 20)

/* svga_build_block_map without a workspace argument, for callers that cannot allocate
 * device memory when they build a map: plugin hosts whose execute callback forbids
 * allocation, servers that fix their memory budget at start-up, code that must not take
 * the implicit device synchronisation of cudaMalloc / cudaFree.  The paper has no
 * counterpart; it is a deployment convenience.
 *   - The caller still provides every output buffer of `map` (svga_block_map_size).
 *   - The build's scratch lives in one static device array of
 *     SVGA_MAP_STATIC_SCRATCH_BYTES that each GPU loading the library keeps until the
 *     process exits.  A problem needing more scratch (svga_block_map_size's
 *     workspace_bytes) is rejected with SVGA_ERR_WORKSPACE and nothing is launched.
 *   - Every call looks up the array's device address in the CUDA context current at
 *     that call (cudaGetSymbolAddress: no allocation, no synchronisation), so the call
 *     stays correct after a cudaDeviceReset or with another context of the device
 *     current.  The first call in a context may load the library's device code into
 *     it: make that first call before any stream capture.
 *   - The call allocates nothing.  All calls share the array: calls that overlap on the
 *     GPU (unordered streams) race; calls ordered on one stream are safe.
 * Results are identical to svga_build_block_map's. */
SVGA_API svga_status svga_build_block_map_static(const svga_problem *problem,
                                                 svga_block_map *map, svga_stream_t stream);

/* Host-side consistency check of a built map, the stand-in for a race detector:
 * copies the map to the host (synchronises `stream`) and checks that the status word
 * is 0, classes are 0 / 1 / 2 and no tile holding padding is full, the CSR offsets
 * start at 0, never decrease and fit the capacities, every list is strictly ascending,
 * in range and agrees with the classes (complete, nothing extra), and the plan matches
 * the problem: header, head info, one item per (head, query-block pair), items longest
 * first, each item's entries exactly the visited key chunks in ascending order with
 * visit / full flags recomputed from the classes.  Returns SVGA_OK, or
 * SVGA_ERR_INVALID_ARG naming the first violation in svga_last_error. */
SVGA_API svga_status svga_validate_block_map(const svga_problem *problem,
                                             const svga_block_map *map, svga_stream_t stream);

/* Token permutation of one tensor [heads, tokens, head_dim] bf16: for every head h,
 * dst[h, pos] = src[h, t] where pos is the position of frame-major token t in
 * order[h] (spatial heads usually stay frame-major: a plain copy).  The pages move
 * temporal heads to temporal-major order (ainews.tenesys.com, "Co sie zmienilo?"
 * item 5).  src and dst must not overlap.  Bit-exact copy.  With frame_pad, dst has
 * svga_problem_rows rows per head and its positions without a token are set to 0. */
SVGA_API svga_status svga_permute_tokens(const void *src, void *dst, const svga_problem *problem,
                                svga_stream_t stream);

/* Inverse of svga_permute_tokens: dst[h, t] = src[h, pos] (src with
 * svga_problem_rows rows per head). */
SVGA_API svga_status svga_unpermute_tokens(const void *src, void *dst, const svga_problem *problem,
                                  svga_stream_t stream);

/* Block-sparse attention forward.  For head h and query position i (order[h]):
 *   O[h,i,:] = sum_{k in K(i)} exp(x_ik - m_i) V[h,k,:] / sum_{k in K(i)} exp(x_ik - m_i)
 *   x_ik = scale * Q[h,i,:] . K[h,k,:],   m_i = max_{k in K(i)} x_ik,
 *   lse[h,i] = m_i + ln sum_{k in K(i)} exp(x_ik - m_i)      (natural log)
 * where K(i) is the set of keys the head's mask keeps, evaluated on the tokens'
 * original (frame, in-frame index) coordinates.  Skipped tiles hold no kept pair,
 * full tiles run without mask arithmetic, boundary tiles are masked element by
 * element (aihirek.info, section "A TPU-kernel kialakitasa ...").  An empty row
 * gives O = 0 and lse = -inf.
 *   q, k, v, o : DEVICE bf16 [heads, rows, head_dim], every head in order[h], rows
 *                = svga_problem_rows (q and o frame-major [heads, tokens, head_dim]
 *                instead with SVGA_FLAG_QO_FRAME_MAJOR, k and v with
 *                SVGA_FLAG_KV_FRAME_MAJOR)
 *   lse        : DEVICE float [heads, rows] or NULL (frame-major with that flag)
 *   map        : built by svga_build_block_map (or _routed / _static) for this problem;
 *                the per-head type, band and order are read from the map's plan.  The
 *                kernel first compares the plan's header (magic, heads, tokens, frames,
 *                grid, anchor, tiles, chunk size and item count) and each work item
 *                with this call: a map built for another problem sets map->status to
 *                SVGA_ERR_INVALID_ARG and nothing is written (O and lse untouched)
 *   scale      : softmax scale, usually 1/sqrt(head_dim)
 *   flags      : 0 or a combination of SVGA_FLAG_NAIVE_B1 / SVGA_FLAG_TILE_ALIGNED
 *                (not both), SVGA_FLAG_QO_FRAME_MAJOR, SVGA_FLAG_KV_FRAME_MAJOR,
 *                SVGA_FLAG_CTA_PAIR and the
 *                test hook
 *                SVGA_FLAG_TEST_STALL; other bits give SVGA_ERR_INVALID_ARG
 * bf16 inputs, fp32 accumulation and softmax, P rounded to bf16 for the PV product. */
SVGA_API svga_status svga_sparse_attention_fwd(const void *q, const void *k, const void *v, void *o,
                                      float *lse, const svga_problem *problem,
                                      const svga_block_map *map, float scale, int flags,
                                      svga_stream_t stream);

/* One part of svga_sparse_attention_fwd, for running one problem on several GPUs
 * (or streams) with no exchange between them.  The work items of the block map (a
 * head and two 128-row query blocks each, longest first) are dealt to num_parts parts
 * in snake order (group g of num_parts consecutive items: part r takes the r-th item
 * when g is even, the (num_parts-1-r)-th when g is odd), so that the parts' work
 * differs by at most about one item.  The call computes and stores the O rows (and
 * lse entries) of its own items only; the parts of 0 .. num_parts-1 together write
 * every row exactly once, with results identical bit for bit to the single call.
 * Heads and query rows are independent in the method (aihirek.info, section
 * "A Sparse VideoGen a figyelmi fejeket osztalyozza": masks are per head and per
 * query), so the split needs no communication.  Arguments as for
 * svga_sparse_attention_fwd, plus
 *   part, num_parts : 1 <= num_parts <= 4096, 0 <= part < num_parts
 *                     (SVGA_ERR_INVALID_ARG otherwise). */
SVGA_API svga_status svga_sparse_attention_fwd_part(const void *q, const void *k, const void *v,
                                           void *o, float *lse, const svga_problem *problem,
                                           const svga_block_map *map, float scale, int flags,
                                           int part, int num_parts, svga_stream_t stream);

/* Dense attention forward (every pair kept): the same-GPU dense baseline, the role
 * dense Splash Attention plays on the pages (aihirek.info, section "A TPU-kernel
 * kialakitasa ..."; oossa.com, "Die Fakten").  Same kernel, every tile unmasked
 * except the ragged last key tile, which is length-masked.
 *   status: DEVICE int32 word or NULL (cleared, then set on a device failure). */
SVGA_API svga_status svga_dense_attention_fwd(const void *q, const void *k, const void *v, void *o,
                                     float *lse, int heads, int tokens, int head_dim,
                                     float scale, int32_t *status, svga_stream_t stream);

/* Workspace for svga_classify_heads with n_rows sampled query rows per head. */
SVGA_API svga_status svga_classify_size(const svga_problem *problem, int n_rows,
                               size_t *workspace_bytes);

/* Online head classification.  For a few query rows per head, compute the dense
 * output and the outputs under the spatial and the temporal mask, and give the head
 * the mask whose output deviates least from the dense one (aihirek.info, section
 * "A Sparse VideoGen a figyelmi fejeket osztalyozza").  Deviation = mean squared
 * error over the sampled rows x head_dim; a tie goes to spatial.
 *   q, k, v     : DEVICE bf16 [heads, tokens, head_dim] in FRAME-MAJOR order
 *   problem     : shape, anchor and head_dim; head_type/band/order are not read
 *   w_spatial   : HOST int32 [heads], spatial band of the candidate mask
 *   w_temporal  : HOST int32 [heads], temporal band of the candidate mask
 *   rows        : DEVICE int32 [n_rows] frame-major token indices shared by all
 *                 heads, or NULL for the default rule r_i = floor((2i+1) N / (2 n_rows))
 *   n_rows      : sampled rows per head, 1 .. N
 *   scale       : softmax scale, usually 1/sqrt(head_dim)
 *   head_type_out : HOST int32 [heads] (written before the call returns)
 *   mse_out     : HOST float [heads][2] (spatial, temporal) or NULL
 *   workspace   : DEVICE scratch of at least svga_classify_size bytes
 * This call synchronises `stream` to return the types to the host. */
SVGA_API svga_status svga_classify_heads(const void *q, const void *k, const void *v,
                                const svga_problem *problem, const int32_t *w_spatial,
                                const int32_t *w_temporal, const int32_t *rows, int n_rows,
                                float scale, int32_t *head_type_out, float *mse_out, void *workspace,
                                size_t workspace_bytes, svga_stream_t stream);

/* ---- Band selection: the classifier over a list of candidate masks ----------------
 * The pages choose between a spatial and a temporal mask per head by the least
 * deviation from dense on a few query rows (aihirek.info, section "A Sparse VideoGen a
 * figyelmi fejeket osztalyozza").  The calls below extend the choice to a list of
 * candidate (type, band) masks.  The pages give no rule for trading a band's deviation
 * against its cost (the least deviation alone always favours the widest band), so this
 * library's reading is a budget: a candidate is eligible when the fraction of all
 * (query, key) pairs its mask keeps is at most max_kept_fraction (the pages report
 * about 39 % kept, aihirek.info, section "A TPU-kernel kialakitasa dontonek
 * bizonyult"), and each head takes the eligible candidate whose output deviates least
 * from dense (mean squared error over the sampled rows x head_dim), the earlier
 * candidate on a tie. */

/* Fraction of the N*N (query, key) pairs one head's mask keeps on this problem (the
 * anchor included), counted exactly in closed form.  Host-only. */
SVGA_API svga_status svga_kept_fraction(const svga_problem *problem, int head_type, int band,
                                        double *fraction);

/* Workspace for svga_autotune_heads with n_rows sampled rows and n_cand candidates
 * (1 .. 16). */
SVGA_API svga_status svga_autotune_size(const svga_problem *problem, int n_rows, int n_cand,
                                        size_t *workspace_bytes);

/* Per-head mask type and band among candidates.
 *   q, k, v          : DEVICE bf16 [heads, tokens, head_dim], frame-major
 *   cand_type/_band  : HOST int32 [n_cand]: SVGA_HEAD_SPATIAL / _TEMPORAL and 0..65535
 *   max_kept_fraction: in (0, 1]; at least one candidate must keep no more than it
 *                      (SVGA_ERR_INVALID_ARG otherwise)
 *   rows, n_rows     : sampled query rows as for svga_classify_heads (NULL: the default
 *                      rule)
 *   head_type_out    : HOST int32 [heads];  band_out: HOST int32 [heads]
 *   mse_out          : HOST float [heads][n_cand] or NULL: every candidate's deviation
 *   workspace        : DEVICE, at least svga_autotune_size bytes, 256-byte aligned
 * Synchronises `stream`.  The problem's head_type, band and order arrays are not read. */
SVGA_API svga_status svga_autotune_heads(const void *q, const void *k, const void *v,
                                         const svga_problem *problem, const int32_t *cand_type,
                                         const int32_t *cand_band, int n_cand,
                                         double max_kept_fraction, const int32_t *rows,
                                         int n_rows, float scale, int32_t *head_type_out,
                                         int32_t *band_out, float *mse_out, void *workspace,
                                         size_t workspace_bytes, svga_stream_t stream);

/* ---- Routed pipeline: the classifier's decision stays on the device -------------
 * The pages profile the heads online and then run the chosen sparse mask (aihirek.info,
 * section "A Sparse VideoGen a figyelmi fejeket osztalyozza").  The four calls below
 * run classification -> block map -> permutation -> attention -> inverse permutation
 * on one stream without returning to the host in between, so a whole attention layer
 * can be replayed from one CUDA graph.  Per head: type from the classifier, band =
 * w_spatial[h] or w_temporal[h] by that type, order = frame-major for spatial heads and
 * anchor-first temporal-major for temporal heads.  The problem's head_type, band and
 * order arrays are not read by these calls (they may be NULL); svga_block_map_size and
 * svga_sparse_attention_fwd(_part) do not read them either. */

/* svga_classify_heads without the host round trip: nothing synchronises.
 *   head_type_dev : DEVICE int32 [heads], written on `stream`
 *   mse_dev       : DEVICE float [heads][2] or NULL
 *   status_dev    : DEVICE int32 or NULL: 0, or the svga_status of a failure found
 *                   on the device (e.g. a row index outside 0..N-1)
 * Other arguments and their checks as for svga_classify_heads. */
SVGA_API svga_status svga_classify_heads_async(const void *q, const void *k, const void *v,
                                      const svga_problem *problem, const int32_t *w_spatial,
                                      const int32_t *w_temporal, const int32_t *rows,
                                      int n_rows, float scale, int32_t *head_type_dev,
                                      float *mse_dev, int32_t *status_dev, void *workspace,
                                      size_t workspace_bytes, svga_stream_t stream);

/* svga_build_block_map with the head types read on the device from head_type_dev
 * (DEVICE int32 [heads], e.g. svga_classify_heads_async's output) and the bands and
 * orders derived from them as described above.  w_spatial, w_temporal: HOST int32
 * [heads], 0 .. 65535.  A type other than 0 / 1 on the device sets map->status to
 * SVGA_ERR_INVALID_ARG (the head is then built as spatial).  The plan records every
 * head's type, band and order for the calls below.  Same buffers as
 * svga_build_block_map. */
SVGA_API svga_status svga_build_block_map_routed(const svga_problem *problem,
                                        const int32_t *head_type_dev, const int32_t *w_spatial,
                                        const int32_t *w_temporal, svga_block_map *map,
                                        void *workspace, size_t workspace_bytes,
                                        svga_stream_t stream);

/* svga_permute_tokens / svga_unpermute_tokens with each head's order read from the
 * plan of `map` on the device instead of problem->order.  The plan's header and head
 * info are checked against the problem on the device first: a map built for another
 * problem sets map->status (when not NULL) to SVGA_ERR_INVALID_ARG and dst is left
 * untouched.  The status word is not cleared by these calls. */
SVGA_API svga_status svga_permute_tokens_mapped(const void *src, void *dst,
                                       const svga_problem *problem, const svga_block_map *map,
                                       svga_stream_t stream);
SVGA_API svga_status svga_unpermute_tokens_mapped(const void *src, void *dst,
                                         const svga_problem *problem,
                                         const svga_block_map *map, svga_stream_t stream);

/* Message of the last failed call on this thread ("" if none). */
SVGA_API const char *svga_last_error(void);

/* Name of a status code. */
SVGA_API const char *svga_status_string(svga_status status);

/* SVGA_VERSION of the built library. */
SVGA_API int svga_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVGA_H */
