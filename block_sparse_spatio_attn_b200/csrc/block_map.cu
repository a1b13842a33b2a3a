// block_map.cu -- tile classification, per-q-tile CSR lists and the attention plan.
//
// "Accelerating Spatio-Temporal Attention for Video Diffusion on TPUs" skips the
// (query tile, key tile) pairs that hold no kept pair and treats the visited tiles
// as full (unmasked fast path) or boundary (masked by coordinates) (aihirek.info,
// section "A TPU-kernel kialakitasa dontonek bizonyult"; ainews.tenesys.com,
// "Co sie zmienilo?" items 1-2).  This file builds that classification for every
// head and the lists the attention kernel walks.
//
// Method: the tokens of a tile are a run of consecutive positions of the head's
// token order.  In every order the run splits into at most four rectangles of
// (frame range) x (in-frame index range).  Whether a rectangle pair keeps all, some or
// none of its pairs follows from the min / max distance of the two ranges, so a tile
// costs a few integer operations instead of tile_q * tile_k predicate evaluations.
// A tile holding padding (positions >= N) is never full.
#include <cuda_runtime.h>

#include "svga_device.cuh"
#include "svga_internal.h"

namespace svga {
namespace {

struct Rect {
    int f0, f1, s0, s1;  // inclusive ranges
};

// Positions [u0, u1) of a grid with period P (major = u / P, minor = u % P) as at
// most three rectangles: the first partial major row (h), the whole rows between (m)
// and the last partial row (t).  major_is_f: frames follow the major index; otherwise
// the in-frame index does and frames follow the minor index plus foff.  Returns the
// valid ones as bits (1 = h, 2 = m, 4 = t).  Fixed slots, not a count, so that the
// rectangles stay in registers.
__host__ __device__ __forceinline__ uint32_t run_rects(int u0, int u1, int P, bool major_is_f,
                                                      int foff, Rect &h, Rect &m, Rect &t)
{
    const int M0 = u0 / P, m0 = u0 - M0 * P;
    const int M1 = (u1 - 1) / P, m1 = (u1 - 1) - M1 * P;
    auto emit = [&](int Ma, int Mb, int ma, int mb) {
        return major_is_f ? Rect{Ma, Mb, ma, mb} : Rect{ma + foff, mb + foff, Ma, Mb};
    };
    if (M0 == M1) {
        h = emit(M0, M0, m0, m1);
        return 1u;
    }
    h = emit(M0, M0, m0, P - 1);
    t = emit(M1, M1, 0, m1);
    if (M1 > M0 + 1) {
        m = emit(M0 + 1, M1 - 1, 0, P - 1);
        return 7u;
    }
    return 5u;
}

// Tokens at positions [a, b) of `order` (0 <= a < b) as at most 4 rectangles in fixed
// slots: r[0] the frame-0 part of the anchor-first order, r[1..3] the run's head,
// middle and tail.  Returns the valid slots as bits.  Frame-major frames lie at stride
// Sp >= S (the padded layout when Sp > S); temporal-major tokens end at N.  *holes is
// set when a position of [a, b) holds no token.
__host__ __device__ __forceinline__ uint32_t tile_rects(int order, int a, int b, int F, int S,
                                                       int Sp, int N, Rect (&r)[4], bool &holes)
{
    if (order == ORDER_FM) {
        uint32_t mk = run_rects(a, b, Sp, true, 0, r[1], r[2], r[3]) << 1;
        if (Sp > S)
#pragma unroll
            for (int i = 1; i < 4; ++i)
                if (((mk >> i) & 1u) && r[i].s1 >= S) {  // the frame's empty tail
                    holes = true;
                    r[i].s1 = S - 1;
                    if (r[i].s0 > r[i].s1) mk &= ~(1u << i);
                }
        return mk;
    }
    if (b > N) {
        holes = true;
        b = N;
    }
    if (a >= b) return 0u;
    if (order == ORDER_TM_STRICT) return run_rects(a, b, F, false, 0, r[1], r[2], r[3]) << 1;
    uint32_t mask = 0;  // anchor-first: frame 0 at positions [0, S), then s-major over f >= 1
    if (a < S) {
        r[0] = Rect{0, 0, a, (b < S ? b : S) - 1};
        mask = 1u;
    }
    if (b > S)
        mask |= run_rects((a > S ? a : S) - S, b - S, F - 1, false, 1, r[1], r[2], r[3]) << 1;
    return mask;
}

// Does the rectangle pair keep all / any of its (q, k) pairs?
__host__ __device__ __forceinline__ void rect_pair(int type, int band, int anchor, const Rect &q,
                                          const Rect &k, bool &all, bool &any)
{
    const bool k_has_anchor = anchor && k.f0 == 0;
    if (type == MASK_SPATIAL) {
        const int mind = max(0, max(k.f0 - q.f1, q.f0 - k.f1));
        any = k_has_anchor || mind <= band;
        const int kf0 = k_has_anchor ? 1 : k.f0;  // key frames the anchor does not cover
        all = (kf0 > k.f1) || max(q.f1 - kf0, k.f1 - q.f0) <= band;
    } else {
        const int mind = max(0, max(k.s0 - q.s1, q.s0 - k.s1));
        any = k_has_anchor || mind <= band;
        all = (anchor && k.f1 == 0) || max(q.s1 - k.s0, k.s1 - q.s0) <= band;
    }
}

struct HeadParams {
    uint32_t packed[kMaxHeads];  // type | order << 2 | band << 8
};
__host__ __device__ __forceinline__ int hp_type(uint32_t x) { return x & 3; }
__host__ __device__ __forceinline__ int hp_order(uint32_t x) { return (x >> 2) & 3; }
__host__ __device__ __forceinline__ int hp_band(uint32_t x) { return (int)(x >> 8); }

// Plan header and per-head info, written from kernel parameters (no host staging).
__global__ void write_plan_header_kernel(PlanHeader hdr, HeadParams hp, int4 *head_info)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<PlanHeader *>(head_info - 4) = hdr;
    for (int h = blockIdx.x * blockDim.x + threadIdx.x; h < hdr.heads; h += gridDim.x * blockDim.x) {
        uint32_t x = hp.packed[h];
        head_info[h] = make_int4(hp_type(x), hp_band(x), hp_order(x), 0);
    }
}

// The same from head types on the device (the online classifier's output): the band is
// the candidate of the chosen type, temporal heads read the anchor-first temporal-major
// order, spatial heads frame-major.  An invalid type is reported in the status word and
// the head is treated as spatial.
struct BandPairs {
    uint32_t packed[kMaxHeads];  // w_spatial | w_temporal << 16
};

__global__ void write_plan_header_routed_kernel(PlanHeader hdr, BandPairs bp,
                                                const int32_t *types, int4 *head_info,
                                                int32_t *status)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) *reinterpret_cast<PlanHeader *>(head_info - 4) = hdr;
    for (int h = blockIdx.x * blockDim.x + threadIdx.x; h < hdr.heads; h += gridDim.x * blockDim.x) {
        int t = types[h];
        if (t != MASK_SPATIAL && t != MASK_TEMPORAL) {
            if (status) atomicCAS(status, 0, 1);  // SVGA_ERR_INVALID_ARG
            t = MASK_SPATIAL;
        }
        const uint32_t x = bp.packed[h];
        const int band = t == MASK_SPATIAL ? (int)(x & 0xFFFFu) : (int)(x >> 16);
        head_info[h] = make_int4(t, band, t == MASK_SPATIAL ? ORDER_FM : ORDER_TM, 0);
    }
}

__device__ __forceinline__ int block_sum(int v, int *red)
{
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    int t = 0;
    for (int i = 0; i < nw; ++i) t += red[i];
    return t;
}

// One block per (q-tile, head): class of every k-tile and the row's two counts.  The row
// goes in segments of 256 groups of 8 k-tiles.  First each thread asks of one group
// whether the q-tile keeps none, all or some of the pairs with its key positions: the
// rectangles of a range cover exactly its tokens and the test is exact, so a group
// with none has 8 empty tiles, and a group with all of them (and no position without
// a token) has 8 full tiles, bar one reaching past the last position.  Then the threads
// classify the segment's tiles, testing one by one only inside the mixed groups (those
// at the edges of a band).
constexpr int kGroupTiles = 8;
constexpr int kClassifyThreads = 256;

__global__ void __launch_bounds__(kClassifyThreads) classify_tiles_kernel(
    Geometry g, int anchor, const int4 *head_info, uint8_t *cls, int *full_cnt, int *bnd_cnt)
{
    __shared__ int red[8];
    __shared__ uint8_t group_cls[kClassifyThreads];  // 0 none, 1 all, 2 some kept
    const int i = blockIdx.x, h = blockIdx.y;
    const int4 hi = head_info[h];
    const int type = hi.x, band = hi.y, order = hi.z;
    // tiles cover the NP positions; a tile with a position past them or without a token
    // is never full
    const int qa = i * g.tile_q, qb = min(g.NP, qa + g.tile_q);
    bool qpad = qa + g.tile_q > g.NP;
    Rect qr[4];
    const uint32_t qm = tile_rects(order, qa, qb, g.F, g.S, g.Sp, g.N, qr, qpad);
    // does the q-tile keep any pair with the keys at positions [ka, kb)?  (all: all of
    // them, holes aside)
    auto test = [&](int ka, int kb, bool &all) {
        bool kpad = false;
        Rect kr[4];
        const uint32_t km = tile_rects(order, ka, kb, g.F, g.S, g.Sp, g.N, kr, kpad);
        bool any = false;
        all = !kpad;
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (((qm >> a) & 1u) && ((km >> b) & 1u)) {
                    bool all_, any_;
                    rect_pair(type, band, anchor, qr[a], kr[b], all_, any_);
                    all = all && all_;
                    any = any || any_;
                }
        return any;
    };
    int nf = 0, nb = 0;
    uint8_t *row = cls + ((size_t)h * g.n_q + i) * g.n_k;
    constexpr int kSegTiles = kClassifyThreads * kGroupTiles;
    for (int seg = 0; seg < g.n_k; seg += kSegTiles) {
        {
            const int j0 = seg + threadIdx.x * kGroupTiles;
            uint8_t gc = 0;
            if (j0 < g.n_k) {
                bool all;
                if (test(j0 * g.tile_k, min(g.NP, min(g.n_k, j0 + kGroupTiles) * g.tile_k), all))
                    gc = (all && !qpad) ? 1 : 2;
            }
            group_cls[threadIdx.x] = gc;
        }
        __syncthreads();
        const int seg_end = min(g.n_k, seg + kSegTiles);
        for (int j = seg + threadIdx.x; j < seg_end; j += kClassifyThreads) {
            const uint8_t gc = group_cls[(j - seg) / kGroupTiles];
            const int ka = j * g.tile_k;
            uint8_t c = gc;
            if (gc == 1) {
                // every pair kept: full, unless the tile reaches past the positions
                if (ka + g.tile_k > g.NP) c = 2;
            } else if (gc == 2) {
                const int kb = min(g.NP, ka + g.tile_k);
                bool all;
                const bool any = test(ka, kb, all);
                // a tile reaching past the positions is never full
                const bool full = all && !qpad && ka + g.tile_k <= g.NP;
                c = any ? (full ? 1 : 2) : 0;
            }
            row[j] = c;
            nf += c == 1;
            nb += c == 2;
        }
        __syncthreads();  // group_cls is rewritten by the next segment
    }
    nf = block_sum(nf, red);
    nb = block_sum(nb, red);
    if (threadIdx.x == 0) {
        full_cnt[h * g.n_q + i] = nf;
        bnd_cnt[h * g.n_q + i] = nb;
    }
}

// Exclusive scan of n counts into ptr[0..n] by one block; flags an overflow of cap.
__global__ void __launch_bounds__(1024) scan_kernel(const int *cnt, int n, int *ptr, int64_t cap,
                                                    int32_t *status)
{
    __shared__ long long part[1024];
    const int t = threadIdx.x, per = (n + 1023) / 1024;
    const int lo = min(n, t * per), hi = min(n, lo + per);
    long long s = 0;
    for (int x = lo; x < hi; ++x) s += cnt[x];
    part[t] = s;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        long long v = t >= o ? part[t - o] : 0;
        __syncthreads();
        part[t] += v;
        __syncthreads();
    }
    long long run = part[t] - s;
    for (int x = lo; x < hi; ++x) {
        ptr[x] = (int)run;
        run += cnt[x];
    }
    if (t == 1023) {
        ptr[n] = (int)part[1023];
        if (part[1023] > cap && status) atomicExch(status, (int32_t)SVGA_ERR_WORKSPACE);
    }
}

// Exclusive prefix sum over the block of one value per thread (warp shuffles, then the
// warp totals); *total gets the block's sum.  Values may pack two 16-bit counts as long
// as neither half overflows.
__device__ __forceinline__ int block_exclusive_scan(int v, int *wsum, int *total)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    __syncthreads();  // wsum may still be read by the previous call
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    int off = 0, tot = 0;
    for (int i = 0; i < nw; ++i) {
        off += i < w ? wsum[i] : 0;
        tot += wsum[i];
    }
    *total = tot;
    return off + inc - v;
}

// Elements a thread of the list and plan builders takes per step (consecutive ones).
constexpr int kPerThread = 8;

__global__ void __launch_bounds__(256) compact_lists_kernel(Geometry g, const uint8_t *cls,
                                                            const int *full_ptr, const int *bnd_ptr,
                                                            int *full_idx, int *bnd_idx,
                                                            int64_t full_cap, int64_t bnd_cap)
{
    __shared__ int wsum[8];
    const int i = blockIdx.x, h = blockIdx.y, r = h * g.n_q + i;
    const uint8_t *row = cls + (size_t)r * g.n_k;
    long long fo = full_ptr[r], bo = bnd_ptr[r];
    // each step: kPerThread consecutive tiles per thread, one scan of both counts
    for (int base = 0; base < g.n_k; base += blockDim.x * kPerThread) {
        const int j0 = base + threadIdx.x * kPerThread;
        uint8_t c[kPerThread];
        int nf = 0, nb = 0;
#pragma unroll
        for (int u = 0; u < kPerThread; ++u) {
            c[u] = j0 + u < g.n_k ? row[j0 + u] : 0;
            nf += c[u] == 1;
            nb += c[u] == 2;
        }
        int tot;
        const int pos = block_exclusive_scan(nf | (nb << 16), wsum, &tot);
        long long pf = fo + (pos & 0xFFFF), pb = bo + (pos >> 16);
#pragma unroll
        for (int u = 0; u < kPerThread; ++u) {
            if (c[u] == 1) {
                if (pf < full_cap) full_idx[pf] = j0 + u;
                ++pf;
            } else if (c[u] == 2) {
                if (pb < bnd_cap) bnd_idx[pb] = j0 + u;
                ++pb;
            }
        }
        fo += tot & 0xFFFF;
        bo += tot >> 16;
    }
}

// Flags of (128-row block b, key chunk c) from the tile classes.
__device__ __forceinline__ uint32_t block_chunk_flags(const Geometry &g, const uint8_t *cls_h,
                                                      int b, int c, int naive)
{
    if (b >= g.n_qblk) return 0;
    int i0, i1;
    if (g.tile_q == 64) {
        i0 = 2 * b;
        i1 = min(2 * b + 1, g.n_q - 1);
    } else if (g.tile_q == 128) {
        i0 = i1 = b;
    } else {
        i0 = i1 = b / 2;
    }
    const int j = (g.tile_k > g.kn) ? c / (g.tile_k / g.kn) : c;
    const uint8_t x0 = cls_h[(size_t)i0 * g.n_k + j], x1 = cls_h[(size_t)i1 * g.n_k + j];
    const bool visit = x0 != 0 || x1 != 0;
    const bool full = x0 == 1 && x1 == 1 && !naive;
    return visit ? (1u | (full ? 2u : 0u)) : 0u;
}

__device__ __forceinline__ uint32_t entry_of(const Geometry &g, const uint8_t *cls_h, int p, int c)
{
    const uint32_t a = block_chunk_flags(g, cls_h, 2 * p, c, 0);
    const uint32_t b = block_chunk_flags(g, cls_h, 2 * p + 1, c, 0);
    if (!(a | b)) return 0;
    return (uint32_t)c | (a << 24) | (b << 26);
}

__global__ void __launch_bounds__(256) plan_count_kernel(Geometry g, const uint8_t *cls,
                                                         int *item_cnt)
{
    __shared__ int red[8];
    const int item = blockIdx.x, h = item / g.n_pairs, p = item - h * g.n_pairs;
    const uint8_t *cls_h = cls + (size_t)h * g.n_q * g.n_k;
    int n = 0;
    for (int c = threadIdx.x; c < g.n_kc; c += blockDim.x) n += entry_of(g, cls_h, p, c) != 0;
    n = block_sum(n, red);
    if (threadIdx.x == 0) item_cnt[item] = n;
}

__global__ void __launch_bounds__(256) plan_write_kernel(Geometry g, const uint8_t *cls,
                                                         const int *item_off, uint32_t *entries,
                                                         int64_t cap)
{
    __shared__ int wsum[8];
    const int item = blockIdx.x, h = item / g.n_pairs, p = item - h * g.n_pairs;
    const uint8_t *cls_h = cls + (size_t)h * g.n_q * g.n_k;
    long long off = item_off[item];
    // each step: kPerThread consecutive chunks per thread, one scan of the entry counts
    for (int base = 0; base < g.n_kc; base += blockDim.x * kPerThread) {
        const int c0 = base + threadIdx.x * kPerThread;
        uint32_t e[kPerThread];
        int n = 0;
#pragma unroll
        for (int u = 0; u < kPerThread; ++u) {
            e[u] = c0 + u < g.n_kc ? entry_of(g, cls_h, p, c0 + u) : 0u;
            n += e[u] != 0;
        }
        int tot;
        long long pos = off + block_exclusive_scan(n, wsum, &tot);
#pragma unroll
        for (int u = 0; u < kPerThread; ++u)
            if (e[u] != 0) {
                if (pos < cap) entries[pos] = e[u];
                ++pos;
            }
        off += tot;
    }
}

// Longest-first order of the work items (ties: lower item index first), so that a
// launch in plan order hands the long items out first.  One warp per item counts the
// items that go before it (a rank); the counts are read from L1.
__global__ void __launch_bounds__(256) plan_sort_kernel(Geometry g, const int *item_cnt,
                                                        const int *item_off, int4 *items)
{
    const int me = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (me >= g.n_items) return;  // whole warps leave together
    const int my = item_cnt[me];
    int rank = 0;
#pragma unroll 4
    for (int o = lane; o < g.n_items; o += 32) {
        const int x = __ldg(item_cnt + o);
        rank += (x > my) || (x == my && o < me);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    if (lane == 0) {
        const int h = me / g.n_pairs, p = me - h * g.n_pairs;
        items[rank] = make_int4(h, 2 * p, item_off[me], my);
    }
}

}  // namespace

size_t block_map_workspace_bytes(const Geometry &g)
{
    const size_t rows = (size_t)g.heads * g.n_q;
    return align_up(sizeof(int) * rows, 256) * 2 + align_up(sizeof(int) * (g.n_items + 1), 256) * 2;
}

svga_status launch_build_block_map(const svga_problem *p, const Geometry &g, svga_block_map *map,
                                   void *ws, size_t ws_bytes, void *stream_,
                                   const int32_t *types_dev, const int32_t *w_spatial,
                                   const int32_t *w_temporal)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream_);
    const size_t rows = (size_t)g.heads * g.n_q;
    char *w = static_cast<char *>(ws);
    int *full_cnt = reinterpret_cast<int *>(w);
    w += align_up(sizeof(int) * rows, 256);
    int *bnd_cnt = reinterpret_cast<int *>(w);
    w += align_up(sizeof(int) * rows, 256);
    int *item_cnt = reinterpret_cast<int *>(w);
    w += align_up(sizeof(int) * (g.n_items + 1), 256);
    int *item_off = reinterpret_cast<int *>(w);
    (void)ws_bytes;

    char *plan = static_cast<char *>(map->plan);
    int4 *head_info = reinterpret_cast<int4 *>(plan + sizeof(PlanHeader));
    int4 *items = head_info + g.heads;
    uint32_t *entries = reinterpret_cast<uint32_t *>(plan + plan_header_bytes(g));
    const int64_t entry_cap =
        (int64_t)((map->plan_bytes - plan_header_bytes(g)) / sizeof(uint32_t));

    if (map->status && cudaMemsetAsync(map->status, 0, sizeof(int32_t), st) != cudaSuccess) {
        set_error("cudaMemsetAsync of the status word failed");
        return SVGA_ERR_CUDA;
    }
    PlanHeader hdr{};
    hdr.magic = kPlanMagic;
    hdr.heads = g.heads;
    hdr.tokens = g.N;
    hdr.frames = g.F;
    hdr.tokens_per_frame = g.S;
    hdr.anchor = p->anchor_frame0;
    hdr.tile_q = g.tile_q;
    hdr.tile_k = g.tile_k;
    hdr.kn = g.kn;
    hdr.n_qblk = g.n_qblk;
    hdr.n_kc = g.n_kc;
    hdr.n_items = g.n_items;
    hdr.entry_cap = entry_cap;
    hdr.frame_stride = g.Sp;
    if (types_dev) {
        BandPairs bp;  // 16 KB: travels as kernel parameters
        for (int h = 0; h < g.heads; ++h)
            bp.packed[h] = (uint32_t)w_spatial[h] | ((uint32_t)w_temporal[h] << 16);
        write_plan_header_routed_kernel<<<(g.heads + 255) / 256, 256, 0, st>>>(
            hdr, bp, types_dev, head_info, map->status);
    } else {
        HeadParams local;  // 16 KB: travels as kernel parameters
        for (int h = 0; h < g.heads; ++h)
            local.packed[h] = (uint32_t)p->head_type[h] | ((uint32_t)p->order[h] << 2) |
                              ((uint32_t)p->band[h] << 8);
        write_plan_header_kernel<<<(g.heads + 255) / 256, 256, 0, st>>>(hdr, local, head_info);
    }
    classify_tiles_kernel<<<dim3(g.n_q, g.heads), kClassifyThreads, 0, st>>>(g, p->anchor_frame0, head_info,
                                                                map->cls, full_cnt, bnd_cnt);
    scan_kernel<<<1, 1024, 0, st>>>(full_cnt, (int)rows, map->full_ptr, map->full_cap, map->status);
    scan_kernel<<<1, 1024, 0, st>>>(bnd_cnt, (int)rows, map->bnd_ptr, map->bnd_cap, map->status);
    compact_lists_kernel<<<dim3(g.n_q, g.heads), 256, 0, st>>>(
        g, map->cls, map->full_ptr, map->bnd_ptr, map->full_idx, map->bnd_idx, map->full_cap,
        map->bnd_cap);
    plan_count_kernel<<<g.n_items, 256, 0, st>>>(g, map->cls, item_cnt);
    scan_kernel<<<1, 1024, 0, st>>>(item_cnt, g.n_items, item_off, entry_cap, map->status);
    plan_write_kernel<<<g.n_items, 256, 0, st>>>(g, map->cls, item_off, entries, entry_cap);
    // one warp per item
    plan_sort_kernel<<<(g.n_items + 7) / 8, 256, 0, st>>>(g, item_cnt, item_off, items);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("block map launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    return SVGA_OK;
}

}  // namespace svga
