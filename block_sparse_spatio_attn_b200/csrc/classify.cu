// classify.cu -- online spatial / temporal head classification and band selection.
//
// Sparse VideoGen profiles the heads while it runs: for a few query rows it computes
// the dense, the spatial and the temporal outputs and keeps the sparse mask whose
// output deviates least from the dense one ("Accelerating Spatio-Temporal Attention for
// Video Diffusion on TPUs", aihirek.info, section "A Sparse VideoGen a figyelmi
// fejeket osztalyozza").  Here, for a list of candidate masks (type, band):
//   1. the sampled rows of Q are gathered into a compact [heads, n_rows, d] tensor (and
//      a second time grouped by in-frame index, for the temporal candidates);
//   2. the tcgen05 attention kernel runs with the gathered rows as queries (their
//      original coordinates ride along), writing fp32 outputs: once dense over all
//      keys, then once per candidate through a small plan of its own: each 128-row block
//      of sampled rows is bounded by the min / max of its rows' frame and in-frame index,
//      which decides per key chunk whether it can hold a kept pair (conservative) and
//      whether every pair is kept (exact), so that a masked pass skips empty chunks and
//      runs full ones unmasked.  Every pass splits each work item's key range over
//      several CTAs and merges their partial rows exactly;
//   3. each candidate's squared deviation from dense is reduced in fp64, first over
//      slices of each head's outputs by many blocks, then per head in a fixed order
//      (deterministic), and per head the eligible candidate with the smallest one is
//      chosen, the earlier candidate on a tie.
// The classifier proper has two candidates, spatial then temporal, with per-head bands
// (a tie goes to spatial).  The band selection takes a caller's list of (type, band)
// candidates; the pages give no rule for trading deviation against cost (the least
// deviation alone always favours the widest band), so a candidate is eligible when the
// fraction of pairs its mask keeps stays within a caller's budget, the pages reporting
// about 39 % of pairs kept (aihirek.info, "A TPU-kernel kialakitasa dontonek bizonyult").
#include <cuda_runtime.h>

#include "svga_device.cuh"
#include "svga_internal.h"

namespace svga {
namespace {

struct BandParams {
    uint16_t w_spatial[kMaxHeads];
    uint16_t w_temporal[kMaxHeads];
};

// The default sampled rows r_i = floor((2i + 1) N / (2 n)) (one per row stratum).
__global__ void default_rows_kernel(int N, int n_rows, int32_t *rows)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_rows; i += gridDim.x * blockDim.x)
        rows[i] = (int32_t)(((2ll * i + 1) * (long long)N) / (2ll * n_rows));
}

// Head info of one candidate's pass plan: its mask type for every head, its band either
// shared (band >= 0) or per head from the classifier's band arrays (band < 0: the
// spatial or the temporal array by type); keys stay frame-major.
__global__ void candidate_info_kernel(int heads, int type, int band, BandParams bp, int4 *info)
{
    for (int h = blockIdx.x * blockDim.x + threadIdx.x; h < heads; h += gridDim.x * blockDim.x) {
        const int b = band >= 0 ? band : (type == MASK_SPATIAL ? bp.w_spatial[h] : bp.w_temporal[h]);
        info[h] = make_int4(type, b, ORDER_FM, 0);
    }
}

template <int VPR>
__global__ void gather_rows_kernel(const uint4 *__restrict__ q, uint4 *__restrict__ qg,
                                   const int32_t *__restrict__ rows, int N, int n_rows,
                                   int32_t *status)
{
    const int h = blockIdx.y;
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < n_rows * VPR;
         idx += gridDim.x * blockDim.x) {
        const int r = idx / VPR, v = idx - r * VPR;
        const int t = __ldg(rows + r);
        if (t < 0 || t >= N) {
            if (status) atomicExch(status, (int32_t)SVGA_ERR_INVALID_ARG);
            qg[((size_t)h * n_rows + r) * VPR + v] = make_uint4(0, 0, 0, 0);
            continue;
        }
        qg[((size_t)h * n_rows + r) * VPR + v] = __ldg(q + ((size_t)h * N + t) * VPR + v);
    }
}

constexpr int kMseParts = 32;  // blocks per head in the first reduction stage

// Frame and in-frame index bounds (min f, max f, min s, max s) of each 128-row block of
// sampled rows.  Rows outside 0..N-1 are clamped here (the gather reports them).
__global__ void __launch_bounds__(128) row_bounds_kernel(const int32_t *rows, int n_rows, int N,
                                                         int S, int4 *bounds)
{
    __shared__ int red[4][4];
    const int r = blockIdx.x * 128 + threadIdx.x;
    int fmin = 0x7fffffff, fmax = -1, smin = 0x7fffffff, smax = -1;
    if (r < n_rows) {
        int t = __ldg(rows + r);
        t = t < 0 ? 0 : (t >= N ? N - 1 : t);
        const int f = t / S, s = t - f * S;
        fmin = fmax = f;
        smin = smax = s;
    }
    for (int o = 16; o > 0; o >>= 1) {
        fmin = min(fmin, __shfl_xor_sync(0xffffffffu, fmin, o));
        fmax = max(fmax, __shfl_xor_sync(0xffffffffu, fmax, o));
        smin = min(smin, __shfl_xor_sync(0xffffffffu, smin, o));
        smax = max(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    }
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        red[w][0] = fmin;
        red[w][1] = fmax;
        red[w][2] = smin;
        red[w][3] = smax;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < 4; ++i) {
            fmin = min(fmin, red[i][0]);
            fmax = max(fmax, red[i][1]);
            smin = min(smin, red[i][2]);
            smax = max(smax, red[i][3]);
        }
        bounds[blockIdx.x] = make_int4(fmin, fmax, smin, smax);
    }
}

// Visit / full flags (1 | 2) of key chunk c (128 frame-major keys) for a block of rows
// with bounds bb, under a mask of `type` and `band`.  A chunk is at most three
// rectangles (frame x in-frame range): the first partial frame, whole frames, the last
// partial frame; only the first can be frame 0.  "Visit" from the distance between the
// bound intervals is a superset of the chunks that hold kept pairs; "full" compares the
// farthest pair, which is exact.
__device__ uint32_t chunk_flags(int4 bb, int type, int band, int anchor, int c, int N, int S)
{
    if (bb.y < 0) return 0u;
    const int ka = c * 128, kb = min(N, ka + 128);
    const int F0 = ka / S, m0 = ka - F0 * S, F1 = (kb - 1) / S, m1 = (kb - 1) - F1 * S;
    bool any = false, all = ka + 128 <= N;  // a chunk holding padding is never full
    auto rect = [&](int f0, int f1, int s0, int s1) {
        const bool anch = anchor && f0 == 0;
        int dist, far;
        if (type == MASK_SPATIAL) {
            dist = max(0, max(f0 - bb.y, bb.x - f1));
            far = max(bb.y - f0, f1 - bb.x);
        } else {
            dist = max(0, max(s0 - bb.w, bb.z - s1));
            far = max(bb.w - s0, s1 - bb.z);
        }
        any = any || anch || dist <= band;
        all = all && (anch || far <= band);
    };
    if (F0 == F1) {
        rect(F0, F0, m0, m1);
    } else {
        rect(F0, F0, m0, S - 1);
        if (F1 > F0 + 1) rect(F0 + 1, F1 - 1, 0, S - 1);
        rect(F1, F1, 0, m1);
    }
    return any ? (1u | (all ? 2u : 0u)) : 0u;
}

// The attention plan's entry for work item (head info hi, row-block pair p) and chunk c.
__device__ __forceinline__ uint32_t pass_entry(const int4 &hi, int anchor, const int4 *bounds,
                                               int n_qblk, int p, int c, int N, int S)
{
    const uint32_t a =
        2 * p < n_qblk ? chunk_flags(bounds[2 * p], hi.x, hi.y, anchor, c, N, S) : 0u;
    const uint32_t b =
        2 * p + 1 < n_qblk ? chunk_flags(bounds[2 * p + 1], hi.x, hi.y, anchor, c, N, S) : 0u;
    if (!(a | b)) return 0u;
    return (uint32_t)c | (a << 24) | (b << 26);
}

// Entries per work item (a head and two row blocks) of one pass plan.
__global__ void __launch_bounds__(256) pass_count_kernel(int n_pairs, int n_qblk, int n_kc, int N,
                                                         int S, int anchor, const int4 *head_info,
                                                         const int4 *bounds, int *cnt)
{
    __shared__ int red[8];
    const int item = blockIdx.x, h = item / n_pairs, p = item - h * n_pairs;
    const int4 hi = head_info[h];
    int n = 0;
    for (int c = threadIdx.x; c < n_kc; c += blockDim.x)
        n += pass_entry(hi, anchor, bounds, n_qblk, p, c, N, S) != 0u;
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = n;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
        for (int w = 0; w < 8; ++w) t += red[w];
        cnt[item] = t;
    }
}

// Exclusive offsets of the items' entries, the items and the plan header (one block).
__global__ void __launch_bounds__(1024) pass_items_kernel(int heads, int n_pairs, int n_items,
                                                          int N, int n_kc, const int *cnt,
                                                          int *off, int4 *items, char *plan)
{
    __shared__ int wsum[32];
    __shared__ int carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int base = 0; base < n_items; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int v = i < n_items ? cnt[i] : 0;
        int x = v;  // inclusive scan inside the warp
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[w] = x;
        __syncthreads();
        int before = carry;
        for (int j = 0; j < w; ++j) before += wsum[j];
        if (i < n_items) {
            const int start = before + x - v;
            off[i] = start;
            const int h = i / n_pairs, p = i - h * n_pairs;
            items[i] = make_int4(h, 2 * p, start, v);
        }
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = before + x;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        PlanHeader hdr{};
        hdr.magic = kPlanMagic;
        hdr.heads = heads;
        hdr.tokens = N;
        hdr.kn = 128;
        hdr.n_kc = n_kc;
        hdr.n_items = n_items;
        *reinterpret_cast<PlanHeader *>(plan) = hdr;
    }
}

// The entries of each item, in ascending chunk order.
__global__ void __launch_bounds__(128) pass_write_kernel(int n_pairs, int n_qblk, int n_kc, int N,
                                                         int S, int anchor, const int4 *head_info,
                                                         const int4 *bounds, const int *off,
                                                         uint32_t *entries)
{
    __shared__ int wsum[4];
    const int item = blockIdx.x, h = item / n_pairs, p = item - h * n_pairs;
    const int4 hi = head_info[h];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int o = off[item];
    for (int base = 0; base < n_kc; base += 128) {
        const int c = base + threadIdx.x;
        const uint32_t e = c < n_kc ? pass_entry(hi, anchor, bounds, n_qblk, p, c, N, S) : 0u;
        const uint32_t bal = __ballot_sync(0xffffffffu, e != 0u);
        const int pos = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) wsum[w] = __popc(bal);
        __syncthreads();
        int before = 0, tot = 0;
        for (int i = 0; i < 4; ++i) {
            before += i < w ? wsum[i] : 0;
            tot += wsum[i];
        }
        if (e != 0u) entries[o + before + pos] = e;
        o += tot;
        __syncthreads();
    }
}

// The temporal pass takes the sampled rows grouped by in-frame index s (a counting sort
// over the S positions), so that a 128-row block spans few positions and its plan skips
// the key chunks out of band.  Each row's output does not depend on its block.
__global__ void s_hist_kernel(const int32_t *rows, int n_rows, int N, int S, int *hist)
{
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < n_rows; r += gridDim.x * blockDim.x) {
        int t = __ldg(rows + r);
        t = t < 0 ? 0 : (t >= N ? N - 1 : t);
        atomicAdd(hist + t % S, 1);
    }
}

// Exclusive scan of the S counts in place (one block).
__global__ void __launch_bounds__(1024) s_scan_kernel(int *hist, int S)
{
    __shared__ int wsum[32];
    __shared__ int carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int base = 0; base < S; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int v = i < S ? hist[i] : 0;
        int x = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[w] = x;
        __syncthreads();
        int before = carry;
        for (int j = 0; j < w; ++j) before += wsum[j];
        if (i < S) hist[i] = before + x - v;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = before + x;
        __syncthreads();
    }
}

// rows_t[pos] = rows[r] with the rows of equal s contiguous; pos_t[r] = pos.  The order
// among rows of one s follows the atomics and may change from call to call: a row's
// output does not depend on the rows it shares a block with, the block's in-frame range
// (all the temporal plan reads) does not change, and the deviation sums run in the
// original row order, so the results are the same on every call.
__global__ void s_scatter_kernel(const int32_t *rows, int n_rows, int N, int S, int *cursor,
                                 int32_t *rows_t, int32_t *pos_t)
{
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < n_rows; r += gridDim.x * blockDim.x) {
        const int t0 = __ldg(rows + r);
        const int t = t0 < 0 ? 0 : (t0 >= N ? N - 1 : t0);
        const int pos = atomicAdd(cursor + t % S, 1);
        rows_t[pos] = t0;
        pos_t[r] = pos;
    }
}

// Stage 1: block (part, h) sums the squared deviations of one slice of head h between
// the dense output od and one candidate's output ox.  With pos (a temporal candidate's
// pass, which took the rows grouped by in-frame index) row r of od is row pos[r] of ox.
__global__ void __launch_bounds__(256) mse_partial_kernel(const float *od, const float *ox,
                                                          const int32_t *pos, int d, int n,
                                                          double *partial)
{
    __shared__ double red[8];
    const int part = blockIdx.x, h = blockIdx.y;
    const size_t base = (size_t)h * n;
    const int per = (n + kMseParts - 1) / kMseParts;
    const int i0 = part * per, i1 = min(n, i0 + per);
    double acc = 0.0;
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
        const int r = i / d, c = i - r * d;
        const size_t j = pos ? (size_t)__ldg(pos + r) * d + c : (size_t)i;
        const double dv = od[base + i];
        const double x = ox[base + j] - dv;
        acc += x * x;
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += red[w];
        partial[(size_t)h * kMseParts + part] = t;
    }
}

constexpr int kMaxCand = 16;  // candidates of one selection

struct CandParams {
    int n;
    int type[kMaxCand];
    int band[kMaxCand];  // shared band, or -1 (per-head bands: no band output)
    uint32_t eligible;   // bit c: candidate c may be chosen
};

// Stage 2: per head, each candidate's partial sums in part order (deterministic), its
// mean, and the choice: the eligible candidate with the least deviation, the earlier
// one on a tie.
__global__ void select_kernel(const double *partial, CandParams cp, int heads, int n,
                              int32_t *type_out, int32_t *band_out, float *mse_out)
{
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= heads) return;
    int best = -1;
    double best_mse = 0.0;
    for (int c = 0; c < cp.n; ++c) {
        const double *pc = partial + ((size_t)c * heads + h) * kMseParts;
        double t = 0.0;
        for (int part = 0; part < kMseParts; ++part) t += pc[part];
        t /= n;
        mse_out[(size_t)h * cp.n + c] = (float)t;
        if (((cp.eligible >> c) & 1u) && (best < 0 || t < best_mse)) {
            best = c;
            best_mse = t;
        }
    }
    type_out[h] = best >= 0 ? cp.type[best] : -1;
    if (band_out) band_out[h] = best >= 0 ? cp.band[best] : -1;
}

// Key-range split of the passes.  With 1% of the rows sampled the passes have few work
// items (a head and two 128-row blocks each), fewer than the 148 SMs of a B200 at
// 302,400 tokens and 10 heads (120 items), each with thousands of key chunks.  Splitting
// every item's chunks over P CTAs (P <= kMaxSplit) that write partial outputs, merged
// afterwards, fills the GPU: P minimises the waves per unit of work,
// ceil(items P / 148) / P, the smallest P on a tie.  The choice depends on the item
// count only, so the workspace size does too; on a part with other SM counts the split
// is still correct, only less well balanced.
constexpr int kMaxSplit = 8;
constexpr int kSplitSms = 148;

int classify_ksplit(int n_items)
{
    int best = 1;
    double best_cost = 1e30;
    for (int P = 1; P <= kMaxSplit; ++P) {
        const double waves = (double)(((long long)n_items * P + kSplitSms - 1) / kSplitSms);
        const double cost = waves / P;
        if (cost < best_cost - 1e-12) {
            best_cost = cost;
            best = P;
        }
    }
    return best;
}

struct ClassifyLayout {
    size_t plan, plan_hdr, bounds, bounds_t, cnt, off, rows, rows_t, pos_t, s_hist, qg, qg_t, od,
        ox, part_o, part_ml, partial, types, bands, mse, status, total;
    int ksplit;
};

ClassifyLayout classify_layout(int heads, int d, int n_rows, int N, int S, int n_cand)
{
    ClassifyLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    // one pass plan in the attention plan's layout, rebuilt for each candidate
    const int n_qblk = (n_rows + kBlockM - 1) / kBlockM, n_items = heads * ((n_qblk + 1) / 2);
    const int n_kc = (N + 127) / 128;
    L.plan_hdr = align_up(sizeof(PlanHeader) + sizeof(int4) * ((size_t)heads + n_items), 256);
    L.plan = take(L.plan_hdr + sizeof(uint32_t) * (size_t)n_items * n_kc);
    L.bounds = take(sizeof(int4) * n_qblk);
    L.bounds_t = take(sizeof(int4) * n_qblk);
    L.cnt = take(sizeof(int) * n_items);
    L.off = take(sizeof(int) * (n_items + 1));
    L.rows = take(sizeof(int32_t) * n_rows);
    L.rows_t = take(sizeof(int32_t) * n_rows);
    L.pos_t = take(sizeof(int32_t) * n_rows);
    L.s_hist = take(sizeof(int) * (size_t)S);
    L.qg = take((size_t)heads * n_rows * d * 2);
    L.qg_t = take((size_t)heads * n_rows * d * 2);
    L.od = take((size_t)heads * n_rows * d * 4);
    L.ox = take((size_t)heads * n_rows * d * 4);
    L.ksplit = classify_ksplit(n_items);
    // shared by the passes, each merged before the next starts
    L.part_o = L.ksplit > 1 ? take((size_t)L.ksplit * heads * n_rows * d * 4) : 0;
    L.part_ml = L.ksplit > 1 ? take((size_t)L.ksplit * heads * n_rows * 8) : 0;
    L.partial = take(sizeof(double) * (size_t)n_cand * kMseParts * heads);
    L.types = take(sizeof(int32_t) * heads);
    L.bands = take(sizeof(int32_t) * heads);
    L.mse = take(sizeof(float) * (size_t)n_cand * heads);
    L.status = take(sizeof(int32_t));
    L.total = o;
    return L;
}

}  // namespace

size_t classify_workspace_bytes(const svga_problem *p, int n_rows, int n_cand)
{
    return classify_layout(p->heads, p->head_dim, n_rows,
                           p->num_frames * p->grid_h * p->grid_w, p->grid_h * p->grid_w, n_cand)
        .total;
}

int max_candidates() { return kMaxCand; }

svga_status run_select(const void *q, const void *k, const void *v, const svga_problem *p,
                       int n_cand, const int32_t *cand_type, const int32_t *cand_band,
                       uint32_t eligible, const int32_t *w_spatial, const int32_t *w_temporal,
                       const int32_t *rows, int n_rows, float scale, int32_t *type_out,
                       int32_t *band_out, float *mse_out, int32_t *status_out, int device_out,
                       void *ws, size_t ws_bytes, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int H = p->heads, d = p->head_dim, S = p->grid_h * p->grid_w, N = p->num_frames * S;
    const ClassifyLayout L = classify_layout(H, d, n_rows, N, S, n_cand);
    (void)ws_bytes;
    char *w = static_cast<char *>(ws);
    char *plan = w + L.plan;
    int4 *info = reinterpret_cast<int4 *>(plan + sizeof(PlanHeader));
    int4 *bounds = reinterpret_cast<int4 *>(w + L.bounds);
    int4 *bounds_t = reinterpret_cast<int4 *>(w + L.bounds_t);
    int32_t *rows_t = reinterpret_cast<int32_t *>(w + L.rows_t);
    int32_t *pos_t = reinterpret_cast<int32_t *>(w + L.pos_t);
    int *s_hist = reinterpret_cast<int *>(w + L.s_hist);
    void *qg_t = w + L.qg_t;
    int *cnt = reinterpret_cast<int *>(w + L.cnt);
    int *off = reinterpret_cast<int *>(w + L.off);
    int32_t *rows_ws = reinterpret_cast<int32_t *>(w + L.rows);
    void *qg = w + L.qg;
    float *od = reinterpret_cast<float *>(w + L.od);
    float *ox = reinterpret_cast<float *>(w + L.ox);
    double *partial = reinterpret_cast<double *>(w + L.partial);
    int32_t *types = reinterpret_cast<int32_t *>(w + L.types);
    int32_t *bands = reinterpret_cast<int32_t *>(w + L.bands);
    float *mse = reinterpret_cast<float *>(w + L.mse);
    int32_t *status = reinterpret_cast<int32_t *>(w + L.status);

    BandParams bp{};
    if (w_spatial && w_temporal)
        for (int h = 0; h < H; ++h) {
            bp.w_spatial[h] = (uint16_t)w_spatial[h];
            bp.w_temporal[h] = (uint16_t)w_temporal[h];
        }
    CandParams cp{};
    cp.n = n_cand;
    cp.eligible = eligible;
    for (int c = 0; c < n_cand; ++c) {
        cp.type[c] = cand_type[c];
        cp.band[c] = cand_band ? cand_band[c] : -1;
    }
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess ||
        cudaMemsetAsync(s_hist, 0, sizeof(int) * (size_t)S, st) != cudaSuccess) {
        set_error("cudaMemsetAsync failed");
        return SVGA_ERR_CUDA;
    }
    const int32_t *rows_use = rows ? rows : rows_ws;
    if (!rows) default_rows_kernel<<<n_rows / 256 + 1, 256, 0, st>>>(N, n_rows, rows_ws);
    const int vpr = d / 8;
    dim3 grid((n_rows * vpr + 255) / 256 < 1184 ? (n_rows * vpr + 255) / 256 : 1184, H);
    auto gather = [&](const int32_t *r, void *dst) {
        if (vpr == 16)
            gather_rows_kernel<16><<<grid, 256, 0, st>>>(static_cast<const uint4 *>(q),
                                                        static_cast<uint4 *>(dst), r, N, n_rows,
                                                        status);
        else
            gather_rows_kernel<8><<<grid, 256, 0, st>>>(static_cast<const uint4 *>(q),
                                                       static_cast<uint4 *>(dst), r, N, n_rows,
                                                       status);
    };
    gather(rows_use, qg);
    const int n_qblk = (n_rows + kBlockM - 1) / kBlockM, n_pairs = (n_qblk + 1) / 2;
    const int n_items = H * n_pairs, n_kc = (N + 127) / 128;
    // rows grouped by in-frame index for the temporal passes, their Q rows gathered so
    const int sblocks = (n_rows + 255) / 256 < 1184 ? (n_rows + 255) / 256 : 1184;
    s_hist_kernel<<<sblocks, 256, 0, st>>>(rows_use, n_rows, N, S, s_hist);
    s_scan_kernel<<<1, 1024, 0, st>>>(s_hist, S);
    s_scatter_kernel<<<sblocks, 256, 0, st>>>(rows_use, n_rows, N, S, s_hist, rows_t, pos_t);
    gather(rows_t, qg_t);
    row_bounds_kernel<<<n_qblk, 128, 0, st>>>(rows_use, n_rows, N, S, bounds);
    row_bounds_kernel<<<n_qblk, 128, 0, st>>>(rows_t, n_rows, N, S, bounds_t);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("classifier setup launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    AttnLaunch a{};
    a.k = k;
    a.v = v;
    a.lse = nullptr;
    a.heads = H;
    a.nq_rows = n_rows;
    a.nk_rows = N;
    a.d = d;
    a.F = p->num_frames;
    a.S = S;
    a.anchor = p->anchor_frame0;
    a.scale = scale;
    a.kn = 128;
    a.out_f32 = 1;
    a.n_items = n_items;
    a.status = status;
    a.ksplit = L.ksplit;
    a.part_o = L.ksplit > 1 ? reinterpret_cast<float *>(w + L.part_o) : nullptr;
    a.part_ml = L.ksplit > 1 ? reinterpret_cast<float *>(w + L.part_ml) : nullptr;
    svga_status rc;
    auto pass = [&]() {
        svga_status r = launch_attention(a, stream);
        return r != SVGA_OK ? r : merge_attention_parts(a, stream);
    };
    // the dense pass over every key
    a.mode = 1;
    a.q = qg;
    a.qrow_tokens = rows_use;
    a.o = od;
    if ((rc = pass()) != SVGA_OK) return rc;
    // one masked pass per candidate through its own plan, and its deviation from dense
    int4 *items = info + H;
    uint32_t *entries = reinterpret_cast<uint32_t *>(plan + L.plan_hdr);
    a.mode = 0;
    a.plan = plan;
    a.o = ox;
    for (int c = 0; c < n_cand; ++c) {
        const bool temporal = cp.type[c] == MASK_TEMPORAL;
        const int4 *bnd = temporal ? bounds_t : bounds;
        candidate_info_kernel<<<H / 256 + 1, 256, 0, st>>>(H, cp.type[c], cp.band[c], bp, info);
        pass_count_kernel<<<n_items, 256, 0, st>>>(n_pairs, n_qblk, n_kc, N, S,
                                                   p->anchor_frame0, info, bnd, cnt);
        pass_items_kernel<<<1, 1024, 0, st>>>(H, n_pairs, n_items, N, n_kc, cnt, off, items, plan);
        pass_write_kernel<<<n_items, 128, 0, st>>>(n_pairs, n_qblk, n_kc, N, S,
                                                   p->anchor_frame0, info, bnd, off, entries);
        if ((e = cudaGetLastError()) != cudaSuccess) {
            set_error("classifier plan launch failed: %s", cudaGetErrorString(e));
            return SVGA_ERR_CUDA;
        }
        a.q = temporal ? qg_t : qg;
        a.qrow_tokens = temporal ? rows_t : rows_use;
        if ((rc = pass()) != SVGA_OK) return rc;
        mse_partial_kernel<<<dim3(kMseParts, H), 256, 0, st>>>(
            od, ox, temporal ? pos_t : nullptr, d, n_rows * d, partial + (size_t)c * H * kMseParts);
    }
    select_kernel<<<(H + 127) / 128, 128, 0, st>>>(partial, cp, H, n_rows * d, types,
                                                   band_out ? bands : nullptr, mse);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("classifier reduction launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    const size_t mse_bytes = sizeof(float) * (size_t)n_cand * H;
    if (device_out) {
        // results stay on the device: no host round trip, nothing waits
        if (cudaMemcpyAsync(type_out, types, sizeof(int32_t) * H, cudaMemcpyDeviceToDevice,
                            st) != cudaSuccess ||
            (band_out && cudaMemcpyAsync(band_out, bands, sizeof(int32_t) * H,
                                         cudaMemcpyDeviceToDevice, st) != cudaSuccess) ||
            (mse_out &&
             cudaMemcpyAsync(mse_out, mse, mse_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess) ||
            (status_out && cudaMemcpyAsync(status_out, status, sizeof(int32_t),
                                           cudaMemcpyDeviceToDevice, st) != cudaSuccess)) {
            set_error("classifier result copy failed: %s", cudaGetErrorString(cudaGetLastError()));
            return SVGA_ERR_CUDA;
        }
        return SVGA_OK;
    }
    int32_t dev_status = 0;
    if (cudaMemcpyAsync(type_out, types, sizeof(int32_t) * H, cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        (band_out && cudaMemcpyAsync(band_out, bands, sizeof(int32_t) * H, cudaMemcpyDeviceToHost,
                                     st) != cudaSuccess) ||
        (mse_out &&
         cudaMemcpyAsync(mse_out, mse, mse_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) ||
        cudaMemcpyAsync(&dev_status, status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        set_error("classifier result copy failed: %s", cudaGetErrorString(cudaGetLastError()));
        return SVGA_ERR_CUDA;
    }
    if (dev_status != 0) {
        set_error("classifier kernels reported %d on the device", dev_status);
        return (svga_status)dev_status;
    }
    return SVGA_OK;
}

svga_status run_classify(const void *q, const void *k, const void *v, const svga_problem *p,
                         const int32_t *w_spatial, const int32_t *w_temporal, const int32_t *rows,
                         int n_rows, float scale, int32_t *head_type_out, float *mse_out,
                         int32_t *status_out, int device_out, void *ws, size_t ws_bytes,
                         void *stream)
{
    // two candidates with per-head bands: spatial first, so that a tie goes to spatial
    const int32_t types[2] = {MASK_SPATIAL, MASK_TEMPORAL};
    return run_select(q, k, v, p, 2, types, nullptr, 3u, w_spatial, w_temporal, rows, n_rows,
                      scale, head_type_out, nullptr, mse_out, status_out, device_out, ws, ws_bytes,
                      stream);
}

}  // namespace svga
