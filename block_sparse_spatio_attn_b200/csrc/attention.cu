// attention.cu -- block-sparse flash-attention forward for B200 (sm_100a).
//
// Computes, per head and query row, the masked softmax(scale * q k^T) v over the keys
// the head's mask keeps, walking only the key tiles that hold kept pairs.  Full tiles
// run with no mask arithmetic; boundary tiles are masked element by element from the
// tokens' (frame, in-frame index) coordinates.  This is the full/boundary tile
// specialisation of "Accelerating Spatio-Temporal Attention for Video Diffusion on
// TPUs" (aihirek.info, section "A TPU-kernel kialakitasa dontonek bizonyult";
// ainews.tenesys.com, "Co sie zmienilo?" items 1-2), written for Blackwell:
//
//   * one CTA per work item = two consecutive 128-row query blocks (Q0, Q1) that share
//     one stream of key chunks (the merged lists of the two blocks); a visit is one
//     (chunk, block) pair the block's list holds, taken chunk by chunk, Q0 before Q1;
//   * warp 0 streams K and V chunks with TMA (128-byte swizzle) through a ring of
//     shared-memory stages;
//   * TMEM: S | P0 | P1 | O0 | O1 (128, 64, 64, 128, 128 columns).  The S tile is shared
//     by the two groups and P has columns of its own, so the S of the next visit can be
//     computed as soon as the previous S has been read into registers; a group's next S
//     does not wait for its P V product (with P written over S it would);
//   * two threads issue tcgen05.mma: warp 1 the products S = Q_i K^T (A, B from shared
//     memory, D in TMEM, fp32) visit after visit, warp 3 the products O_i += P_i V
//     (A = P from TMEM as bf16, B = V from shared memory), each P V right behind the S
//     two visits ahead of it, where it runs while that S is being read.  Neither waits
//     for the other; the hazards between the streams go through the softmax barriers;
//   * warps 4-7 and 8-11 hold one query row per thread (TMEM lane = row): they read S,
//     run the online softmax in the exp2 domain with packed fp32x2 arithmetic and the
//     MUFU exponential, and write P as bf16 into their P columns.  The reference maximum
//     is the exact maximum of the row's first visited tile and is kept: later tiles
//     need no maximum pass; a tile whose P sum would exceed 2^16 is redone with its own
//     maximum after O is rescaled in TMEM;
//   * boundary tiles build a 128-bit keep mask per row from the runs of the key chunk
//     (at most a few intervals per run), then mask with one select per element;
//   * the producer/MMA warpgroup gives registers to the softmax warpgroups (setmaxnreg);
//   * a launch may run one part of the plan's items (snake order), so one problem can
//     be split over several GPUs; the tile-aligned traversal (B3) treats every visited
//     chunk as full;
//   * with Q and O frame-major, the softmax threads of a temporal-major head copy their
//     own Q rows into the swizzled Q tile (frame-major heads keep the TMA load) and
//     every head writes O and LSE rows back to their frame-major tokens;
//   * with K and V frame-major, warps 0 and 2 gather the key chunks of a temporal-major
//     head row by row (16-byte cp.async into the same swizzled stage layout) in place of
//     warp 0's tile loads;
//   * plan entries are read one step ahead and used only at the next step, so that no
//     warp waits for a global load in its loop.
//
// Every mbarrier wait gives up after about a second: the CTA raises a shared abort
// flag, drains its MMAs and copies, frees TMEM, writes SVGA_ERR_TIMEOUT to the
// caller's status word and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>
#include <type_traits>

#include "svga_device.cuh"
#include "svga_internal.h"


namespace svga {
namespace {

constexpr int kThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;
// a tile's P sum above this (2^16) triggers a new reference maximum; every P then stays
// below it, far inside the range of bf16 P and of the fp32 sums
constexpr float kTileSumLimit = 65536.0f;

constexpr uint32_t kNegInfBits = 0xff800000u;
// Register split: the producer / MMA warpgroup drops to kRegsLow, the two softmax
// warpgroups rise to kRegsHigh.  128 * kRegsLow + 256 * kRegsHigh must not exceed the
// 384 * kRegsLaunch registers the CTA is launched with (checked on the host).
constexpr int kRegsLaunch = 168, kRegsLow = 120, kRegsHigh = 192;
// TMEM columns: the S tile shared by the two groups, a P tile per group, an O per group
constexpr uint32_t kTmS = 0, kTmP = 128, kTmO = 256;
constexpr int kGatherThreads = 64;  // warps 0 and 2, when K / V rows are gathered
constexpr int kGatherRows = kGatherThreads / 8;  // chunk rows one gather step covers
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split");

struct KParams {
    int heads, nq_rows, nk_rows, F, S, anchor;
    int N, Sp;  // tokens and frame stride: frame-major frame f starts at position f * Sp
    float scale_log2;
    int mode, naive, aligned, n_pairs, n_qblk, n_kc;
    int n_items, part, num_parts;  // plan mode: this launch runs the items of one part
    int test_stall;                // test hook: the first K chunk is never loaded
    int qo_fm;                     // Q and O frame-major: Q rows gathered, O rows scattered
    int kv_fm;                     // K and V frame-major: key rows gathered
    const void *q, *k, *v;         // bases for the gathers
    int check_plan;                // compare the plan with this launch before using it
    int tile_q, tile_k;            // the map tiles the plan must have been built with
    const PlanHeader *hdr;
    const int4 *items;
    const uint32_t *entries;
    const int4 *head_info;
    const int32_t *qrow_tokens;
    void *o;
    float *lse;
    int32_t *status;
    // Key-range split: each work item runs as ksplit CTAs, CTA part r taking the item's
    // entries [r E / ksplit, (r + 1) E / ksplit).  With ksplit > 1 a CTA writes its rows'
    // unnormalised O (fp32) to part_o and (reference maximum, sum) to part_ml, both
    // indexed [(r * heads + head) * nq_rows + row], for a merge kernel to combine.
    int ksplit;
    float *part_o;
    float2 *part_ml;
    // plan mode after the pair kernel: run only the items the pair kernel leaves
    int pair_rest;
};

template <int D, int KN>
struct Cfg {
    static constexpr int kQBytes = kBlockM * D * 2;             // one 128-row Q tile
    static constexpr int kQChunk = kBlockM * 128;               // 64 columns x 128 rows
    static constexpr int kKVBytes = KN * D * 2;                  // one K or V chunk
    static constexpr int kKVChunk = KN * 128;                    // 64 columns x KN rows
    static constexpr int kStages = (kKVBytes >= 32768) ? 5 : 8;
    static constexpr int kSmemData = 2 * kQBytes + kStages * kKVBytes;
    static constexpr int kSmemBar = 1024;
    static constexpr int kSmemAlloc = kSmemData + kSmemBar + 1024;  // + alignment slack
    static constexpr int kSmemLaunch = kSmemAlloc < 120 * 1024 ? 120 * 1024 : kSmemAlloc;
    static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");
};

struct Barriers {
    uint64_t q_full;
    uint64_t kv_full[8];
    uint64_t kv_empty[8];
    uint64_t s_full[2];  // [group]: that group's S is in the shared S columns
    uint64_t s_free;     // the S columns were read into registers by their owner (4 warps)
    uint64_t s_issued[4];  // [visit % 4]: the S issuer has issued the S of that visit
    uint64_t p_full[2];  // [group]: P of the group's tile is in its P columns (4 warps)
    uint64_t o_done[2];  // [group]: the group's last P V product is done
    uint64_t drain[2];   // abort: [issuer]: the MMAs that issuer started are done
    uint32_t tmem_base;
    int abort;
};

struct Item {
    int h, b0, E;
    const uint32_t *ent;
    bool valid1, ragged;
    int mode, naive, n_kc;
    int n0;  // dense: chunk of this part's first entry (key-range split)

    // Entry n as stored (plan mode: a global load).  A prefetched entry is read with
    // raw() and passed through fix() only where it is used: an instruction that depends on
    // the load right after it would hold the warp for the whole load latency.
    __device__ __forceinline__ uint32_t raw(int n) const
    {
        // dense: every chunk, full except a last one that runs past the final token
        const int c = n + n0;
        const bool full = !(ragged && c == n_kc - 1);
        uint32_t e = (uint32_t)c | kEntV0 | (full ? kEntF0 : 0u);
        if (valid1) e |= kEntV1 | (full ? kEntF1 : 0u);
        // plan mode: a predicated load over that value (a select between the two would
        // wait for the load at once)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.eq.s32 p, %2, 0;\n\t@p ld.global.nc.u32 %0, [%1];\n\t}"
            : "+r"(e)
            : "l"(ent + n), "r"(mode));
        return e;
    }
    // The naive traversal clears the full flags (visit flags and chunk are unchanged).
    __device__ __forceinline__ uint32_t fix(uint32_t e) const
    {
        return (mode == 0 && naive) ? (e & ~(kEntF0 | kEntF1)) : e;
    }
    __device__ __forceinline__ uint32_t entry(int n) const { return fix(raw(n)); }
};

// Plan items (sorted longest first) are dealt to the parts in snake order: in group g of
// num_parts consecutive items, part r takes item r when g is even and num_parts-1-r when
// g is odd, which keeps the parts' total work within one item of each other.  Under a
// key-range split the ksplit consecutive CTAs of one item share its g.
__device__ __forceinline__ int plan_item_of_slot(const KParams &p, int g)
{
    const int r = p.part, n = p.num_parts;
    return g * n + ((g & 1) ? n - 1 - r : r);
}

// The CTAs of one work item: ksplit key-range parts, or the two CTAs of a pair.
__device__ __forceinline__ int item_slot(const KParams &p) { return blockIdx.x / p.ksplit; }
__device__ __forceinline__ int plan_item_of_block(const KParams &p)
{
    return plan_item_of_slot(p, item_slot(p));
}

// A caller's plan must describe this launch before any of its offsets is used: the
// header against the launch's shape, tiles, anchor and item count, then this CTA's work
// item (head, even first block, entry range inside the plan) and the head's info.
// Every thread of the CTA reads the same words, so the outcome is uniform.
__device__ __forceinline__ bool plan_matches(const KParams &p, int kn, int slot)
{
    const int4 *h4 = reinterpret_cast<const int4 *>(p.hdr);
    // {magic, heads, tokens, frames}, {tokens_per_frame, anchor, tile_q, tile_k},
    // {kn, n_qblk, n_kc, n_items}, {entry_cap (low, high), frame stride, reserved}
    const int4 a = __ldg(h4), b = __ldg(h4 + 1), c = __ldg(h4 + 2), d = __ldg(h4 + 3);
    const long long entry_cap = (long long)(uint32_t)d.x | ((long long)d.y << 32);
    if (!(a.x == kPlanMagic && a.y == p.heads && a.z == p.N && a.w == p.F && b.x == p.S &&
          b.y == p.anchor && b.z == p.tile_q && b.w == p.tile_k && c.x == kn &&
          c.y == p.n_qblk && c.z == p.n_kc && c.w == p.n_items && d.z == p.Sp &&
          p.nq_rows == p.F * p.Sp && p.nk_rows == p.nq_rows))
        return false;
    const int4 x = __ldg(p.items + plan_item_of_slot(p, slot));
    if (!(x.x >= 0 && x.x < p.heads && x.y >= 0 && !(x.y & 1) && x.y < p.n_qblk && x.z >= 0 &&
          x.w >= 0 && x.w <= p.n_kc && (long long)x.z + x.w <= entry_cap))
        return false;
    const int4 hi = __ldg(p.head_info + x.x);
    return (hi.x == MASK_SPATIAL || hi.x == MASK_TEMPORAL) && hi.y >= 0 && hi.z >= ORDER_FM &&
           hi.z <= ORDER_TM_STRICT;
}

__device__ __forceinline__ Item make_item(const KParams &p, int kn, int slot, int kpart)
{
    Item it;
    it.mode = p.mode;
    it.naive = p.naive;
    it.n_kc = p.n_kc;
    it.ragged = (p.nk_rows % kn) != 0;
    int e_all;  // entries of the whole item
    if (p.mode == 0) {
        const int4 x = __ldg(p.items + plan_item_of_slot(p, slot));
        it.h = x.x;
        it.b0 = x.y;
        it.ent = p.entries + x.z;
        e_all = x.w;
    } else {
        const int item = slot;
        it.h = item / p.n_pairs;
        it.b0 = 2 * (item - it.h * p.n_pairs);
        it.ent = nullptr;
        e_all = p.n_kc;
    }
    // this CTA's share of the entries (all of them without a key-range split)
    const int r = kpart;
    const int e0 = (int)((long long)r * e_all / p.ksplit);
    const int e1 = (int)((long long)(r + 1) * e_all / p.ksplit);
    if (it.ent) it.ent += e0;
    it.n0 = e0;
    it.E = e1 - e0;
    it.valid1 = it.b0 + 1 < p.n_qblk;
    return it;
}

// Does the CTA pair run this item?  It takes items whose two 128-row blocks both exist
// and both visit at least one key chunk; the rest (the last item of a head with an odd
// number of blocks, items one of whose blocks visits nothing) run in the one-CTA kernel.
// Every thread of the CTA calls it; the entries are scanned by all threads together.
__device__ __forceinline__ bool item_fits_pair(const Item &it)
{
    if (!it.valid1) return false;
    uint32_t any = 0u;
    for (int n = threadIdx.x; n < it.E; n += blockDim.x) any |= it.raw(n);
    const int has0 = __syncthreads_or((int)(any & kEntV0));
    const int has1 = __syncthreads_or((int)(any & kEntV1));
    return has0 && has1;
}

// Set bits [c0, c1) of a mask of NW 32-bit words (0 <= c0 < c1 <= 32 * NW).
template <int NW>
__device__ __forceinline__ void mask_set(uint32_t (&m)[NW], int c0, int c1)
{
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int lo = max(c0 - 32 * w, 0), hi = min(c1 - 32 * w, 32);
        if (lo < hi) {
            const uint32_t upto = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
            m[w] |= upto & ~((1u << lo) - 1u);
        }
    }
}

// Keep mask of the key positions [k0, k0 + KN) for one query (fq, sq): bit c is set
// when position k0 + c holds a key and the head's mask keeps it.  The positions of a
// chunk are walked row by row of the order's grid (a frame in frame-major order, an
// in-frame index in the temporal-major orders); in each row the kept keys form at most
// two intervals, so the mask costs a handful of integer operations per row.  Keys end
// at position N_end (frame-major: F * Sp, temporal-major: the token count); frame f of
// a frame-major head starts at f * Sp and holds S keys (Sp > S: the padded layout).  A
// query without a token (q_tok false) keeps nothing.
template <int KN>
__device__ __forceinline__ void keep_mask(int order, int type, int band, int anchor, int F, int S,
                                          int Sp, int N_end, bool q_tok, int fq, int sq, int k0,
                                          uint32_t (&m)[KN / 32])
{
#pragma unroll
    for (int w = 0; w < KN / 32; ++w) m[w] = 0u;
    if (!q_tok) return;
    const int kend = min(k0 + KN, N_end);
    int pos = k0, fixed, row_start, row_len, row_stride, fbase;
    bool f_fixed;
    if (order == ORDER_FM) {
        fixed = pos / Sp;
        row_start = fixed * Sp;
        row_len = S;
        row_stride = Sp;
        f_fixed = true;
        fbase = 0;
    } else if (order == ORDER_TM_STRICT) {
        fixed = pos / F;
        row_start = fixed * F;
        row_len = row_stride = F;
        f_fixed = false;
        fbase = 0;
    } else if (pos < S) {
        fixed = 0;
        row_start = 0;
        row_len = row_stride = S;
        f_fixed = true;
        fbase = 0;
    } else {
        fixed = (pos - S) / (F - 1);
        row_start = S + fixed * (F - 1);
        row_len = row_stride = F - 1;
        f_fixed = false;
        fbase = 1;
    }
    // kept intervals are merged while they touch, so runs of fully kept rows cost one
    // mask_set
    int plo = 0, phi = 0;
    auto flush = [&]() {
        if (plo < phi) mask_set<KN / 32>(m, plo - k0, phi - k0);
        plo = phi = 0;
    };
#pragma unroll 1
    while (true) {
        pos = max(pos, row_start);  // the positions between a padded frame's end and the next
        if (pos >= kend) break;
        const int b = min(kend, row_start + row_len);
        auto add = [&](int lo, int hi) {
            lo = max(lo, pos);
            hi = min(hi, b);
            if (lo >= hi) return;
            if (plo < phi && lo == phi) {
                phi = hi;
            } else {
                flush();
                plo = lo;
                phi = hi;
            }
        };
        if (type == MASK_DENSE) {
            add(pos, b);
        } else if (f_fixed) {  // one frame: s runs along the row
            const int ff = fixed;
            if ((anchor && ff == 0) || (type == MASK_SPATIAL && abs(fq - ff) <= band))
                add(pos, b);
            else if (type == MASK_TEMPORAL)
                add(row_start + sq - band, row_start + sq + band + 1);
        } else {  // one in-frame index: f runs along the row from fbase
            const int sf = fixed;
            if (type == MASK_TEMPORAL) {
                if (abs(sq - sf) <= band)
                    add(pos, b);
                else if (anchor && fbase == 0)
                    add(row_start, row_start + 1);
            } else {
                add(row_start + (fq - band) - fbase, row_start + (fq + band) - fbase + 1);
                if (anchor && fbase == 0) add(row_start, row_start + 1);
            }
        }
        pos = max(pos, b);
        if (order == ORDER_TM && f_fixed) {  // leave the frame-0 block
            f_fixed = false;
            fbase = 1;
            fixed = 0;
            row_start = S;
            row_len = row_stride = F - 1;
        } else {
            ++fixed;
            row_start += row_stride;
        }
    }
    flush();
}

template <int D, int KN, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const KParams p)
{
    using C = Cfg<D, KN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *sQ = smem;                                  // 2 x kQBytes
    uint8_t *sKV = smem + 2 * C::kQBytes;                // kStages x kKVBytes
    Barriers *bar = reinterpret_cast<Barriers *>(smem + C::kSmemData);
    volatile int *abort_flag = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (p.mode == 0 && plan_item_of_block(p) >= p.n_items) return;  // the last group ran out
    if (p.mode == 0 && p.check_plan && !plan_matches(p, KN, item_slot(p))) {
        // a map built for another problem: report it and touch nothing
        if (threadIdx.x == 0 && p.status) atomicCAS(p.status, 0, (int32_t)SVGA_ERR_INVALID_ARG);
        return;
    }
    const Item it = make_item(p, KN, item_slot(p), blockIdx.x % p.ksplit);
    if (p.pair_rest && item_fits_pair(it)) return;  // the pair kernel ran this item
    // keys of a head in a temporal-major order, read from frame-major K and V: warps 0 and
    // 2 gather the chunk rows instead of the TMA producer's tile loads
    const bool kv_gather = p.kv_fm && p.mode == 0 && __ldg(p.head_info + it.h).z != ORDER_FM;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar->q_full), 1);  // the TMA load, or the last gathering warp
        for (int s = 0; s < C::kStages; ++s) {
            // the TMA load, or one arrival per gathering thread
            mbar_init(smem_u32(&bar->kv_full[s]), kv_gather ? kGatherThreads : 1);
            mbar_init(smem_u32(&bar->kv_empty[s]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bar->s_full[i]), 1);
            mbar_init(smem_u32(&bar->p_full[i]), 4);  // one arrival per softmax warp
            mbar_init(smem_u32(&bar->o_done[i]), 1);
        }
        mbar_init(smem_u32(&bar->s_free), 4);  // one arrival per softmax warp of the owner
        for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bar->s_issued[i]), 1);
        mbar_init(smem_u32(&bar->drain[0]), 1);
        mbar_init(smem_u32(&bar->drain[1]), 1);
        bar->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&bar->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp < 4) {
        setmaxnreg_dec<kRegsLow>();
        if (warp == 0 && lane == 0) {
            // -------------------------------------------------------- TMA producer
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const uint32_t qf = smem_u32(&bar->q_full);
            // frame-major Q of a head in frame-major order is already in the head's order
            const bool q_tma = !p.qo_fm || __ldg(p.head_info + it.h).z == ORDER_FM;
            if (q_tma) {
                mbar_arrive_expect_tx(qf, (it.valid1 ? 2 : 1) * C::kQBytes);
                for (int i = 0; i < (it.valid1 ? 2 : 1); ++i)
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(smem_u32(sQ + i * C::kQBytes + c * C::kQChunk), &tmQ, qf,
                                    64 * c, (it.b0 + i) * kBlockM, it.h);
            }
            int issued = 0;
            bool ok = true;
            uint32_t e_nxt = (!kv_gather && it.E > 0) ? it.raw(0) : 0u;  // one entry ahead
            for (int n = 0; n < (kv_gather ? 0 : it.E) && ok; ++n) {
                const int kc = (int)(e_nxt & kEntChunkMask);
                e_nxt = it.raw(min(n + 1, it.E - 1));
                for (int t = 0; t < 2; ++t) {
                    const int idx = 2 * n + t, s = idx % C::kStages, round = idx / C::kStages;
                    if (round > 0 &&
                        !mbar_wait(smem_u32(&bar->kv_empty[s]), (round - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (p.test_stall && idx == 0) {  // nothing ever completes this stage
                        issued = idx + 1;
                        continue;
                    }
                    const uint32_t fb = smem_u32(&bar->kv_full[s]);
                    mbar_arrive_expect_tx(fb, C::kKVBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(smem_u32(sKV + s * C::kKVBytes + c * C::kKVChunk),
                                    t ? &tmV : &tmK, fb, 64 * c, kc * KN, it.h);
                    issued = idx + 1;
                }
            }
            {
                // Every copy this thread issued lands before the CTA can exit, whichever
                // role aborts (in a normal run they have all landed already).
                if (q_tma) mbar_wait_bounded(qf, 0);
                for (int idx = (issued > C::kStages ? issued - C::kStages : 0); idx < issued; ++idx)
                    if (!(p.test_stall && idx == 0))
                        mbar_wait_bounded(smem_u32(&bar->kv_full[idx % C::kStages]),
                                          (idx / C::kStages) & 1);
            }
        }
        if ((warp == 0 || warp == 2) && kv_gather) {
            // ---------------------------------------------------- K/V row gather
            // Chunk row r holds the key at position kc * KN + r of the head's order; its
            // frame-major token is found by walking the order's grid.  Eight lanes copy one
            // 128-byte half row, 16 bytes each, into the 128-byte-swizzled stage (the
            // layout the TMA load gives); rows past the last token are zero-filled.  Each
            // thread's copies arrive on the stage's barrier when they land, so the gather
            // never waits for its own copies and keeps every free stage in flight; the MMA
            // issuers order the landed rows before their reads with a proxy fence.
            // warp 0 joins once its lane 0 has issued the Q load (no K / V tile loads then)
            const int gt = (warp == 0 ? 0 : 32) + lane;
            const int u = gt & 7, r0 = gt >> 3;  // rows r0 + kGatherRows * g
            const int korder = __ldg(p.head_info + it.h).z;
            // within a head the row offsets fit 32 bits (at most 2^24 rows of 256 bytes)
            const size_t head_off = (size_t)it.h * p.nk_rows * (D * 2);
            const char *kb = static_cast<const char *>(p.k) + head_off;
            const char *vb = static_cast<const char *>(p.v) + head_off;
            const uint32_t dst_base = smem_u32(sKV);
            const int total = 2 * it.E;
            int tok[KN / kGatherRows];
            int issued = 0;
            bool ok = true;
            for (int idx = 0; idx < total; ++idx) {
                const int s = idx % C::kStages, round = idx / C::kStages;
                if (round > 0 &&
                    !mbar_wait(smem_u32(&bar->kv_empty[s]), (round - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                issued = idx + 1;
                if (!(idx & 1)) {  // the K stage of a chunk: its rows' tokens
                    const int pos0 = (int)(it.entry(idx >> 1) & kEntChunkMask) * KN + r0;
                    int f = 0, sx = 0;
                    if (pos0 < p.nk_rows) pos_to_coord(korder, pos0, p.F, p.S, f, sx);
#pragma unroll
                    for (int g = 0; g < KN / kGatherRows; ++g) {
                        const int pos = pos0 + kGatherRows * g;
                        tok[g] = pos < p.nk_rows ? f * p.S + sx : -1;
                        if (korder == ORDER_FM) {
                            for (sx += kGatherRows; sx >= p.S; sx -= p.S) ++f;
                        } else if (korder == ORDER_TM_STRICT) {
                            for (f += kGatherRows; f >= p.F; f -= p.F) ++sx;
                        } else if (f == 0) {  // the anchor frame leads the order
                            sx += kGatherRows;
                            if (sx >= p.S && pos + kGatherRows < p.nk_rows)
                                pos_to_coord(korder, pos + kGatherRows, p.F, p.S, f, sx);
                        } else {
                            for (f += kGatherRows; f >= p.F; f -= p.F - 1) ++sx;
                        }
                    }
                }
                if (!(p.test_stall && idx == 0)) {  // the test hook never loads stage 0
                    const char *base = (idx & 1) ? vb : kb;
                    const uint32_t dst = dst_base + s * C::kKVBytes;
#pragma unroll
                    for (int g = 0; g < KN / kGatherRows; ++g) {
                        const int row = r0 + kGatherRows * g;  // swizzle: 16-byte unit ^ row % 8
                        const char *src =
                            base + ((uint32_t)(tok[g] < 0 ? 0 : tok[g]) * (D * 2) + u * 16);
#pragma unroll
                        for (int c = 0; c < D / 64; ++c)
                            cp_async_16(dst + c * C::kKVChunk + row * 128 + ((u ^ (row & 7)) << 4),
                                        src + c * 128, tok[g] < 0 ? 0u : 16u);
                    }
                }
                // the stage's barrier counts this thread once its copies have landed
                if (!(p.test_stall && idx == 0))
                    cp_async_arrive_noinc(smem_u32(&bar->kv_full[s]));
            }
            cp_async_wait_all();  // nothing in flight when the CTA exits
            if (!ok)  // and no arrival still to come: the stages issued last have completed
                for (int idx = (issued > C::kStages ? issued - C::kStages : 0); idx < issued; ++idx)
                    if (!(p.test_stall && idx == 0))
                        mbar_wait_bounded(smem_u32(&bar->kv_full[idx % C::kStages]),
                                          (idx / C::kStages) & 1);
        } else if ((warp == 1 || warp == 3) && lane == 0) {
            // ------------------------------------------------------- MMA issuers
            // TMEM: S (shared by both groups, kTmS) | P0 | P1 (kTmP + 64 g) | O0 | O1 (kTmO + 128 g)
            // Two threads issue the tcgen05.mma, each waiting on its own barriers with no
            // warp-wide votes: warp 1 the S = Q K^T products, warp 3 the O += P V
            // products.  The two streams touch different TMEM columns, and every hazard
            // between them goes through a barrier the softmax groups complete (the S
            // columns are rewritten only after their owner has read them, P only after its
            // P V product is done), so neither issuer waits for the other: while one waits
            // or does its bookkeeping the other keeps the tensor pipe fed.
            const bool s_role = warp == 1;
            constexpr uint32_t idS = idesc_bf16_f32(kBlockM, KN, 0);
            constexpr uint32_t idO = idesc_bf16_f32(kBlockM, D, 1);
            // Descriptors with an empty address field; an operand's start address
            // (>> 4) is added to the low word, offsets inside a tile are constants.
            const uint64_t dK = smem_desc_sw128(0, 16, 1024);
            const uint64_t dV = smem_desc_sw128(0, C::kKVChunk, 1024);
            const uint32_t q_addr = smem_u32(sQ) >> 4, kv_addr = smem_u32(sKV) >> 4;
            bool ok = !s_role || mbar_wait(smem_u32(&bar->q_full), 0, abort_flag);
            tc_fence_after();
            const int total = 2 * it.E;
            // TMA completion on the barrier makes the stage visible to the MMA (both async
            // proxy); no tcgen05 fence is needed after these waits.  Rows gathered with
            // cp.async are generic-proxy writes: the proxy fence after the wait orders them
            // before the MMA's reads.
            auto wait_full = [&](int idx) {
                const bool r = mbar_wait(smem_u32(&bar->kv_full[idx % C::kStages]),
                                         (idx / C::kStages) & 1, abort_flag);
                if (kv_gather) fence_proxy_async_smem();
                return r;
            };
            auto release = [&](int idx) {
                if (idx + C::kStages < total)
                    mma_commit(smem_u32(&bar->kv_empty[idx % C::kStages]));
            };
            // A cursor over the visits of the item: (entry n, group g) for each group
            // whose block visits entry n, entries ascending, group 0 before group 1.  It
            // holds its entry and, already requested, the next one, so that stepping to
            // the next entry waits for no global load.
            struct Cursor {
                int n, g;
                uint32_t e, e1;
            };
            auto last_of_chunk = [](const Cursor &c) { return !(c.g == 0 && (c.e & kEntV1)); };
            auto advance = [&](Cursor &c) {
                if (!last_of_chunk(c)) {
                    c.g = 1;
                    return;
                }
                ++c.n;
                c.e = c.e1;
                // unconditional load from a clamped index: a select on the loaded value
                // would wait for it here (only visit flags are used from it)
                c.e1 = it.raw(min(c.n + 1, it.E - 1));
                c.g = (c.e & kEntV0) ? 0 : 1;  // every entry is visited by some block
            };
            Cursor c;
            c.n = 0;
            c.e = it.E > 0 ? it.raw(0) : 0u;
            c.e1 = it.E > 0 ? it.raw(min(1, it.E - 1)) : 0u;
            c.g = (c.e & kEntV0) ? 0 : 1;
            int k = 0;              // visits done
            int need_chunk = -1;    // last entry whose K (or V) stage was waited for
            int pvn0 = 0, pvn1 = 0;  // P V products issued per group
            // one loop per role, specialised at compile time (less live state each)
            auto run = [&](auto role_tag) {
            constexpr bool kSRole = decltype(role_tag)::value;
            while (ok && c.n < it.E) {
                if constexpr (kSRole) {
                    // S of visit k into the shared S columns, once the owner of visit k-1
                    // has read its S into registers
                    if (k > 0 && !(ok = mbar_wait(smem_u32(&bar->s_free), (k - 1) & 1, abort_flag)))
                        break;
                    tc_fence_after();
                    if (c.n != need_chunk) {
                        if (!(ok = wait_full(2 * c.n))) break;
                        need_chunk = c.n;
                    }
                    const uint64_t a0 = dK + (q_addr + c.g * (C::kQBytes >> 4));
                    const uint64_t b0 =
                        dK + (kv_addr + ((2 * c.n) % C::kStages) * (C::kKVBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + kTmS,
                               a0 + (uint32_t)(((kk >> 2) * C::kQChunk + (kk & 3) * 32) >> 4),
                               b0 + (uint32_t)(((kk >> 2) * C::kKVChunk + (kk & 3) * 32) >> 4),
                               idS, kk > 0 ? 1u : 0u);
                    mma_commit(smem_u32(&bar->s_full[c.g]));
                    if (last_of_chunk(c)) release(2 * c.n);
                    mbar_arrive(smem_u32(&bar->s_issued[k & 3]));
                } else {
                    // O_g += P_g V of visit k, once the group has written P
                    if (c.n != need_chunk) {
                        if (!(ok = wait_full(2 * c.n + 1))) break;
                        need_chunk = c.n;
                    }
                    int &pvn = c.g ? pvn1 : pvn0;
                    ok = mbar_wait(smem_u32(&bar->p_full[c.g]), pvn & 1, abort_flag);
                    // Behind the S of visit k + 2 in the pipe: the S stream is the chain
                    // (each S waits until the previous one was read), and a P V product
                    // issued right after an S runs while that S is being read.
                    // The S of visit m completes phase m / 4 of s_issued[m % 4].  While
                    // this P V is not issued, the S of visit k + 5 cannot be: an S waits
                    // for the previous S to be read, which waits for its group's P
                    // columns, which wait for that group's previous P V; so at most S of
                    // visits up to k + 4 are issued, and the barrier of visit k + 2 is at
                    // most one phase past the one waited for (a parity wait would take a
                    // barrier two phases ahead for one behind).  (After its last S the S
                    // issuer arrives for two more visits.)
                    ok = ok && mbar_wait(smem_u32(&bar->s_issued[(k + 2) & 3]),
                                         ((k + 2) >> 2) & 1, abort_flag);
                    tc_fence_after();
                    if (!ok) break;
                    const uint64_t b0 =
                        dV + (kv_addr + ((2 * c.n + 1) % C::kStages) * (C::kKVBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < KN / 16; ++kk)
                        mma_ts(tmem + kTmO + c.g * 128, tmem + kTmP + c.g * 64 + kk * 8,
                               b0 + (uint32_t)(kk * (2048 >> 4)), idO,
                               (pvn != 0 || kk > 0) ? 1u : 0u);
                    mma_commit(smem_u32(&bar->o_done[c.g]));
                    if (last_of_chunk(c)) release(2 * c.n + 1);
                    ++pvn;
                }
                ++k;
                advance(c);
            }
            };
            if (s_role)
                run(std::true_type{});
            else
                run(std::false_type{});
            if (ok && s_role) {  // the last two P V products wait for no later S
                mbar_arrive(smem_u32(&bar->s_issued[k & 3]));
                mbar_arrive(smem_u32(&bar->s_issued[(k + 1) & 3]));
            }
            if (!ok) {
                // Abort: wait for every MMA this thread issued before TMEM is freed.
                const uint32_t drain = smem_u32(s_role ? &bar->drain[0] : &bar->drain[1]);
                mma_commit(drain);
                mbar_wait_bounded(drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------ softmax warpgroups
        setmaxnreg_inc<kRegsHigh>();
        const int wg = (warp - 4) >> 2, quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + lane_base + kTmS;            // shared by both groups
        const uint32_t tP = tmem + lane_base + kTmP + wg * 64;  // this group's P
        const uint32_t tO = tmem + lane_base + kTmO + wg * 128;
        const int blk = it.b0 + wg;
        const int qpos = blk * kBlockM + row;
        const bool row_valid = qpos < p.nq_rows;
        int type = MASK_DENSE, band = 0, korder = ORDER_FM;
        if (p.mode != 1) {
            const int4 hi = __ldg(p.head_info + it.h);
            type = hi.x;
            band = hi.y;
            korder = hi.z;
        }
        int fq = 0, sq = 0;
        bool q_tok = row_valid;  // false: a position of the padded layout without a token
        if (row_valid && type != MASK_DENSE) {
            if (p.qrow_tokens) {
                const int t = __ldg(p.qrow_tokens + qpos);
                fq = t / p.S;
                sq = t - fq * p.S;
            } else if (korder == ORDER_FM) {
                fq = qpos / p.Sp;
                sq = qpos - fq * p.Sp;
                q_tok = sq < p.S;
            } else {
                q_tok = qpos < p.N;
                if (q_tok) pos_to_coord(korder, qpos, p.F, p.S, fq, sq);
            }
        }
        // Q and O frame-major: each thread copies its own Q row from the row's frame-major
        // token into the 128-byte-swizzled Q tile (the layout the TMA load would give),
        // and O / LSE go back to that token.
        int tok = qpos;
        if (p.qo_fm && row_valid) tok = fq * p.S + sq;
        if (p.qo_fm && korder != ORDER_FM) {
            const uint32_t qs = smem_u32(sQ + wg * C::kQBytes) + row * 128;
            const uint4 *src = static_cast<const uint4 *>(p.q) +
                               ((size_t)it.h * p.nq_rows + (row_valid ? tok : 0)) * (D / 8);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 x = row_valid ? __ldg(src + c * 8 + u) : make_uint4(0, 0, 0, 0);
                    st_shared_v4(qs + c * C::kQChunk + ((u ^ (row & 7)) << 4), x.x, x.y, x.z,
                                 x.w);
                }
            fence_proxy_async_smem();  // generic-proxy stores -> visible to the MMA
            named_bar_sync(1, 256);    // both groups' rows are in place
            if (warp == 4 && lane == 0) mbar_arrive(smem_u32(&bar->q_full));
        }
        const uint32_t vbit = wg ? kEntV1 : kEntV0, fbit = wg ? kEntF1 : kEntF0;
        const float sl2 = p.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        int visit = 0;
        bool ok = true;
        uint32_t e_next = it.E > 0 ? it.raw(0) : 0u;  // prefetched, fixed where used
        for (int n = 0; n < it.E; ++n) {
            const uint32_t e = it.fix(e_next);
            e_next = it.raw(min(n + 1, it.E - 1));  // unconditional: see the MMA cursors
            if (!(e & vbit)) continue;
            ok = __all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&bar->s_full[wg]), visit & 1, abort_flag));
            tc_fence_after();
            if (!ok) break;
            uint32_t r[KN];
#pragma unroll
            for (int j = 0; j < KN / 32; ++j)
                tmem_ld32(tS + j * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[j * 32]));
            const int kc = (int)(e & kEntChunkMask);
            // Tile-aligned traversal: a visited chunk keeps every key; only a chunk that
            // runs past the last token still needs its range mask.
            const bool full = p.aligned ? (kc + 1) * KN <= p.nk_rows : (e & fbit) != 0;
            uint32_t keep[KN / 32];
            if (!full)  // mask computed while the TMEM load is in flight
                keep_mask<KN>(korder, p.aligned ? MASK_DENSE : type, band, p.anchor, p.F, p.S,
                              p.Sp, korder == ORDER_FM ? p.nk_rows : p.N, q_tok, fq, sq,
                              kc * KN, keep);
            tmem_wait_ld();
            // S is in registers: the shared S columns may take the next visit's S
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar->s_free));

            // Boundary tiles drop the keys their rows do not keep; full tiles skip this and
            // share the rest of the code (one copy of the exponential loop, which keeps
            // the loop small enough to stay in the instruction cache with the MMA issuer).
            if (!full) {
#pragma unroll
                for (int c = 0; c < KN; ++c)
                    if (!((keep[c >> 5] >> (c & 31)) & 1u)) r[c] = kNegInfBits;
            }
            // exact row maximum of the tile, in the exp2 domain
            auto tile_max = [&]() {
                float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
                for (int c = 0; c < KN; c += 8) {
                    a0 = fmax3(a0, __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
                    a1 = fmax3(a1, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
                    a2 = fmax3(a2, __uint_as_float(r[c + 4]), __uint_as_float(r[c + 5]));
                    a3 = fmax3(a3, __uint_as_float(r[c + 6]), __uint_as_float(r[c + 7]));
                }
                return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * sl2;
            };
            // The reference maximum m_used is the exact maximum of the row's first visited
            // tile and is kept afterwards: softmax is the same for any reference, so later
            // tiles need no maximum pass.  A tile whose P sum exceeds kTileSumLimit (a
            // value far above the reference, or an overflow) is done a second time with its
            // exact maximum as the new reference, after O and the running sum are rescaled;
            // every P then stays below the limit.
            if (m_used == -INFINITY) m_used = tile_max();
            // O += P V of the previous visit reads the P columns this tile writes: it must
            // be complete first (in steady state it finished long ago)
            if (visit > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar->o_done[wg]),
                                                       (visit - 1) & 1, abort_flag));
                tc_fence_after();
                if (!ok) break;
            }
            float lt;
#pragma unroll 1
            for (int attempt = 0;; ++attempt) {
                // P = 2^(x sl2 - m_used) of every column, packed to bf16 into this group's
                // P columns; lt = the tile's sum of P
                const float ms = (m_used == -INFINITY) ? 0.f : m_used;
                const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-ms, -ms);
                float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < KN / 32; ++j) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c2 = 0; c2 < 16; ++c2) {
                        const int c = j * 32 + 2 * c2;
                        const float2 x = ffma2(
                            make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sc2, nm2);
                        const float2 ev = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                        if (c2 & 1)
                            s1 = fadd2(s1, ev);
                        else
                            s0 = fadd2(s0, ev);
                        pk[c2] = pack_bf16x2_int(ev.x, ev.y);
                    }
                    tmem_st16(tP + j * 16, pk);
                }
                lt = (s0.x + s0.y) + (s1.x + s1.y);
                const bool need = !(lt <= kTileSumLimit);
                if (attempt > 0 || !__any_sync(0xffffffffu, need)) break;
                // rare: O (complete up to the previous visit, see above) is rescaled to the
                // tile's exact maximum and the tile is done again
                const float m_new = need ? fmaxf(m_used, tile_max()) : m_used;
                const float fac = need ? fast_exp2(m_used - m_new) : 1.f;
                l *= fac;
                m_used = m_new;
#pragma unroll 1
                for (int j = 0; j < D / 32; ++j) {
                    uint32_t o[32];
                    tmem_ld32(tO + j * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * fac);
                    tmem_st32(tO + j * 32, o);
                }
                tmem_wait_st();
            }
            l += lt;
            if (!ok) break;
            tmem_wait_st();
            // every lane's P is in TMEM (wait::st + fence); after the warp-level sync one
            // arrival per warp hands the tile to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar->p_full[wg]));
            ++visit;
        }
        // ----------------------------------------------------------------- epilogue
        if (ok && visit > 0) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&bar->o_done[wg]), (visit - 1) & 1, abort_flag));
            tc_fence_after();
        }
        // a key-range part (fp32 output only) leaves its rows unnormalised, with their
        // reference maximum and sum, for the merge
        const bool split = OUT_F32 && p.part_o != nullptr;
        if (ok && (blk < p.n_qblk)) {
            const float inv = split ? 1.f : (l > 0.f ? 1.f / l : 0.f);
            const size_t prow =
                split ? (size_t)(blockIdx.x % p.ksplit) * p.heads * p.nq_rows : (size_t)0;
            const size_t orow = (prow + (size_t)it.h * p.nq_rows + (row_valid ? tok : 0)) * D;
#pragma unroll 1
            for (int j = 0; j < D / 32; ++j) {
                uint32_t o[32];
                if (visit > 0) {
                    tmem_ld32(tO + j * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = 0u;
                }
                if (row_valid) {
                    if (OUT_F32) {
                        float4 *dst = reinterpret_cast<float4 *>(
                            (split ? p.part_o : static_cast<float *>(p.o)) + orow + j * 32);
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            dst[c] = make_float4(__uint_as_float(o[4 * c]) * inv,
                                                 __uint_as_float(o[4 * c + 1]) * inv,
                                                 __uint_as_float(o[4 * c + 2]) * inv,
                                                 __uint_as_float(o[4 * c + 3]) * inv);
                    } else {
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) + orow +
                                                               j * 32);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            dst[c] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * c]) * inv,
                                                            __uint_as_float(o[8 * c + 1]) * inv),
                                                pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv,
                                                            __uint_as_float(o[8 * c + 3]) * inv),
                                                pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv,
                                                            __uint_as_float(o[8 * c + 5]) * inv),
                                                pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv,
                                                            __uint_as_float(o[8 * c + 7]) * inv));
                    }
                }
            }
            if (row_valid && split)
                p.part_ml[prow + (size_t)it.h * p.nq_rows + tok] = make_float2(m_used, l);
            else if (row_valid && p.lse)
                p.lse[(size_t)it.h * p.nq_rows + tok] =
                    l > 0.f ? (m_used + log2f(l)) * 0.6931471805599453f : -INFINITY;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && bar->abort && p.status) atomicExch(p.status, (int32_t)SVGA_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// [heads, rows, d] bf16, box = 64 columns x box_rows rows x 1 head, 128-byte swizzle.
// ============================================================================
// The pair kernel (SVGA_FLAG_CTA_PAIR): a work item (two 128-row query blocks) runs on a
// CTA pair over two SMs.  Each tcgen05.mma covers M = 256 rows (both blocks); CTA r
// holds block r's Q rows, S and O, and half of every K chunk (keys r*64 .. r*64+63) and
// of every V chunk (head-dim columns r*64 .. r*64+63), so each SM loads half the K/V
// bytes the one-CTA kernel loads per item.  The TMEM this frees (one block per CTA)
// holds two S tiles, so the S of a visit is computed while the softmax works on the
// previous one.
//   * TMEM per CTA: S0 | S1 (128 columns each) | P0 | P1 (64 each, bf16 pairs) | O (128);
//     visit k uses S and P buffer k % 2;
//   * warp 0: TMA producer (own Q rows, own halves of K / V) into 16 KB stages; a
//     stage's copies complete on this CTA's barrier;
//   * rank 0: warp 1 issues the S products, warp 2 the P V products (the issuing warps
//     slow the softmax warps that share their SM sub-partition, so they sit on two
//     different ones).  Rank 1, warp 1: forwards its Q and stage completions to rank 0
//     (one remote arrival each);
//   * warps 4-7 and 8-11: two softmax groups of whole rows (TMEM lane = row); group g
//     takes the visits k with k % 2 == g, and the groups pass each row's reference
//     maximum from visit to visit;
//   * every wait is bounded; an abort stops every role of the CTA, drains its copies
//     and (rank 0) its MMAs, and the pair meets at a cluster barrier before TMEM is
//     released.
// Arrivals on the peer's barriers use the default (CTA-scope) release: what they hand
// over is tensor memory the caller completed and fenced, or copies complete on the
// caller's own barrier.  A cluster-scope release there cost a memory barrier per
// hand-off and made the kernel 40 % slower.
namespace pair {

constexpr int kThreads = 384;
constexpr int kD = 128, kKN = 128;
constexpr int kQBytes = 128 * kD * 2;        // the CTA's 128 Q rows
constexpr int kQChunk = 128 * 64 * 2;         // one 64-column half of the Q rows
constexpr int kStageBytes = 16384;            // a K half (64 keys x 128) or V half (128 x 64)
constexpr int kKHalfChunk = 64 * 64 * 2;      // 64 keys x 64 columns of a K half
constexpr int kStages = 10;
constexpr uint32_t kPS = 0, kPP = 256, kPO = 384;  // TMEM columns: S0|S1, P0|P1, O
constexpr int kRows = 128;                    // rows of the CTA's block
constexpr float kRaiseLog2 = 8.f;             // a tile this far above the reference raises it

struct Bars {
    uint64_t q_full;              // own Q rows landed (TMA bytes, or the gather's arrival)
    uint64_t peer_q;              // rank 0: rank 1's Q landed
    uint64_t kv_full[kStages];    // own half of the stage landed
    uint64_t peer_full[kStages];  // rank 0: rank 1's half landed
    uint64_t kv_empty[kStages];   // the MMAs reading the stage are done (both CTAs)
    uint64_t s_full[2];           // S buffer b computed (both CTAs)
    uint64_t s_free[2];           // rank 0: S buffer b read by its group's 8 warps (2 CTAs)
    uint64_t p_full[2];           // rank 0: P buffer b written by its group's 8 warps
    uint64_t o_done[2];           // the P V reading P buffer b is done (both CTAs)
    uint64_t o_final;             // every P V of the item is done (both CTAs)
    uint64_t ref_bar[2];          // the reference after visit k (k % 2 = b) is in m_ref
    uint64_t p_local[2];          // this CTA's group wrote P buffer b
    uint64_t fin_bar;             // both groups' sums are in fin_m / fin_l
    uint64_t drain[2];            // rank 0's issuers, after an abort
    uint32_t tmem_base;
    int abort;
    float m_ref[kRows];           // each row's reference maximum (exp2 domain)
    float fin_m[2][kRows];        // per group: the reference of its sum
    float fin_l[2][kRows];        // per group: its sum of P
};
constexpr int kSmemData = kQBytes + kStages * kStageBytes;
constexpr int kSmemLaunch = kSmemData + (int)sizeof(Bars) + 1024;

}  // namespace pair

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::kThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK64,
                         const __grid_constant__ CUtensorMap tmV, const KParams p)
{
    using namespace pair;
    constexpr int D = kD, KN = kKN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem;
    uint8_t *sKV = smem + kQBytes;
    Bars *bar = reinterpret_cast<Bars *>(smem + kSmemData);
    volatile int *abort_flag = &bar->abort;

    const uint32_t rank = cluster_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = blockIdx.x >> 1;
    // both CTAs of the pair take the same decisions here: same item, same plan
    if (plan_item_of_slot(p, slot) >= p.n_items) return;  // the last group ran out
    if (p.check_plan && !plan_matches(p, KN, slot)) {
        if (threadIdx.x == 0 && rank == 0 && p.status)
            atomicCAS(p.status, 0, (int32_t)SVGA_ERR_INVALID_ARG);
        return;
    }
    const Item it = make_item(p, KN, slot, 0);
    if (!item_fits_pair(it)) return;  // both CTAs decide alike: the one-CTA kernel runs it
    const int4 hinfo = __ldg(p.head_info + it.h);
    const bool q_tma = !p.qo_fm || hinfo.z == ORDER_FM;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar->q_full), 1);
        mbar_init(smem_u32(&bar->peer_q), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bar->kv_full[s]), 1);
            mbar_init(smem_u32(&bar->peer_full[s]), 1);
            mbar_init(smem_u32(&bar->kv_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bar->s_full[b]), 1);
            mbar_init(smem_u32(&bar->s_free[b]), 8);
            mbar_init(smem_u32(&bar->p_full[b]), 8);
            mbar_init(smem_u32(&bar->ref_bar[b]), 4);
            mbar_init(smem_u32(&bar->p_local[b]), 4);
            mbar_init(smem_u32(&bar->o_done[b]), 1);
            mbar_init(smem_u32(&bar->drain[b]), 1);
        }
        mbar_init(smem_u32(&bar->o_final), 1);
        mbar_init(smem_u32(&bar->fin_bar), 8);
        bar->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&bar->tmem_base), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    const int total = 2 * it.E;  // stages: K then V of each entry
    const int blk = it.b0 + (int)rank;

    if (warp < 4) {
        setmaxnreg_dec<kRegsLow>();
        if (warp == 0 && lane == 0) {
            // -------------------------------------------------------- TMA producer
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK64);
            prefetch_tmap(&tmV);
            const uint32_t qf = smem_u32(&bar->q_full);
            if (q_tma) {
                // a block past the last one reads zeros (the box is out of range)
                mbar_arrive_expect_tx(qf, kQBytes);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(smem_u32(sQ + c * kQChunk), &tmQ, qf, 64 * c, blk * kBlockM, it.h);
            }
            int issued = 0;
            bool ok = true;
            uint32_t e_nxt = it.E > 0 ? it.raw(0) : 0u;
            for (int n = 0; n < it.E && ok; ++n) {
                const int kc = (int)(e_nxt & kEntChunkMask);
                e_nxt = it.raw(min(n + 1, it.E - 1));
                for (int t = 0; t < 2; ++t) {
                    const int idx = 2 * n + t, s = idx % kStages, round = idx / kStages;
                    if (round > 0 &&
                        !mbar_wait(smem_u32(&bar->kv_empty[s]), (round - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (p.test_stall && idx == 0) {  // nothing ever completes this stage
                        issued = idx + 1;
                        continue;
                    }
                    const uint32_t fb = smem_u32(&bar->kv_full[s]);
                    const uint32_t dst = smem_u32(sKV + s * kStageBytes);
                    const int krow = kc * KN + (int)rank * 64;
                    if (t == 0 && krow >= p.nk_rows) {
                        // This half of the last chunk holds no key: no copy is issued, the
                        // stage keeps stale rows, and every key of it is masked (the last
                        // chunk is never a full one), so its P is zero; its V rows are
                        // zeros, read by a box that starts inside the tensor.
                        mbar_arrive(fb);
                    } else if (t == 0) {  // keys kc*128 + rank*64 .. +63, both column halves
                        mbar_arrive_expect_tx(fb, kStageBytes);
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_3d(dst + c * kKHalfChunk, &tmK64, fb, 64 * c, krow, it.h);
                    } else {  // all 128 keys, columns rank*64 .. +63
                        mbar_arrive_expect_tx(fb, kStageBytes);
                        tma_load_3d(dst, &tmV, fb, 64 * (int)rank, kc * KN, it.h);
                    }
                    issued = idx + 1;
                }
            }
            {  // every copy issued lands before the CTA can exit, whichever role aborts
                if (q_tma) mbar_wait_bounded(qf, 0);
                for (int idx = (issued > kStages ? issued - kStages : 0); idx < issued; ++idx)
                    if (!(p.test_stall && idx == 0))
                        mbar_wait_bounded(smem_u32(&bar->kv_full[idx % kStages]),
                                          (idx / kStages) & 1);
            }
        } else if (warp == 1 && lane == 0 && rank == 1) {
            // ------------------------------------ rank 1: completions to rank 0
            const uint32_t peer_q = cluster_addr(smem_u32(&bar->peer_q), 0);
            if (mbar_wait(smem_u32(&bar->q_full), 0, abort_flag)) {
                mbar_arrive_cluster(peer_q);
                for (int idx = 0; idx < total; ++idx) {
                    const int s = idx % kStages;
                    if (!mbar_wait(smem_u32(&bar->kv_full[s]), (idx / kStages) & 1, abort_flag))
                        break;
                    mbar_arrive_cluster(cluster_addr(smem_u32(&bar->peer_full[s]), 0));
                }
            }
        } else if ((warp == 1 || warp == 2) && lane == 0 && rank == 0) {
            // ------------------------------------------------ rank 0: MMA issuers
            const bool s_role = warp == 1;
            constexpr uint32_t idS = idesc_bf16_f32(256, KN, 0);
            constexpr uint32_t idO = idesc_bf16_f32(256, D, 1);
            const uint64_t dK = smem_desc_sw128(0, 16, 1024);
            const uint64_t dV = smem_desc_sw128(0, 16, 1024);
            const uint32_t q_addr = smem_u32(sQ) >> 4, kv_addr = smem_u32(sKV) >> 4;
            bool ok = true;
            if (s_role)
                ok = mbar_wait(smem_u32(&bar->q_full), 0, abort_flag) &&
                     mbar_wait(smem_u32(&bar->peer_q), 0, abort_flag);
            tc_fence_after();
            // both halves of stage idx are in place
            auto wait_full = [&](int idx) {
                const int s = idx % kStages;
                const uint32_t ph = (idx / kStages) & 1;
                return mbar_wait(smem_u32(&bar->kv_full[s]), ph, abort_flag) &&
                       mbar_wait(smem_u32(&bar->peer_full[s]), ph, abort_flag);
            };
            auto release = [&](int idx) {
                if (idx + kStages < total) mma_commit_pair(smem_u32(&bar->kv_empty[idx % kStages]));
            };
            for (int k = 0; k < it.E && ok; ++k) {
                const int b = k & 1;
                if (s_role) {
                    // S of visit k into S buffer b, once visit k-2's S was read there
                    if (k >= 2 &&
                        !(ok = mbar_wait(smem_u32(&bar->s_free[b]), ((k >> 1) - 1) & 1, abort_flag)))
                        break;
                    if (!(ok = wait_full(2 * k))) break;
                    tc_fence_after();
                    const uint64_t a0 = dK + q_addr;
                    const uint64_t b0 = dK + (kv_addr + ((2 * k) % kStages) * (kStageBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss_pair(tmem + kPS + b * 128,
                                    a0 + (uint32_t)(((kk >> 2) * kQChunk + (kk & 3) * 32) >> 4),
                                    b0 + (uint32_t)(((kk >> 2) * kKHalfChunk + (kk & 3) * 32) >> 4),
                                    idS, kk > 0 ? 1u : 0u);
                    mma_commit_pair(smem_u32(&bar->s_full[b]));
                    release(2 * k);
                } else {
                    // O += P V of visit k, once both CTAs wrote P buffer b
                    if (!(ok = mbar_wait(smem_u32(&bar->p_full[b]), (k >> 1) & 1, abort_flag)))
                        break;
                    if (!(ok = wait_full(2 * k + 1))) break;
                    tc_fence_after();
                    const uint64_t b0 =
                        dV + (kv_addr + ((2 * k + 1) % kStages) * (kStageBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < KN / 16; ++kk)
                        mma_ts_pair(tmem + kPO, tmem + kPP + b * 64 + kk * 8,
                                    b0 + (uint32_t)((kk * 2048) >> 4), idO,
                                    (k > 0 || kk > 0) ? 1u : 0u);
                    mma_commit_pair(smem_u32(&bar->o_done[b]));
                    release(2 * k + 1);
                }
            }
            // the epilogue's signal: every P V of the item is done
            if (ok && !s_role && it.E > 0) mma_commit_pair(smem_u32(&bar->o_final));
            if (!ok) {  // every MMA this thread issued is done before TMEM is released
                const uint32_t drain = smem_u32(s_role ? &bar->drain[0] : &bar->drain[1]);
                mma_commit_pair_self(drain);
                mbar_wait_bounded(drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------ softmax groups
        // Group g (warps 4-7 or 8-11) takes the visits k with k % 2 == g, whole rows
        // (thread = TMEM lane = row of this CTA's block).  The groups run half a visit
        // apart, so the exponentials of one overlap the waits of the other.  They share
        // each row's reference maximum: the group of visit k reads the reference visit
        // k-1 left, raises it when the tile's maximum lies more than kRaiseLog2 above it
        // (the row's first kept keys set it), and passes it on.  Every P is then at most
        // 2^kRaiseLog2.  Each group keeps its own running sum; the epilogue adds them.
        setmaxnreg_inc<kRegsHigh>();
        const int g = (warp - 4) >> 2, quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const uint32_t tO = tmem + lane_base + kPO;
        const int qpos = blk * kBlockM + row;
        const bool row_valid = qpos < p.nq_rows;
        const int type = hinfo.x, band = hinfo.y, korder = hinfo.z;
        int fq = 0, sq = 0;
        bool q_tok = row_valid;  // false: a position of the padded layout without a token
        if (row_valid) {
            if (korder == ORDER_FM) {
                fq = qpos / p.Sp;
                sq = qpos - fq * p.Sp;
                q_tok = sq < p.S;
            } else {
                q_tok = qpos < p.N;
                if (q_tok) pos_to_coord(korder, qpos, p.F, p.S, fq, sq);
            }
        }
        int tok = qpos;
        if (p.qo_fm && row_valid) tok = fq * p.S + sq;
        if (!q_tma) {
            // Q rows gathered from their frame-major tokens: group g copies head-dim
            // columns g*64 .. g*64+63 of its row into the swizzled Q tile
            const uint32_t qs = smem_u32(sQ + g * kQChunk) + row * 128;
            const uint4 *src = static_cast<const uint4 *>(p.q) +
                               ((size_t)it.h * p.nq_rows + (row_valid ? tok : 0)) * (D / 8) + g * 8;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 x = row_valid ? __ldg(src + u) : make_uint4(0, 0, 0, 0);
                st_shared_v4(qs + ((u ^ (row & 7)) << 4), x.x, x.y, x.z, x.w);
            }
            fence_proxy_async_smem();  // generic-proxy stores -> visible to the MMA
            named_bar_sync(1, 256);    // every row of the tile is in place
            if (warp == 4 && lane == 0) mbar_arrive(smem_u32(&bar->q_full));
        }
        const uint32_t vbit = rank ? kEntV1 : kEntV0, fbit = rank ? kEntF1 : kEntF0;
        const uint32_t s_free0 = cluster_addr(smem_u32(&bar->s_free[0]), 0);
        const uint32_t p_full0 = cluster_addr(smem_u32(&bar->p_full[0]), 0);
        const float sl2 = p.scale_log2;
        float m_seen = -INFINITY, l = 0.f;  // this group's sum, in units of 2^m_seen
        bool ok = true;
        // all lanes wait (bounded) for a phase; tensor-memory reads may follow
        auto wait_all = [&](uint32_t b_addr, uint32_t parity) {
            const bool w = __all_sync(0xffffffffu, mbar_wait(b_addr, parity, abort_flag));
            tc_fence_after();
            return w;
        };
        uint32_t r[KN];
        auto tile_max = [&]() {
            float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
            for (int c = 0; c < KN; c += 8) {
                a0 = fmax3(a0, __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
                a1 = fmax3(a1, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
                a2 = fmax3(a2, __uint_as_float(r[c + 4]), __uint_as_float(r[c + 5]));
                a3 = fmax3(a3, __uint_as_float(r[c + 6]), __uint_as_float(r[c + 7]));
            }
            return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * sl2;
        };
        uint32_t e_next = g < it.E ? it.raw(g) : 0u;  // prefetched, fixed where used
        for (int k = g; k < it.E; k += 2) {
            const int b = k & 1;  // this group's S and P buffers
            const uint32_t e = it.fix(e_next);
            e_next = it.raw(min(k + 2, it.E - 1));
            const bool visits = (e & vbit) != 0;  // the same for the whole CTA
            if (!(ok = wait_all(smem_u32(&bar->s_full[b]), (k >> 1) & 1))) break;
            const int kc = (int)(e & kEntChunkMask);
            const bool full = p.aligned ? (kc + 1) * KN <= p.nk_rows : (e & fbit) != 0;
            uint32_t keep[KN / 32];
            if (visits) {
                const uint32_t tS = tmem + lane_base + kPS + b * 128;
#pragma unroll
                for (int j = 0; j < KN / 32; ++j)
                    tmem_ld32(tS + j * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[j * 32]));
                if (!full)  // mask computed while the TMEM load is in flight
                    keep_mask<KN>(korder, p.aligned ? MASK_DENSE : type, band, p.anchor, p.F,
                                  p.S, p.Sp, korder == ORDER_FM ? p.nk_rows : p.N, q_tok, fq,
                                  sq, kc * KN, keep);
                tmem_wait_ld();
            }
            // S is in registers: S buffer b may take visit k+2's S
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(s_free0 + b * 8);
            if (visits && !full) {
#pragma unroll
                for (int c = 0; c < KN; ++c)
                    if (!((keep[c >> 5] >> (c & 31)) & 1u)) r[c] = kNegInfBits;
            }
            float m_cur = -INFINITY;  // the reference visit k-1 left
            if (k >= 1) {
                if (!(ok = wait_all(smem_u32(&bar->ref_bar[b ^ 1]), ((k - 1) >> 1) & 1))) break;
                m_cur = bar->m_ref[row];
            }
            if (m_cur != m_seen) {  // raised by the other group: this group's sum follows
                l *= fast_exp2(m_seen - m_cur);
                m_seen = m_cur;
            }
            float m_new = m_cur;
            if (visits) {
                const float t = tile_max();
                if (t > m_cur + kRaiseLog2) m_new = t;
            }
            // A raised reference rescales O, which holds the P V of visits up to k-1 in
            // units of 2^m_cur, once the last of them is done.  A row whose reference is
            // set for the first time has a zero O row and needs none.  (Rare.)  A warp
            // that raises first waits for the other group's P of visit k-1, which that
            // group wrote after it saw the P V of visit k-3 done; and it passes the
            // reference on only then, so that group cannot write the P of visit k+1 in
            // the meantime.  Both barriers waited for here are thus one phase from the
            // phase they are at.
            const bool raise = m_new > m_cur && m_cur != -INFINITY;
            const bool any_raise = __any_sync(0xffffffffu, raise);
            if (any_raise &&
                !(ok = wait_all(smem_u32(&bar->p_local[b ^ 1]), ((k - 1) >> 1) & 1)))
                break;
            bar->m_ref[row] = m_new;
            __threadfence_block();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar->ref_bar[b]));
            if (any_raise) {
                if (!(ok = wait_all(smem_u32(&bar->o_done[b ^ 1]), ((k - 1) >> 1) & 1))) break;
                const float fac = raise ? fast_exp2(m_cur - m_new) : 1.f;
#pragma unroll 1
                for (int j = 0; j < D / 32; ++j) {
                    uint32_t o[32];
                    tmem_ld32(tO + j * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * fac);
                    tmem_st32(tO + j * 32, o);
                }
                tmem_wait_st();
            }
            if (m_new != m_seen) {
                l *= fast_exp2(m_seen - m_new);
                m_seen = m_new;
            }
            // P buffer b: the P V of visit k-2 read it
            if (k >= 2 && !(ok = wait_all(smem_u32(&bar->o_done[b]), ((k - 2) >> 1) & 1))) break;
            const uint32_t tP = tmem + lane_base + kPP + b * 64;
            if (!visits) {  // the other block's chunk: this block adds nothing
                uint32_t z[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) z[c] = 0u;
                tmem_st32(tP, z);
                tmem_st32(tP + 32, z);
            } else {
                // P = 2^(x sl2 - m_new) of every column, packed to bf16 into P buffer b
                const float ms = (m_new == -INFINITY) ? 0.f : m_new;
                const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-ms, -ms);
                float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < KN / 32; ++j) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c2 = 0; c2 < 16; ++c2) {
                        const int c = j * 32 + 2 * c2;
                        const float2 x = ffma2(
                            make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sc2, nm2);
                        const float2 ev = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                        if (c2 & 1)
                            s1 = fadd2(s1, ev);
                        else
                            s0 = fadd2(s0, ev);
                        pk[c2] = pack_bf16x2_int(ev.x, ev.y);
                    }
                    tmem_st16(tP + j * 16, pk);
                }
                l += (s0.x + s0.y) + (s1.x + s1.y);
            }
            tmem_wait_st();
            // this warp's P is in TMEM; one arrival per warp on rank 0's barrier, and one
            // on this CTA's
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_cluster(p_full0 + b * 8);
                mbar_arrive(smem_u32(&bar->p_local[b]));
            }
        }
        // ----------------------------------------------------------------- epilogue
        // every P V is done (one commit after the last); the groups then add their sums
        // under the final reference, the larger of theirs (references only rise)
        if (ok && it.E > 0) ok = wait_all(smem_u32(&bar->o_final), 0);
        if (ok) {
            bar->fin_m[g][row] = m_seen;
            bar->fin_l[g][row] = l;
            __threadfence_block();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar->fin_bar));
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar->fin_bar), 0, abort_flag));
        }
        if (ok && blk < p.n_qblk) {
            const float m0 = bar->fin_m[0][row], m1 = bar->fin_m[1][row];
            const float m_fin = fmaxf(m0, m1);
            const float lt = m_fin == -INFINITY
                                 ? 0.f
                                 : bar->fin_l[0][row] * fast_exp2(m0 - m_fin) +
                                       bar->fin_l[1][row] * fast_exp2(m1 - m_fin);
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const size_t orow = ((size_t)it.h * p.nq_rows + (row_valid ? tok : 0)) * D + g * 64;
#pragma unroll 1
            for (int j = 0; j < 2; ++j) {
                uint32_t o[32];
                if (it.E > 0) {
                    tmem_ld32(tO + g * 64 + j * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = 0u;
                }
                if (row_valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) + orow +
                                                           j * 32);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        dst[c] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * c]) * inv,
                                                        __uint_as_float(o[8 * c + 1]) * inv),
                                            pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv,
                                                        __uint_as_float(o[8 * c + 3]) * inv),
                                            pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv,
                                                        __uint_as_float(o[8 * c + 5]) * inv),
                                            pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv,
                                                        __uint_as_float(o[8 * c + 7]) * inv));
                }
            }
            if (row_valid && g == 0 && p.lse)
                p.lse[(size_t)it.h * p.nq_rows + tok] =
                    lt > 0.f ? (m_fin + log2f(lt)) * 0.6931471805599453f : -INFINITY;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && bar->abort && p.status) atomicExch(p.status, (int32_t)SVGA_ERR_TIMEOUT);
    cluster_sync_all();  // no MMA of the pair and no remote arrival is still in flight
    if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

bool make_tmap(CUtensorMap *m, const void *base, int heads, int rows, int d, int box_rows)
{
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KN, bool OUT_F32>
svga_status launch_t(const AttnLaunch &a, const KParams &kp, cudaStream_t st)
{
    using C = Cfg<D, KN>;
    auto kfn = attn_fwd_kernel<D, KN, OUT_F32>;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kfn) != cudaSuccess) {
        set_error("cudaFuncGetAttributes failed: %s", cudaGetErrorString(cudaGetLastError()));
        return SVGA_ERR_CUDA;
    }
    if (fa.numRegs < kRegsLaunch) {
        // the setmaxnreg split assumes the CTA is launched with kRegsLaunch registers/thread
        set_error("attention kernel built with %d registers/thread, the register split needs %d",
                  fa.numRegs, kRegsLaunch);
        return SVGA_ERR_UNSUPPORTED;
    }
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, a.q, a.heads, a.nq_rows, D, kBlockM) ||
        !make_tmap(&tk, a.k, a.heads, a.nk_rows, D, KN) ||
        !make_tmap(&tv, a.v, a.heads, a.nk_rows, D, KN)) {
        set_error("cuTensorMapEncodeTiled failed (driver entry point or arguments)");
        return SVGA_ERR_CUDA;
    }
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemLaunch) !=
        cudaSuccess) {
        set_error("cudaFuncSetAttribute(max dynamic shared memory) failed");
        return SVGA_ERR_CUDA;
    }
    const int groups = a.mode == 0 ? (a.n_items + kp.num_parts - 1) / kp.num_parts : a.n_items;
    const int grid = groups * kp.ksplit;
    if (grid > 0) kfn<<<grid, kThreads, C::kSmemLaunch, st>>>(tq, tk, tv, kp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("attention launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    return SVGA_OK;
}

// The pair kernel: plan mode, head_dim 128, 128-key chunks, bf16 output, K and V in
// each head's order.  Two CTAs (one cluster) per work item.
svga_status launch_pair(const AttnLaunch &a, const KParams &kp, cudaStream_t st)
{
    constexpr int D = pair::kD;
    auto kfn = attn_fwd_pair_kernel;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kfn) != cudaSuccess) {
        set_error("cudaFuncGetAttributes failed: %s", cudaGetErrorString(cudaGetLastError()));
        return SVGA_ERR_CUDA;
    }
    if (fa.numRegs < kRegsLaunch) {
        set_error("pair attention kernel built with %d registers/thread, the register split "
                  "needs %d",
                  fa.numRegs, kRegsLaunch);
        return SVGA_ERR_UNSUPPORTED;
    }
    CUtensorMap tq, tk64, tv;
    if (!make_tmap(&tq, a.q, a.heads, a.nq_rows, D, kBlockM) ||
        !make_tmap(&tk64, a.k, a.heads, a.nk_rows, D, 64) ||
        !make_tmap(&tv, a.v, a.heads, a.nk_rows, D, pair::kKN)) {
        set_error("cuTensorMapEncodeTiled failed (driver entry point or arguments)");
        return SVGA_ERR_CUDA;
    }
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pair::kSmemLaunch) != cudaSuccess) {
        set_error("cudaFuncSetAttribute(max dynamic shared memory) failed");
        return SVGA_ERR_CUDA;
    }
    const int groups = (a.n_items + kp.num_parts - 1) / kp.num_parts;
    if (groups > 0)
        kfn<<<2 * groups, pair::kThreads, pair::kSmemLaunch, st>>>(tq, tk64, tv, kp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("pair attention launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    return SVGA_OK;
}

// One thread per 4 output columns of a row: the parts' maxima give the common scale
// 2^(m_r - m), the weighted sums add in part order (deterministic), and the row is
// divided by the weighted total.  A part that saw no key of the row has l = 0 and adds
// nothing.
__global__ void __launch_bounds__(256) merge_parts_kernel(const float4 *__restrict__ part_o,
                                                          const float2 *__restrict__ part_ml,
                                                          int ksplit, size_t rows, int d4,
                                                          float4 *__restrict__ o)
{
    const size_t n = rows * d4;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / d4;
        float m = -INFINITY;
        for (int r = 0; r < ksplit; ++r) {
            const float2 ml = __ldg(part_ml + r * rows + row);
            if (ml.y > 0.f) m = fmaxf(m, ml.x);
        }
        float l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < ksplit; ++r) {
            const float2 ml = __ldg(part_ml + r * rows + row);
            if (!(ml.y > 0.f)) continue;
            const float w = exp2f(ml.x - m);
            const float4 x = __ldg(part_o + r * n + i);
            l += w * ml.y;
            acc.x += w * x.x;
            acc.y += w * x.y;
            acc.z += w * x.z;
            acc.w += w * x.w;
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
        o[i] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
}

}  // namespace

svga_status merge_attention_parts(const AttnLaunch &a, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (a.ksplit <= 1) return SVGA_OK;
    const size_t rows = (size_t)a.heads * a.nq_rows;
    const int d4 = a.d / 4;
    const size_t n = rows * d4;
    const int blocks = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
    if (blocks > 0)
        merge_parts_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4 *>(a.part_o),
                                                   reinterpret_cast<const float2 *>(a.part_ml),
                                                   a.ksplit, rows, d4,
                                                   static_cast<float4 *>(a.o));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("attention part merge launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    return SVGA_OK;
}

svga_status launch_attention(const AttnLaunch &a, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    KParams kp{};
    kp.heads = a.heads;
    kp.nq_rows = a.nq_rows;
    kp.nk_rows = a.nk_rows;
    kp.F = a.F;
    kp.S = a.S;
    kp.N = a.N > 0 ? a.N : a.nk_rows;  // without a padded layout every row is a token
    kp.Sp = a.Sp > 0 ? a.Sp : a.S;
    kp.anchor = a.anchor;
    kp.scale_log2 = a.scale * kLog2e;
    kp.mode = a.mode;
    kp.naive = a.naive;
    kp.aligned = a.aligned;
    kp.n_items = a.n_items;
    kp.part = a.part;
    kp.num_parts = a.num_parts > 0 ? a.num_parts : 1;
    kp.test_stall = a.test_stall;
    kp.qo_fm = a.qo_fm;
    kp.kv_fm = a.kv_fm;
    kp.q = a.q;
    kp.k = a.k;
    kp.v = a.v;
    kp.n_qblk = (a.nq_rows + kBlockM - 1) / kBlockM;
    kp.n_pairs = (kp.n_qblk + 1) / 2;
    kp.n_kc = (a.nk_rows + a.kn - 1) / a.kn;
    kp.check_plan = a.check_plan;
    kp.tile_q = a.tile_q;
    kp.tile_k = a.tile_k;
    if (a.mode == 0) {
        const char *plan = static_cast<const char *>(a.plan);
        kp.hdr = reinterpret_cast<const PlanHeader *>(plan);
        kp.head_info = reinterpret_cast<const int4 *>(plan + sizeof(PlanHeader));
        kp.items = kp.head_info + a.heads;
        // entries start after header + head_info + items, 256-byte aligned
        const size_t hdr =
            align_up(sizeof(PlanHeader) + sizeof(int4) * ((size_t)a.heads + a.n_items), 256);
        kp.entries = reinterpret_cast<const uint32_t *>(plan + hdr);
    } else {
        kp.hdr = nullptr;
        kp.head_info = nullptr;  // dense: no head info is read
        kp.items = nullptr;
        kp.entries = nullptr;
    }
    kp.qrow_tokens = a.qrow_tokens;
    kp.o = a.o;
    kp.lse = a.lse;
    kp.status = a.status;
    const bool split = a.ksplit > 1;
    if (split && (!a.out_f32 || !a.part_o || !a.part_ml)) {
        set_error("a key-range split needs fp32 output and part buffers");
        return SVGA_ERR_INVALID_ARG;
    }
    kp.ksplit = split ? a.ksplit : 1;
    kp.part_o = split ? a.part_o : nullptr;
    kp.part_ml = split ? reinterpret_cast<float2 *>(a.part_ml) : nullptr;
    const int d = a.d, kn = a.kn;
    if (a.cta_pair && a.mode == 0 && d == 128 && kn == 128 && !a.out_f32 && !a.kv_fm && !split) {
        svga_status rc = launch_pair(a, kp, st);
        if (rc != SVGA_OK) return rc;
        KParams rest = kp;  // the items the pair kernel left
        rest.pair_rest = 1;
        return launch_t<128, 128, false>(a, rest, st);
    }
    if (d == 128 && kn == 128)
        return a.out_f32 ? launch_t<128, 128, true>(a, kp, st) : launch_t<128, 128, false>(a, kp, st);
    if (d == 128 && kn == 64)
        return a.out_f32 ? launch_t<128, 64, true>(a, kp, st) : launch_t<128, 64, false>(a, kp, st);
    if (d == 64 && kn == 128)
        return a.out_f32 ? launch_t<64, 128, true>(a, kp, st) : launch_t<64, 128, false>(a, kp, st);
    if (d == 64 && kn == 64)
        return a.out_f32 ? launch_t<64, 64, true>(a, kp, st) : launch_t<64, 64, false>(a, kp, st);
    set_error("unsupported head_dim %d / key chunk %d", d, kn);
    return SVGA_ERR_UNSUPPORTED;
}

}  // namespace svga
