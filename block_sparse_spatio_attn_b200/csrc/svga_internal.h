// svga_internal.h -- definitions shared by the library's translation units.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/svga.h"

namespace svga {

// token orders (values of svga.h's SVGA_ORDER_*)
enum { ORDER_FM = 0, ORDER_TM = 1, ORDER_TM_STRICT = 2 };
// mask kinds used inside kernels (SVGA_HEAD_* plus dense)
enum { MASK_SPATIAL = 0, MASK_TEMPORAL = 1, MASK_DENSE = 2 };

constexpr int kMaxHeads = 4096;
constexpr int kMaxTokens = 1 << 24;
constexpr int kBlockM = 128;     // query rows per tcgen05 tile (one TMEM lane per row)
constexpr int kMaxParts = 4096;  // largest num_parts of a partitioned attention call

// Execution plan of the attention kernel, stored in svga_block_map::plan.
//   PlanHeader, then int4 head_info[heads] = {mask type, band, order, 0},
//   then int4 items[n_items] = {head, first 128-row block, entry offset, entry count}
//   in longest-first order, then uint32 entries[].
// A work item is a pair of consecutive 128-row query blocks; an entry is one key
// chunk of kn keys visited by at least one of the two blocks:
//   bits 0-23 key chunk index, bit 24 block 0 visits, bit 25 block 0 full,
//   bit 26 block 1 visits, bit 27 block 1 full.
struct PlanHeader {
    int32_t magic;
    int32_t heads, tokens, frames, tokens_per_frame, anchor;
    int32_t tile_q, tile_k, kn, n_qblk, n_kc, n_items;
    int64_t entry_cap;
    int32_t frame_stride;  // Sp: S rounded up to the problem's frame_pad (S without)
    int32_t reserved;
};
static_assert(sizeof(PlanHeader) == 64, "plan header is 64 bytes");
constexpr int32_t kPlanMagic = 0x53564741;  // "SVGA"

constexpr uint32_t kEntChunkMask = 0x00FFFFFFu;
constexpr uint32_t kEntV0 = 1u << 24, kEntF0 = 1u << 25, kEntV1 = 1u << 26, kEntF1 = 1u << 27;

struct Geometry {
    int heads, F, S, N, d;
    int Sp, NP;  // frame stride and positions per head (S and N without frame_pad)
    int tile_q, tile_k, n_q, n_k;
    int kn, n_qblk, n_pairs, n_kc, n_items;
};

// ----------------------------------------------------------- host-side helpers
void set_error(const char *fmt, ...);
svga_status validate_problem(const svga_problem *p, Geometry *g);
// Shape checks and geometry only (per-head arrays not read).
svga_status validate_geometry(const svga_problem *p, Geometry *g);
size_t plan_header_bytes(const Geometry &g);  // header + head_info + items, 256-aligned
int64_t plan_entry_cap(const Geometry &g);
// Plan bytes a map of this geometry needs (header + worst-case entries): what
// svga_block_map_size reports and every call that takes a map requires.
size_t plan_bytes_needed(const Geometry &g);
size_t align_up(size_t x, size_t a);
// Output buffers of a map build (everything but the workspace): non-NULL, aligned, and a
// plan of at least plan_bytes_needed.  Shared by the workspace and the static builds.
svga_status check_map_outputs(const Geometry &g, const svga_block_map *map);
// The plan of a map handed to a call that reads it (attention, mapped permutations).
svga_status check_map_plan(const Geometry &g, const svga_block_map *map);

// block_map.cu
// Per-head type, band and order come from the problem's host arrays, or, when types_dev
// is set, from the device (type) and the two candidate band arrays (band by type; order
// frame-major for spatial, anchor-first temporal-major for temporal heads).
svga_status launch_build_block_map(const svga_problem *p, const Geometry &g, svga_block_map *map,
                                   void *ws, size_t ws_bytes, void *stream,
                                   const int32_t *types_dev = nullptr,
                                   const int32_t *w_spatial = nullptr,
                                   const int32_t *w_temporal = nullptr);
size_t block_map_workspace_bytes(const Geometry &g);

// permute.cu
// Per-head order from the problem's host array, or from a plan's head info when set.
// With a plan, its header is checked against the geometry on the device first: on a
// mismatch nothing is written and `status` (when not NULL) is set to SVGA_ERR_INVALID_ARG.
svga_status launch_permute(const void *src, void *dst, const svga_problem *p, const Geometry &g,
                           int inverse, void *stream, const void *plan = nullptr,
                           int32_t *status = nullptr);

// attention.cu
struct AttnLaunch {
    const void *q, *k, *v;
    void *o;
    float *lse;
    int heads, nq_rows, nk_rows, d;
    int F, S, anchor;
    // token positions: frame-major heads put frame f at f * Sp (Sp = S unless padded),
    // temporal-major heads' tokens fill positions 0 .. N-1; other positions hold none
    int N, Sp;
    float scale;
    int mode;                  // 0 plan, 1 dense (every chunk of every block pair)
    int naive;                 // plan mode: visit full tiles through the masked path
    int aligned;               // plan mode: keep every key of a visited tile (mask snapped to tiles)
    int part, num_parts;       // plan mode: run only the items of part `part` (0 of 1: all)
    int test_stall;            // SVGA_FLAG_TEST_STALL: withhold the first K load
    int qo_fm;                 // SVGA_FLAG_QO_FRAME_MAJOR: q, o, lse frame-major
    int kv_fm;                 // SVGA_FLAG_KV_FRAME_MAJOR: k, v frame-major
    int cta_pair;              // SVGA_FLAG_CTA_PAIR: work items on CTA pairs where it applies
    int kn;                    // keys per chunk: 64 or 128
    int tile_q, tile_k;        // plan mode: the problem's map tiles
    int check_plan;            // plan mode: compare the plan's header and items with the call
    const void *plan;          // device plan (mode 0)
    const int32_t *qrow_tokens;  // device [nq_rows] frame-major token of each query row (shared by all heads) or null
    int out_f32;               // o is float32 instead of bf16
    int n_items;
    int32_t *status;
    // key-range split (out_f32 only): each item runs as ksplit CTAs writing unnormalised
    // fp32 O to part_o [ksplit][heads][nq_rows][d] and (max, sum) to part_ml
    // [ksplit][heads][nq_rows]; merge_attention_parts combines them into o.  ksplit <= 1: off.
    int ksplit;
    float *part_o;
    float *part_ml;
};
svga_status launch_attention(const AttnLaunch &a, void *stream);

// Combine the ksplit parts of a key-range split launch into normalised fp32 o
// [heads][nq_rows][d]; a row no part visited reads 0.
svga_status merge_attention_parts(const AttnLaunch &a, void *stream);

// classify.cu
size_t classify_workspace_bytes(const svga_problem *p, int n_rows, int n_cand);
int max_candidates();
// Dense pass, then one masked pass per candidate (type, band: shared, or per head from
// w_spatial / w_temporal when cand_band is NULL), each one's squared deviation from
// dense, and per head the eligible candidate with the least (the earlier on a tie).
svga_status run_select(const void *q, const void *k, const void *v, const svga_problem *p,
                       int n_cand, const int32_t *cand_type, const int32_t *cand_band,
                       uint32_t eligible, const int32_t *w_spatial, const int32_t *w_temporal,
                       const int32_t *rows, int n_rows, float scale, int32_t *type_out,
                       int32_t *band_out, float *mse_out, int32_t *status_out, int device_out,
                       void *ws, size_t ws_bytes, void *stream);
svga_status run_classify(const void *q, const void *k, const void *v, const svga_problem *p,
                         const int32_t *w_spatial, const int32_t *w_temporal,
                         const int32_t *rows, int n_rows, float scale, int32_t *head_type_out,
                         float *mse_out, int32_t *status_out, int device_out, void *ws,
                         size_t ws_bytes, void *stream);

}  // namespace svga
