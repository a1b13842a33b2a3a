// validate.cu -- host-side consistency check of a built block map.
//
// The block map is what the attention kernel trusts to skip tiles ("Accelerating
// Spatio-Temporal Attention for Video Diffusion on TPUs", aihirek.info, section "A
// TPU-kernel kialakitasa dontonek bizonyult": empty tiles are skipped, full tiles run
// unmasked, boundary tiles are masked).  A full tile that is not really full, or a
// list that misses a visited tile, silently changes the result, so this check copies
// the map to the host and verifies every invariant the kernels rely on.  It stands in
// for a device race detector, which this library does not use.
#include <cuda_runtime.h>

#include <cstring>
#include <vector>

#include "svga_internal.h"

namespace svga {
namespace {

// The visit / full flags of (128-row block b, key chunk c), recomputed from the tile
// classes: the block's q-tiles and the chunk's k-tile, visited if any is non-empty,
// full if all are full.
uint32_t expect_flags(const Geometry &g, const uint8_t *cls_h, int b, int c)
{
    if (b >= g.n_qblk) return 0;
    int i0 = b, i1 = b;
    if (g.tile_q == 64) {
        i0 = 2 * b;
        i1 = 2 * b + 1 < g.n_q ? 2 * b + 1 : g.n_q - 1;
    } else if (g.tile_q == 256) {
        i0 = i1 = b / 2;
    }
    const int j = (g.tile_k > g.kn) ? c / (g.tile_k / g.kn) : c;
    bool visit = false, full = true;
    for (int i = i0; i <= i1; ++i) {
        const uint8_t x = cls_h[(size_t)i * g.n_k + j];
        visit = visit || x != 0;
        full = full && x == 1;
    }
    return visit ? (1u | (full ? 2u : 0u)) : 0u;
}

template <class T>
bool fetch(std::vector<T> &dst, const void *src, size_t n, cudaStream_t st)
{
    dst.resize(n);
    if (n == 0) return true;
    return cudaMemcpyAsync(dst.data(), src, n * sizeof(T), cudaMemcpyDeviceToHost, st) ==
           cudaSuccess;
}

}  // namespace
}  // namespace svga

using namespace svga;

extern "C" svga_status svga_validate_block_map(const svga_problem *problem,
                                               const svga_block_map *map, svga_stream_t stream)
{
    Geometry g;
    svga_status rc = validate_geometry(problem, &g);
    if (rc != SVGA_OK) return rc;
    if (!map || !map->cls || !map->full_ptr || !map->bnd_ptr || !map->plan ||
        map->plan_bytes < plan_bytes_needed(g)) {
        set_error("block map buffers missing or plan smaller than svga_block_map_size");
        return SVGA_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t rows = (size_t)g.heads * g.n_q;
    std::vector<uint8_t> cls, head;
    std::vector<int32_t> fptr, bptr, fidx, bidx, status(1, 0);
    bool ok = fetch(cls, map->cls, rows * g.n_k, st) && fetch(fptr, map->full_ptr, rows + 1, st) &&
              fetch(bptr, map->bnd_ptr, rows + 1, st) &&
              fetch(head, map->plan, plan_header_bytes(g), st) &&
              (!map->status || fetch(status, map->status, 1, st));
    if (!ok || cudaStreamSynchronize(st) != cudaSuccess) {
        set_error("copying the block map to the host failed: %s",
                  cudaGetErrorString(cudaGetLastError()));
        return SVGA_ERR_CUDA;
    }
    auto fail = [](const char *what, long long a, long long b) {
        set_error("block map invalid: %s (%lld, %lld)", what, a, b);
        return SVGA_ERR_INVALID_ARG;
    };
    if (status[0] != 0) return fail("status word set by the build", status[0], 0);

    // head info first: a tile's "holds a position without a token" depends on the order
    const int4 *hinfo = reinterpret_cast<const int4 *>(head.data() + sizeof(PlanHeader));
    for (int h = 0; h < g.heads; ++h)
        if (hinfo[h].x < 0 || hinfo[h].x > 1 || hinfo[h].y < 0 || hinfo[h].z < 0 || hinfo[h].z > 2)
            return fail("plan head info invalid (head, type)", h, hinfo[h].x);
    // holes[order][0 / 1][tile]: the q-tile / k-tile holds a position past the NP
    // positions or one without a token (frame-major: the padding after each frame;
    // temporal-major: the positions from N on)
    std::vector<uint8_t> holes[3][2];
    for (int od = 0; od < 3; ++od)
        for (int side = 0; side < 2; ++side) {
            const int t = side ? g.tile_k : g.tile_q, n = side ? g.n_k : g.n_q;
            holes[od][side].assign(n, 0);
            for (int i = 0; i < n; ++i)
                for (long long pos = (long long)i * t; pos < (long long)(i + 1) * t; ++pos) {
                    const bool tok = pos < g.NP && (od == ORDER_FM ? (pos % g.Sp) < g.S : pos < g.N);
                    if (!tok) {
                        holes[od][side][i] = 1;
                        break;
                    }
                }
        }

    // ---- classes and CSR lists
    for (size_t t = 0; t < cls.size(); ++t)
        if (cls[t] > 2) return fail("tile class outside 0..2 at tile", (long long)t, cls[t]);
    if (fptr[0] != 0 || bptr[0] != 0) return fail("list offsets do not start at 0", fptr[0], bptr[0]);
    for (size_t r = 0; r < rows; ++r)
        if (fptr[r + 1] < fptr[r] || bptr[r + 1] < bptr[r])
            return fail("list offsets decrease at row", (long long)r, 0);
    if (fptr[rows] > map->full_cap || bptr[rows] > map->bnd_cap)
        return fail("lists longer than their capacity", fptr[rows], bptr[rows]);
    ok = fetch(fidx, map->full_idx, (size_t)fptr[rows], st) &&
         fetch(bidx, map->bnd_idx, (size_t)bptr[rows], st);
    if (!ok || cudaStreamSynchronize(st) != cudaSuccess) {
        set_error("copying the lists to the host failed");
        return SVGA_ERR_CUDA;
    }
    for (size_t r = 0; r < rows; ++r) {
        const uint8_t *row = cls.data() + r * g.n_k;
        const int i = (int)(r % g.n_q), od = hinfo[r / g.n_q].z;
        const bool qpad = holes[od][0][i] != 0;
        int nf = 0, nb = 0;
        for (int j = 0; j < g.n_k; ++j) {
            nf += row[j] == 1;
            nb += row[j] == 2;
            const bool kpad = holes[od][1][j] != 0;
            if (row[j] == 1 && (qpad || kpad))
                return fail("tile holding padding marked full (row, k-tile)", (long long)r, j);
        }
        if (fptr[r + 1] - fptr[r] != nf || bptr[r + 1] - bptr[r] != nb)
            return fail("list lengths differ from the class counts of row", (long long)r, nf);
        for (int k = fptr[r]; k < fptr[r + 1]; ++k) {
            const int j = fidx[k];
            if (j < 0 || j >= g.n_k || row[j] != 1 || (k > fptr[r] && j <= fidx[k - 1]))
                return fail("full list entry out of range, not full or not ascending", (long long)r, j);
        }
        for (int k = bptr[r]; k < bptr[r + 1]; ++k) {
            const int j = bidx[k];
            if (j < 0 || j >= g.n_k || row[j] != 2 || (k > bptr[r] && j <= bidx[k - 1]))
                return fail("boundary list entry out of range, not boundary or not ascending",
                            (long long)r, j);
        }
    }

    // ---- execution plan
    PlanHeader hdr;
    std::memcpy(&hdr, head.data(), sizeof hdr);
    if (hdr.magic != kPlanMagic || hdr.heads != g.heads || hdr.tokens != g.N ||
        hdr.frames != g.F || hdr.tokens_per_frame != g.S ||
        hdr.anchor != problem->anchor_frame0 || hdr.tile_q != g.tile_q ||
        hdr.tile_k != g.tile_k || hdr.kn != g.kn || hdr.n_qblk != g.n_qblk ||
        hdr.n_kc != g.n_kc || hdr.n_items != g.n_items || hdr.frame_stride != g.Sp)
        return fail("plan header does not match the problem", hdr.magic, hdr.n_items);
    const int4 *items = hinfo + g.heads;
    const long long entry_cap =
        (long long)((map->plan_bytes - plan_header_bytes(g)) / sizeof(uint32_t));
    std::vector<uint8_t> seen(g.n_items, 0);
    long long need = 0;  // entries up to the end of the furthest item
    for (int it = 0; it < g.n_items; ++it) {
        const int4 x = items[it];
        if (x.x < 0 || x.x >= g.heads || x.y < 0 || (x.y & 1) || x.y / 2 >= g.n_pairs)
            return fail("plan item outside the problem (item, head)", it, x.x);
        const int id = x.x * g.n_pairs + x.y / 2;
        if (seen[id]++) return fail("plan item listed twice (item, head)", it, x.x);
        if (it > 0 && x.w > items[it - 1].w) return fail("plan items not longest first", it, x.w);
        if (x.z < 0 || x.w < 0 || (long long)x.z + x.w > entry_cap)
            return fail("plan item entries outside the plan (item, offset)", it, x.z);
        if ((long long)x.z + x.w > need) need = (long long)x.z + x.w;
    }
    std::vector<uint32_t> ent;
    if (!fetch(ent, static_cast<const char *>(map->plan) + plan_header_bytes(g), (size_t)need,
               st) ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        set_error("copying the plan entries to the host failed");
        return SVGA_ERR_CUDA;
    }
    for (int it = 0; it < g.n_items; ++it) {
        const int4 x = items[it];
        const uint8_t *cls_h = cls.data() + (size_t)x.x * g.n_q * g.n_k;
        const int p = x.y / 2;
        int n = 0;
        for (int c = 0; c < g.n_kc; ++c) {
            const uint32_t a = expect_flags(g, cls_h, 2 * p, c), b = expect_flags(g, cls_h, 2 * p + 1, c);
            if (!(a | b)) continue;
            const uint32_t want = (uint32_t)c | (a << 24) | (b << 26);
            if (n >= x.w) return fail("plan item misses a visited chunk (item, chunk)", it, c);
            if (ent[(size_t)x.z + n] != want)
                return fail("plan entry differs from the tile classes (item, chunk)", it, c);
            ++n;
        }
        if (n != x.w) return fail("plan item has extra entries (item, count)", it, x.w);
    }
    return SVGA_OK;
}
