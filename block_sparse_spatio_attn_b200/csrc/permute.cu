// permute.cu -- token permutation between frame-major and a head's token order.
//
// The pages move the tokens of temporal heads from frame-major to temporal-major
// order so that a temporal head's band lines up with the tiles ("Accelerating
// Spatio-Temporal Attention for Video Diffusion on TPUs", ainews.tenesys.com,
// "Co sie zmienilo?" item 5).  Both directions are gathers: every thread writes one
// 16-byte piece of a destination row (coalesced) and reads the matching piece of the
// source row the order maps it to (a whole 128- or 256-byte row per warp quarter or
// half, so reads stay full cache lines).  Pure data movement: bound by HBM bandwidth.
#include <cuda_runtime.h>

#include "svga_device.cuh"
#include "svga_internal.h"

namespace svga {
namespace {

struct OrderParams {
    uint8_t order[kMaxHeads];
};

// Does a block map's plan (header, then head info) describe this launch?  Checked by
// every block before anything is written, so a map of another problem changes nothing.
__device__ __forceinline__ bool plan_fits(const int4 *plan, int heads, int N, int F, int S, int Sp,
                                          int h)
{
    // {magic, heads, tokens, frames}, {S, ..}, .., {entry_cap, frame stride, ..}
    const int4 a = __ldg(plan), b = __ldg(plan + 1), d = __ldg(plan + 3);
    if (!(a.x == kPlanMagic && a.y == heads && a.z == N && a.w == F && b.x == S && d.z == Sp))
        return false;
    const int order = __ldg(plan + 4 + h).z;  // head info follows the 64-byte header
    return order >= ORDER_FM && order <= ORDER_TM_STRICT;
}

// Both directions gather into the destination's rows: forward, dst has NP positions
// per head (frame-major frames at stride Sp; positions without a token get zeros),
// src N frame-major tokens; inverse, the other way round.
template <int VPR>  // 16-byte vectors per row (head_dim / 8)
__global__ void __launch_bounds__(256) permute_kernel(const uint4 *__restrict__ src,
                                                      uint4 *__restrict__ dst, int N, int F, int S,
                                                      int Sp, int inverse, OrderParams op,
                                                      const int4 *__restrict__ plan,
                                                      int32_t *status)
{
    const int h = blockIdx.y;
    if (plan && !plan_fits(plan, gridDim.y, N, F, S, Sp, h)) {
        if (threadIdx.x == 0 && status) atomicCAS(status, 0, (int32_t)SVGA_ERR_INVALID_ARG);
        return;
    }
    const int order = plan ? __ldg(plan + 4 + h).z : op.order[h];
    const int NP = F * Sp;
    const int src_rows = inverse ? NP : N, dst_rows = inverse ? N : NP;
    const size_t src_off = (size_t)h * src_rows * VPR, dst_off = (size_t)h * dst_rows * VPR;
    const int total = dst_rows * VPR;
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
        const int drow = idx / VPR, v = idx - drow * VPR;
        int srow;  // -1: a position without a token
        if (order == ORDER_FM && Sp == S) {  // unpadded frame-major: a plain copy
            srow = drow;
        } else if (!inverse) {  // dst position -> its token's frame-major row
            if (order == ORDER_FM) {
                const int f = drow / Sp, s = drow - f * Sp;
                srow = s < S ? f * S + s : -1;
            } else if (drow < N) {
                int f, s;
                pos_to_coord(order, drow, F, S, f, s);
                srow = f * S + s;
            } else {
                srow = -1;
            }
        } else {  // dst is frame-major token drow: where the order put it
            const int f = drow / S, s = drow - f * S;
            srow = order == ORDER_FM ? f * Sp + s : coord_to_pos(order, f, s, F, S);
        }
        dst[dst_off + (size_t)drow * VPR + v] =
            srow >= 0 ? __ldg(src + src_off + (size_t)srow * VPR + v) : make_uint4(0, 0, 0, 0);
    }
}

}  // namespace

svga_status launch_permute(const void *src, void *dst, const svga_problem *p, const Geometry &g,
                           int inverse, void *stream, const void *plan, int32_t *status)
{
    static_assert(sizeof(PlanHeader) == 4 * sizeof(int4), "head info starts at int4 index 4");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    OrderParams op;
    const int4 *hi = static_cast<const int4 *>(plan);
    for (int h = 0; h < g.heads; ++h) op.order[h] = hi ? 0 : (uint8_t)p->order[h];
    const int vpr = g.d / 8;
    const int total = (inverse ? g.N : g.NP) * vpr;
    int blocks = (total + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    dim3 grid(blocks, g.heads);
    if (vpr == 16)
        permute_kernel<16><<<grid, 256, 0, st>>>(static_cast<const uint4 *>(src),
                                                 static_cast<uint4 *>(dst), g.N, g.F, g.S, g.Sp, inverse, op,
                                                 hi, status);
    else
        permute_kernel<8><<<grid, 256, 0, st>>>(static_cast<const uint4 *>(src),
                                                static_cast<uint4 *>(dst), g.N, g.F, g.S, g.Sp, inverse, op,
                                                hi, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("permute launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    return SVGA_OK;
}

}  // namespace svga
