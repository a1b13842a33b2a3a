// classify.cu -- online spatial / temporal head classification.
//
// Sparse VideoGen profiles the heads while it runs: for a few query rows it computes
// the dense, the spatial and the temporal outputs and keeps the sparse mask whose
// output deviates least from the dense one ("Accelerating Spatio-Temporal Attention for
// Video Diffusion on TPUs", aihirek.info, section "A Sparse VideoGen a figyelmi
// fejeket osztalyozza").  Here:
//   1. the sampled rows of Q are gathered into a compact [heads, n_rows, d] tensor;
//   2. the tcgen05 attention kernel runs three times over all keys with the gathered
//      rows as queries (their original coordinates ride along): dense, spatial-masked
//      and temporal-masked, writing fp32 outputs;
//   3. the two squared deviations are reduced in fp64, first over slices of each head's
//      outputs by many blocks, then per head in a fixed order (deterministic), and the
//      smaller one picks the mask (a tie goes to spatial).
#include <cuda_runtime.h>

#include "svga_device.cuh"
#include "svga_internal.h"

namespace svga {
namespace {

struct BandParams {
    uint16_t w_spatial[kMaxHeads];
    uint16_t w_temporal[kMaxHeads];
};

__global__ void classify_setup_kernel(int heads, int N, int n_rows, int make_rows, BandParams bp,
                                      int4 *info_s, int4 *info_t, int32_t *rows)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    for (int h = t; h < heads; h += gridDim.x * blockDim.x) {
        info_s[h] = make_int4(MASK_SPATIAL, bp.w_spatial[h], ORDER_FM, 0);
        info_t[h] = make_int4(MASK_TEMPORAL, bp.w_temporal[h], ORDER_FM, 0);
    }
    if (make_rows)
        for (int i = t; i < n_rows; i += gridDim.x * blockDim.x)
            rows[i] = (int32_t)(((2ll * i + 1) * (long long)N) / (2ll * n_rows));
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

// Stage 1: block (part, h) sums the squared deviations of one slice of head h.
__global__ void __launch_bounds__(256) mse_partial_kernel(const float *od, const float *os,
                                                          const float *ot, int n, double *partial)
{
    __shared__ double red[2][8];
    const int part = blockIdx.x, h = blockIdx.y;
    const size_t base = (size_t)h * n;
    const int per = (n + kMseParts - 1) / kMseParts;
    const int i0 = part * per, i1 = min(n, i0 + per);
    double as = 0.0, at = 0.0;
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
        const double d = od[base + i];
        const double a = os[base + i] - d, b = ot[base + i] - d;
        as += a * a;
        at += b * b;
    }
    for (int o = 16; o > 0; o >>= 1) {
        as += __shfl_xor_sync(0xffffffffu, as, o);
        at += __shfl_xor_sync(0xffffffffu, at, o);
    }
    if ((threadIdx.x & 31) == 0) {
        red[0][threadIdx.x >> 5] = as;
        red[1][threadIdx.x >> 5] = at;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0, t = 0.0;
        for (int w = 0; w < 8; ++w) {
            s += red[0][w];
            t += red[1][w];
        }
        partial[((size_t)h * kMseParts + part) * 2] = s;
        partial[((size_t)h * kMseParts + part) * 2 + 1] = t;
    }
}

// Stage 2: per head, the partial sums in part order, the means and the decision.
__global__ void mse_final_kernel(const double *partial, int heads, int n, int32_t *type_out,
                                 float *mse_out)
{
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= heads) return;
    double s = 0.0, t = 0.0;
    for (int part = 0; part < kMseParts; ++part) {
        s += partial[((size_t)h * kMseParts + part) * 2];
        t += partial[((size_t)h * kMseParts + part) * 2 + 1];
    }
    s /= n;
    t /= n;
    mse_out[2 * h] = (float)s;
    mse_out[2 * h + 1] = (float)t;
    type_out[h] = s <= t ? MASK_SPATIAL : MASK_TEMPORAL;
}

struct ClassifyLayout {
    size_t info_s, info_t, rows, qg, od, os, ot, partial, types, mse, status, total;
};

ClassifyLayout classify_layout(int heads, int d, int n_rows)
{
    ClassifyLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    L.info_s = take(sizeof(int4) * heads);
    L.info_t = take(sizeof(int4) * heads);
    L.rows = take(sizeof(int32_t) * n_rows);
    L.qg = take((size_t)heads * n_rows * d * 2);
    L.od = take((size_t)heads * n_rows * d * 4);
    L.os = take((size_t)heads * n_rows * d * 4);
    L.ot = take((size_t)heads * n_rows * d * 4);
    L.partial = take(sizeof(double) * 2 * kMseParts * heads);
    L.types = take(sizeof(int32_t) * heads);
    L.mse = take(sizeof(float) * 2 * heads);
    L.status = take(sizeof(int32_t));
    L.total = o;
    return L;
}

}  // namespace

size_t classify_workspace_bytes(const svga_problem *p, int n_rows)
{
    return classify_layout(p->heads, p->head_dim, n_rows).total;
}

svga_status run_classify(const void *q, const void *k, const void *v, const svga_problem *p,
                         const int32_t *w_spatial, const int32_t *w_temporal, const int32_t *rows,
                         int n_rows, float scale, int32_t *head_type_out, float *mse_out,
                         int32_t *status_out, int device_out, void *ws, size_t ws_bytes,
                         void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int H = p->heads, d = p->head_dim, S = p->grid_h * p->grid_w, N = p->num_frames * S;
    const ClassifyLayout L = classify_layout(H, d, n_rows);
    (void)ws_bytes;
    char *w = static_cast<char *>(ws);
    int4 *info_s = reinterpret_cast<int4 *>(w + L.info_s);
    int4 *info_t = reinterpret_cast<int4 *>(w + L.info_t);
    int32_t *rows_ws = reinterpret_cast<int32_t *>(w + L.rows);
    void *qg = w + L.qg;
    float *od = reinterpret_cast<float *>(w + L.od);
    float *os = reinterpret_cast<float *>(w + L.os);
    float *ot = reinterpret_cast<float *>(w + L.ot);
    int32_t *types = reinterpret_cast<int32_t *>(w + L.types);
    float *mse = reinterpret_cast<float *>(w + L.mse);
    int32_t *status = reinterpret_cast<int32_t *>(w + L.status);

    BandParams bp;
    for (int h = 0; h < H; ++h) {
        bp.w_spatial[h] = (uint16_t)w_spatial[h];
        bp.w_temporal[h] = (uint16_t)w_temporal[h];
    }
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) {
        set_error("cudaMemsetAsync failed");
        return SVGA_ERR_CUDA;
    }
    const int32_t *rows_use = rows ? rows : rows_ws;
    classify_setup_kernel<<<(H > n_rows ? H : n_rows) / 256 + 1, 256, 0, st>>>(
        H, N, n_rows, rows ? 0 : 1, bp, info_s, info_t, rows_ws);
    const int vpr = d / 8;
    dim3 grid((n_rows * vpr + 255) / 256 < 1184 ? (n_rows * vpr + 255) / 256 : 1184, H);
    if (vpr == 16)
        gather_rows_kernel<16><<<grid, 256, 0, st>>>(static_cast<const uint4 *>(q),
                                                    static_cast<uint4 *>(qg), rows_use, N, n_rows,
                                                    status);
    else
        gather_rows_kernel<8><<<grid, 256, 0, st>>>(static_cast<const uint4 *>(q),
                                                   static_cast<uint4 *>(qg), rows_use, N, n_rows,
                                                   status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("classifier setup launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    AttnLaunch a{};
    a.q = qg;
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
    a.qrow_tokens = rows_use;
    a.out_f32 = 1;
    const int n_qblk = (n_rows + kBlockM - 1) / kBlockM;
    a.n_items = H * ((n_qblk + 1) / 2);
    a.status = status;
    svga_status rc;
    a.mode = 1;
    a.head_info = nullptr;
    a.o = od;
    if ((rc = launch_attention(a, stream)) != SVGA_OK) return rc;
    a.mode = 2;
    a.head_info = reinterpret_cast<const int32_t *>(info_s);
    a.o = os;
    if ((rc = launch_attention(a, stream)) != SVGA_OK) return rc;
    a.head_info = reinterpret_cast<const int32_t *>(info_t);
    a.o = ot;
    if ((rc = launch_attention(a, stream)) != SVGA_OK) return rc;
    double *partial = reinterpret_cast<double *>(w + L.partial);
    mse_partial_kernel<<<dim3(kMseParts, H), 256, 0, st>>>(od, os, ot, n_rows * d, partial);
    mse_final_kernel<<<(H + 127) / 128, 128, 0, st>>>(partial, H, n_rows * d, types, mse);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_error("classifier reduction launch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    if (device_out) {
        // results stay on the device: no host round trip, nothing waits
        if (cudaMemcpyAsync(head_type_out, types, sizeof(int32_t) * H, cudaMemcpyDeviceToDevice,
                            st) != cudaSuccess ||
            (mse_out && cudaMemcpyAsync(mse_out, mse, sizeof(float) * 2 * H,
                                        cudaMemcpyDeviceToDevice, st) != cudaSuccess) ||
            (status_out && cudaMemcpyAsync(status_out, status, sizeof(int32_t),
                                           cudaMemcpyDeviceToDevice, st) != cudaSuccess)) {
            set_error("classifier result copy failed: %s", cudaGetErrorString(cudaGetLastError()));
            return SVGA_ERR_CUDA;
        }
        return SVGA_OK;
    }
    int32_t dev_status = 0;
    if (cudaMemcpyAsync(head_type_out, types, sizeof(int32_t) * H, cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        (mse_out && cudaMemcpyAsync(mse_out, mse, sizeof(float) * 2 * H, cudaMemcpyDeviceToHost,
                                    st) != cudaSuccess) ||
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

}  // namespace svga
