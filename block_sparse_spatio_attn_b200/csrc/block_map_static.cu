// block_map_static.cu -- svga_build_block_map_static: the block-map build without a
// caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory when they build a map.
// Examples are plugin hosts whose execute callback forbids allocation, servers that fix
// their memory budget at start-up, and code that must not take the implicit device
// synchronisation cudaMalloc / cudaFree can cause.  Such a caller still owns the map's
// output buffers (allocated once, up front), but has no place to put the build's
// scratch.  This variant keeps that scratch in a file-scope device array of
// kStaticScratchBytes, which every GPU that loads the library holds until the process
// exits.
//
// The array is a host-side stand-in in host code: its device address is looked up once
// per device (cudaGetSymbolAddress, with that device current) on the first call made on
// that device, and cached.  That first call should therefore happen before any stream
// capture.  All calls share the one array and it keeps the previous call's contents;
// the build writes every scratch word it reads before reading it, so nothing needs
// clearing, but two calls that overlap on the GPU (different streams, no ordering
// between them) race on the array.
#include <cuda_runtime.h>

#include <mutex>

#include "svga_internal.h"

namespace svga {
namespace {

constexpr size_t kStaticScratchBytes = 1u << 20;  // SVGA_MAP_STATIC_SCRATCH_BYTES
static_assert(kStaticScratchBytes == SVGA_MAP_STATIC_SCRATCH_BYTES, "header and file agree");

__device__ __align__(256) unsigned char g_map_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_map_scratch on the current device (looked up once per device).
svga_status scratch_address(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        set_error("cudaGetDevice failed or device ordinal out of range: %s",
                  cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_map_scratch);
        if (e != cudaSuccess || !p) {
            set_error("cudaGetSymbolAddress of the static scratch failed: %s",
                      cudaGetErrorString(e));
            return SVGA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SVGA_OK;
}

}  // namespace
}  // namespace svga

using namespace svga;

extern "C" svga_status svga_build_block_map_static(const svga_problem *problem,
                                                   svga_block_map *map, svga_stream_t stream)
{
    Geometry g;
    svga_status rc = validate_problem(problem, &g);
    if (rc != SVGA_OK) return rc;
    if (!map || !map->cls || !map->full_ptr || !map->full_idx || !map->bnd_ptr || !map->bnd_idx ||
        !map->plan) {
        set_error("block map buffers must be non-NULL device pointers");
        return SVGA_ERR_INVALID_ARG;
    }
    const size_t need = block_map_workspace_bytes(g);
    if (need > kStaticScratchBytes) {
        set_error("this problem needs %zu bytes of build scratch, more than the %zu bytes of the "
                  "static array; use svga_build_block_map with a workspace",
                  need, kStaticScratchBytes);
        return SVGA_ERR_WORKSPACE;
    }
    auto misaligned = [](const void *p, uintptr_t a) {
        return (reinterpret_cast<uintptr_t>(p) % a) != 0;
    };
    if (misaligned(map->plan, 256) || misaligned(map->full_ptr, 4) || misaligned(map->bnd_ptr, 4) ||
        misaligned(map->full_idx, 4) || misaligned(map->bnd_idx, 4)) {
        set_error("plan must be 256-byte aligned, CSR arrays 4-byte aligned");
        return SVGA_ERR_ALIGNMENT;
    }
    if (map->plan_bytes < plan_header_bytes(g) || map->full_cap < 0 || map->bnd_cap < 0) {
        set_error("plan (%zu bytes) smaller than svga_block_map_size", map->plan_bytes);
        return SVGA_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    if ((rc = scratch_address(&scratch)) != SVGA_OK) return rc;
    return launch_build_block_map(problem, g, map, scratch, kStaticScratchBytes, stream);
}
