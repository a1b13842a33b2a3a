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
// In host code the name g_map_scratch does not denote device memory: it is a host-side
// stand-in for the array, and a kernel given it would fault or read the wrong memory.
// The device address is therefore asked for with cudaGetSymbolAddress on every call, in
// the CUDA context current at that call (one host call, no allocation, no
// synchronisation).  Looking it up each time keeps the address right after a
// cudaDeviceReset or when another context of the device is current.  The first call in
// a context may load the library's device code into it, so make that first call before
// any stream capture.
//
// All calls share the one array and it keeps the previous call's contents; the build
// writes every scratch word it reads before reading it, so nothing needs clearing, but
// two calls that overlap on the GPU (different streams, no ordering between them) race
// on the array.
#include <cuda_runtime.h>

#include "svga_internal.h"

namespace svga {
namespace {

constexpr size_t kStaticScratchBytes = 1u << 20;  // SVGA_MAP_STATIC_SCRATCH_BYTES
static_assert(kStaticScratchBytes == SVGA_MAP_STATIC_SCRATCH_BYTES, "header and file agree");

__device__ __align__(256) unsigned char g_map_scratch[kStaticScratchBytes];

// Device address of g_map_scratch in the current context.
svga_status scratch_address(void **out)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_map_scratch);
    if (e != cudaSuccess || !p) {
        set_error("cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
        return SVGA_ERR_CUDA;
    }
    *out = p;
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
    const size_t need = block_map_workspace_bytes(g);
    if (need > kStaticScratchBytes) {
        set_error("this problem needs %zu bytes of build scratch, more than the %zu bytes of the "
                  "static array; use svga_build_block_map with a workspace",
                  need, kStaticScratchBytes);
        return SVGA_ERR_WORKSPACE;
    }
    if ((rc = check_map_outputs(g, map)) != SVGA_OK) return rc;
    void *scratch = nullptr;
    if ((rc = scratch_address(&scratch)) != SVGA_OK) return rc;
    return launch_build_block_map(problem, g, map, scratch, kStaticScratchBytes, stream);
}
