// sf_fwd_noalloc: the forward of one sequence piece for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace: code that runs under a
// framework which plans all device memory before it starts and hands a plugin
// only its input and output buffers, code that runs inside a memory
// allocator's own callbacks, or latency-critical loops that must not call
// cudaMalloc (which can synchronise the whole device).  For them this entry
// point takes the scratch that sf_fwd would take from its `ws` argument from a
// fixed array compiled into the library instead.
//
// The array lives in device global memory of every GPU that loads the
// library, for as long as the process runs.  All calls share it, so two calls
// whose work overlaps on the GPU (different streams, or different host
// threads) race on it; calls that are ordered on one stream are safe.  The
// array keeps whatever the previous call left in it; each call clears the one
// word that must start at zero (the error word that bounded device waits set)
// and every other byte it reads is written by an earlier kernel of the same
// call.  sf_check_noalloc reads that error word.

#include <cuda_runtime.h>

#include "../../include/sf.h"
#include "sf_internal.h"

namespace sf {
namespace {

constexpr size_t kScratchBytes = (size_t)32 << 20;  // 32 MiB

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch in the current device's context.  In host code
// g_scratch names a host-side stand-in, so kernels must be given this address.
// It is looked up on every call (cheap once the module is loaded), so that a new
// context after cudaDeviceReset, in which the module may land elsewhere, gets
// its own address; the first lookup on a device may load the module, which is
// why the first call should come before any stream capture.
cudaError_t scratch_address(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace sf

extern "C" {

sf_status sf_fwd_noalloc(const sf_shape* s, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* S_in, void* o,
                         float* S_out, void* stream) {
    const size_t need = sf_workspace_bytes(s, SF_OP_FWD);
    if (need == 0)  // invalid shape: sf_fwd reports which error, before any CUDA call
        return sf_fwd(s, q, k, v, g, beta, S_in, o, S_out, nullptr, 0, stream);
    if (need > sf::kScratchBytes) return SF_ERR_WORKSPACE;
    void* ws = nullptr;
    if (sf::scratch_address(&ws) != cudaSuccess) return SF_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(int), (cudaStream_t)stream) != cudaSuccess) return SF_ERR_CUDA;
    return sf_fwd(s, q, k, v, g, beta, S_in, o, S_out, ws, sf::kScratchBytes, stream);
}

sf_status sf_check_noalloc(void* stream) {
    void* ws = nullptr;
    if (sf::scratch_address(&ws) != cudaSuccess) return SF_ERR_CUDA;
    return sf_check(ws, stream);
}

}  // extern "C"
