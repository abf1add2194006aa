// Forward entry point for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code running under
// an allocator it does not own (an inference engine or framework plugin whose
// memory is planned up front and that exposes no allocation hook), code that
// must not call cudaMalloc on its hot path because it would synchronise the
// device, and small tools linking only this C ABI without a memory manager.
// For them, sf_gdn_fwd_noalloc runs exactly the forward of sf_gdn_fwd but takes
// its scratch from a fixed array in device memory that belongs to this
// library, so it allocates nothing at all.
//
// Costs and limits of that choice:
//   * every GPU that loads the library holds the array (SF_NOALLOC_SCRATCH_BYTES)
//     until the process exits, whether or not this entry point is used;
//   * shapes whose forward workspace is larger than the array are rejected with
//     SF_ERR_WORKSPACE before anything is enqueued;
//   * all calls share the one array per device, so calls whose work overlaps on
//     the GPU (different streams, or different host threads on one device)
//     race on it; serialise them (one stream, or events between streams);
//   * the array keeps whatever the previous call left in it.  The forward writes
//     every scratch element it later reads, so nothing needs clearing first.
// The first call on each device looks up the array's device address
// (cudaGetSymbolAddress) with that device current; make that first call
// outside of any stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/sf_gdn.h"

namespace {

// The scratch array.  In host code this name is only a stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SF_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device), or an error status.
sf_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SF_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SF_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return SF_OK;
}

}  // namespace

extern "C" sf_status sf_gdn_fwd_noalloc(const sf_gdn_shape* shape, const void* q, const void* k,
                                        const void* v, const float* g, const float* beta,
                                        const float* S_in, void* o, float* S_out, void* stream) {
    if (!shape) return SF_ERR_INVALID_ARG;
    const size_t need = sf_gdn_fwd_workspace_bytes(shape);
    if (need > (size_t)SF_NOALLOC_SCRATCH_BYTES) return SF_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0) {
        const sf_status st = scratch_address(&ws);
        if (st != SF_OK) return st;
    }
    return sf_gdn_fwd(shape, q, k, v, g, beta, S_in, o, S_out, ws,
                      need > 0 ? (size_t)SF_NOALLOC_SCRATCH_BYTES : 0, stream);
}
