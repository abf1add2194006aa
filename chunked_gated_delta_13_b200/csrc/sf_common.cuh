// Shared declarations of the CUDA side of libsf_gdn: the per-call parameter
// block, element load/store helpers and the internal launcher entry points.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sf {

// One call's view of a (segment of a) sequence.  Element (bh, t, d) of a
// [B,H,T_full,d] tensor sits at base[bh * hs + t * d]; base already points at
// the first token of the segment, so a segment is a strided view of the full
// sequence and nothing is copied.
struct SeqView {
    int BH;          // batch * heads
    int T;           // tokens in this segment
    int dk, dv;      // head sizes
    int C;           // kernel chunk length
    int NC;          // chunks = ceil(T / C)
    int use_beta;    // 0: recurrence without the delta term
    float scale;     // multiplies q
    long long hs_k;  // head stride of q, k, dq, dk (elements)
    long long hs_v;  // head stride of v, o, dO, dv
    long long hs_g;  // head stride of g, beta, dg, dbeta
};

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float* p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device pointers of one forward call (segment view applied).
struct FwdArgs {
    const void* q; const void* k; const void* v;
    const float* g; const float* beta; const float* S_in;
    void* o; float* S_out;
};

// Device pointers of one backward call (segment view applied).
struct BwdArgs {
    const void* q; const void* k; const void* v;
    const float* g; const float* beta; const float* S_in;
    const void* dO; const float* dS_out;
    void* dq; void* dk; void* dv; float* dg; float* dbeta; float* dS_in;
};

// Launch observer (see sf_set_launch_hook): called before (after = 0) and
// after (after = 1) every kernel launch.
void launch_hook(const char* kernel, int after, cudaStream_t st);

#define SF_LAUNCH(name, stream, ...)            \
    do {                                        \
        ::sf::launch_hook(name, 0, stream);     \
        __VA_ARGS__;                            \
        ::sf::launch_hook(name, 1, stream);     \
    } while (0)

// Fp32 CUDA-core kernel family (any supported shape, both I/O dtypes).
size_t simt_workspace_bytes(const SeqView& s, bool backward);
cudaError_t simt_fwd(const SeqView& s, bool bf16, const FwdArgs& a, void* ws, cudaStream_t st);
cudaError_t simt_bwd(const SeqView& s, bool bf16, const BwdArgs& a, void* ws, cudaStream_t st);
int simt_launches(bool backward);

}  // namespace sf
