// Short causal depthwise convolution with a boundary state: the second state a
// sequence chunk hands to the next (StateFlow, arXiv 2608.06838, section 1:
// chunks must "maintain boundary states from local convolution modules";
// section 3.3: the boundary tensor holds "recurrent and local-convolution
// boundary states").  Per (batch b, head h, channel c) with taps w[h][c][j]
// (tap j multiplies the input j steps back) and the extended input
// xe_p = conv_in[K-1+p] for p < 0, x_p otherwise:
//     pre_t = sum_j w_j xe_{t-j},   y_t = act(pre_t),   conv_out = xe_{T-K+1 .. T-1}
// Backward (gradients of sum <y, dy> + <conv_out, dconv_out>), delta_t = dy_t act'(pre_t):
//     g_p = [p >= T-K+1] dconv_out[p-T+K-1] + sum_j w_j delta_{p+j}   (0 <= p+j < T)
//     dx_p = g_p (p >= 0),  dconv_in[p+K-1] = g_p (p < 0),  dw_j = sum_t delta_t xe_{t-j}
// Summation orders are fixed so that splitting the sequence changes no bit:
//   pre_t: j ascending; g_p: starting from the dconv_out term, j descending
//   (the terms a later segment contributes are exactly the highest taps, which
//   it folds first and hands back as its dconv_in); dw: per 64-token chunk, t
//   descending, then the chunks in descending order starting from dw_in (so a
//   chain running its segments backwards continues the same fold).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>
#include <vector>

#include "../../include/sf_gdn.h"
#include "sf_common.cuh"

namespace sf {
namespace {

constexpr int kConvChunk = 64;  // tokens per CTA (and per weight-gradient partial)
constexpr int kMaxTaps = 8;

struct ConvView {
    int BH, H, T, d, K, NC;
    long long hs;  // head stride of x, y, dy, dx (elements): T_full * d
};

__device__ __forceinline__ float2 ld2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 ld2(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ void st2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void st2(__nv_bfloat16* p, float2 v) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}

template <int ACT>
__device__ __forceinline__ float act_f(float z) {
    return ACT ? z / (1.f + __expf(-z)) : z;
}
template <int ACT>
__device__ __forceinline__ float dact_f(float z) {
    if (!ACT) return 1.f;
    const float s = 1.f / (1.f + __expf(-z));
    return s * (1.f + z * (1.f - s));
}

// xe_p of channels (c, c+1): x for p >= 0, the boundary state for p < 0.
template <typename IO>
__device__ __forceinline__ float2 xe2(const IO* xb, const IO* cib, int p, int K, int d, int c) {
    if (p >= 0) return ld2(xb + (size_t)p * d + c);
    if (!cib) return make_float2(0.f, 0.f);
    return ld2(cib + (size_t)(p + K - 1) * d + c);
}

// Forward: one CTA per (64-token chunk, batch-head); thread i owns channels 2i, 2i+1.
template <typename IO, int ACT>
__global__ void conv_fwd_kernel(ConvView s, const IO* __restrict__ x, const float* __restrict__ w,
                                const IO* __restrict__ conv_in, IO* __restrict__ y) {
    const int c = 2 * threadIdx.x, bh = blockIdx.y, h = bh % s.H;
    const int t0 = blockIdx.x * kConvChunk, t1 = min(s.T, t0 + kConvChunk);
    const IO* xb = x + bh * s.hs;
    const IO* cib = conv_in ? conv_in + (size_t)bh * (s.K - 1) * s.d : nullptr;
    IO* yb = y + bh * s.hs;
    float w0[kMaxTaps], w1[kMaxTaps];
    float2 win[kMaxTaps];  // win[j] = xe_{t-j}
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j) {
        w0[j] = j < s.K ? w[((size_t)h * s.d + c) * s.K + j] : 0.f;
        w1[j] = j < s.K ? w[((size_t)h * s.d + c + 1) * s.K + j] : 0.f;
        win[j] = (j >= 1 && j < s.K) ? xe2(xb, cib, t0 - j, s.K, s.d, c) : make_float2(0.f, 0.f);
    }
    for (int t = t0; t < t1; ++t) {
        win[0] = ld2(xb + (size_t)t * s.d + c);
        float p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxTaps; ++j)
            if (j < s.K) {
                p0 = fmaf(w0[j], win[j].x, p0);
                p1 = fmaf(w1[j], win[j].y, p1);
            }
        st2(yb + (size_t)t * s.d + c, make_float2(act_f<ACT>(p0), act_f<ACT>(p1)));
#pragma unroll
        for (int j = kMaxTaps - 1; j > 0; --j) win[j] = win[j - 1];
    }
}

// conv_out = xe_{T-K+1 .. T-1}: one CTA per batch-head, one thread per channel pair.
template <typename IO>
__global__ void conv_state_kernel(ConvView s, const IO* __restrict__ x, const IO* __restrict__ conv_in,
                                  IO* __restrict__ conv_out) {
    const int c = 2 * threadIdx.x, bh = blockIdx.x;
    const IO* xb = x + bh * s.hs;
    const IO* cib = conv_in ? conv_in + (size_t)bh * (s.K - 1) * s.d : nullptr;
    IO* cob = conv_out + (size_t)bh * (s.K - 1) * s.d;
    for (int m = 0; m < s.K - 1; ++m) st2(cob + (size_t)m * s.d + c, xe2(xb, cib, s.T - (s.K - 1) + m, s.K, s.d, c));
}

// Backward: one CTA per (chunk, batch-head), positions handled in descending
// order with windows of the extended input and of delta in registers.  Chunk 0
// also produces dconv_in (positions -K+1 .. -1).  Writes dx, dconv_in and the
// chunk's weight-gradient partial part[chunk][bh][c][j].
template <typename IO, int ACT>
__global__ void conv_bwd_kernel(ConvView s, const IO* __restrict__ x, const float* __restrict__ w,
                                const IO* __restrict__ conv_in, const IO* __restrict__ dy,
                                const float* __restrict__ dconv_out, IO* __restrict__ dx,
                                float* __restrict__ dconv_in, float* __restrict__ part) {
    const int c = 2 * threadIdx.x, bh = blockIdx.y, h = bh % s.H, K = s.K;
    const int t0 = blockIdx.x * kConvChunk, t1 = min(s.T, t0 + kConvChunk);
    const IO* xb = x + bh * s.hs;
    const IO* dyb = dy + bh * s.hs;
    const IO* cib = conv_in ? conv_in + (size_t)bh * (K - 1) * s.d : nullptr;
    const float* dcob = dconv_out ? dconv_out + (size_t)bh * (K - 1) * s.d : nullptr;
    float w0[kMaxTaps], w1[kMaxTaps];
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j) {
        w0[j] = j < K ? w[((size_t)h * s.d + c) * K + j] : 0.f;
        w1[j] = j < K ? w[((size_t)h * s.d + c + 1) * K + j] : 0.f;
    }
    // delta_t for t in [0, T): dy_t act'(pre_t)
    auto delta = [&](int t) {
        float p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxTaps; ++j)
            if (j < K) {
                const float2 xv = xe2(xb, cib, t - j, K, s.d, c);
                p0 = fmaf(w0[j], xv.x, p0);
                p1 = fmaf(w1[j], xv.y, p1);
            }
        const float2 g = ld2(dyb + (size_t)t * s.d + c);
        return make_float2(g.x * dact_f<ACT>(p0), g.y * dact_f<ACT>(p1));
    };
    // dwin[j] = delta_{p+j} (0 outside [0, T)) once shifted at the top of the
    // loop: before the first position it holds delta_{t1}, delta_{t1+1}, ...
    // (the next chunk's first K-1 positions, recomputed here)
    float2 dwin[kMaxTaps];
#pragma unroll
    for (int i = 0; i < kMaxTaps; ++i)
        dwin[i] = (i < K - 1 && t1 + i < s.T) ? delta(t1 + i) : make_float2(0.f, 0.f);
    float a0[kMaxTaps], a1[kMaxTaps];  // weight-gradient partial of this chunk
#pragma unroll
    for (int j = 0; j < kMaxTaps; ++j) a0[j] = a1[j] = 0.f;
    const int lo = blockIdx.x == 0 ? -(K - 1) : t0;
    for (int p = t1 - 1; p >= lo; --p) {
#pragma unroll
        for (int j = kMaxTaps - 1; j > 0; --j) dwin[j] = dwin[j - 1];
        dwin[0] = p >= 0 ? delta(p) : make_float2(0.f, 0.f);
        float g0 = 0.f, g1 = 0.f;
        if (dcob && p >= s.T - K + 1) {
            const float* q = dcob + (size_t)(p - (s.T - K + 1)) * s.d + c;
            g0 = q[0];
            g1 = q[1];
        }
#pragma unroll
        for (int j = kMaxTaps - 1; j >= 0; --j)
            if (j < K && p + j >= 0 && p + j < s.T) {
                g0 = fmaf(w0[j], dwin[j].x, g0);
                g1 = fmaf(w1[j], dwin[j].y, g1);
            }
        if (p >= 0) {
            st2(dx + bh * s.hs + (size_t)p * s.d + c, make_float2(g0, g1));
#pragma unroll
            for (int j = 0; j < kMaxTaps; ++j)
                if (j < K) {
                    const float2 xv = xe2(xb, cib, p - j, K, s.d, c);
                    a0[j] = fmaf(dwin[0].x, xv.x, a0[j]);
                    a1[j] = fmaf(dwin[0].y, xv.y, a1[j]);
                }
        } else {
            float* q = dconv_in + ((size_t)bh * (K - 1) + (p + K - 1)) * s.d + c;
            q[0] = g0;
            q[1] = g1;
        }
    }
    float* pb = part + (((size_t)blockIdx.x * s.BH + bh) * s.d + c) * K;
    for (int j = 0; j < K; ++j) {
        pb[j] = a0[j];
        pb[K + j] = a1[j];
    }
}

// dconv_in for T == 0 and the chunk-0 positions when there is no token: the
// state gradient passes through (dconv_in = dconv_out).
__global__ void conv_pass_kernel(int n, const float* __restrict__ src, float* __restrict__ dst) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = src ? src[i] : 0.f;
}

// dw_out[h][c][j] = dw_in + the partials, chunks descending, batches ascending.
__global__ void conv_dw_fold_kernel(ConvView s, int B, const float* __restrict__ part,
                                    const float* __restrict__ dw_in, float* __restrict__ dw_out) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;  // (h, c, j)
    const int n = s.H * s.d * s.K;
    if (i >= n) return;
    const int h = i / (s.d * s.K), rem = i % (s.d * s.K);
    float acc = dw_in ? dw_in[i] : 0.f;
    for (int ch = s.NC - 1; ch >= 0; --ch)
        for (int b = 0; b < B; ++b) acc += part[((size_t)ch * s.BH + (size_t)b * s.H + h) * s.d * s.K + rem];
    dw_out[i] = acc;
}

bool conv_shape_ok(const sf_conv_shape* s) {
    return s && s->B >= 0 && s->H >= 0 && s->T >= 0 && (s->io == SF_F32 || s->io == SF_BF16) &&
           (s->act == 0 || s->act == 1);
}
bool conv_supported(const sf_conv_shape* s) {
    return s->d >= 2 && s->d <= 1024 && s->d % 2 == 0 && s->K >= 2 && s->K <= kMaxTaps &&
           (long long)s->B * s->H <= 65535;
}
ConvView conv_view(const sf_conv_shape& s, int T, long long T_full) {
    ConvView v{};
    v.BH = s.B * s.H;
    v.H = s.H;
    v.T = T;
    v.d = s.d;
    v.K = s.K;
    v.NC = (T + kConvChunk - 1) / kConvChunk;
    v.hs = T_full * s.d;
    return v;
}
size_t conv_ws(const sf_conv_shape& s, int T) {
    const size_t nc = (T + kConvChunk - 1) / kConvChunk;
    return nc * (size_t)s.B * s.H * s.d * s.K * sizeof(float);
}
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }
bool all_al8(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (p && !al8(p)) return false;
    return true;
}

cudaError_t fwd_launch(const sf_conv_shape& sh, const ConvView& v, const void* x, const float* w,
                       const void* ci, void* y, void* co, cudaStream_t st) {
    const dim3 grid(v.NC, v.BH);
    const int nt = v.d / 2;
    if (v.NC > 0) {
        if (sh.io == SF_BF16) {
            auto* xx = static_cast<const __nv_bfloat16*>(x);
            auto* cc = static_cast<const __nv_bfloat16*>(ci);
            auto* yy = static_cast<__nv_bfloat16*>(y);
            if (sh.act) SF_LAUNCH("conv_fwd", st, conv_fwd_kernel<__nv_bfloat16, 1><<<grid, nt, 0, st>>>(v, xx, w, cc, yy));
            else SF_LAUNCH("conv_fwd", st, conv_fwd_kernel<__nv_bfloat16, 0><<<grid, nt, 0, st>>>(v, xx, w, cc, yy));
        } else {
            auto* xx = static_cast<const float*>(x);
            auto* cc = static_cast<const float*>(ci);
            auto* yy = static_cast<float*>(y);
            if (sh.act) SF_LAUNCH("conv_fwd", st, conv_fwd_kernel<float, 1><<<grid, nt, 0, st>>>(v, xx, w, cc, yy));
            else SF_LAUNCH("conv_fwd", st, conv_fwd_kernel<float, 0><<<grid, nt, 0, st>>>(v, xx, w, cc, yy));
        }
    }
    if (co) {
        if (sh.io == SF_BF16)
            SF_LAUNCH("conv_state", st, conv_state_kernel<__nv_bfloat16><<<v.BH, nt, 0, st>>>(
                                            v, static_cast<const __nv_bfloat16*>(x),
                                            static_cast<const __nv_bfloat16*>(ci), static_cast<__nv_bfloat16*>(co)));
        else
            SF_LAUNCH("conv_state", st, conv_state_kernel<float><<<v.BH, nt, 0, st>>>(
                                            v, static_cast<const float*>(x), static_cast<const float*>(ci),
                                            static_cast<float*>(co)));
    }
    return cudaGetLastError();
}

cudaError_t bwd_launch(const sf_conv_shape& sh, const ConvView& v, int B, const void* x, const float* w,
                       const void* ci, const void* dy, const float* dco, void* dx, const float* dw_in,
                       float* dw_out, float* dci, float* part, cudaStream_t st) {
    const int nt = v.d / 2;
    const int nstate = v.BH * (v.K - 1) * v.d;
    if (v.NC == 0) {
        if (dci) SF_LAUNCH("conv_pass", st, conv_pass_kernel<<<(nstate + 255) / 256, 256, 0, st>>>(nstate, dco, dci));
    } else {
        // dconv_in is written by chunk 0; without a caller buffer it goes to the
        // workspace's spare state slot
        const dim3 grid(v.NC, v.BH);
        if (sh.io == SF_BF16) {
            auto* xx = static_cast<const __nv_bfloat16*>(x);
            auto* cc = static_cast<const __nv_bfloat16*>(ci);
            auto* gy = static_cast<const __nv_bfloat16*>(dy);
            auto* gx = static_cast<__nv_bfloat16*>(dx);
            if (sh.act) SF_LAUNCH("conv_bwd", st, conv_bwd_kernel<__nv_bfloat16, 1><<<grid, nt, 0, st>>>(v, xx, w, cc, gy, dco, gx, dci, part));
            else SF_LAUNCH("conv_bwd", st, conv_bwd_kernel<__nv_bfloat16, 0><<<grid, nt, 0, st>>>(v, xx, w, cc, gy, dco, gx, dci, part));
        } else {
            auto* xx = static_cast<const float*>(x);
            auto* cc = static_cast<const float*>(ci);
            auto* gy = static_cast<const float*>(dy);
            auto* gx = static_cast<float*>(dx);
            if (sh.act) SF_LAUNCH("conv_bwd", st, conv_bwd_kernel<float, 1><<<grid, nt, 0, st>>>(v, xx, w, cc, gy, dco, gx, dci, part));
            else SF_LAUNCH("conv_bwd", st, conv_bwd_kernel<float, 0><<<grid, nt, 0, st>>>(v, xx, w, cc, gy, dco, gx, dci, part));
        }
    }
    const int n = v.H * v.d * v.K;
    if (n > 0 && dw_out)
        SF_LAUNCH("conv_dw_fold", st, conv_dw_fold_kernel<<<(n + 127) / 128, 128, 0, st>>>(v, B, part, dw_in, dw_out));
    return cudaGetLastError();
}

sf_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SF_OK : SF_ERR_CUDA; }

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" {

size_t sf_conv_workspace_bytes(const sf_conv_shape* s) {
    if (!conv_shape_ok(s) || !conv_supported(s)) return 0;
    // the weight-gradient partials plus one spare state-gradient slot
    return align_up(conv_ws(*s, s->T), 256) + align_up((size_t)s->B * s->H * (s->K - 1) * s->d * 4, 256) + 256;
}

sf_status sf_conv_fwd(const sf_conv_shape* s, const void* x, const float* w, const void* conv_in, void* y,
                      void* conv_out, void* stream) {
    if (!conv_shape_ok(s)) return SF_ERR_INVALID_ARG;
    if (!conv_supported(s)) return SF_ERR_UNSUPPORTED;
    const bool empty = (long long)s->B * s->H == 0;
    if (!empty && (!w || (s->T > 0 && (!x || !y)))) return SF_ERR_INVALID_ARG;
    if (!all_al8({x, w, conv_in, y, conv_out})) return SF_ERR_ALIGNMENT;
    if (empty) return SF_OK;
    const ConvView v = conv_view(*s, s->T, s->T);
    return cuda_status(fwd_launch(*s, v, x, w, conv_in, y, conv_out, static_cast<cudaStream_t>(stream)));
}

sf_status sf_conv_bwd(const sf_conv_shape* s, const void* x, const float* w, const void* conv_in, const void* dy,
                      const float* dconv_out, void* dx, const float* dw_in, float* dw_out, float* dconv_in,
                      void* ws, size_t ws_bytes, void* stream) {
    if (!conv_shape_ok(s)) return SF_ERR_INVALID_ARG;
    if (!conv_supported(s)) return SF_ERR_UNSUPPORTED;
    const bool empty = (long long)s->B * s->H == 0;
    if (!empty && (!w || !dw_out || (s->T > 0 && (!x || !dy || !dx)))) return SF_ERR_INVALID_ARG;
    if (!all_al8({x, w, conv_in, dy, dconv_out, dx, dw_in, dw_out, dconv_in})) return SF_ERR_ALIGNMENT;
    const size_t need = sf_conv_workspace_bytes(s);
    if (!ws || ws_bytes < need) return SF_ERR_WORKSPACE;
    if (!al16(ws)) return SF_ERR_ALIGNMENT;
    if (empty) return SF_OK;
    char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
    float* part = reinterpret_cast<float*>(base);
    float* spare = reinterpret_cast<float*>(base + align_up(conv_ws(*s, s->T), 256));
    const ConvView v = conv_view(*s, s->T, s->T);
    return cuda_status(bwd_launch(*s, v, s->B, x, w, conv_in, dy, dconv_out, dx, dw_in, dw_out,
                                  dconv_in ? dconv_in : spare, part, static_cast<cudaStream_t>(stream)));
}

size_t sf_conv_segment_workspace_bytes(const sf_conv_shape* s, int N, const int* seg_len) {
    if (!conv_shape_ok(s) || !conv_supported(s) || N <= 0) return 0;
    long long sum = 0;
    int lmax = 0;
    for (int i = 0; i < N; ++i) {
        const int L = seg_len ? seg_len[i] : s->T / N + (i < s->T % N ? 1 : 0);
        if (L < 0) return 0;
        sum += L;
        lmax = L > lmax ? L : lmax;
    }
    if (sum != s->T) return 0;
    const size_t es = s->io == SF_BF16 ? 2 : 4;
    const size_t nstate = (size_t)s->B * s->H * (s->K - 1) * s->d;
    sf_conv_shape one = *s;
    one.T = lmax;
    // N+1 boundary states (I/O dtype), two state gradients (fp32), the per-segment workspace
    return align_up(nstate * es, 256) * (N + 1) + align_up(nstate * 4, 256) * 2 + sf_conv_workspace_bytes(&one);
}

sf_status sf_conv_segment_run(const sf_conv_shape* s, int N, const int* seg_len, const void* x, const float* w,
                              const void* conv_in, const void* dy, const float* dconv_out, void* y,
                              void* conv_out, void* dx, float* dw, float* dconv_in, void* ws, size_t ws_bytes,
                              void* stream) {
    if (!conv_shape_ok(s) || N <= 0) return SF_ERR_INVALID_ARG;
    if (!conv_supported(s)) return SF_ERR_UNSUPPORTED;
    const size_t need = sf_conv_segment_workspace_bytes(s, N, seg_len);
    if (need == 0) return SF_ERR_INVALID_ARG;
    const bool empty = (long long)s->B * s->H == 0;
    if (!empty && (!w || (s->T > 0 && (!x || !y)) || (dy && (!dw || (s->T > 0 && !dx)))))
        return SF_ERR_INVALID_ARG;
    if (!all_al8({x, w, conv_in, dy, dconv_out, y, conv_out, dx, dw, dconv_in})) return SF_ERR_ALIGNMENT;
    if (!ws || ws_bytes < need) return SF_ERR_WORKSPACE;
    if (!al16(ws)) return SF_ERR_ALIGNMENT;
    if (empty) return SF_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t es = s->io == SF_BF16 ? 2 : 4;
    const size_t nstate = (size_t)s->B * s->H * (s->K - 1) * s->d;
    char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
    const size_t sstr = align_up(nstate * es, 256), gstr = align_up(nstate * 4, 256);
    auto state = [&](int i) { return static_cast<void*>(base + sstr * i); };
    float* gA = reinterpret_cast<float*>(base + sstr * (N + 1));
    float* gB = reinterpret_cast<float*>(base + sstr * (N + 1) + gstr);
    float* part = reinterpret_cast<float*>(base + sstr * (N + 1) + 2 * gstr);
    std::vector<int> lens(N);
    std::vector<long long> t0(N);
    long long t = 0;
    for (int i = 0; i < N; ++i) {
        lens[i] = seg_len ? seg_len[i] : s->T / N + (i < s->T % N ? 1 : 0);
        t0[i] = t;
        t += lens[i];
    }
    auto at = [&](const void* p, long long tok) {
        return p ? static_cast<const void*>(static_cast<const char*>(p) + (size_t)tok * s->d * es) : p;
    };
    auto atm = [&](void* p, long long tok) {
        return p ? static_cast<void*>(static_cast<char*>(p) + (size_t)tok * s->d * es) : p;
    };
    cudaError_t e = conv_in ? cudaMemcpyAsync(state(0), conv_in, nstate * es, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(state(0), 0, nstate * es, st);
    for (int i = 0; i < N && e == cudaSuccess; ++i) {
        sf_conv_shape one = *s;
        one.T = lens[i];
        const ConvView v = conv_view(one, lens[i], s->T);
        e = fwd_launch(one, v, at(x, t0[i]), w, state(i), atm(y, t0[i]), state(i + 1), st);
    }
    if (e == cudaSuccess && conv_out)
        e = cudaMemcpyAsync(conv_out, state(N), nstate * es, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && dy) {
        float* cur = gA;
        float* nxt = gB;
        e = dconv_out ? cudaMemcpyAsync(cur, dconv_out, nstate * 4, cudaMemcpyDeviceToDevice, st)
                      : cudaMemsetAsync(cur, 0, nstate * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dw, 0, (size_t)s->H * s->d * s->K * 4, st);
        for (int i = N - 1; i >= 0 && e == cudaSuccess; --i) {
            sf_conv_shape one = *s;
            one.T = lens[i];
            const ConvView v = conv_view(one, lens[i], s->T);
            e = bwd_launch(one, v, s->B, at(x, t0[i]), w, state(i), at(dy, t0[i]), cur, atm(dx, t0[i]), dw, dw,
                           nxt, part, st);
            float* tmp = cur;
            cur = nxt;
            nxt = tmp;
        }
        if (e == cudaSuccess && dconv_in) e = cudaMemcpyAsync(dconv_in, cur, nstate * 4, cudaMemcpyDeviceToDevice, st);
    }
    return cuda_status(e);
}

}  // extern "C"
