// Delta rule with a per-channel (diagonal) decay: the diagonal-plus-low-rank
// member of the structured transitions StateFlow lists (arXiv 2608.06838,
// section 2.1: Kimi Delta Attention's F_t), in the state orientation of this
// library (S in R^{dk x dv}, rows = key channels):
//     S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T,  o_t = scale S_t^T q_t
//     (beta off: S_t = Diag(exp(g_t)) S_{t-1} + k_t v_t^T)
// with g_t in R^{dk}.  This family is fp32 on the CUDA cores, token by token:
// with an independent decay per channel the chunked (WY) form needs the pairwise
// factors exp(G_ic - G_jc) per channel, and the workloads' decay (about -2.2 per
// token) takes exp(-G) out of fp32 range within one chunk, so the recurrence is
// run as it is defined.  The columns of S are independent, so a CTA owns one
// head and 32 state columns: warp w holds key rows DK/8 * w.., lane j holds
// column j; the per-token sums over the key rows (u = S'^T k, o = S^T q,
// w = D^T k) go through shared memory in a fixed warp order.
// Backward: the forward is replayed from checkpoints every 64 tokens (a first
// pass stores them), each 64-token window's states go to an L2-resident
// scratch, and the reverse-time adjoint runs over the window; the sums over
// state columns (dq, dk, dg, dbeta) are written per 32-column block and added
// in block order by a second kernel.  Every sum has a fixed order, so the
// results do not depend on where a sequence is split.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>

#include "../../include/sf_gdn.h"
#include "sf_common.cuh"

namespace sf {
namespace {

constexpr int kWin = 64;     // tokens per staged window and per checkpoint
constexpr int kCols = 32;    // state columns per CTA
constexpr int kWarps = 8;    // warps per CTA

struct KView {
    int BH, T, dk, dv, NB, use_beta;
    float scale;
};

template <typename IO>
__device__ __forceinline__ float ldf(const IO* p) {
    return sf::ld(p);
}

// Per-window staging of the token data the CTA needs (fp32).
template <int DK>
struct Stage {
    float k[kWin][DK], q[kWin][DK], a[kWin][DK];  // a = exp(g)
    float v[kWin][kCols], dO[kWin][kCols];
    float b[kWin];
};

template <int DK, typename IO>
__device__ void stage_window(Stage<DK>& st, const KView& s, int bh, int c0, int t0, int n, const IO* q,
                             const IO* k, const IO* v, const float* g, const float* beta, const IO* dO) {
    const int tid = threadIdx.x;
    for (int e = tid; e < kWin * DK; e += kWarps * 32) {
        const int i = e / DK, c = e % DK;
        const bool ok = i < n;
        const size_t o = ((size_t)bh * s.T + t0 + i) * DK + c;
        st.k[i][c] = ok ? ldf(k + o) : 0.f;
        st.q[i][c] = ok ? ldf(q + o) : 0.f;
        st.a[i][c] = ok ? __expf(g[o]) : 1.f;
    }
    for (int e = tid; e < kWin * kCols; e += kWarps * 32) {
        const int i = e / kCols, j = e % kCols;
        const bool ok = i < n;
        const size_t o = ((size_t)bh * s.T + t0 + i) * s.dv + c0 + j;
        st.v[i][j] = ok ? ldf(v + o) : 0.f;
        if (dO) st.dO[i][j] = ok ? ldf(dO + o) : 0.f;
    }
    for (int i = tid; i < kWin; i += kWarps * 32)
        st.b[i] = (s.use_beta && i < n) ? beta[(size_t)bh * s.T + t0 + i] : 0.f;
}

// Sum over the key rows of per-warp partials: red[w][lane] -> every thread of column lane.
__device__ __forceinline__ float rows_sum(float* red, float part, int w, int lane) {
    red[w * 32 + lane] = part;
    __syncthreads();
    float x = 0.f;
#pragma unroll
    for (int u = 0; u < kWarps; ++u) x += red[u * 32 + lane];
    __syncthreads();
    return x;
}

// One token of the forward on this thread's R rows of column j.
template <int R>
__device__ __forceinline__ void fwd_token(float (&S)[R], const float* k, const float* a, float v, float b,
                                          bool use_beta, float* red, int w, int lane) {
    float pu = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        S[r] *= a[r];
        pu = fmaf(k[r], S[r], pu);
    }
    if (use_beta) {
        const float u = rows_sum(red, pu, w, lane);
        const float d = b * (v - u);
#pragma unroll
        for (int r = 0; r < R; ++r) S[r] = fmaf(k[r], d, S[r]);
    } else {
#pragma unroll
        for (int r = 0; r < R; ++r) S[r] = fmaf(k[r], v, S[r]);
    }
}

template <int DK, typename IO>
__global__ void __launch_bounds__(kWarps * 32, 1)
kda_fwd_kernel(KView s, const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
               const float* __restrict__ g, const float* __restrict__ beta, const float* __restrict__ S_in,
               IO* __restrict__ o, float* __restrict__ S_out, float* __restrict__ ckpt) {
    constexpr int R = DK / kWarps;
    extern __shared__ __align__(16) unsigned char smem[];
    Stage<DK>& sg = *reinterpret_cast<Stage<DK>*>(smem);
    float* red = reinterpret_cast<float*>(smem + sizeof(Stage<DK>));
    const int bh = blockIdx.x / s.NB, c0 = (blockIdx.x % s.NB) * kCols;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, j = c0 + lane, r0 = w * R;
    float S[R];
#pragma unroll
    for (int r = 0; r < R; ++r) S[r] = S_in ? S_in[((size_t)bh * DK + r0 + r) * s.dv + j] : 0.f;
    for (int t0 = 0; t0 < s.T; t0 += kWin) {
        const int n = min(kWin, s.T - t0);
        if (ckpt) {
            float* cp = ckpt + (((size_t)bh * ((s.T + kWin - 1) / kWin) + t0 / kWin) * DK + r0) * s.dv + j;
#pragma unroll
            for (int r = 0; r < R; ++r) cp[(size_t)r * s.dv] = S[r];
        }
        __syncthreads();  // the previous window's stage is no longer read
        stage_window<DK, IO>(sg, s, bh, c0, t0, n, q, k, v, g, beta, nullptr);
        __syncthreads();
        for (int i = 0; i < n; ++i) {
            fwd_token<R>(S, &sg.k[i][r0], &sg.a[i][r0], sg.v[i][lane], sg.b[i], s.use_beta, red, w, lane);
            if (o) {
                float po = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) po = fmaf(sg.q[i][r0 + r], S[r], po);
                const float ov = rows_sum(red, po, w, lane);
                if (w == 0) sf::st(o + ((size_t)bh * s.T + t0 + i) * s.dv + j, s.scale * ov);
            }
        }
    }
    if (S_out) {
#pragma unroll
        for (int r = 0; r < R; ++r) S_out[((size_t)bh * DK + r0 + r) * s.dv + j] = S[r];
    }
}

// Backward.  Pass 1 (the forward kernel above, ckpt != NULL, o == NULL) wrote
// the state at the start of every window.  Per window, last first: stage the
// token data, replay the window forward into the scratch (the state before
// each token), then run the adjoint over the window in reverse.
template <int DK, typename IO>
__global__ void __launch_bounds__(kWarps * 32, 1)
kda_bwd_kernel(KView s, const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
               const float* __restrict__ g, const float* __restrict__ beta, const IO* __restrict__ dO,
               const float* __restrict__ dS_out, const float* __restrict__ ckpt, float* __restrict__ scratch,
               IO* __restrict__ dv, float* __restrict__ dS_in, float* __restrict__ part) {
    constexpr int R = DK / kWarps;
    extern __shared__ __align__(16) unsigned char smem[];
    Stage<DK>& sg = *reinterpret_cast<Stage<DK>*>(smem);
    float* red = reinterpret_cast<float*>(smem + sizeof(Stage<DK>));
    const int bh = blockIdx.x / s.NB, nb = blockIdx.x % s.NB, c0 = nb * kCols;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, j = c0 + lane, r0 = w * R;
    const int nck = (s.T + kWin - 1) / kWin;
    // scratch of this CTA: [kWin + 1][threads][R] (state before token i of the window)
    float* scr = scratch + (size_t)blockIdx.x * (kWin + 1) * kWarps * 32 * R + threadIdx.x * R;
    auto scr_at = [&](int i) { return scr + (size_t)i * kWarps * 32 * R; };
    // partial sums of this column block: [4][BH][T][DK]-style planes: dq, dk, dg ([T][DK]) and dbeta ([T])
    const size_t plane = (size_t)s.BH * s.T * DK;
    float* pq = part + ((size_t)nb * 3 + 0) * plane;
    float* pk = part + ((size_t)nb * 3 + 1) * plane;
    float* pg = part + ((size_t)nb * 3 + 2) * plane;
    float* pb = part + (size_t)s.NB * 3 * plane + (size_t)nb * s.BH * s.T;
    float D[R];
#pragma unroll
    for (int r = 0; r < R; ++r) D[r] = dS_out ? dS_out[((size_t)bh * DK + r0 + r) * s.dv + j] : 0.f;
    for (int wi = nck - 1; wi >= 0; --wi) {
        const int t0 = wi * kWin, n = min(kWin, s.T - t0);
        __syncthreads();
        stage_window<DK, IO>(sg, s, bh, c0, t0, n, q, k, v, g, beta, dO);
        __syncthreads();
        {  // replay
            float S[R];
            const float* cp = ckpt + (((size_t)bh * nck + wi) * DK + r0) * s.dv + j;
#pragma unroll
            for (int r = 0; r < R; ++r) S[r] = cp[(size_t)r * s.dv];
            for (int i = 0; i < n; ++i) {
                float* o = scr_at(i);
#pragma unroll
                for (int r = 0; r < R; ++r) o[r] = S[r];
                fwd_token<R>(S, &sg.k[i][r0], &sg.a[i][r0], sg.v[i][lane], sg.b[i], s.use_beta, red, w, lane);
            }
            float* o = scr_at(n);
#pragma unroll
            for (int r = 0; r < R; ++r) o[r] = S[r];
        }
        for (int i = n - 1; i >= 0; --i) {
            const size_t tok = (size_t)bh * s.T + t0 + i;
            const float* kk = &sg.k[i][r0];
            const float* qq = &sg.q[i][r0];
            const float* aa = &sg.a[i][r0];
            const float dOj = sg.dO[i][lane], vj = sg.v[i][lane], b = sg.b[i];
            float Sp[R], St[R];
            {
                const float* sp = scr_at(i);
                const float* stt = scr_at(i + 1);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    Sp[r] = sp[r];  // S_{t-1}
                    St[r] = stt[r];
                }
            }
            // D = carry + scale q dO^T; w = D^T k; u = (Diag(a) S_{t-1})^T k
            float pw = 0.f, pu = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                D[r] = fmaf(s.scale * qq[r], dOj, D[r]);
                pw = fmaf(kk[r], D[r], pw);
                pu = fmaf(kk[r], aa[r] * Sp[r], pu);
            }
            const float wj = rows_sum(red, pw, w, lane);
            const float uj = s.use_beta ? rows_sum(red, pu, w, lane) : 0.f;
            if (w == 0) sf::st(dv + tok * s.dv + j, s.use_beta ? b * wj : wj);
            // per-row terms, summed over this block's 32 columns by the warp
            float dqr[R], dkr[R], dgr[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float sp = aa[r] * Sp[r];  // S'
                dqr[r] = s.scale * St[r] * dOj;
                float dsp;
                if (s.use_beta) {
                    dkr[r] = b * (D[r] * (vj - uj) - sp * wj);
                    dsp = D[r] - b * kk[r] * wj;
                } else {
                    dkr[r] = D[r] * vj;
                    dsp = D[r];
                }
                dgr[r] = aa[r] * dsp * Sp[r];
                D[r] = aa[r] * dsp;  // carry to the previous token
            }
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    dqr[r] += __shfl_xor_sync(0xffffffffu, dqr[r], off);
                    dkr[r] += __shfl_xor_sync(0xffffffffu, dkr[r], off);
                    dgr[r] += __shfl_xor_sync(0xffffffffu, dgr[r], off);
                }
            if (lane < R) {  // lane r writes row r0 + r (registers indexed by a constant after the unroll)
#pragma unroll
                for (int r = 0; r < R; ++r)
                    if (lane == r) {
                        pq[tok * DK + r0 + r] = dqr[r];
                        pk[tok * DK + r0 + r] = dkr[r];
                        pg[tok * DK + r0 + r] = dgr[r];
                    }
            }
            if (s.use_beta) {
                float db = wj * (vj - uj);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) db += __shfl_xor_sync(0xffffffffu, db, off);
                if (w == 0 && lane == 0) pb[tok] = db;
            }
        }
    }
    if (dS_in) {
#pragma unroll
        for (int r = 0; r < R; ++r) dS_in[((size_t)bh * DK + r0 + r) * s.dv + j] = D[r];
    }
}

// dq, dk, dg, dbeta = the column blocks' partial sums, added in block order.
template <typename IO>
__global__ void kda_sum_kernel(KView s, const float* __restrict__ part, IO* __restrict__ dq, IO* __restrict__ dk,
                               float* __restrict__ dg, float* __restrict__ dbeta) {
    const size_t plane = (size_t)s.BH * s.T * s.dk;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < plane) {
        float a = 0.f, b = 0.f, c = 0.f;
        for (int nb = 0; nb < s.NB; ++nb) {
            a += part[((size_t)nb * 3 + 0) * plane + i];
            b += part[((size_t)nb * 3 + 1) * plane + i];
            c += part[((size_t)nb * 3 + 2) * plane + i];
        }
        sf::st(dq + i, a);
        sf::st(dk + i, b);
        dg[i] = c;
    }
    if (s.use_beta && i < (size_t)s.BH * s.T) {
        float d = 0.f;
        for (int nb = 0; nb < s.NB; ++nb) d += part[(size_t)s.NB * 3 * plane + (size_t)nb * s.BH * s.T + i];
        dbeta[i] = d;
    }
}

template <int DK>
constexpr size_t kda_smem() { return sizeof(Stage<DK>) + kWarps * 32 * 4; }

bool kda_ok(const sf_kda_shape* s) {
    return s && s->B >= 0 && s->H >= 0 && s->T >= 0 && (s->io == SF_F32 || s->io == SF_BF16) &&
           (s->use_beta == 0 || s->use_beta == 1) && s->scale == s->scale;
}
bool kda_supported(const sf_kda_shape* s) {
    return (s->dk == 32 || s->dk == 64 || s->dk == 128) && s->dv >= kCols && s->dv % kCols == 0 && s->dv <= 1024 &&
           (long long)s->B * s->H * (s->dv / kCols) <= 65535 * 32;
}
KView kview(const sf_kda_shape& s) {
    return KView{s.B * s.H, s.T, s.dk, s.dv, s.dv / kCols, s.use_beta, s.scale};
}
struct KdaWs {
    float* ckpt;
    float* scratch;
    float* part;
    size_t total;
};
KdaWs kda_layout(const sf_kda_shape& s, char* base) {
    KdaWs w{};
    const KView v = kview(s);
    const size_t nck = (size_t)(s.T + kWin - 1) / kWin;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* p = base ? base + off : nullptr;
        off = align_up(off + bytes, 256);
        return reinterpret_cast<float*>(p);
    };
    w.ckpt = take((size_t)v.BH * nck * s.dk * s.dv * 4);
    w.scratch = take((size_t)v.BH * v.NB * (kWin + 1) * kWarps * 32 * (s.dk / kWarps) * 4);
    w.part = take(((size_t)v.NB * 3 * v.BH * s.T * s.dk + (size_t)v.NB * v.BH * s.T) * 4);
    w.total = off + 256;
    return w;
}

template <int DK, typename IO>
cudaError_t kda_fwd_launch(const KView& v, const void* q, const void* k, const void* vv, const float* g,
                           const float* beta, const float* S_in, void* o, float* S_out, float* ckpt,
                           cudaStream_t st) {
    constexpr size_t sm = kda_smem<DK>();
    cudaError_t e = cudaFuncSetAttribute(kda_fwd_kernel<DK, IO>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    SF_LAUNCH("kda_fwd", st, kda_fwd_kernel<DK, IO><<<v.BH * v.NB, kWarps * 32, sm, st>>>(
                                 v, static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(vv),
                                 g, beta, S_in, static_cast<IO*>(o), S_out, ckpt));
    return cudaGetLastError();
}

template <int DK, typename IO>
cudaError_t kda_bwd_launch(const KView& v, const void* q, const void* k, const void* vv, const float* g,
                           const float* beta, const float* S_in, const void* dO, const float* dS_out, void* dq,
                           void* dk, void* dvv, float* dg, float* dbeta, float* dS_in, const KdaWs& w,
                           cudaStream_t st) {
    cudaError_t e = kda_fwd_launch<DK, IO>(v, q, k, vv, g, beta, S_in, nullptr, nullptr, w.ckpt, st);
    if (e != cudaSuccess) return e;
    constexpr size_t sm = kda_smem<DK>();
    e = cudaFuncSetAttribute(kda_bwd_kernel<DK, IO>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    SF_LAUNCH("kda_bwd", st, kda_bwd_kernel<DK, IO><<<v.BH * v.NB, kWarps * 32, sm, st>>>(
                                 v, static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(vv),
                                 g, beta, static_cast<const IO*>(dO), dS_out, w.ckpt, w.scratch,
                                 static_cast<IO*>(dvv), dS_in, w.part));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t n = (size_t)v.BH * v.T * v.dk;
    SF_LAUNCH("kda_sum", st, kda_sum_kernel<IO><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
                                 v, w.part, static_cast<IO*>(dq), static_cast<IO*>(dk), dg, dbeta));
    return cudaGetLastError();
}

template <typename IO>
cudaError_t kda_fwd_any(const KView& v, const void* q, const void* k, const void* vv, const float* g,
                        const float* beta, const float* S_in, void* o, float* S_out, cudaStream_t st) {
    switch (v.dk) {
        case 32: return kda_fwd_launch<32, IO>(v, q, k, vv, g, beta, S_in, o, S_out, nullptr, st);
        case 64: return kda_fwd_launch<64, IO>(v, q, k, vv, g, beta, S_in, o, S_out, nullptr, st);
        default: return kda_fwd_launch<128, IO>(v, q, k, vv, g, beta, S_in, o, S_out, nullptr, st);
    }
}
template <typename IO>
cudaError_t kda_bwd_any(const KView& v, const void* q, const void* k, const void* vv, const float* g,
                        const float* beta, const float* S_in, const void* dO, const float* dS_out, void* dq,
                        void* dk, void* dvv, float* dg, float* dbeta, float* dS_in, const KdaWs& w,
                        cudaStream_t st) {
    switch (v.dk) {
        case 32: return kda_bwd_launch<32, IO>(v, q, k, vv, g, beta, S_in, dO, dS_out, dq, dk, dvv, dg, dbeta, dS_in, w, st);
        case 64: return kda_bwd_launch<64, IO>(v, q, k, vv, g, beta, S_in, dO, dS_out, dq, dk, dvv, dg, dbeta, dS_in, w, st);
        default: return kda_bwd_launch<128, IO>(v, q, k, vv, g, beta, S_in, dO, dS_out, dq, dk, dvv, dg, dbeta, dS_in, w, st);
    }
}

bool a16(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (p && (reinterpret_cast<uintptr_t>(p) & 15u)) return false;
    return true;
}

}  // namespace
}  // namespace sf

using namespace sf;

extern "C" {

size_t sf_kda_workspace_bytes(const sf_kda_shape* s, int backward) {
    if (!kda_ok(s) || !kda_supported(s)) return 0;
    if (!backward || (long long)s->B * s->H * s->T == 0) return 0;
    return kda_layout(*s, nullptr).total;
}

sf_status sf_kda_fwd(const sf_kda_shape* s, const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* S_in, void* o, float* S_out, void* stream) {
    if (!kda_ok(s)) return SF_ERR_INVALID_ARG;
    if (!kda_supported(s)) return SF_ERR_UNSUPPORTED;
    const bool empty = (long long)s->B * s->H * s->T == 0;
    if (!empty && (!q || !k || !v || !g || !o || (s->use_beta && !beta))) return SF_ERR_INVALID_ARG;
    if (!s->use_beta && beta) return SF_ERR_INVALID_ARG;
    if (!a16({q, k, v, g, beta, S_in, o, S_out})) return SF_ERR_ALIGNMENT;
    if ((long long)s->B * s->H == 0) return SF_OK;
    const KView kv = kview(*s);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = s->io == SF_BF16 ? kda_fwd_any<__nv_bfloat16>(kv, q, k, v, g, beta, S_in, s->T ? o : nullptr, S_out, st)
                                           : kda_fwd_any<float>(kv, q, k, v, g, beta, S_in, s->T ? o : nullptr, S_out, st);
    return e == cudaSuccess ? SF_OK : SF_ERR_CUDA;
}

sf_status sf_kda_bwd(const sf_kda_shape* s, const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* S_in, const void* dO, const float* dS_out, void* dq, void* dk,
                     void* dv, float* dg, float* dbeta, float* dS_in, void* ws, size_t ws_bytes, void* stream) {
    if (!kda_ok(s)) return SF_ERR_INVALID_ARG;
    if (!kda_supported(s)) return SF_ERR_UNSUPPORTED;
    const bool empty = (long long)s->B * s->H * s->T == 0;
    if (!empty && (!q || !k || !v || !g || !dO || !dq || !dk || !dv || !dg || (s->use_beta && (!beta || !dbeta))))
        return SF_ERR_INVALID_ARG;
    if (!s->use_beta && (beta || dbeta)) return SF_ERR_INVALID_ARG;
    if (!a16({q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in})) return SF_ERR_ALIGNMENT;
    const size_t need = sf_kda_workspace_bytes(s, 1);
    if (need && (!ws || ws_bytes < need)) return SF_ERR_WORKSPACE;
    if (need && (reinterpret_cast<uintptr_t>(ws) & 15u)) return SF_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((long long)s->B * s->H == 0) return SF_OK;
    if (s->T == 0) {  // no token: the state gradient passes through
        if (!dS_in) return SF_OK;
        const size_t n = (size_t)s->B * s->H * s->dk * s->dv * 4;
        const cudaError_t e = dS_out ? cudaMemcpyAsync(dS_in, dS_out, n, cudaMemcpyDeviceToDevice, st)
                                     : cudaMemsetAsync(dS_in, 0, n, st);
        return e == cudaSuccess ? SF_OK : SF_ERR_CUDA;
    }
    char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
    const KdaWs w = kda_layout(*s, base);
    const KView kv = kview(*s);
    const cudaError_t e =
        s->io == SF_BF16 ? kda_bwd_any<__nv_bfloat16>(kv, q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in, w, st)
                         : kda_bwd_any<float>(kv, q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in, w, st);
    return e == cudaSuccess ? SF_OK : SF_ERR_CUDA;
}

}  // extern "C"
