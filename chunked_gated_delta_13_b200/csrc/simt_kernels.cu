// Fp32 CUDA-core kernels for the gated delta-rule chunk forward and backward.
//
// This family runs every supported shape in both I/O dtypes with fp32
// arithmetic throughout; it is the path of the fp32 I/O mode, whose tolerance
// (1e-4 against fp64) bf16 tensor-core operands cannot meet.  Each kernel is a
// direct, per-element rendering of one stage of the chunk form of StateFlow
// (arXiv 2608.06838) section 2.2, Omega_i = Pre(X_i); (S_next, V_new) =
// ST(S, Omega_i); Y_i = Out(V_new, S, Omega_i), with the Gated DeltaNet Pre
// being the UT/WY transform of the chunk:
//
//   G_i = sum_{s<=i} g_s (chunk-local), gamma_i = exp(G_i),
//   Gamma_ij = exp(G_i - G_j) for j <= i, else 0
//   A = strictly-lower(diag(beta) (K K^T * Gamma)),  Linv = (I + A)^{-1}
//   W = Linv diag(beta) (gamma * K),  U = Linv diag(beta) V
//   V_new = U - W S0;  S_C = gamma_C S0 + (K * exp(G_C - G))^T V_new
//   O = (gamma * Qs) S0 + ((Qs K^T) * Gamma) V_new,   Qs = scale * Q
//
// Backward (adjoint of the same operations; section 3.1 Bwd recomputes from
// the inputs and S_in):  prep again -> forward state recompute -> intra-chunk
// dV_new = P^T dO -> reverse state-gradient scan (dV_new += Khat dS,
// dS <- gamma_C dS + (gamma*Qs)^T dO - W^T dV_new) -> per-chunk gradients.
//
// Ragged tails: tokens past the end of the segment are treated as k = q = v = 0,
// g = 0, beta = 0, which is an exact identity step of the recurrence.
#include <algorithm>

#include "sf_common.cuh"

namespace sf {
namespace {

constexpr int kThreads = 256;
constexpr int kBV = 32;  // state columns per scan block

struct SimtWs {
    float* Gc;    // [BH, Tp]          chunk-local cumulative log-decay
    float* W;     // [BH, Tp, dk]
    float* U;     // [BH, Tp, dv]
    float* Vn;    // [BH, Tp, dv]      V_new
    float* S0;    // [BH, NC, dk, dv]  state entering each chunk
    float* Li;    // [BH, NC, C, C]    (I + A)^{-1}
    float* dVn;   // [BH, Tp, dv]
    float* dSc;   // [BH, NC, dk, dv]  gradient of the state leaving each chunk
    float* scr;   // [BH, NC, kScrMats*C*C + kScrRows*C*dk]
    size_t total;
};

constexpr int kScrMats = 6;  // QK, KK, M, dT, X, dA
constexpr int kScrRows = 4;  // dW, VdS, dOS, dKt

SimtWs simt_layout(const SeqView& s, bool backward, char* base) {
    SimtWs w{};
    const size_t BH = (size_t)s.BH, NC = (size_t)s.NC, C = (size_t)s.C;
    const size_t Tp = NC * C;
    size_t off = 0;
    auto take = [&](size_t n) {
        float* p = base ? reinterpret_cast<float*>(base + off) : nullptr;
        off = align_up(off + n * sizeof(float), 256);
        return p;
    };
    w.Gc = take(BH * Tp);
    w.W = take(BH * Tp * s.dk);
    w.U = take(BH * Tp * s.dv);
    w.Vn = take(BH * Tp * s.dv);
    w.S0 = take(BH * NC * s.dk * s.dv);
    w.Li = take(BH * NC * C * C);
    if (backward) {
        w.dVn = take(BH * Tp * s.dv);
        w.dSc = take(BH * NC * s.dk * s.dv);
        w.scr = take(BH * NC * (kScrMats * C * C + kScrRows * C * s.dk));
    }
    w.total = off + 256;  // room to align the caller's base up to 256
    return w;
}

// ---------------------------------------------------------------- Pre -----
// One block per (chunk, head).  Writes G (chunk-local cumsum), and with the
// beta path on also Linv = (I+A)^{-1}, W and U.
template <typename TI>
__global__ void __launch_bounds__(kThreads)
simt_prep_kernel(SeqView s, const TI* __restrict__ k, const TI* __restrict__ v,
                 const float* __restrict__ g, const float* __restrict__ beta,
                 float* __restrict__ Gc, float* __restrict__ Wo, float* __restrict__ Uo,
                 float* __restrict__ Lio) {
    extern __shared__ float smem[];
    const int C = s.C, dk = s.dk, dv = s.dv;
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t Tp = (size_t)s.NC * C;
    const TI* kb = k + bh * s.hs_k + (size_t)t0 * dk;
    const TI* vb = v + bh * s.hs_v + (size_t)t0 * dv;
    float* G = smem;            // [C]
    float* sb = G + C;          // [C]
    float* A = sb + C;          // [C][C]
    float* L = A + C * C;       // [C][C]
    if (tid == 0) {
        float acc = 0.f;
        for (int i = 0; i < C; ++i) {
            acc += (i < nval) ? g[bh * s.hs_g + t0 + i] : 0.f;
            G[i] = acc;
        }
    }
    for (int i = tid; i < C; i += blockDim.x)
        sb[i] = (s.use_beta && i < nval) ? beta[bh * s.hs_g + t0 + i] : 0.f;
    __syncthreads();
    for (int i = tid; i < C; i += blockDim.x) Gc[bh * Tp + t0 + i] = G[i];
    if (!s.use_beta) return;

    for (int e = tid; e < C * C; e += blockDim.x) {
        const int i = e / C, j = e % C;
        float a = 0.f;
        if (j < i && i < nval) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += ld(kb + (size_t)i * dk + d) * ld(kb + (size_t)j * dk + d);
            a = sb[i] * expf(G[i] - G[j]) * dot;
        }
        A[e] = a;
    }
    __syncthreads();
    // forward substitution, one row at a time: Linv_i = e_i - sum_{j<i} A_ij Linv_j
    for (int i = 0; i < C; ++i) {
        for (int col = tid; col < C; col += blockDim.x) {
            float x = (i == col) ? 1.f : 0.f;
            for (int j = col; j < i; ++j) x -= A[i * C + j] * L[j * C + col];
            L[i * C + col] = x;
        }
        __syncthreads();
    }
    float* Lg = Lio + ((size_t)bh * s.NC + c) * C * C;
    for (int e = tid; e < C * C; e += blockDim.x) Lg[e] = L[e];
    // W_i = sum_j Linv_ij beta_j gamma_j k_j ;  U_i = sum_j Linv_ij beta_j v_j
    for (int e = tid; e < C * dk; e += blockDim.x) {
        const int i = e / dk, d = e % dk;
        float x = 0.f;
        for (int j = 0; j <= i && j < nval; ++j)
            x += L[i * C + j] * sb[j] * expf(G[j]) * ld(kb + (size_t)j * dk + d);
        Wo[(bh * Tp + t0 + i) * dk + d] = x;
    }
    for (int e = tid; e < C * dv; e += blockDim.x) {
        const int i = e / dv, d = e % dv;
        float x = 0.f;
        for (int j = 0; j <= i && j < nval; ++j) x += L[i * C + j] * sb[j] * ld(vb + (size_t)j * dv + d);
        Uo[(bh * Tp + t0 + i) * dv + d] = x;
    }
}

// ------------------------------------------------------------- ST (fwd) ---
// One block per (state column tile, head); sequential over chunks.
template <typename TI>
__global__ void __launch_bounds__(kThreads)
simt_scan_fwd_kernel(SeqView s, const TI* __restrict__ k, const TI* __restrict__ v,
                     const float* __restrict__ Gc, const float* __restrict__ W,
                     const float* __restrict__ U, const float* __restrict__ S_in,
                     float* __restrict__ Vn, float* __restrict__ S0, float* __restrict__ S_out) {
    extern __shared__ float smem[];
    const int C = s.C, dk = s.dk, dv = s.dv;
    const int bh = blockIdx.y, tid = threadIdx.x;
    const int b0 = blockIdx.x * kBV;
    const int nb = min(kBV, dv - b0);
    const size_t Tp = (size_t)s.NC * C;
    float* S = smem;              // [dk][kBV]
    float* vn = S + dk * kBV;     // [C][kBV]
    float* dec = vn + C * kBV;    // [C]
    for (int e = tid; e < dk * kBV; e += blockDim.x) {
        const int a = e / kBV, bb = e % kBV;
        S[e] = (S_in && bb < nb) ? S_in[((size_t)bh * dk + a) * dv + b0 + bb] : 0.f;
    }
    __syncthreads();
    for (int c = 0; c < s.NC; ++c) {
        const int t0 = c * C;
        const int nval = min(C, s.T - t0);
        const float gC = Gc[bh * Tp + t0 + C - 1];
        for (int i = tid; i < C; i += blockDim.x) dec[i] = expf(gC - Gc[bh * Tp + t0 + i]);
        if (S0) {
            float* S0c = S0 + ((size_t)bh * s.NC + c) * dk * dv;
            for (int e = tid; e < dk * kBV; e += blockDim.x) {
                const int a = e / kBV, bb = e % kBV;
                if (bb < nb) S0c[(size_t)a * dv + b0 + bb] = S[e];
            }
        }
        for (int e = tid; e < C * kBV; e += blockDim.x) {
            const int i = e / kBV, bb = e % kBV;
            float x = 0.f;
            if (bb < nb && i < nval) {
                if (s.use_beta) {
                    const size_t row = bh * Tp + t0 + i;
                    x = U[row * dv + b0 + bb];
                    for (int a = 0; a < dk; ++a) x -= W[row * dk + a] * S[a * kBV + bb];
                } else {
                    x = ld(v + bh * s.hs_v + (size_t)(t0 + i) * dv + b0 + bb);
                }
                Vn[(bh * Tp + t0 + i) * dv + b0 + bb] = x;
            } else if (bb < nb) {
                Vn[(bh * Tp + t0 + i) * dv + b0 + bb] = 0.f;
            }
            vn[e] = x;
        }
        __syncthreads();
        const float gamC = expf(gC);
        const TI* kb = k + bh * s.hs_k + (size_t)t0 * dk;
        for (int e = tid; e < dk * kBV; e += blockDim.x) {
            const int a = e / kBV, bb = e % kBV;
            float x = gamC * S[e];
            for (int i = 0; i < nval; ++i) x += dec[i] * ld(kb + (size_t)i * dk + a) * vn[i * kBV + bb];
            S[e] = x;
        }
        __syncthreads();
    }
    if (S_out) {
        for (int e = tid; e < dk * kBV; e += blockDim.x) {
            const int a = e / kBV, bb = e % kBV;
            if (bb < nb) S_out[((size_t)bh * dk + a) * dv + b0 + bb] = S[e];
        }
    }
}

// ---------------------------------------------------------------- Out -----
template <typename TI>
__global__ void __launch_bounds__(kThreads)
simt_out_kernel(SeqView s, const TI* __restrict__ q, const TI* __restrict__ k,
                const float* __restrict__ Gc, const float* __restrict__ Vn,
                const float* __restrict__ S0, TI* __restrict__ o) {
    extern __shared__ float smem[];
    const int C = s.C, dk = s.dk, dv = s.dv;
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t Tp = (size_t)s.NC * C;
    const TI* qb = q + bh * s.hs_k + (size_t)t0 * dk;
    const TI* kb = k + bh * s.hs_k + (size_t)t0 * dk;
    const float* G = Gc + bh * Tp + t0;
    const float* S0c = S0 + ((size_t)bh * s.NC + c) * dk * dv;
    float* P = smem;  // [C][C]
    for (int e = tid; e < C * C; e += blockDim.x) {
        const int i = e / C, j = e % C;
        float p = 0.f;
        if (j <= i && i < nval) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += ld(qb + (size_t)i * dk + d) * ld(kb + (size_t)j * dk + d);
            p = s.scale * dot * expf(G[i] - G[j]);
        }
        P[e] = p;
    }
    __syncthreads();
    for (int e = tid; e < nval * dv; e += blockDim.x) {
        const int i = e / dv, b = e % dv;
        float inter = 0.f;
        for (int a = 0; a < dk; ++a) inter += ld(qb + (size_t)i * dk + a) * S0c[(size_t)a * dv + b];
        float x = s.scale * expf(G[i]) * inter;
        for (int j = 0; j <= i; ++j) x += P[i * C + j] * Vn[(bh * Tp + t0 + j) * dv + b];
        st(o + bh * s.hs_v + (size_t)(t0 + i) * dv + b, x);
    }
}

// -------------------------------------------------- backward: intra part ---
// dV_new_j = sum_{i >= j} P_ij dO_i  (P = (Qs K^T) * Gamma), the part of the
// value gradient that does not depend on the state gradient.
template <typename TI>
__global__ void __launch_bounds__(kThreads)
simt_bwd_intra_kernel(SeqView s, const TI* __restrict__ q, const TI* __restrict__ k,
                      const float* __restrict__ Gc, const TI* __restrict__ dO,
                      float* __restrict__ dVn) {
    extern __shared__ float smem[];
    const int C = s.C, dk = s.dk, dv = s.dv;
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t Tp = (size_t)s.NC * C;
    const TI* qb = q + bh * s.hs_k + (size_t)t0 * dk;
    const TI* kb = k + bh * s.hs_k + (size_t)t0 * dk;
    const TI* dOb = dO + bh * s.hs_v + (size_t)t0 * dv;
    const float* G = Gc + bh * Tp + t0;
    float* P = smem;
    for (int e = tid; e < C * C; e += blockDim.x) {
        const int i = e / C, j = e % C;
        float p = 0.f;
        if (j <= i && i < nval) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += ld(qb + (size_t)i * dk + d) * ld(kb + (size_t)j * dk + d);
            p = s.scale * dot * expf(G[i] - G[j]);
        }
        P[e] = p;
    }
    __syncthreads();
    for (int e = tid; e < C * dv; e += blockDim.x) {
        const int j = e / dv, b = e % dv;
        float x = 0.f;
        for (int i = j; i < nval; ++i) x += P[i * C + j] * ld(dOb + (size_t)i * dv + b);
        dVn[(bh * Tp + t0 + j) * dv + b] = x;
    }
}

// ----------------------------------------------------------- ST (bwd) -----
// Reverse chain of the state gradient, sequential over chunks from the last.
template <typename TI>
__global__ void __launch_bounds__(kThreads)
simt_scan_bwd_kernel(SeqView s, const TI* __restrict__ q, const TI* __restrict__ k,
                     const float* __restrict__ Gc, const float* __restrict__ W,
                     const TI* __restrict__ dO, const float* __restrict__ dS_out,
                     float* __restrict__ dVn, float* __restrict__ dSc, float* __restrict__ dS_in) {
    extern __shared__ float smem[];
    const int C = s.C, dk = s.dk, dv = s.dv;
    const int bh = blockIdx.y, tid = threadIdx.x;
    const int b0 = blockIdx.x * kBV;
    const int nb = min(kBV, dv - b0);
    const size_t Tp = (size_t)s.NC * C;
    float* dS = smem;              // [dk][kBV]
    float* dvn = dS + dk * kBV;    // [C][kBV]
    float* dec = dvn + C * kBV;    // [C]
    float* gam = dec + C;          // [C]
    for (int e = tid; e < dk * kBV; e += blockDim.x) {
        const int a = e / kBV, bb = e % kBV;
        dS[e] = (dS_out && bb < nb) ? dS_out[((size_t)bh * dk + a) * dv + b0 + bb] : 0.f;
    }
    __syncthreads();
    for (int c = s.NC - 1; c >= 0; --c) {
        const int t0 = c * C;
        const int nval = min(C, s.T - t0);
        const float gC = Gc[bh * Tp + t0 + C - 1];
        for (int i = tid; i < C; i += blockDim.x) {
            const float Gi = Gc[bh * Tp + t0 + i];
            dec[i] = expf(gC - Gi);
            gam[i] = expf(Gi);
        }
        float* dScc = dSc + ((size_t)bh * s.NC + c) * dk * dv;
        for (int e = tid; e < dk * kBV; e += blockDim.x) {
            const int a = e / kBV, bb = e % kBV;
            if (bb < nb) dScc[(size_t)a * dv + b0 + bb] = dS[e];
        }
        __syncthreads();
        const TI* kb = k + bh * s.hs_k + (size_t)t0 * dk;
        const TI* qb = q + bh * s.hs_k + (size_t)t0 * dk;
        const TI* dOb = dO + bh * s.hs_v + (size_t)t0 * dv;
        for (int e = tid; e < C * kBV; e += blockDim.x) {
            const int i = e / kBV, bb = e % kBV;
            float x = 0.f;
            if (bb < nb && i < nval) {
                float acc = 0.f;
                for (int a = 0; a < dk; ++a) acc += ld(kb + (size_t)i * dk + a) * dS[a * kBV + bb];
                float* p = dVn + (bh * Tp + t0 + i) * dv + b0 + bb;
                x = *p + dec[i] * acc;
                *p = x;
            }
            dvn[e] = x;
        }
        __syncthreads();
        const float gamC = expf(gC);
        for (int e = tid; e < dk * kBV; e += blockDim.x) {
            const int a = e / kBV, bb = e % kBV;
            float x = gamC * dS[e];
            if (bb < nb) {
                float acc = 0.f;
                for (int i = 0; i < nval; ++i)
                    acc += gam[i] * ld(qb + (size_t)i * dk + a) * ld(dOb + (size_t)i * dv + b0 + bb);
                x += s.scale * acc;
                if (s.use_beta) {
                    const float* Wc = W + (bh * Tp + t0) * dk;
                    float w = 0.f;
                    for (int i = 0; i < nval; ++i) w += Wc[(size_t)i * dk + a] * dvn[i * kBV + bb];
                    x -= w;
                }
            }
            dS[e] = x;
        }
        __syncthreads();
    }
    if (dS_in) {
        for (int e = tid; e < dk * kBV; e += blockDim.x) {
            const int a = e / kBV, bb = e % kBV;
            if (bb < nb) dS_in[((size_t)bh * dk + a) * dv + b0 + bb] = dS[e];
        }
    }
}

// ------------------------------------------------- backward: gradients ----
// One block per (chunk, head).  Given the state entering the chunk S0, the
// state gradient leaving it dS_C, V_new and dV_new, forms every input gradient
// of the chunk (adjoint of Pre, the intra-chunk output and the state update).
template <typename TI>
__global__ void __launch_bounds__(kThreads)
simt_grad_kernel(SeqView s, const TI* __restrict__ q, const TI* __restrict__ k,
                 const TI* __restrict__ v, const float* __restrict__ beta,
                 const TI* __restrict__ dO, const float* __restrict__ Gc,
                 const float* __restrict__ Vn, const float* __restrict__ dVn,
                 const float* __restrict__ S0, const float* __restrict__ dSc,
                 const float* __restrict__ Li, float* __restrict__ scr, TI* __restrict__ dq,
                 TI* __restrict__ dk_, TI* __restrict__ dv_, float* __restrict__ dg,
                 float* __restrict__ dbeta) {
    extern __shared__ float smem[];
    const int C = s.C, dk = s.dk, dv = s.dv;
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t Tp = (size_t)s.NC * C;
    const bool ub = s.use_beta != 0;
    const float sc = s.scale;
    const TI* qb = q + bh * s.hs_k + (size_t)t0 * dk;
    const TI* kb = k + bh * s.hs_k + (size_t)t0 * dk;
    const TI* vb = v + bh * s.hs_v + (size_t)t0 * dv;
    const TI* dOb = dO + bh * s.hs_v + (size_t)t0 * dv;
    const float* Vnc = Vn + (bh * Tp + t0) * dv;
    const float* dVnc = dVn + (bh * Tp + t0) * dv;
    const float* S0c = S0 + ((size_t)bh * s.NC + c) * dk * dv;
    const float* dSC = dSc + ((size_t)bh * s.NC + c) * dk * dv;
    const float* L = Li + ((size_t)bh * s.NC + c) * C * C;
    float* base = scr + ((size_t)bh * s.NC + c) * ((size_t)kScrMats * C * C + (size_t)kScrRows * C * dk);
    float* QK = base;
    float* KK = QK + C * C;
    float* M = KK + C * C;
    float* dT = M + C * C;
    float* X = dT + C * C;
    float* dA = X + C * C;
    float* dW = dA + C * C;
    float* VdS = dW + C * dk;
    float* dOS = VdS + C * dk;
    float* dKt = dOS + C * dk;

    float* G = smem;          // [C]
    float* gam = G + C;       // [C]
    float* dec = gam + C;     // [C]
    float* bt = dec + C;      // [C]
    float* dG = bt + C;       // [C]
    float* red = dG + C;      // [kThreads]
    for (int i = tid; i < C; i += blockDim.x) {
        G[i] = Gc[bh * Tp + t0 + i];
        bt[i] = (ub && i < nval) ? beta[bh * s.hs_g + t0 + i] : 0.f;
    }
    __syncthreads();
    const float gC = G[C - 1];
    for (int i = tid; i < C; i += blockDim.x) {
        gam[i] = expf(G[i]);
        dec[i] = expf(gC - G[i]);
    }
    __syncthreads();

    // phase 1: C x C products
    for (int e = tid; e < C * C; e += blockDim.x) {
        const int i = e / C, j = e % C;
        float qk = 0.f, kk = 0.f, m = 0.f;
        if (i < nval && j < nval) {
            for (int d = 0; d < dk; ++d) {
                const float kj = ld(kb + (size_t)j * dk + d);
                qk += ld(qb + (size_t)i * dk + d) * kj;
                kk += ld(kb + (size_t)i * dk + d) * kj;
            }
            qk *= sc;
            if (j <= i) {
                float dp = 0.f;
                for (int b = 0; b < dv; ++b) dp += ld(dOb + (size_t)i * dv + b) * Vnc[(size_t)j * dv + b];
                m = dp * expf(G[i] - G[j]);
            }
        }
        QK[e] = qk;
        KK[e] = kk;
        M[e] = m;
    }
    // phase 1b: C x dk products against the states
    for (int e = tid; e < C * dk; e += blockDim.x) {
        const int i = e / dk, a = e % dk;
        float w = 0.f, vd = 0.f, os = 0.f;
        if (i < nval) {
            for (int b = 0; b < dv; ++b) {
                const float s0 = S0c[(size_t)a * dv + b];
                w += dVnc[(size_t)i * dv + b] * s0;
                vd += Vnc[(size_t)i * dv + b] * dSC[(size_t)a * dv + b];
                os += ld(dOb + (size_t)i * dv + b) * s0;
            }
        }
        dW[e] = -w;
        VdS[e] = vd;
        dOS[e] = os;
    }
    __syncthreads();
    if (ub) {
        // phase 2: dT = dW (gamma*K)^T + dU V^T
        for (int e = tid; e < C * C; e += blockDim.x) {
            const int r = e / C, j = e % C;
            float x = 0.f;
            if (r < nval && j < nval) {
                for (int a = 0; a < dk; ++a) x += dW[r * dk + a] * gam[j] * ld(kb + (size_t)j * dk + a);
                for (int b = 0; b < dv; ++b) x += dVnc[(size_t)r * dv + b] * ld(vb + (size_t)j * dv + b);
            }
            dT[e] = x;
        }
        // phase 2b: dKt = T^T dW, T = Linv diag(beta)
        for (int e = tid; e < C * dk; e += blockDim.x) {
            const int j = e / dk, a = e % dk;
            float x = 0.f;
            for (int r = j; r < nval; ++r) x += L[r * C + j] * dW[r * dk + a];
            dKt[e] = bt[j] * x;
        }
        __syncthreads();
        // phase 3: X = Linv^T (dT diag(beta))
        for (int e = tid; e < C * C; e += blockDim.x) {
            const int i = e / C, j = e % C;
            float x = 0.f;
            for (int r = i; r < C; ++r) x += L[r * C + i] * dT[r * C + j];
            X[e] = x * bt[j];
        }
        __syncthreads();
        // phase 4: dA = strictly-lower(-X Linv^T)
        for (int e = tid; e < C * C; e += blockDim.x) {
            const int i = e / C, j = e % C;
            float x = 0.f;
            if (j < i) {
                for (int m = 0; m <= j; ++m) x += X[i * C + m] * L[j * C + m];
                x = -x;
            }
            dA[e] = x;
        }
        __syncthreads();
    }
    // phase 5: per-token reductions -> dG, dbeta
    for (int i = tid; i < C; i += blockDim.x) {
        float x = 0.f, db = 0.f;
        if (i < nval) {
            float inter = 0.f;
            for (int a = 0; a < dk; ++a) inter += ld(qb + (size_t)i * dk + a) * dOS[i * dk + a];
            x += sc * gam[i] * inter;
            for (int j = 0; j < C; ++j) x += M[i * C + j] * QK[i * C + j] - M[j * C + i] * QK[j * C + i];
            float z = 0.f;
            for (int a = 0; a < dk; ++a) z += ld(kb + (size_t)i * dk + a) * VdS[i * dk + a];
            x -= dec[i] * z;
            if (ub) {
                for (int j = 0; j < C; ++j) {
                    const float zij = (j < i) ? dA[i * C + j] * bt[i] * expf(G[i] - G[j]) : 0.f;
                    const float zji = (i < j) ? dA[j * C + i] * bt[j] * expf(G[j] - G[i]) : 0.f;
                    x += zij * KK[i * C + j] - zji * KK[j * C + i];
                }
                float kt = 0.f;
                for (int a = 0; a < dk; ++a) kt += ld(kb + (size_t)i * dk + a) * dKt[i * dk + a];
                x += gam[i] * kt;
                for (int r = 0; r < C; ++r) db += dT[r * C + i] * L[r * C + i];
                for (int j = 0; j < i; ++j) db += dA[i * C + j] * expf(G[i] - G[j]) * KK[i * C + j];
            }
        }
        dG[i] = x;
        if (ub && i < nval) dbeta[bh * s.hs_g + t0 + i] = db;
    }
    // terms of the last position: gamma_C <S0, dS_C> + sum_j z_j
    float part = 0.f;
    for (int e = tid; e < dk * dv; e += blockDim.x) part += S0c[e] * dSC[e];
    red[tid] = part;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if (tid < w) red[tid] += red[tid + w];
        __syncthreads();
    }
    if (tid == 0) {
        float zs = 0.f;
        for (int j = 0; j < nval; ++j) {
            float z = 0.f;
            for (int a = 0; a < dk; ++a) z += ld(kb + (size_t)j * dk + a) * VdS[j * dk + a];
            zs += dec[j] * z;
        }
        dG[C - 1] += expf(gC) * red[0] + zs;
        // dg_s = sum_{i >= s} dG_i
        float acc = 0.f;
        for (int i = C - 1; i >= 0; --i) {
            acc += dG[i];
            if (i < nval) dg[bh * s.hs_g + t0 + i] = acc;
        }
    }
    // phase 6: element gradients
    for (int e = tid; e < nval * dk; e += blockDim.x) {
        const int j = e / dk, a = e % dk;
        float xq = gam[j] * dOS[j * dk + a];
        for (int i = 0; i <= j; ++i) xq += M[j * C + i] * ld(kb + (size_t)i * dk + a);
        st(dq + bh * s.hs_k + (size_t)(t0 + j) * dk + a, sc * xq);
        float xk = dec[j] * VdS[j * dk + a];
        for (int i = j; i < nval; ++i) xk += M[i * C + j] * sc * ld(qb + (size_t)i * dk + a);
        if (ub) {
            xk += gam[j] * dKt[j * dk + a];
            for (int i = 0; i < nval; ++i) {
                const float zij = (j < i) ? dA[i * C + j] * bt[i] * expf(G[i] - G[j]) : 0.f;
                const float zji = (i < j) ? dA[j * C + i] * bt[j] * expf(G[j] - G[i]) : 0.f;
                xk += (zij + zji) * ld(kb + (size_t)i * dk + a);
            }
        }
        st(dk_ + bh * s.hs_k + (size_t)(t0 + j) * dk + a, xk);
    }
    for (int e = tid; e < nval * dv; e += blockDim.x) {
        const int j = e / dv, b = e % dv;
        float x;
        if (ub) {
            x = 0.f;
            for (int r = j; r < nval; ++r) x += L[r * C + j] * dVnc[(size_t)r * dv + b];
            x *= bt[j];
        } else {
            x = dVnc[(size_t)j * dv + b];
        }
        st(dv_ + bh * s.hs_v + (size_t)(t0 + j) * dv + b, x);
    }
}

template <typename F>
cudaError_t set_smem(F* kern, size_t bytes) {
    if (bytes > 48 * 1024)
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    return cudaSuccess;
}

#define SF_TRY(x)                              \
    do {                                       \
        cudaError_t e_ = (x);                  \
        if (e_ != cudaSuccess) return e_;      \
    } while (0)

template <typename TI>
cudaError_t fwd_impl(const SeqView& s, const FwdArgs& a, void* ws, cudaStream_t st) {
    char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
    SimtWs w = simt_layout(s, false, base);
    const TI* q = static_cast<const TI*>(a.q);
    const TI* k = static_cast<const TI*>(a.k);
    const TI* v = static_cast<const TI*>(a.v);
    const dim3 gc(s.NC, s.BH), gt((s.dv + kBV - 1) / kBV, s.BH);
    const size_t sm_prep = sizeof(float) * (2 * s.C + 2 * s.C * s.C);
    const size_t sm_scan = sizeof(float) * (s.dk * kBV + s.C * kBV + s.C);
    const size_t sm_out = sizeof(float) * (s.C * s.C);
    SF_TRY(set_smem(simt_prep_kernel<TI>, sm_prep));
    SF_TRY(set_smem(simt_scan_fwd_kernel<TI>, sm_scan));
    SF_TRY(set_smem(simt_out_kernel<TI>, sm_out));
    SF_LAUNCH("simt_prep", st, simt_prep_kernel<TI><<<gc, kThreads, sm_prep, st>>>(s, k, v, a.g, a.beta, w.Gc, w.W, w.U, w.Li));
    SF_TRY(cudaGetLastError());
    SF_LAUNCH("simt_scan_fwd", st, simt_scan_fwd_kernel<TI><<<gt, kThreads, sm_scan, st>>>(
        s, k, v, w.Gc, w.W, w.U, a.S_in, w.Vn, w.S0, a.S_out));
    SF_TRY(cudaGetLastError());
    SF_LAUNCH("simt_out", st, simt_out_kernel<TI><<<gc, kThreads, sm_out, st>>>(
        s, q, k, w.Gc, w.Vn, w.S0, static_cast<TI*>(a.o)));
    return cudaGetLastError();
}

template <typename TI>
cudaError_t bwd_impl(const SeqView& s, const BwdArgs& a, void* ws, cudaStream_t st) {
    char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
    SimtWs w = simt_layout(s, true, base);
    const TI* q = static_cast<const TI*>(a.q);
    const TI* k = static_cast<const TI*>(a.k);
    const TI* v = static_cast<const TI*>(a.v);
    const TI* dO = static_cast<const TI*>(a.dO);
    const dim3 gc(s.NC, s.BH), gt((s.dv + kBV - 1) / kBV, s.BH);
    const size_t sm_prep = sizeof(float) * (2 * s.C + 2 * s.C * s.C);
    const size_t sm_scan = sizeof(float) * (s.dk * kBV + s.C * kBV + s.C);
    const size_t sm_intra = sizeof(float) * (s.C * s.C);
    const size_t sm_sbwd = sizeof(float) * (s.dk * kBV + s.C * kBV + 2 * s.C);
    const size_t sm_grad = sizeof(float) * (5 * s.C + kThreads);
    SF_TRY(set_smem(simt_prep_kernel<TI>, sm_prep));
    SF_TRY(set_smem(simt_scan_fwd_kernel<TI>, sm_scan));
    SF_TRY(set_smem(simt_bwd_intra_kernel<TI>, sm_intra));
    SF_TRY(set_smem(simt_scan_bwd_kernel<TI>, sm_sbwd));
    SF_TRY(set_smem(simt_grad_kernel<TI>, sm_grad));
    SF_LAUNCH("simt_prep", st, simt_prep_kernel<TI><<<gc, kThreads, sm_prep, st>>>(s, k, v, a.g, a.beta, w.Gc, w.W, w.U, w.Li));
    SF_TRY(cudaGetLastError());
    SF_LAUNCH("simt_scan_fwd", st, simt_scan_fwd_kernel<TI><<<gt, kThreads, sm_scan, st>>>(
        s, k, v, w.Gc, w.W, w.U, a.S_in, w.Vn, w.S0, nullptr));
    SF_TRY(cudaGetLastError());
    SF_LAUNCH("simt_bwd_intra", st, simt_bwd_intra_kernel<TI><<<gc, kThreads, sm_intra, st>>>(
        s, q, k, w.Gc, dO, w.dVn));
    SF_TRY(cudaGetLastError());
    SF_LAUNCH("simt_scan_bwd", st, simt_scan_bwd_kernel<TI><<<gt, kThreads, sm_sbwd, st>>>(
        s, q, k, w.Gc, w.W, dO, a.dS_out, w.dVn, w.dSc, a.dS_in));
    SF_TRY(cudaGetLastError());
    SF_LAUNCH("simt_grad", st, simt_grad_kernel<TI><<<gc, kThreads, sm_grad, st>>>(
        s, q, k, v, a.beta, dO, w.Gc, w.Vn, w.dVn, w.S0, w.dSc, w.Li, w.scr,
        static_cast<TI*>(a.dq), static_cast<TI*>(a.dk), static_cast<TI*>(a.dv), a.dg, a.dbeta));
    return cudaGetLastError();
}

}  // namespace

size_t simt_workspace_bytes(const SeqView& s, bool backward) {
    return simt_layout(s, backward, nullptr).total;
}

cudaError_t simt_fwd(const SeqView& s, bool bf16, const FwdArgs& a, void* ws, cudaStream_t st) {
    return bf16 ? fwd_impl<__nv_bfloat16>(s, a, ws, st) : fwd_impl<float>(s, a, ws, st);
}

cudaError_t simt_bwd(const SeqView& s, bool bf16, const BwdArgs& a, void* ws, cudaStream_t st) {
    return bf16 ? bwd_impl<__nv_bfloat16>(s, a, ws, st) : bwd_impl<float>(s, a, ws, st);
}

int simt_launches(bool backward) { return backward ? 5 : 3; }

}  // namespace sf
