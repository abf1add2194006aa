// Tensor-core kernel family of libsf_gdn: bf16 I/O, fp32 state and
// accumulation, key head size 128, value head size 64 or 128, chunk length 64.
//
// Decomposition (StateFlow, arXiv 2608.06838, section 2.2: Pre / ST / Out per
// chunk; section 3.4.2: the backward stages SR, OG, STB, PG):
//   forward  : prep (Pre: UT/WY transform, also L for the gradients)
//              -> scan (ST, sequential over chunks) -> out (Out)
//   backward : prep (Pre again) -> intra (OG: dVi = P^T dO, and the
//              chain-independent term D = (gamma dO)^T Q of the reverse scan)
//              -> one launch running the forward state recompute (SR) and the
//                 reverse state-gradient scan (STB) side by side: the two
//                 chains do not depend on each other
//              -> grad (PG: every input gradient of every chunk)
//   segment chain (sf_segment_run): per segment prep, scan, out with OG fused
//              into the same launch; then per segment, in reverse, STB and PG
//              on the kept forward intermediates (no second Pre, no SR).
// With G_i = sum_{s<=i} g_s inside a chunk, gamma_i = exp(G_i),
// Gamma_ij = exp(G_i - G_j) (j <= i), Khat = K * exp(G_C - G):
//   A = strictly-lower(diag(beta)(K K^T * Gamma)), L = (I + A)^{-1}, T = L diag(beta)
//   W = T (gamma * K), U = T V;  V_new = U - W S0;  S_C = gamma_C S0 + Khat^T V_new
//   O = scale (gamma * Q) S0 + scale ((Q K^T) * Gamma) V_new
// The state chains keep S (or dS) in fp32 registers as the accumulator of
// warp-level m16n8k16 products: each 16-column slice of the state is held by a
// warp pair, so the recurrence never leaves the register file; only the
// operands (W, Khat, U or dVi and D) stream in, through bulk copies three
// (forward) or two (backward) chunks deep.
#include <algorithm>

#include "tc_kernels.cuh"
#include "tc_mma.cuh"

namespace sf {
namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int C = 64;        // chunk length
constexpr int DK = 128;      // key head size
constexpr int LDK = DK + 8;  // shared row stride of [*][DK] tiles
constexpr int LDC = C + 8;   // shared row stride of [*][C] tiles
constexpr int LDF = 72;      // shared row stride of fp32 [C][C] tiles

// Set (bit 0) by a kernel that gave up waiting for one of its own bulk copies;
// read and cleared by sf_device_check().
__device__ int g_tc_status = 0;

struct TcWs {
    float* Gc;   // [BH][Tp]           chunk-local cumulative log-decay G
    float* Gm;   // [BH][Tp]           exp(G)
    bf16* W;     // [BH][Tp][DK]       -W (negated: the scans only ever subtract W products; permuted, see swz)
    float* Lm;   // [BH][NC][C][C]     L = (I + A)^{-1} per chunk (delta path), for the gradient kernel
    bf16* Kh;    // [BH][Tp][DK]       K * exp(G_C - G) (permuted)
    bf16* Ut;    // [BH][NC][DV][C]    U transposed per chunk, V^T without the beta path (permuted)
    bf16* Vnt;   // [BH][NC][DV][C]    V_new transposed per chunk (pieces permuted, see swz)
    bf16* S0t;   // [BH][NC][DV][DK]   state entering each chunk, transposed (permuted)
    bf16* dVit;  // [BH][NC][DV][C]    intra-chunk part of dV_new, transposed (permuted)
    bf16* dVnt;  // [BH][NC][DV][C]    dV_new transposed (permuted)
    bf16* dSCt;  // [BH][NC][DV][DK]   gradient of the state leaving each chunk, transposed (permuted)
    bf16* Dt;    // [BH][NC][DV][DK]   scale (gamma * dO)^T Q per chunk, transposed (permuted)
    int* ticket;  // chunk counter of the persistent gradient kernel
    size_t total;
};

// The buffers fall in three parts: what the forward produces and the
// backward reads again (Gc .. S0t, "keep"), what the intra-chunk kernel of the
// backward produces for the reverse scan (dVit, Dt, "og"), and the reverse
// scan's own tiles (dVnt, dSCt, "slot").  A base may be null to size its part.
// Returns the bytes of each part (multiples of 256; bases 256-byte aligned).
TcWs tc_parts(const SeqView& s, char* keep, char* og, char* slot, size_t* keep_bytes, size_t* og_bytes,
              size_t* slot_bytes) {
    TcWs w{};
    const size_t BH = s.BH, NC = s.NC, Tp = NC * C, DV = s.dv;
    char* base = keep;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* p = base ? base + off : nullptr;
        off = align_up(off + bytes, 256);
        return p;
    };
    w.Gc = reinterpret_cast<float*>(take(BH * Tp * 4));
    w.Gm = reinterpret_cast<float*>(take(BH * Tp * 4));
    w.W = reinterpret_cast<bf16*>(take(s.use_beta ? BH * Tp * DK * 2 : 0));
    w.Lm = reinterpret_cast<float*>(take(s.use_beta ? BH * NC * C * C * 4 : 0));
    w.Kh = reinterpret_cast<bf16*>(take(BH * Tp * DK * 2));
    w.Ut = reinterpret_cast<bf16*>(take(BH * NC * DV * C * 2));
    w.Vnt = reinterpret_cast<bf16*>(take(BH * NC * DV * C * 2));
    w.S0t = reinterpret_cast<bf16*>(take(BH * NC * DV * DK * 2));
    if (keep_bytes) *keep_bytes = off;
    base = og;
    off = 0;
    w.dVit = reinterpret_cast<bf16*>(take(BH * NC * DV * C * 2));
    w.Dt = reinterpret_cast<bf16*>(take(BH * NC * DV * DK * 2));
    if (og_bytes) *og_bytes = off;
    base = slot;
    off = 0;
    w.dVnt = reinterpret_cast<bf16*>(take(BH * NC * DV * C * 2));
    w.dSCt = reinterpret_cast<bf16*>(take(BH * NC * DV * DK * 2));
    w.ticket = reinterpret_cast<int*>(take(sizeof(int)));
    if (slot_bytes) *slot_bytes = off;
    return w;
}

// One call's workspace: the keep part, then (backward) the og and slot parts.
TcWs tc_layout(const SeqView& s, bool backward, char* base) {
    size_t kb = 0, ob = 0, sb = 0;
    tc_parts(s, nullptr, nullptr, nullptr, &kb, &ob, &sb);
    TcWs w = tc_parts(s, base, base ? base + kb : nullptr, base ? base + kb + ob : nullptr, nullptr, nullptr,
                      nullptr);
    if (!backward) {
        w.dVit = w.dVnt = w.dSCt = w.Dt = nullptr;
        w.ticket = nullptr;
    }
    w.total = kb + (backward ? ob + sb : 0) + 256;
    return w;
}

// Inclusive cumulative sum of the 64 log-decays of a chunk by warp 0 (fixed
// shuffle order, so every launch adds in the same order).  Tokens past the end
// contribute g = 0.
__device__ __forceinline__ void chunk_cumsum(const float* g, int nval, float* Gs, int lane) {
    const float x0 = (2 * lane < nval) ? g[2 * lane] : 0.f;
    const float x1 = (2 * lane + 1 < nval) ? g[2 * lane + 1] : 0.f;
    float inc = x0 + x1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    float exc = __shfl_up_sync(0xffffffffu, inc, 1);
    if (lane == 0) exc = 0.f;
    const float a = exc + x0;
    Gs[2 * lane] = a;
    Gs[2 * lane + 1] = a + x1;
}

// (I + A)^{-1} of a strictly lower-triangular 64x64 fp32 matrix A (row stride
// la) into L (row stride ll; the blocks strictly above the block diagonal must
// be zero on entry).  Each 16x16 diagonal block is inverted by forward
// substitution with one column per thread held in registers (threads 0-63);
// the off-diagonal blocks follow in three rounds by distance from the
// diagonal: L_IJ = -L_II * sum_{m=J}^{I-1} A_Im L_mJ.  Y: 768 floats of scratch.
__device__ void block_inverse(const float* A, int la, float* L, int ll, float* Y, int tid, int nthr) {
    if (tid < 64) {
        const int o = 16 * (tid >> 4), c = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == c) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < r; ++j) acc = fmaf(-A[(o + r) * la + o + j], x[j], acc);
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) L[(o + r) * ll + o + c] = x[r];
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;  // blocks (I, J = I - d) of this round; one item = a row and 4 columns
        for (int e = tid; e < nb * 64; e += nthr) {
            const int J = e >> 6, I = J + d, r = (e >> 2) & 15, c4 = (e & 3) * 4;
            float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int m = J; m < I; ++m) {
                const float* Ar = A + (16 * I + r) * la + 16 * m;
                const float* Lc = L + (16 * m) * ll + 16 * J + c4;
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    const float a = Ar[p];
                    const float4 l = *reinterpret_cast<const float4*>(Lc + p * ll);
                    y.x = fmaf(a, l.x, y.x);
                    y.y = fmaf(a, l.y, y.y);
                    y.z = fmaf(a, l.z, y.z);
                    y.w = fmaf(a, l.w, y.w);
                }
            }
            *reinterpret_cast<float4*>(Y + (J << 8) + r * 16 + c4) = y;
        }
        __syncthreads();
        for (int e = tid; e < nb * 64; e += nthr) {
            const int J = e >> 6, I = J + d, r = (e >> 2) & 15, c4 = (e & 3) * 4;
            const float* Lr = L + (16 * I + r) * ll + 16 * I;
            const float* Yc = Y + (J << 8) + c4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const float a = Lr[p];
                const float4 yy = *reinterpret_cast<const float4*>(Yc + p * 16);
                x.x = fmaf(a, yy.x, x.x);
                x.y = fmaf(a, yy.y, x.y);
                x.z = fmaf(a, yy.z, x.z);
                x.w = fmaf(a, yy.w, x.w);
            }
            *reinterpret_cast<float4*>(L + (16 * I + r) * ll + 16 * J + c4) = make_float4(-x.x, -x.y, -x.z, -x.w);
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ prep ---
template <int DV>
constexpr size_t prep_smem() {  // 75.5 KB: three CTAs per SM
    return (size_t)C * LDK * 2 * 2 + (size_t)C * LDF * 4 * 2 + 768 * 4 + 3 * C * 4;
}

// One CTA (8 warps: rows 16*(w%4), column half w/4) per (chunk, head).  Writes
// G, exp(G), Khat, -W, L and U^T.
template <int DV, bool BETA>
__global__ void __launch_bounds__(256)
tc_prep_kernel(SeqView s, const bf16* __restrict__ k, const bf16* __restrict__ v, const float* __restrict__ g,
               const float* __restrict__ beta, float* __restrict__ Gc, float* __restrict__ Gmo,
               bf16* __restrict__ Wo, float* __restrict__ Lmo, bf16* __restrict__ Kho, bf16* __restrict__ Uto) {
    constexpr int LDV = DV + 8;
    extern __shared__ __align__(16) unsigned char smem[];
    // Regions are reused as the chunk advances: V's region (sized for a
    // [C][LDK] tile) holds the W staging once U is done, A's region holds the
    // bf16 T tiles once L is known, L's region the U^T staging.
    bf16* Ks = reinterpret_cast<bf16*>(smem);
    bf16* Vs = Ks + C * LDK;                                  // later: W staging [C][LDK]
    float* Af = reinterpret_cast<float*>(Vs + C * LDK);      // later: T tiles
    float* Lf = Af + C * LDF;                                 // later: U^T staging
    bf16* Tw = reinterpret_cast<bf16*>(Af);
    bf16* Tu = Tw + C * LDC;
    float* Yb = Lf + C * LDF;
    float* Gs = Yb + 768;
    float* Bs = Gs + C;
    float* BGs = Bs + C;  // beta_j exp(G_j)

    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int mw = w & 3, nw = w >> 2;
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t Tp = (size_t)s.NC * C;
    load_tile<C, DK, 256>(Ks, LDK, k + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
    load_tile<C, DV, 256>(Vs, LDV, v + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
    cp_async_commit();
    if (w == 0) chunk_cumsum(g + bh * s.hs_g + t0, nval, Gs, lane);
    for (int i = tid; i < C; i += 256) Bs[i] = (BETA && i < nval) ? beta[bh * s.hs_g + t0 + i] : 0.f;
    if (BETA)
        for (int e = tid; e < C * LDF; e += 256) Lf[e] = 0.f;
    cp_async_wait<0>();
    __syncthreads();

    for (int i = tid; i < C; i += 256) {
        const float e = __expf(Gs[i]);
        Gc[bh * Tp + t0 + i] = Gs[i];
        Gmo[bh * Tp + t0 + i] = e;
        BGs[i] = Bs[i] * e;
    }
    const float gC = Gs[C - 1];
    for (int e = tid; e < C * (DK / 8); e += 256) {
        const int r = e >> 4, cc = (e & 15) * 8;
        const float d = __expf(gC - Gs[r]);
        uint4 x = *reinterpret_cast<const uint4*>(Ks + r * LDK + cc);
        x.x = scale2(x.x, d, d);
        x.y = scale2(x.y, d, d);
        x.z = scale2(x.z, d, d);
        x.w = scale2(x.w, d, d);
        *reinterpret_cast<uint4*>(Kho + (bh * Tp + t0) * DK + swz(r, cc, DK)) = x;
    }

    bf16* Ust = reinterpret_cast<bf16*>(Lf);  // [DV][LDC]
    if (BETA) {
        {  // A = strictly-lower(diag(beta) (K K^T * Gamma))
            float acc[4][4] = {};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t a[4];
                ldA(a, Ks, LDK, 16 * mw, 16 * kk, lane);
#pragma unroll
                for (int nn = 0; nn < 4; nn += 2) {
                    uint32_t b[4];
                    ldBnk(b, Ks, LDK, 32 * nw + 8 * nn, 16 * kk, lane);
                    mma(acc[nn], a, b[0], b[1]);
                    mma(acc[nn + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nn = 0; nn < 4; ++nn)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 16 * mw + gq + 8 * (e >> 1), j = 32 * nw + 8 * nn + 2 * tq + (e & 1);
                    Af[i * LDF + j] = (j < i) ? Bs[i] * __expf(Gs[i] - Gs[j]) * acc[nn][e] : 0.f;
                }
        }
        __syncthreads();
        block_inverse(Af, LDF, Lf, LDF, Yb, tid, 256);
        float* Lg = Lmo + ((size_t)bh * s.NC + c) * C * C;
        for (int e = tid; e < C * C / 4; e += 256) {
            const int i = e >> 4, j = (e & 15) * 4;
            *reinterpret_cast<float4*>(Lg + i * C + j) = *reinterpret_cast<const float4*>(Lf + i * LDF + j);
        }
        for (int e = tid; e < C * C; e += 256) {  // A is dead: its region takes the T tiles
            const int i = e >> 6, j = e & 63;
            const float l = Lf[i * LDF + j];
            Tw[i * LDC + j] = __float2bfloat16_rn(l * BGs[j]);
            Tu[i * LDC + j] = __float2bfloat16_rn(l * Bs[j]);
        }
        __syncthreads();
        {  // U = T V, staged transposed into L's region
            float acc[DV / 16][4] = {};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a[4];
                ldA(a, Tu, LDC, 16 * mw, 16 * kk, lane);
#pragma unroll
                for (int nn = 0; nn < DV / 16; nn += 2) {
                    uint32_t b[4];
                    ldBkn(b, Vs, LDV, (DV / 2) * nw + 8 * nn, 16 * kk, lane);
                    mma(acc[nn], a, b[0], b[1]);
                    mma(acc[nn + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nn = 0; nn < DV / 16; ++nn)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 16 * mw + gq + 8 * (e >> 1), col = (DV / 2) * nw + 8 * nn + 2 * tq + (e & 1);
                    Ust[col * LDC + i] = __float2bfloat16_rn(acc[nn][e]);
                }
        }
        __syncthreads();  // V is dead: its region takes the W staging
        bf16* Wst = Vs;  // [C][LDK]
        {  // W = T (gamma * K), staged negated
            float acc[8][4] = {};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a[4];
                ldA(a, Tw, LDC, 16 * mw, 16 * kk, lane);
#pragma unroll
                for (int nn = 0; nn < 8; nn += 2) {
                    uint32_t b[4];
                    ldBkn(b, Ks, LDK, 64 * nw + 8 * nn, 16 * kk, lane);
                    mma(acc[nn], a, b[0], b[1]);
                    mma(acc[nn + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nn = 0; nn < 8; ++nn) {
                const int i = 16 * mw + gq, col = 64 * nw + 8 * nn + 2 * tq;
                *reinterpret_cast<uint32_t*>(Wst + i * LDK + col) = pack(-acc[nn][0], -acc[nn][1]);
                *reinterpret_cast<uint32_t*>(Wst + (i + 8) * LDK + col) = pack(-acc[nn][2], -acc[nn][3]);
            }
        }
        __syncthreads();
        for (int e = tid; e < C * (DK / 8); e += 256) {
            const int r = e >> 4, cc = (e & 15) * 8;
            *reinterpret_cast<uint4*>(Wo + (bh * Tp + t0) * DK + swz(r, cc, DK)) =
                *reinterpret_cast<const uint4*>(Wst + r * LDK + cc);
        }
    } else {
        for (int e = tid; e < C * DV; e += 256) {
            const int i = e / DV, col = e % DV;
            Ust[col * LDC + i] = Vs[i * LDV + col];
        }
        __syncthreads();
    }
    bf16* Utg = Uto + ((size_t)bh * s.NC + c) * DV * C;
    for (int e = tid; e < DV * (C / 8); e += 256) {
        const int r = e >> 3, cc = (e & 7) * 8;
        *reinterpret_cast<uint4*>(Utg + swz(r, cc, C)) = *reinterpret_cast<const uint4*>(Ust + r * LDC + cc);
    }
}

// ----------------------------------------------------------------- intra ---
// Intra-chunk parts of the backward that only read inputs: dVi^T = (P^T dO)^T
// and D^T = (scale (gamma * dO)^T Q)^T, 4 warps, P in shared memory.
template <int DV>
__device__ __forceinline__ void og_products(const SeqView& s, const bf16* Qs, const bf16* dOs, const bf16* Ps,
                                            const float* Gs, bf16* dVi, bf16* Dg, int w, int lane) {
    constexpr int LDV = DV + 8;
    constexpr int MT = DV / 64;  // 16-row m-tiles per warp
    const int gq = lane >> 2, tq = lane & 3;
    // dVi^T[v][j] = sum_i dO[i][v] P[i][j]
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m0 = (w * MT + mt) * 16;
        float acc[8][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t a[4];
            ldAt(a, dOs, LDV, m0, 16 * kk, lane);
#pragma unroll
            for (int nn = 0; nn < 8; nn += 2) {
                uint32_t b[4];
                ldBkn(b, Ps, LDC, 8 * nn, 16 * kk, lane);
                mma(acc[nn], a, b[0], b[1]);
                mma(acc[nn + 1], a, b[2], b[3]);
            }
        }
#pragma unroll
        for (int nn = 0; nn < 8; ++nn) {
            const int r = m0 + gq, j = 8 * nn + 2 * tq;
            *reinterpret_cast<uint32_t*>(dVi + swz(r, j, C)) = pack(acc[nn][0], acc[nn][1]);
            *reinterpret_cast<uint32_t*>(dVi + swz(r + 8, j, C)) = pack(acc[nn][2], acc[nn][3]);
        }
    }
    // D^T[v][d] = sum_t scale gamma_t dO[t][v] Q[t][d]
#pragma unroll 1
    for (int mt = 0; mt < MT; ++mt) {
        const int m0 = (w * MT + mt) * 16;
        uint32_t a[4][4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            ldAt(a[kk], dOs, LDV, m0, 16 * kk, lane);
            const int tk = 16 * kk + 2 * tq;
            const float g0 = s.scale * __expf(Gs[tk]), g1 = s.scale * __expf(Gs[tk + 1]);
            const float g2 = s.scale * __expf(Gs[tk + 8]), g3 = s.scale * __expf(Gs[tk + 9]);
            a[kk][0] = scale2(a[kk][0], g0, g1);
            a[kk][1] = scale2(a[kk][1], g0, g1);
            a[kk][2] = scale2(a[kk][2], g2, g3);
            a[kk][3] = scale2(a[kk][3], g2, g3);
        }
#pragma unroll 1
        for (int nh = 0; nh < 2; ++nh) {
            float acc[8][4] = {};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int nn = 0; nn < 8; nn += 2) {
                    uint32_t b[4];
                    ldBkn(b, Qs, LDK, 64 * nh + 8 * nn, 16 * kk, lane);
                    mma(acc[nn], a[kk], b[0], b[1]);
                    mma(acc[nn + 1], a[kk], b[2], b[3]);
                }
            }
#pragma unroll
            for (int nn = 0; nn < 8; ++nn) {
                const int r = m0 + gq, d = 64 * nh + 8 * nn + 2 * tq;
                *reinterpret_cast<uint32_t*>(Dg + swz(r, d, DK)) = pack(acc[nn][0], acc[nn][1]);
                *reinterpret_cast<uint32_t*>(Dg + swz(r + 8, d, DK)) = pack(acc[nn][2], acc[nn][3]);
            }
        }
    }
}

template <int DV>
constexpr size_t intra_smem() {
    return (size_t)C * LDK * 2 * 2 + (size_t)C * (DV + 8) * 2 + (size_t)C * LDC * 2 + C * 4;
}

// Intra-chunk output gradient (OG): dVi^T = (P^T dO)^T with
// P = scale (Q K^T) * Gamma, and the chain-independent term of the reverse
// state scan, D^T = (scale (gamma * dO)^T Q)^T; one CTA (4 warps) per (chunk, head).
template <int DV>
__global__ void __launch_bounds__(128)
tc_intra_kernel(SeqView s, const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ dO,
                const float* __restrict__ Gc, bf16* __restrict__ dVito, bf16* __restrict__ Dto) {
    constexpr int LDV = DV + 8;
    extern __shared__ __align__(16) unsigned char smem[];
    bf16* Qs = reinterpret_cast<bf16*>(smem);
    bf16* Ks = Qs + C * LDK;
    bf16* dOs = Ks + C * LDK;
    bf16* Ps = dOs + C * LDV;
    float* Gs = reinterpret_cast<float*>(Ps + C * LDC);
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t Tp = (size_t)s.NC * C;
    load_tile<C, DK, 128>(Qs, LDK, q + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
    load_tile<C, DK, 128>(Ks, LDK, k + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
    load_tile<C, DV, 128>(dOs, LDV, dO + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
    if (tid < 16) cp_async16(Gs + tid * 4, Gc + bh * Tp + t0 + tid * 4, true);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    {
        float acc[8][4] = {};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t a[4];
            ldA(a, Qs, LDK, 16 * w, 16 * kk, lane);
#pragma unroll
            for (int nn = 0; nn < 8; nn += 2) {
                uint32_t b[4];
                ldBnk(b, Ks, LDK, 8 * nn, 16 * kk, lane);
                mma(acc[nn], a, b[0], b[1]);
                mma(acc[nn + 1], a, b[2], b[3]);
            }
        }
#pragma unroll
        for (int nn = 0; nn < 8; ++nn)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 16 * w + gq + 8 * (e >> 1), j = 8 * nn + 2 * tq + (e & 1);
                const float p = (j <= i) ? s.scale * __expf(Gs[i] - Gs[j]) * acc[nn][e] : 0.f;
                Ps[i * LDC + j] = __float2bfloat16_rn(p);
            }
    }
    __syncthreads();
    const size_t ci = (size_t)bh * s.NC + c;
    og_products<DV>(s, Qs, dOs, Ps, Gs, dVito + ci * DV * C, Dto + ci * DV * DK, w, lane);
}

// ------------------------------------------------------------ state scans ---
// Operand stages of the chains are filled by one thread with bulk copies that
// complete on an mbarrier per stage; tiles produced by the prep kernel are
// stored permuted (swz), so the linear copies land bank-conflict-free.
constexpr uint32_t kTileK = C * DK * 2;   // a [C][DK] bf16 tile
constexpr uint32_t kTileV = 64 * C * 2;   // 64 rows of a [DV][C] bf16 tile
template <bool BETA>
constexpr size_t fwd_stage_bytes() {
    return (size_t)kTileK * (BETA ? 2 : 1) + kTileV + C * 4;
}
template <bool BETA>
constexpr size_t bwd_stage_bytes() {  // + the 64 rows of D^T of this block
    return (size_t)kTileK * (BETA ? 2 : 1) + kTileV + C * 4 + kTileK;
}
// Output staging of one chunk step of a 64-column block: the state tile
// (64 x DK) and the value tile (64 x C), in the permuted layout of swz().
constexpr size_t out_stage_bytes() { return (size_t)64 * DK * 2 + (size_t)64 * C * 2; }
constexpr int kOutBufs = 3;  // staged outputs of chunk c are flushed during step c+1 and must be read by step c+3
constexpr int kFwdStages = 3;  // operand stages of the forward chain: chunk c+2 is in flight during step c
constexpr size_t xch_bytes();
template <bool BETA>
constexpr size_t fwd_scan_smem() {
    return kFwdStages * fwd_stage_bytes<BETA>() + kOutBufs * out_stage_bytes() + xch_bytes() + 8 * kFwdStages;
}
template <bool BETA>
constexpr size_t bwd_scan_smem() { return 2 * bwd_stage_bytes<BETA>() + kOutBufs * out_stage_bytes() + xch_bytes() + 16; }

// Per-lane parts of the addresses into permuted [rows][128] tiles.
//   B fragments (stored [n][k], k = 16kk..): row = n0 + lr, piece 2kk + pb
//   B fragments (stored [k][n], trans):      row = k0 + lr, piece nn + pb (nn even)
// with lr, pb the lane's row/piece offsets; the piece is XOR-ed with lr & 7.
struct SwLane {
    int row;   // lane row offset inside a 16-row group (times the row length is added by callers)
    int lo;    // (pb ^ (lr & 1)) * 8   element offset of the low bit of the permuted piece
    int hi8;   // (lr & 6) * 8          XOR mask for the even part of the piece
};
__device__ __forceinline__ SwLane sw_lane_nk(int lane) {  // ldmatrix non-trans, row = n, piece from k
    const int lr = (lane & 7) + ((lane >> 4) << 3), pb = (lane >> 3) & 1;
    return {lr, (pb ^ (lr & 1)) * 8, (lr & 6) * 8};
}
__device__ __forceinline__ SwLane sw_lane_kn(int lane) {  // ldmatrix trans, row = k, piece from n
    const int lr = (lane & 7) + (((lane >> 3) & 1) << 3), pb = lane >> 4;
    return {lr, (pb ^ (lr & 1)) * 8, (lr & 6) * 8};
}
// Element offset of the fragment row/piece for an even logical piece `pe`.
__device__ __forceinline__ int sw_off(const SwLane& L, int rowbase, int pe, int rowlen) {
    return (rowbase + L.row) * rowlen + ((pe * 8) ^ L.hi8) + L.lo;
}

// Write a bf16 A-fragment block (16 rows x 16 cols at [r0, c0]) into a permuted
// staging tile of row length `cols` with one stmatrix.
__device__ __forceinline__ void stage_afrag(bf16* t, int cols, int r0, int c0, const uint32_t (&a)[4], int lane) {
    const int lr = (lane & 7) + (((lane >> 3) & 1) << 3), pb = lane >> 4;
    const int piece = ((c0 >> 3) + pb) ^ (lr & 7);
    stsm_x4(t + (r0 + lr) * cols + piece * 8, a);
}

// The chains use 8 warps per 64-column block: warps w and w+4 (which share an
// SM sub-partition) own the same 16 state columns and split every chunk step,
// the first warp taking tokens 0-31 of V_new and state rows 0-63 (of d_k),
// the second tokens 32-63 and rows 64-127.  Each product needs the partner's
// half of its left operand, which the pair swaps as bf16 fragments through
// shared memory.  One warp alone can issue a warp-level MMA only every ~18
// cycles, so two warps per sub-partition halve the step's issue time.
constexpr size_t xch_bytes() { return (size_t)4 * 2 * (4 + 2) * 32 * 16; }  // per pair: 4 state + 2 value fragments

// Pair barrier of the two warps that share a column group.
__device__ __forceinline__ void pair_sync(int cg) { asm volatile("bar.sync %0, 64;\n" ::"r"(cg + 1) : "memory"); }

// Fragment exchange slots (16 bytes per lane): [cg][half][slot 0-5][lane].
__device__ __forceinline__ uint4* xslot(unsigned char* xch, int cg, int half, int slot, int lane) {
    return reinterpret_cast<uint4*>(xch) + (((cg * 2 + half) * 6 + slot) * 32 + lane);
}
__device__ __forceinline__ void put_frag(uint4* p, const uint32_t (&a)[4]) { *p = make_uint4(a[0], a[1], a[2], a[3]); }
__device__ __forceinline__ void get_frag(const uint4* p, uint32_t (&a)[4]) {
    const uint4 v = *p;
    a[0] = v.x;
    a[1] = v.y;
    a[2] = v.z;
    a[3] = v.w;
}


// Forward chain for one (head, 64 state columns): per chunk
// V_new^T = U^T + S^T (-W)^T, S^T <- gamma_C S^T + V_new^T Khat.
// Optional outputs: V_new^T and S0^T per chunk (bf16, bulk-stored from a
// staging area by one thread), S_out (fp32).
template <int DV, bool BETA>
__device__ __forceinline__ void scan_fwd_cta(const SeqView& s, int bh, int vb, const float* __restrict__ Gm,
                                             const bf16* __restrict__ Wn, const bf16* __restrict__ Kh,
                                             const bf16* __restrict__ Ut, const float* __restrict__ S_in,
                                             bf16* __restrict__ Vnt, bf16* __restrict__ S0t,
                                             float* __restrict__ S_out, unsigned char* smem) {
    constexpr size_t STAGE = fwd_stage_bytes<BETA>();
    constexpr uint32_t TX = (BETA ? 2 : 1) * kTileK + kTileV + C * 4;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, gq = lane >> 2, tq = lane & 3;
    const int cg = w & 3, half = w >> 2, oth = half ^ 1;
    const int vl = 16 * cg;           // first state column of this warp pair inside the block
    const int v0 = vb * 64 + vl;      // ... and inside the head
    const size_t Tp = (size_t)s.NC * C;
    unsigned char* outs = smem + kFwdStages * STAGE;
    unsigned char* xch = outs + kOutBufs * out_stage_bytes();
    uint64_t* bars = reinterpret_cast<uint64_t*>(xch + xch_bytes());
    bool failed = false;

    auto stage = [&](int buf, bf16*& Khs, bf16*& Ws, bf16*& Uts, float*& Gs) {
        unsigned char* p = smem + buf * STAGE;
        Khs = reinterpret_cast<bf16*>(p);
        p += kTileK;
        Ws = reinterpret_cast<bf16*>(p);
        if (BETA) p += kTileK;
        Uts = reinterpret_cast<bf16*>(p);
        p += kTileV;
        Gs = reinterpret_cast<float*>(p);
    };
    auto load = [&](int cc) {  // thread 0 only
        bf16 *Khs, *Ws, *Uts;
        float* Gs;
        const int buf = cc % kFwdStages;
        stage(buf, Khs, Ws, Uts, Gs);
        const size_t row0 = (size_t)bh * Tp + (size_t)cc * C;
        mbar_expect_tx(&bars[buf], TX);
        bulk_load(Khs, Kh + row0 * DK, kTileK, &bars[buf]);
        if (BETA) bulk_load(Ws, Wn + row0 * DK, kTileK, &bars[buf]);
        bulk_load(Uts, Ut + (((size_t)bh * s.NC + cc) * DV + vb * 64) * C, kTileV, &bars[buf]);
        bulk_load(Gs, Gm + row0, C * 4, &bars[buf]);
    };
    auto flush = [&](int cc) {  // thread 0 only: bulk-store the staged outputs of chunk cc
        unsigned char* o = outs + (cc % kOutBufs) * out_stage_bytes();
        const size_t blk = ((size_t)bh * s.NC + cc) * DV + vb * 64;
        if (S0t) bulk_store(S0t + blk * DK, o, 64 * DK * 2);
        if (Vnt) bulk_store(Vnt + blk * C, o + 64 * DK * 2, 64 * C * 2);
        bulk_commit();
    };

    float st[8][4];  // S^T rows vl.., state rows 64*half + 8j..
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int vv = v0 + gq + 8 * (e >> 1), d = 64 * half + 8 * j + 2 * tq + (e & 1);
            st[j][e] = S_in ? S_in[((size_t)bh * DK + d) * DV + vv] : 0.f;
        }
    const SwLane Lnk = sw_lane_nk(lane), Lkn = sw_lane_kn(lane);
    const bool outputs = S0t || Vnt;

    if (tid == 0) {
        for (int i = 0; i < kFwdStages; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (tid == 0)
        for (int i = 0; i < kFwdStages - 1 && i < s.NC; ++i) load(i);
    for (int cc = 0; cc < s.NC; ++cc) {
        if (tid == 0) {
            if (cc + kFwdStages - 1 < s.NC) load(cc + kFwdStages - 1);  // buffer released by the barrier ending step cc-1
            if (outputs && cc > 0) flush(cc - 1);
        }
        bf16 *Khs, *Ws, *Uts;
        float* Gs;
        stage(cc % kFwdStages, Khs, Ws, Uts, Gs);
        bf16* S0s = reinterpret_cast<bf16*>(outs + (cc % kOutBufs) * out_stage_bytes());
        bf16* Vns = S0s + 64 * DK;
        // own half of S^T as bf16 fragments, swapped with the partner
        uint32_t sa[4][4], sp[4][4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            c2a(sa[kk], st[2 * kk], st[2 * kk + 1]);
            put_frag(xslot(xch, cg, half, kk, lane), sa[kk]);
        }
        mbar_wait(&bars[cc % kFwdStages], (cc / kFwdStages) & 1, &g_tc_status, failed);
        const float gamC = Gs[C - 1];
        float vn[4][4];  // V_new^T, tokens 32*half + 8nn..
#pragma unroll
        for (int nn = 0; nn < 4; ++nn) {
            const int po = (((4 * half + nn) ^ gq) << 3) + 2 * tq;
            const float2 u0 = unpack(*reinterpret_cast<const uint32_t*>(Uts + (vl + gq) * C + po));
            const float2 u1 = unpack(*reinterpret_cast<const uint32_t*>(Uts + (vl + gq + 8) * C + po));
            vn[nn][0] = u0.x;
            vn[nn][1] = u0.y;
            vn[nn][2] = u1.x;
            vn[nn][3] = u1.y;
        }
        // own state rows first (no wait for the partner), the partner's rows into
        // separate accumulators once its fragments are in
        if (BETA) {
            uint32_t bw[4][2][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2)
                    ldsm_x4(bw[j][n2], Ws + sw_off(Lnk, 8 * (4 * half + 2 * n2), 2 * (4 * half + j), DK));
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2) {
                    mma(vn[2 * n2], sa[j], bw[j][n2][0], bw[j][n2][1]);
                    mma(vn[2 * n2 + 1], sa[j], bw[j][n2][2], bw[j][n2][3]);
                }
        }
        pair_sync(cg);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) get_frag(xslot(xch, cg, oth, kk, lane), sp[kk]);
        if (BETA) {
            uint32_t bw[4][2][4];
            float vq[4][4] = {};
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2)
                    ldsm_x4(bw[j][n2], Ws + sw_off(Lnk, 8 * (4 * half + 2 * n2), 2 * (4 * oth + j), DK));
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2) {
                    mma(vq[2 * n2], sp[j], bw[j][n2][0], bw[j][n2][1]);
                    mma(vq[2 * n2 + 1], sp[j], bw[j][n2][2], bw[j][n2][3]);
                }
#pragma unroll
            for (int nn = 0; nn < 4; ++nn)
#pragma unroll
                for (int e = 0; e < 4; ++e) vn[nn][e] += vq[nn][e];
        }
        uint32_t va[2][4], vp[2][4];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            c2a(va[kk], vn[2 * kk], vn[2 * kk + 1]);
            put_frag(xslot(xch, cg, half, 4 + kk, lane), va[kk]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[j][e] *= gamC;
        {  // own token tiles first (no wait for the partner)
            uint32_t bk[2][4][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2)
                    ldsm_x4_t(bk[j][n2], Khs + sw_off(Lkn, 16 * (2 * half + j), 8 * half + 2 * n2, DK));
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2) {
                    mma(st[2 * n2], va[j], bk[j][n2][0], bk[j][n2][1]);
                    mma(st[2 * n2 + 1], va[j], bk[j][n2][2], bk[j][n2][3]);
                }
        }
        pair_sync(cg);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) get_frag(xslot(xch, cg, oth, 4 + kk, lane), vp[kk]);
        {  // then the partner's
            uint32_t bk[2][4][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2)
                    ldsm_x4_t(bk[j][n2], Khs + sw_off(Lkn, 16 * (2 * oth + j), 8 * half + 2 * n2, DK));
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2) {
                    mma(st[2 * n2], vp[j], bk[j][n2][0], bk[j][n2][1]);
                    mma(st[2 * n2 + 1], vp[j], bk[j][n2][2], bk[j][n2][3]);
                }
        }
        // stage this chunk's outputs (own halves) while the state update is in flight
        if (S0t) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) stage_afrag(S0s, DK, vl, 64 * half + 16 * kk, sa[kk], lane);
        }
        if (Vnt) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) stage_afrag(Vns, C, vl, 32 * half + 16 * kk, va[kk], lane);
        }
        if (outputs) fence_proxy_async_smem();
        if (tid == 0 && outputs) bulk_wait_read<1>();  // chunk cc-2's outputs left their buffer
        __syncthreads();
    }
    if (tid == 0) {
        if (outputs && s.NC > 0) flush(s.NC - 1);
        bulk_wait<0>();
    }
    if (S_out) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int vv = v0 + gq + 8 * (e >> 1), d = 64 * half + 8 * j + 2 * tq + (e & 1);
                S_out[((size_t)bh * DK + d) * DV + vv] = st[j][e];
            }
    }
}

// Reverse chain of the state gradient for one (head, 64 state columns):
// per chunk, from the last, dV_new^T = dVi^T + dS^T Khat^T and
// dS^T <- gamma_C dS^T + D^T + dV_new^T (-W), D^T = (scale (gamma * dO)^T Q)^T
// precomputed by the intra-chunk products.
// Outputs dV_new^T and dS_C^T per chunk (bf16, staged and bulk-stored), dS_in (fp32).
template <int DV, bool BETA>
__device__ __forceinline__ void scan_bwd_cta(const SeqView& s, int bh, int vb, const bf16* __restrict__ Dt,
                                             const float* __restrict__ Gm,
                                             const bf16* __restrict__ Wn, const bf16* __restrict__ Kh,
                                             const bf16* __restrict__ dVit, const float* __restrict__ dS_out,
                                             bf16* __restrict__ dVnt, bf16* __restrict__ dSCt,
                                             float* __restrict__ dS_in, unsigned char* smem) {
    constexpr size_t STAGE = bwd_stage_bytes<BETA>();
    constexpr uint32_t TX = (BETA ? 2 : 1) * kTileK + kTileV + C * 4 + kTileK;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, gq = lane >> 2, tq = lane & 3;
    const int cg = w & 3, half = w >> 2, oth = half ^ 1;
    const int vl = 16 * cg;
    const int v0 = vb * 64 + vl;
    const size_t Tp = (size_t)s.NC * C;
    unsigned char* outs = smem + 2 * STAGE;
    unsigned char* xch = outs + kOutBufs * out_stage_bytes();
    uint64_t* bars = reinterpret_cast<uint64_t*>(xch + xch_bytes());
    bool failed = false;

    auto stage = [&](int buf, bf16*& Khs, bf16*& Ws, bf16*& dVis, float*& Gs, bf16*& Dts) {
        unsigned char* p = smem + buf * STAGE;
        Khs = reinterpret_cast<bf16*>(p);
        p += kTileK;
        Ws = reinterpret_cast<bf16*>(p);
        if (BETA) p += kTileK;
        dVis = reinterpret_cast<bf16*>(p);
        p += kTileV;
        Gs = reinterpret_cast<float*>(p);
        p += C * 4;
        Dts = reinterpret_cast<bf16*>(p);
    };
    auto load = [&](int cc) {  // thread 0: bulk copies of one chunk's operands
        bf16 *Khs, *Ws, *dVis, *Dts;
        float* Gs;
        const int buf = cc & 1;
        stage(buf, Khs, Ws, dVis, Gs, Dts);
        const size_t row0 = (size_t)bh * Tp + (size_t)cc * C;
        const size_t blk = ((size_t)bh * s.NC + cc) * DV + vb * 64;
        if (tid == 0) {
            mbar_expect_tx(&bars[buf], TX);
            bulk_load(Khs, Kh + row0 * DK, kTileK, &bars[buf]);
            if (BETA) bulk_load(Ws, Wn + row0 * DK, kTileK, &bars[buf]);
            bulk_load(dVis, dVit + blk * C, kTileV, &bars[buf]);
            bulk_load(Gs, Gm + row0, C * 4, &bars[buf]);
            bulk_load(Dts, Dt + blk * DK, kTileK, &bars[buf]);
        }
    };
    auto flush = [&](int cc) {
        unsigned char* o = outs + (cc % kOutBufs) * out_stage_bytes();
        const size_t blk = ((size_t)bh * s.NC + cc) * DV + vb * 64;
        if (dSCt) bulk_store(dSCt + blk * DK, o, 64 * DK * 2);
        if (dVnt) bulk_store(dVnt + blk * C, o + 64 * DK * 2, 64 * C * 2);
        bulk_commit();
    };

    float ds[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int vv = v0 + gq + 8 * (e >> 1), d = 64 * half + 8 * j + 2 * tq + (e & 1);
            ds[j][e] = dS_out ? dS_out[((size_t)bh * DK + d) * DV + vv] : 0.f;
        }
    const SwLane Lnk = sw_lane_nk(lane), Lkn = sw_lane_kn(lane);
    const bool outputs = dSCt || dVnt;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init_fence();
    }
    __syncthreads();
    load(s.NC - 1);
    for (int cc = s.NC - 1; cc >= 0; --cc) {
        const int use = s.NC - 1 - cc;  // how many chunks were processed before this one
        if (cc > 0) load(cc - 1);
        if (tid == 0 && outputs && cc < s.NC - 1) flush(cc + 1);
        bf16 *Khs, *Ws, *dVis, *Dts;
        float* Gs;
        stage(cc & 1, Khs, Ws, dVis, Gs, Dts);
        bf16* dSs = reinterpret_cast<bf16*>(outs + (cc % kOutBufs) * out_stage_bytes());
        bf16* dVns = dSs + 64 * DK;
        uint32_t da[4][4], dp[4][4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            c2a(da[kk], ds[2 * kk], ds[2 * kk + 1]);
            put_frag(xslot(xch, cg, half, kk, lane), da[kk]);
        }
        mbar_wait(&bars[cc & 1], (use >> 1) & 1, &g_tc_status, failed);
        const float gamC = Gs[C - 1];
        float dvn[4][4];  // dV_new^T, tokens 32*half + 8nn..
#pragma unroll
        for (int nn = 0; nn < 4; ++nn) {
            const int po = (((4 * half + nn) ^ gq) << 3) + 2 * tq;
            const float2 u0 = unpack(*reinterpret_cast<const uint32_t*>(dVis + (vl + gq) * C + po));
            const float2 u1 = unpack(*reinterpret_cast<const uint32_t*>(dVis + (vl + gq + 8) * C + po));
            dvn[nn][0] = u0.x;
            dvn[nn][1] = u0.y;
            dvn[nn][2] = u1.x;
            dvn[nn][3] = u1.y;
        }
        {  // own state rows first (no wait for the partner)
            uint32_t bk[4][2][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2)
                    ldsm_x4(bk[j][n2], Khs + sw_off(Lnk, 8 * (4 * half + 2 * n2), 2 * (4 * half + j), DK));
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2) {
                    mma(dvn[2 * n2], da[j], bk[j][n2][0], bk[j][n2][1]);
                    mma(dvn[2 * n2 + 1], da[j], bk[j][n2][2], bk[j][n2][3]);
                }
        }
        pair_sync(cg);  // the partner's fragments are visible
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) get_frag(xslot(xch, cg, oth, kk, lane), dp[kk]);
        {  // the partner's rows into separate accumulators
            uint32_t bk[4][2][4];
            float dq[4][4] = {};
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2)
                    ldsm_x4(bk[j][n2], Khs + sw_off(Lnk, 8 * (4 * half + 2 * n2), 2 * (4 * oth + j), DK));
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2) {
                    mma(dq[2 * n2], dp[j], bk[j][n2][0], bk[j][n2][1]);
                    mma(dq[2 * n2 + 1], dp[j], bk[j][n2][2], bk[j][n2][3]);
                }
#pragma unroll
            for (int nn = 0; nn < 4; ++nn)
#pragma unroll
                for (int e = 0; e < 4; ++e) dvn[nn][e] += dq[nn][e];
        }
        uint32_t va[2][4], vp[2][4];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            c2a(va[kk], dvn[2 * kk], dvn[2 * kk + 1]);
            put_frag(xslot(xch, cg, half, 4 + kk, lane), va[kk]);
        }
        // dS <- gamma_C dS + D (D from the intra kernel, independent of the chain)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int col = 64 * half + 8 * j + 2 * tq;
            const float2 d0 = unpack(*reinterpret_cast<const uint32_t*>(Dts + swz(vl + gq, col, DK)));
            const float2 d1 = unpack(*reinterpret_cast<const uint32_t*>(Dts + swz(vl + gq + 8, col, DK)));
            ds[j][0] = fmaf(ds[j][0], gamC, d0.x);
            ds[j][1] = fmaf(ds[j][1], gamC, d0.y);
            ds[j][2] = fmaf(ds[j][2], gamC, d1.x);
            ds[j][3] = fmaf(ds[j][3], gamC, d1.y);
        }
        if (BETA) {  // own token tiles first (no wait for the partner)
            uint32_t bw[2][4][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2)
                    ldsm_x4_t(bw[j][n2], Ws + sw_off(Lkn, 16 * (2 * half + j), 8 * half + 2 * n2, DK));
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2) {
                    mma(ds[2 * n2], va[j], bw[j][n2][0], bw[j][n2][1]);
                    mma(ds[2 * n2 + 1], va[j], bw[j][n2][2], bw[j][n2][3]);
                }
        }
        pair_sync(cg);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) get_frag(xslot(xch, cg, oth, 4 + kk, lane), vp[kk]);
        if (BETA) {  // then the partner's
            uint32_t bw[2][4][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2)
                    ldsm_x4_t(bw[j][n2], Ws + sw_off(Lkn, 16 * (2 * oth + j), 8 * half + 2 * n2, DK));
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2) {
                    mma(ds[2 * n2], vp[j], bw[j][n2][0], bw[j][n2][1]);
                    mma(ds[2 * n2 + 1], vp[j], bw[j][n2][2], bw[j][n2][3]);
                }
        }
        if (dSCt) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) stage_afrag(dSs, DK, vl, 64 * half + 16 * kk, da[kk], lane);
        }
        if (dVnt) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) stage_afrag(dVns, C, vl, 32 * half + 16 * kk, va[kk], lane);
        }
        if (outputs) fence_proxy_async_smem();
        if (tid == 0 && outputs) bulk_wait_read<1>();
        __syncthreads();
    }
    if (tid == 0) {
        if (outputs && s.NC > 0) flush(0);
        bulk_wait<0>();
    }
    if (dS_in) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int vv = v0 + gq + 8 * (e >> 1), d = 64 * half + 8 * j + 2 * tq + (e & 1);
                dS_in[((size_t)bh * DK + d) * DV + vv] = ds[j][e];
            }
    }
}

template <int DV, bool BETA>
__global__ void __launch_bounds__(256, 1)
tc_scan_fwd_kernel(SeqView s, const float* __restrict__ Gm, const bf16* __restrict__ Wn,
                   const bf16* __restrict__ Kh, const bf16* __restrict__ Ut,
                   const float* __restrict__ S_in, bf16* __restrict__ Vnt, bf16* __restrict__ S0t,
                   float* __restrict__ S_out) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NVB = DV / 64;
    scan_fwd_cta<DV, BETA>(s, blockIdx.x / NVB, blockIdx.x % NVB, Gm, Wn, Kh, Ut, S_in, Vnt, S0t, S_out, smem);
}

// Backward chains in one launch: with with_sr, blocks [0, BH*DV/64) recompute
// the forward states (V_new and the chunk-entry states) and the rest run the
// reverse state-gradient scan; the two groups share no data.  Without it (the
// forward's states are kept), every block runs the reverse scan.
template <int DV, bool BETA>
__global__ void __launch_bounds__(256, 1)
tc_scan_bwd_dual_kernel(SeqView s, const bf16* __restrict__ Dt,
                        const float* __restrict__ Gm, const bf16* __restrict__ Wn,
                        const bf16* __restrict__ Kh, const bf16* __restrict__ Ut,
                        const bf16* __restrict__ dVit, const float* __restrict__ S_in,
                        const float* __restrict__ dS_out, bf16* __restrict__ Vnt, bf16* __restrict__ S0t,
                        bf16* __restrict__ dVnt, bf16* __restrict__ dSCt, float* __restrict__ dS_in,
                        int with_sr) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NVB = DV / 64;
    const int nsr = with_sr ? s.BH * NVB : 0;
    int id = blockIdx.x;
    if (id < nsr) {
        scan_fwd_cta<DV, BETA>(s, id / NVB, id % NVB, Gm, Wn, Kh, Ut, S_in, Vnt, S0t, nullptr, smem);
    } else {
        id -= nsr;
        scan_bwd_cta<DV, BETA>(s, id / NVB, id % NVB, Dt, Gm, Wn, Kh, dVit, dS_out, dVnt, dSCt, dS_in, smem);
    }
}

// ------------------------------------------------------------------- out ---
template <int DV, bool OG>
constexpr size_t out_smem() {
    return (size_t)C * LDK * 2 * 2 + (size_t)DV * LDK * 2 + (size_t)DV * LDC * 2 + C * 4 +
           (OG ? (size_t)C * (DV + 8) * 2 : 0);
}

// O = scale (gamma * Q) S0 + (scale (Q K^T) * Gamma) V_new; 4 warps x 16 rows.
// With OG (the forward of a segment whose backward follows), the same CTA also
// writes the intra-chunk backward products of og_products, reusing Q and P.
template <int DV, bool OG>
__global__ void __launch_bounds__(128)
tc_out_kernel(SeqView s, const bf16* __restrict__ q, const bf16* __restrict__ k,
              const float* __restrict__ Gc, const bf16* __restrict__ Vnt,
              const bf16* __restrict__ S0t, bf16* __restrict__ o, const bf16* __restrict__ dO,
              bf16* __restrict__ dVito, bf16* __restrict__ Dto) {
    constexpr int LDV = DV + 8;
    extern __shared__ __align__(16) unsigned char smem[];
    bf16* Qs = reinterpret_cast<bf16*>(smem);
    bf16* Ks = Qs + C * LDK;     // later (OG): P [C][LDC]
    bf16* S0s = Ks + C * LDK;   // [DV][LDK]
    bf16* Vns = S0s + DV * LDK;  // [DV][LDC]
    float* Gs = reinterpret_cast<float*>(Vns + DV * LDC);
    bf16* dOs = reinterpret_cast<bf16*>(Gs + C);  // [C][LDV] (OG)
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t Tp = (size_t)s.NC * C;
    load_tile<C, DK, 128>(Qs, LDK, q + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
    load_tile<C, DK, 128>(Ks, LDK, k + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
    load_tile_swz<DV, DK, 128>(S0s, LDK, S0t + ((size_t)bh * s.NC + c) * DV * DK, tid);
    load_tile_swz<DV, C, 128>(Vns, LDC, Vnt + ((size_t)bh * s.NC + c) * DV * C, tid);
    if (tid < 16) cp_async16(Gs + tid * 4, Gc + bh * Tp + t0 + tid * 4, true);
    cp_async_commit();
    if (OG) {
        load_tile<C, DV, 128>(dOs, LDV, dO + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
        cp_async_commit();
        cp_async_wait<1>();
    } else {
        cp_async_wait<0>();
    }
    __syncthreads();

    float p[8][4] = {};
    float acc[DV / 8][4] = {};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        uint32_t a[4];
        ldA(a, Qs, LDK, 16 * w, 16 * kk, lane);
#pragma unroll
        for (int nn = 0; nn < 8; nn += 2) {
            uint32_t b[4];
            ldBnk(b, Ks, LDK, 8 * nn, 16 * kk, lane);
            mma(p[nn], a, b[0], b[1]);
            mma(p[nn + 1], a, b[2], b[3]);
        }
#pragma unroll
        for (int nn = 0; nn < DV / 8; nn += 2) {
            uint32_t b[4];
            ldBnk(b, S0s, LDK, 8 * nn, 16 * kk, lane);
            mma(acc[nn], a, b[0], b[1]);
            mma(acc[nn + 1], a, b[2], b[3]);
        }
    }
    const int i0 = 16 * w + gq, i1 = i0 + 8;
    const float G0 = Gs[i0], G1 = Gs[i1];
    const float sg0 = s.scale * __expf(G0), sg1 = s.scale * __expf(G1);
#pragma unroll
    for (int nn = 0; nn < DV / 8; ++nn) {
        acc[nn][0] *= sg0;
        acc[nn][1] *= sg0;
        acc[nn][2] *= sg1;
        acc[nn][3] *= sg1;
    }
#pragma unroll
    for (int nn = 0; nn < 8; ++nn)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = (e >> 1) ? i1 : i0, j = 8 * nn + 2 * tq + (e & 1);
            p[nn][e] = (j <= i) ? s.scale * __expf(((e >> 1) ? G1 : G0) - Gs[j]) * p[nn][e] : 0.f;
        }
    bf16* Ps = Ks;
    if (OG) {
        __syncthreads();  // every warp is done reading K
#pragma unroll
        for (int nn = 0; nn < 8; ++nn) {
            const int j = 8 * nn + 2 * tq;
            *reinterpret_cast<uint32_t*>(Ps + i0 * LDC + j) = pack(p[nn][0], p[nn][1]);
            *reinterpret_cast<uint32_t*>(Ps + i1 * LDC + j) = pack(p[nn][2], p[nn][3]);
        }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        c2a(a, p[2 * kk], p[2 * kk + 1]);
#pragma unroll
        for (int nn = 0; nn < DV / 8; nn += 2) {
            uint32_t b[4];
            ldBnk(b, Vns, LDC, 8 * nn, 16 * kk, lane);
            mma(acc[nn], a, b[0], b[1]);
            mma(acc[nn + 1], a, b[2], b[3]);
        }
    }
    bf16* ob = o + bh * s.hs_v + (size_t)t0 * DV;
#pragma unroll
    for (int nn = 0; nn < DV / 8; ++nn) {
        const int col = 8 * nn + 2 * tq;
        if (i0 < nval) *reinterpret_cast<uint32_t*>(ob + (size_t)i0 * DV + col) = pack(acc[nn][0], acc[nn][1]);
        if (i1 < nval) *reinterpret_cast<uint32_t*>(ob + (size_t)i1 * DV + col) = pack(acc[nn][2], acc[nn][3]);
    }
    if (OG) {
        cp_async_wait<0>();
        __syncthreads();  // P and dO are visible
        const size_t ci = (size_t)bh * s.NC + c;
        og_products<DV>(s, Qs, dOs, Ps, Gs, dVito + ci * DV * C, Dto + ci * DV * DK, w, lane);
    }
}

// ------------------------------------------------------------------ grad ---
// Warps of the gradient kernel: 4 row blocks of 16 x GW column groups.
constexpr int GW = 4;
constexpr int GTH = 128 * GW;
constexpr int DKW = DK / GW;  // key columns of one column group
constexpr int CW = C / GW;    // chunk columns of one column group
// Partial-sum rows (each [64] fp32) of the gradient kernel's reductions.
enum GradPart {
    P_INTER = 0,             // [GW] sum_k Q_ik dq_inter_ik
    P_Z = GW,                // [GW] sum_k K_jk dK_state_jk
    P_ROWP = 2 * GW,         // [GW] row sums of M * (Qs K^T)
    P_COLP = 3 * GW,         // [4]  column sums of the same
    P_KT = 3 * GW + 4,       // [GW] gamma_j k_j . dKt_j
    P_DBC = 4 * GW + 4,      // [4]  column sums of dT * L
    P_DBR = 4 * GW + 8,      // [GW] row sums of dA * Gamma * KK
    P_ROWA = 5 * GW + 8,     // [GW] row sums of Z * KK
    P_COLA = 6 * GW + 8,     // [4]  column sums of Z * KK
    P_ROWS = 6 * GW + 12
};

template <int DV>
constexpr size_t grad_region_bytes() {
    const size_t sa = (size_t)DV * LDK * 2 * 2;                                     // S0^T, dS_C^T
    const size_t sb = (size_t)C * LDK * 2 + (size_t)C * LDF * 4 * 2 + (size_t)C * LDC * 2 * 4;  // dW, X/Z, L, T/L/M/dL
    return sa > sb ? sa : sb;
}
template <int DV>
constexpr size_t grad_smem() {
    return (size_t)C * LDK * 2 * 2 + (size_t)C * (DV + 8) * 2 * 2 + (size_t)DV * LDC * 2 * 2 +
           grad_region_bytes<DV>() + (size_t)P_ROWS * C * 4 + GTH * 4 + 4 * C * 4 + 16;
}

// Every input gradient of one chunk (4 x GW warps: rows 16*(w%4), column group w/4).
template <int DV, bool BETA>
__global__ void __launch_bounds__(GTH, 1)
tc_grad_kernel(SeqView s, const bf16* __restrict__ q, const bf16* __restrict__ k,
               const bf16* __restrict__ v, const float* __restrict__ beta,
               const bf16* __restrict__ dO, const float* __restrict__ Gc, const float* __restrict__ Lm,
               const bf16* __restrict__ Vnt, const bf16* __restrict__ dVnt,
               const bf16* __restrict__ S0t, const bf16* __restrict__ dSCt, bf16* __restrict__ dq,
               bf16* __restrict__ dk, bf16* __restrict__ dv, float* __restrict__ dg,
               float* __restrict__ dbeta, int* __restrict__ ticket) {
    constexpr int LDV = DV + 8;
    extern __shared__ __align__(16) unsigned char smem[];
    bf16* Qs = reinterpret_cast<bf16*>(smem);
    bf16* Ks = Qs + C * LDK;
    bf16* Vs = Ks + C * LDK;     // [C][LDV]
    bf16* dOs = Vs + C * LDV;    // [C][LDV]
    bf16* Vns = dOs + C * LDV;   // [DV][LDC]  V_new^T
    bf16* dVns = Vns + DV * LDC;  // [DV][LDC] dV_new^T
    unsigned char* R = reinterpret_cast<unsigned char*>(dVns + DV * LDC);
    bf16* S0s = reinterpret_cast<bf16*>(R);       // [DV][LDK]  (phase S)
    bf16* dSs = S0s + DV * LDK;                   // [DV][LDK]  (phase S)
    bf16* dWs = reinterpret_cast<bf16*>(R);       // [C][LDK]   (after phase S)
    float* XZ = reinterpret_cast<float*>(R + C * LDK * 2);  // X, Z (bf16 [C][LDC] each)
    float* Lf = XZ + C * LDF;                     // [C][LDF] L (fp32)
    bf16* Ts = reinterpret_cast<bf16*>(Lf + C * LDF);  // [C][LDC]; Y scratch during the inverse
    bf16* Ls = Ts + C * LDC;
    bf16* Ms = Ls + C * LDC;
    bf16* dLs = Ms + C * LDC;
    bf16* Xs = reinterpret_cast<bf16*>(XZ);
    bf16* Zs = Xs + C * LDC;
    float* part = reinterpret_cast<float*>(R + grad_region_bytes<DV>());  // [P_ROWS][C]
    float* red = part + P_ROWS * C;                                        // [GTH]
    float* Gsb = red + GTH;  // [2][C] G of this chunk / the next
    float* Bsb = Gsb + 2 * C;  // [2][C] beta of this chunk / the next
    int* tk = reinterpret_cast<int*>(Bsb + 2 * C);

    // Persistent: each CTA takes chunk tickets from `ticket` until none is
    // left.  The next chunk's tiles are copied into regions as they die: dO and
    // V_new after phase S, V and dV_new after C6, Q, K, G, S0 and dS_C after
    // C7; so only the part of the first copy group that C8 cannot cover is
    // waited for at the top of the next iteration.
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int mw = w & 3, nw = w >> 2;
    const size_t Tp = (size_t)s.NC * C;
    const int total = s.NC * s.BH;
    const int r0 = 16 * mw + gq, r1 = r0 + 8;  // the two rows this thread holds
    auto where = [&](int j, int& c, int& bh) {
        bh = j / s.NC;
        c = j - bh * s.NC;
    };
    auto copy_a1 = [&](int j, int gbuf) {  // Q, K, G
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        load_tile<C, DK, GTH>(Qs, LDK, q + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
        load_tile<C, DK, GTH>(Ks, LDK, k + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
        if (tid < 16) cp_async16(Gsb + gbuf * C + tid * 4, Gc + bh * Tp + t0 + tid * 4, true);
    };
    auto copy_a2 = [&](int j) {  // dO, V_new
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        const size_t ci = (size_t)bh * s.NC + c;
        load_tile<C, DV, GTH>(dOs, LDV, dO + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
        load_tile_swz<DV, C, GTH>(Vns, LDC, Vnt + ci * DV * C, tid);
    };
    auto copy_b1 = [&](int j) {  // V, dV_new
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        const size_t ci = (size_t)bh * s.NC + c;
        load_tile_swz<DV, C, GTH>(dVns, LDC, dVnt + ci * DV * C, tid);
        load_tile<C, DV, GTH>(Vs, LDV, v + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
    };
    auto copy_b2 = [&](int j) {  // S0, dS_C
        int c, bh;
        where(j, c, bh);
        const size_t ci = (size_t)bh * s.NC + c;
        load_tile_swz<DV, DK, GTH>(S0s, LDK, S0t + ci * DV * DK, tid);
        load_tile_swz<DV, DK, GTH>(dSs, LDK, dSCt + ci * DV * DK, tid);
    };
    auto beta_of = [&](int j) {
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        return (BETA && tid < nval) ? beta[bh * s.hs_g + t0 + tid] : 0.f;
    };

    if (tid == 0) tk[0] = atomicAdd(ticket, 1);
    __syncthreads();
    int j = tk[0];
    if (j >= total) return;
    // Copy groups of the first chunk: A (C1's operands), then B (the rest).
    copy_a1(j, 0);
    copy_a2(j);
    cp_async_commit();
    copy_b1(j);
    copy_b2(j);
    cp_async_commit();
    if (tid < C) Bsb[tid] = beta_of(j);
    for (int e = tid; e < P_ROWS * C; e += GTH) part[e] = 0.f;
    int buf = 0;
  for (;;) {
    int c, bh;
    where(j, c, bh);
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    const size_t ci = (size_t)bh * s.NC + c;
    float* Gs = Gsb + buf * C;
    float* Bs = Bsb + buf * C;
    cp_async_wait<1>();  // group A of this chunk (the state tiles may still be landing)
    if (tid == 0) tk[1] = atomicAdd(ticket, 1);
    __syncthreads();
    const int jn = tk[1];
    const bool has_next = jn < total;

    const float gam0 = __expf(Gs[r0]), gam1 = __expf(Gs[r1]);
    const float gC = Gs[C - 1];
    const float dec0 = __expf(gC - Gs[r0]), dec1 = __expf(gC - Gs[r1]);

    // ---- phase C1: C x C products (rows 16mw.., columns CW nw..); reads only the first copy group
    float kkr[CW / 8][4] = {};
    {
        float qk[CW / 8][4] = {}, dp[CW / 8][4] = {};
#pragma unroll
        for (int kd = 0; kd < 8; ++kd) {
            uint32_t aQ[4], aK[4];
            ldA(aQ, Qs, LDK, 16 * mw, 16 * kd, lane);
            ldA(aK, Ks, LDK, 16 * mw, 16 * kd, lane);
#pragma unroll
            for (int nn = 0; nn < CW / 8; nn += 2) {
                uint32_t b[4];
                ldBnk(b, Ks, LDK, CW * nw + 8 * nn, 16 * kd, lane);
                mma(qk[nn], aQ, b[0], b[1]);
                mma(qk[nn + 1], aQ, b[2], b[3]);
                mma(kkr[nn], aK, b[0], b[1]);
                mma(kkr[nn + 1], aK, b[2], b[3]);
            }
        }
#pragma unroll
        for (int kv = 0; kv < DV / 16; ++kv) {
            uint32_t aO[4];
            ldA(aO, dOs, LDV, 16 * mw, 16 * kv, lane);
#pragma unroll
            for (int nn = 0; nn < CW / 8; nn += 2) {
                uint32_t b[4];
                ldBkn(b, Vns, LDC, CW * nw + 8 * nn, 16 * kv, lane);
                mma(dp[nn], aO, b[0], b[1]);
                mma(dp[nn + 1], aO, b[2], b[3]);
            }
        }
        float row0 = 0.f, row1 = 0.f;
#pragma unroll
        for (int nn = 0; nn < CW / 8; ++nn) {
            float col[2] = {0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = (e >> 1) ? r1 : r0, j = CW * nw + 8 * nn + 2 * tq + (e & 1);
                const float gm = (j <= i) ? __expf(Gs[i] - Gs[j]) : 0.f;
                const float m = s.scale * dp[nn][e] * gm;
                Ms[i * LDC + j] = __float2bfloat16_rn(m);
                const float zp = m * qk[nn][e];
                if (e >> 1) row1 += zp; else row0 += zp;
                col[e & 1] += zp;
            }
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                col[0] += __shfl_xor_sync(0xffffffffu, col[0], o);
                col[1] += __shfl_xor_sync(0xffffffffu, col[1], o);
            }
            if (gq == 0) {
                const int j = CW * nw + 8 * nn + 2 * tq;
                part[(P_COLP + mw) * C + j] = col[0];
                part[(P_COLP + mw) * C + j + 1] = col[1];
            }
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            row0 += __shfl_xor_sync(0xffffffffu, row0, o);
            row1 += __shfl_xor_sync(0xffffffffu, row1, o);
        }
        if (tq == 0) {
            part[(P_ROWP + nw) * C + r0] = row0;
            part[(P_ROWP + nw) * C + r1] = row1;
        }
    }
    cp_async_wait<0>();
    __syncthreads();  // the state tiles and V have landed

    // ---- phase S: products with the chunk-entry state and the state gradient
    float accQ[DKW / 8][4] = {}, accK[DKW / 8][4] = {};
    {
        float accW[DKW / 8][4] = {};
#pragma unroll
        for (int kv = 0; kv < DV / 16; ++kv) {
            uint32_t aO[4], aN[4], aV[4];
            ldA(aO, dOs, LDV, 16 * mw, 16 * kv, lane);
            ldAt(aN, dVns, LDC, 16 * mw, 16 * kv, lane);
            ldAt(aV, Vns, LDC, 16 * mw, 16 * kv, lane);
#pragma unroll
            for (int nn = 0; nn < DKW / 8; nn += 2) {
                uint32_t b[4];
                ldBkn(b, S0s, LDK, DKW * nw + 8 * nn, 16 * kv, lane);
                mma(accQ[nn], aO, b[0], b[1]);
                mma(accQ[nn + 1], aO, b[2], b[3]);
                mma(accW[nn], aN, b[0], b[1]);
                mma(accW[nn + 1], aN, b[2], b[3]);
                ldBkn(b, dSs, LDK, DKW * nw + 8 * nn, 16 * kv, lane);
                mma(accK[nn], aV, b[0], b[1]);
                mma(accK[nn + 1], aV, b[2], b[3]);
            }
        }
        float pd = 0.f;  // <S0, dS_C>
        for (int e = tid; e < DV * DK; e += GTH) {
            const int r = e / DK, cc = e % DK;
            pd += __bfloat162float(S0s[r * LDK + cc]) * __bfloat162float(dSs[r * LDK + cc]);
        }
        red[tid] = pd;
        // dq_inter = scale gamma (dO S0^T); dK_state = dec (V_new dS_C^T)
        const float sq0 = s.scale * gam0, sq1 = s.scale * gam1;
        float pi0 = 0.f, pi1 = 0.f, pz0 = 0.f, pz1 = 0.f;
#pragma unroll
        for (int nn = 0; nn < DKW / 8; ++nn) {
            const int col = DKW * nw + 8 * nn + 2 * tq;
            const float2 q0 = unpack(*reinterpret_cast<const uint32_t*>(Qs + r0 * LDK + col));
            const float2 q1 = unpack(*reinterpret_cast<const uint32_t*>(Qs + r1 * LDK + col));
            const float2 k0 = unpack(*reinterpret_cast<const uint32_t*>(Ks + r0 * LDK + col));
            const float2 k1 = unpack(*reinterpret_cast<const uint32_t*>(Ks + r1 * LDK + col));
            accQ[nn][0] *= sq0;
            accQ[nn][1] *= sq0;
            accQ[nn][2] *= sq1;
            accQ[nn][3] *= sq1;
            accK[nn][0] *= dec0;
            accK[nn][1] *= dec0;
            accK[nn][2] *= dec1;
            accK[nn][3] *= dec1;
            pi0 += q0.x * accQ[nn][0] + q0.y * accQ[nn][1];
            pi1 += q1.x * accQ[nn][2] + q1.y * accQ[nn][3];
            pz0 += k0.x * accK[nn][0] + k0.y * accK[nn][1];
            pz1 += k1.x * accK[nn][2] + k1.y * accK[nn][3];
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            pi0 += __shfl_xor_sync(0xffffffffu, pi0, o);
            pi1 += __shfl_xor_sync(0xffffffffu, pi1, o);
            pz0 += __shfl_xor_sync(0xffffffffu, pz0, o);
            pz1 += __shfl_xor_sync(0xffffffffu, pz1, o);
        }
        if (tq == 0) {
            part[(P_INTER + nw) * C + r0] = pi0;
            part[(P_INTER + nw) * C + r1] = pi1;
            part[(P_Z + nw) * C + r0] = pz0;
            part[(P_Z + nw) * C + r1] = pz1;
        }
        __syncthreads();  // everyone is done with S0^T and dS_C^T
        if (BETA) {  // L of this chunk (from the prep kernel) into Lf; waited for before phase C2
            const float* Lg = Lm + ci * C * C;
            for (int e = tid; e < C * C / 4; e += GTH) {
                const int i = e >> 4, j = (e & 15) * 4;
                cp_async16(Lf + i * LDF + j, Lg + i * C + j, true);
            }
            cp_async_commit();
        }
        if (has_next) copy_a2(jn);  // dO and V_new are dead
        cp_async_commit();
        // dW = -dV_new S0^T into the freed region
#pragma unroll
        for (int nn = 0; nn < DKW / 8; ++nn) {
            const int col = DKW * nw + 8 * nn + 2 * tq;
            *reinterpret_cast<uint32_t*>(dWs + r0 * LDK + col) = pack(-accW[nn][0], -accW[nn][1]);
            *reinterpret_cast<uint32_t*>(dWs + r1 * LDK + col) = pack(-accW[nn][2], -accW[nn][3]);
        }
    }
    for (int o = GTH / 2; o > 0; o >>= 1) {
        if (tid < o) red[tid] += red[tid + o];
        __syncthreads();
    }
    const float sdot = red[0];

    if (BETA) cp_async_wait<1>();  // L (the next chunk's dO, V_new may still be landing)
    __syncthreads();

    // ---- phase C2: T = L diag(beta), L = (I + A)^{-1} as computed by the prep kernel
    if (BETA) {
        for (int e = tid; e < C * C; e += GTH) {
            const int i = e >> 6, j = e & 63;
            const float l = Lf[i * LDF + j];
            Ts[i * LDC + j] = __float2bfloat16_rn(l * Bs[j]);
            Ls[i * LDC + j] = __float2bfloat16_rn(l);
        }
        __syncthreads();
    }

    // ---- phase C3: dKt = T^T dW (into dK), dV = T^T dV_new
    if (BETA) {
        float acc[DKW / 8][4] = {};
#pragma unroll
        for (int kr = 0; kr < 4; ++kr) {
            uint32_t a[4];
            ldAt(a, Ts, LDC, 16 * mw, 16 * kr, lane);
#pragma unroll
            for (int nn = 0; nn < DKW / 8; nn += 2) {
                uint32_t b[4];
                ldBkn(b, dWs, LDK, DKW * nw + 8 * nn, 16 * kr, lane);
                mma(acc[nn], a, b[0], b[1]);
                mma(acc[nn + 1], a, b[2], b[3]);
            }
        }
        float p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int nn = 0; nn < DKW / 8; ++nn) {
            const int col = DKW * nw + 8 * nn + 2 * tq;
            const float2 k0 = unpack(*reinterpret_cast<const uint32_t*>(Ks + r0 * LDK + col));
            const float2 k1 = unpack(*reinterpret_cast<const uint32_t*>(Ks + r1 * LDK + col));
            const float a0 = gam0 * acc[nn][0], a1 = gam0 * acc[nn][1];
            const float a2 = gam1 * acc[nn][2], a3 = gam1 * acc[nn][3];
            accK[nn][0] += a0;
            accK[nn][1] += a1;
            accK[nn][2] += a2;
            accK[nn][3] += a3;
            p0 += k0.x * a0 + k0.y * a1;
            p1 += k1.x * a2 + k1.y * a3;
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            p0 += __shfl_xor_sync(0xffffffffu, p0, o);
            p1 += __shfl_xor_sync(0xffffffffu, p1, o);
        }
        if (tq == 0) {
            part[(P_KT + nw) * C + r0] = p0;
            part[(P_KT + nw) * C + r1] = p1;
        }
    }
    {
        constexpr int NT = DV / (8 * GW);  // n-tiles of this warp's group of value columns
        bf16* dvb = dv + bh * s.hs_v + (size_t)t0 * DV;
        if (BETA) {
            float acc[NT][4] = {};
#pragma unroll
            for (int kr = 0; kr < 4; ++kr) {
                uint32_t a[4];
                ldAt(a, Ts, LDC, 16 * mw, 16 * kr, lane);
#pragma unroll
                for (int nn = 0; nn < NT; nn += 2) {
                    uint32_t b[4];
                    ldBnk(b, dVns, LDC, (DV / GW) * nw + 8 * nn, 16 * kr, lane);
                    mma(acc[nn], a, b[0], b[1]);
                    mma(acc[nn + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nn = 0; nn < NT; ++nn) {
                const int col = (DV / GW) * nw + 8 * nn + 2 * tq;
                if (r0 < nval) *reinterpret_cast<uint32_t*>(dvb + (size_t)r0 * DV + col) = pack(acc[nn][0], acc[nn][1]);
                if (r1 < nval) *reinterpret_cast<uint32_t*>(dvb + (size_t)r1 * DV + col) = pack(acc[nn][2], acc[nn][3]);
            }
        } else {
            for (int e = tid; e < nval * DV; e += GTH) {
                const int j = e / DV, col = e % DV;
                dvb[(size_t)j * DV + col] = dVns[col * LDC + j];
            }
        }
    }

    // ---- phase C4: dT = dW (gamma K)^T + dV_new V^T; dbeta (column part); dL = dT diag(beta)
    if (BETA) {
        float dt[CW / 8][4] = {};
#pragma unroll
        for (int kd = 0; kd < 8; ++kd) {
            uint32_t a[4];
            ldA(a, dWs, LDK, 16 * mw, 16 * kd, lane);
#pragma unroll
            for (int nn = 0; nn < CW / 8; nn += 2) {
                uint32_t b[4];
                ldBnk(b, Ks, LDK, CW * nw + 8 * nn, 16 * kd, lane);
                mma(dt[nn], a, b[0], b[1]);
                mma(dt[nn + 1], a, b[2], b[3]);
            }
        }
#pragma unroll
        for (int nn = 0; nn < CW / 8; ++nn)
#pragma unroll
            for (int e = 0; e < 4; ++e) dt[nn][e] *= __expf(Gs[CW * nw + 8 * nn + 2 * tq + (e & 1)]);
#pragma unroll
        for (int kv = 0; kv < DV / 16; ++kv) {
            uint32_t a[4];
            ldAt(a, dVns, LDC, 16 * mw, 16 * kv, lane);
#pragma unroll
            for (int nn = 0; nn < CW / 8; nn += 2) {
                uint32_t b[4];
                ldBnk(b, Vs, LDV, CW * nw + 8 * nn, 16 * kv, lane);
                mma(dt[nn], a, b[0], b[1]);
                mma(dt[nn + 1], a, b[2], b[3]);
            }
        }
#pragma unroll
        for (int nn = 0; nn < CW / 8; ++nn) {
            float col[2] = {0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = (e >> 1) ? r1 : r0, j = CW * nw + 8 * nn + 2 * tq + (e & 1);
                col[e & 1] += dt[nn][e] * Lf[r * LDF + j];
                dLs[r * LDC + j] = __float2bfloat16_rn(dt[nn][e] * Bs[j]);
            }
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                col[0] += __shfl_xor_sync(0xffffffffu, col[0], o);
                col[1] += __shfl_xor_sync(0xffffffffu, col[1], o);
            }
            if (gq == 0) {
                const int j = CW * nw + 8 * nn + 2 * tq;
                part[(P_DBC + mw) * C + j] = col[0];
                part[(P_DBC + mw) * C + j + 1] = col[1];
            }
        }
        __syncthreads();
        // ---- phase C5: X = L^T dL
        {
            float x[CW / 8][4] = {};
#pragma unroll
            for (int kr = 0; kr < 4; ++kr) {
                uint32_t a[4];
                ldAt(a, Ls, LDC, 16 * mw, 16 * kr, lane);
#pragma unroll
                for (int nn = 0; nn < CW / 8; nn += 2) {
                    uint32_t b[4];
                    ldBkn(b, dLs, LDC, CW * nw + 8 * nn, 16 * kr, lane);
                    mma(x[nn], a, b[0], b[1]);
                    mma(x[nn + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int nn = 0; nn < CW / 8; ++nn) {
                const int j = CW * nw + 8 * nn + 2 * tq;
                *reinterpret_cast<uint32_t*>(Xs + r0 * LDC + j) = pack(x[nn][0], x[nn][1]);
                *reinterpret_cast<uint32_t*>(Xs + r1 * LDC + j) = pack(x[nn][2], x[nn][3]);
            }
        }
        __syncthreads();
        // ---- phase C6: dA = strictly-lower(-X L^T); Z = dA beta_i Gamma; dbeta (row part)
        {
            float da[CW / 8][4] = {};
#pragma unroll
            for (int km = 0; km < 4; ++km) {
                uint32_t a[4];
                ldA(a, Xs, LDC, 16 * mw, 16 * km, lane);
#pragma unroll
                for (int nn = 0; nn < CW / 8; nn += 2) {
                    uint32_t b[4];
                    ldBnk(b, Ls, LDC, CW * nw + 8 * nn, 16 * km, lane);
                    mma(da[nn], a, b[0], b[1]);
                    mma(da[nn + 1], a, b[2], b[3]);
                }
            }
            float rz0 = 0.f, rz1 = 0.f, rb0 = 0.f, rb1 = 0.f;
#pragma unroll
            for (int nn = 0; nn < CW / 8; ++nn) {
                float col[2] = {0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = (e >> 1) ? r1 : r0, j = CW * nw + 8 * nn + 2 * tq + (e & 1);
                    float z = 0.f, bterm = 0.f;
                    if (j < i) {
                        const float gm = __expf(Gs[i] - Gs[j]);
                        const float dav = -da[nn][e];
                        bterm = dav * gm * kkr[nn][e];
                        z = dav * Bs[i] * gm;
                    }
                    Zs[i * LDC + j] = __float2bfloat16_rn(z);
                    const float za = z * kkr[nn][e];
                    if (e >> 1) {
                        rz1 += za;
                        rb1 += bterm;
                    } else {
                        rz0 += za;
                        rb0 += bterm;
                    }
                    col[e & 1] += za;
                }
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    col[0] += __shfl_xor_sync(0xffffffffu, col[0], o);
                    col[1] += __shfl_xor_sync(0xffffffffu, col[1], o);
                }
                if (gq == 0) {
                    const int j = CW * nw + 8 * nn + 2 * tq;
                    part[(P_COLA + mw) * C + j] = col[0];
                    part[(P_COLA + mw) * C + j + 1] = col[1];
                }
            }
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                rz0 += __shfl_xor_sync(0xffffffffu, rz0, o);
                rz1 += __shfl_xor_sync(0xffffffffu, rz1, o);
                rb0 += __shfl_xor_sync(0xffffffffu, rb0, o);
                rb1 += __shfl_xor_sync(0xffffffffu, rb1, o);
            }
            if (tq == 0) {
                part[(P_ROWA + nw) * C + r0] = rz0;
                part[(P_ROWA + nw) * C + r1] = rz1;
                part[(P_DBR + nw) * C + r0] = rb0;
                part[(P_DBR + nw) * C + r1] = rb1;
            }
        }
    }
    __syncthreads();
    if (has_next) copy_b1(jn);  // V and dV_new are dead
    cp_async_commit();

    // ---- phase C7: dK += (Z + Z^T) K + Ms^T Q ; dq += Ms K
#pragma unroll
    for (int ki = 0; ki < 4; ++ki) {
        uint32_t aM[4], aMt[4];
        ldA(aM, Ms, LDC, 16 * mw, 16 * ki, lane);
        ldAt(aMt, Ms, LDC, 16 * mw, 16 * ki, lane);
        uint32_t aZ[4], aZt[4];
        if (BETA) {
            ldA(aZ, Zs, LDC, 16 * mw, 16 * ki, lane);
            ldAt(aZt, Zs, LDC, 16 * mw, 16 * ki, lane);
        }
#pragma unroll
        for (int nn = 0; nn < DKW / 8; nn += 2) {
            uint32_t bk[4], bq[4];
            ldBkn(bk, Ks, LDK, DKW * nw + 8 * nn, 16 * ki, lane);
            ldBkn(bq, Qs, LDK, DKW * nw + 8 * nn, 16 * ki, lane);
            mma(accQ[nn], aM, bk[0], bk[1]);
            mma(accQ[nn + 1], aM, bk[2], bk[3]);
            mma(accK[nn], aMt, bq[0], bq[1]);
            mma(accK[nn + 1], aMt, bq[2], bq[3]);
            if (BETA) {
                mma(accK[nn], aZ, bk[0], bk[1]);
                mma(accK[nn + 1], aZ, bk[2], bk[3]);
                mma(accK[nn], aZt, bk[0], bk[1]);
                mma(accK[nn + 1], aZt, bk[2], bk[3]);
            }
        }
    }
    __syncthreads();  // the operand reads of C7 are done: Q, K and R are dead
    if (has_next) copy_a1(jn, buf ^ 1);
    cp_async_commit();
    if (has_next) copy_b2(jn);
    cp_async_commit();
    const float beta_next = has_next ? beta_of(jn) : 0.f;
    {
        bf16* dqb = dq + bh * s.hs_k + (size_t)t0 * DK;
        bf16* dkb = dk + bh * s.hs_k + (size_t)t0 * DK;
#pragma unroll
        for (int nn = 0; nn < DKW / 8; ++nn) {
            const int col = DKW * nw + 8 * nn + 2 * tq;
            if (r0 < nval) {
                *reinterpret_cast<uint32_t*>(dqb + (size_t)r0 * DK + col) = pack(accQ[nn][0], accQ[nn][1]);
                *reinterpret_cast<uint32_t*>(dkb + (size_t)r0 * DK + col) = pack(accK[nn][0], accK[nn][1]);
            }
            if (r1 < nval) {
                *reinterpret_cast<uint32_t*>(dqb + (size_t)r1 * DK + col) = pack(accQ[nn][2], accQ[nn][3]);
                *reinterpret_cast<uint32_t*>(dkb + (size_t)r1 * DK + col) = pack(accK[nn][2], accK[nn][3]);
            }
        }
    }

    // ---- phase C8: dG, dg (reverse cumsum), dbeta; warp 0, two tokens per lane
    if (w == 0) {
        auto P = [&](int row, int n, int i) {
            float x = 0.f;
            for (int u = 0; u < n; ++u) x += part[(row + u) * C + i];
            return x;
        };
        float x[2], zs = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i = 2 * lane + h;
            x[h] = P(P_INTER, GW, i) + P(P_ROWP, GW, i) - P(P_COLP, 4, i) - P(P_Z, GW, i);
            zs += P(P_Z, GW, i);
            if (BETA) {
                x[h] += P(P_ROWA, GW, i) - P(P_COLA, 4, i) + P(P_KT, GW, i);
                if (i < nval) dbeta[bh * s.hs_g + t0 + i] = P(P_DBC, 4, i) + P(P_DBR, GW, i);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        if (lane == 31) x[1] += __expf(gC) * sdot + zs;
        // suffix sums over the lanes' pairs: dg_i = sum_{m >= i} dG_m
        float suf = x[0] + x[1];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += y;
        }
        float* dgb = dg + bh * s.hs_g + t0;
        if (2 * lane < nval) dgb[2 * lane] = suf;
        if (2 * lane + 1 < nval) dgb[2 * lane + 1] = suf - x[0];
    }
    __syncthreads();  // C8 is done with the partial sums
    if (!has_next) break;
    for (int e = tid; e < P_ROWS * C; e += GTH) part[e] = 0.f;
    if (tid < C) Bsb[(buf ^ 1) * C + tid] = beta_next;
    j = jn;
    buf ^= 1;
  }
}

template <typename K>
cudaError_t smem_attr(K* kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

#define TC_TRY(x)                          \
    do {                                   \
        cudaError_t e_ = (x);              \
        if (e_ != cudaSuccess) return e_;  \
    } while (0)

// Launches of the stages.  `w` carries the buffers of one segment.
template <int DV, bool BETA>
cudaError_t launch_prep(const char* name, const SeqView& s, const bf16* k, const bf16* v, const float* g,
                        const float* beta, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = prep_smem<DV>();
    TC_TRY(smem_attr(tc_prep_kernel<DV, BETA>, sm));
    SF_LAUNCH(name, st, tc_prep_kernel<DV, BETA><<<dim3(s.NC, s.BH), 256, sm, st>>>(
                            s, k, v, g, beta, w.Gc, w.Gm, w.W, w.Lm, w.Kh, w.Ut));
    return cudaGetLastError();
}

template <int DV, bool BETA>
cudaError_t launch_scan_fwd(const SeqView& s, const float* S_in, float* S_out, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = fwd_scan_smem<BETA>();
    TC_TRY(smem_attr(tc_scan_fwd_kernel<DV, BETA>, sm));
    SF_LAUNCH("tc_scan_fwd", st, tc_scan_fwd_kernel<DV, BETA><<<s.BH * (DV / 64), 256, sm, st>>>(
                                     s, w.Gm, w.W, w.Kh, w.Ut, S_in, w.Vnt, w.S0t, S_out));
    return cudaGetLastError();
}

template <int DV>
cudaError_t launch_out(const SeqView& s, const bf16* q, const bf16* k, bf16* o, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = out_smem<DV, false>();
    TC_TRY(smem_attr(tc_out_kernel<DV, false>, sm));
    SF_LAUNCH("tc_out", st, tc_out_kernel<DV, false><<<dim3(s.NC, s.BH), 128, sm, st>>>(
                                s, q, k, w.Gc, w.Vnt, w.S0t, o, nullptr, nullptr, nullptr));
    return cudaGetLastError();
}

template <int DV>
cudaError_t launch_out_og(const SeqView& s, const bf16* q, const bf16* k, bf16* o, const bf16* dO, const TcWs& w,
                          cudaStream_t st) {
    constexpr size_t sm = out_smem<DV, true>();
    TC_TRY(smem_attr(tc_out_kernel<DV, true>, sm));
    SF_LAUNCH("tc_out_og", st, tc_out_kernel<DV, true><<<dim3(s.NC, s.BH), 128, sm, st>>>(
                                   s, q, k, w.Gc, w.Vnt, w.S0t, o, dO, w.dVit, w.Dt));
    return cudaGetLastError();
}

template <int DV>
cudaError_t launch_intra(const SeqView& s, const bf16* q, const bf16* k, const bf16* dO, const TcWs& w,
                         cudaStream_t st) {
    constexpr size_t sm = intra_smem<DV>();
    TC_TRY(smem_attr(tc_intra_kernel<DV>, sm));
    SF_LAUNCH("tc_intra", st, tc_intra_kernel<DV><<<dim3(s.NC, s.BH), 128, sm, st>>>(s, q, k, dO, w.Gc, w.dVit, w.Dt));
    return cudaGetLastError();
}

template <int DV, bool BETA>
cudaError_t launch_scan_bwd(const SeqView& s, const BwdArgs& a, bool with_sr, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm_f = fwd_scan_smem<BETA>(), sm_b = bwd_scan_smem<BETA>();
    constexpr size_t sm = sm_f > sm_b ? sm_f : sm_b;
    TC_TRY(smem_attr(tc_scan_bwd_dual_kernel<DV, BETA>, sm));
    const int nb = (with_sr ? 2 : 1) * s.BH * (DV / 64);
    SF_LAUNCH("tc_scan_bwd", st, tc_scan_bwd_dual_kernel<DV, BETA><<<nb, 256, sm, st>>>(
                                     s, w.Dt, w.Gm, w.W, w.Kh, w.Ut, w.dVit, a.S_in, a.dS_out, w.Vnt, w.S0t, w.dVnt, w.dSCt,
                                     a.dS_in, with_sr ? 1 : 0));
    return cudaGetLastError();
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            n = v;
        else
            n = 148;
    }
    return n;
}

// Persistent: one CTA per SM at most; the CTAs take chunks from w.ticket, so
// they stay balanced when other kernels hold some of the SMs.
template <int DV, bool BETA>
cudaError_t launch_grad(const SeqView& s, const BwdArgs& a, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = grad_smem<DV>();
    TC_TRY(smem_attr(tc_grad_kernel<DV, BETA>, sm));
    TC_TRY(cudaMemsetAsync(w.ticket, 0, sizeof(int), st));
    const int grid = std::min(s.NC * s.BH, num_sms());
    SF_LAUNCH("tc_grad", st, tc_grad_kernel<DV, BETA><<<grid, GTH, sm, st>>>(
                                 s, static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k),
                                 static_cast<const bf16*>(a.v), a.beta, static_cast<const bf16*>(a.dO), w.Gc,
                                 w.Lm, w.Vnt, w.dVnt, w.S0t, w.dSCt, static_cast<bf16*>(a.dq), static_cast<bf16*>(a.dk),
                                 static_cast<bf16*>(a.dv), a.dg, a.dbeta, w.ticket));
    return cudaGetLastError();
}

template <int DV, bool BETA>
cudaError_t fwd_impl(const SeqView& s, const FwdArgs& a, void* ws, cudaStream_t st) {
    char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
    const TcWs w = tc_layout(s, false, base);
    const bf16* q = static_cast<const bf16*>(a.q);
    const bf16* k = static_cast<const bf16*>(a.k);
    TC_TRY((launch_prep<DV, BETA>("tc_prep", s, k, static_cast<const bf16*>(a.v), a.g, a.beta, w, st)));
    TC_TRY((launch_scan_fwd<DV, BETA>(s, a.S_in, a.S_out, w, st)));
    return launch_out<DV>(s, q, k, static_cast<bf16*>(a.o), w, st);
}

template <int DV, bool BETA>
cudaError_t bwd_impl(const SeqView& s, const BwdArgs& a, void* ws, cudaStream_t st) {
    char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
    const TcWs w = tc_layout(s, true, base);
    const bf16* q = static_cast<const bf16*>(a.q);
    const bf16* k = static_cast<const bf16*>(a.k);
    TC_TRY((launch_prep<DV, BETA>("tc_prep_bwd", s, k, static_cast<const bf16*>(a.v), a.g, a.beta, w, st)));
    TC_TRY((launch_intra<DV>(s, q, k, static_cast<const bf16*>(a.dO), w, st)));
    TC_TRY((launch_scan_bwd<DV, BETA>(s, a, true, w, st)));
    return launch_grad<DV, BETA>(s, a, w, st);
}

template <int DV, bool BETA>
cudaError_t stage_impl(TcStage stage, const SeqView& s, const FwdArgs* f, const BwdArgs* b, void* keep, void* slot,
                       cudaStream_t st) {
    size_t kb = 0;
    tc_parts(s, nullptr, nullptr, nullptr, &kb, nullptr, nullptr);
    const TcWs w = tc_parts(s, static_cast<char*>(keep), static_cast<char*>(keep) + kb, static_cast<char*>(slot),
                            nullptr, nullptr, nullptr);
    switch (stage) {
        case TcStage::Prep:
            return launch_prep<DV, BETA>("tc_prep", s, static_cast<const bf16*>(f->k),
                                         static_cast<const bf16*>(f->v), f->g, f->beta, w, st);
        case TcStage::Scan: return launch_scan_fwd<DV, BETA>(s, f->S_in, f->S_out, w, st);
        case TcStage::Out:
            return launch_out<DV>(s, static_cast<const bf16*>(f->q), static_cast<const bf16*>(f->k),
                                  static_cast<bf16*>(f->o), w, st);
        case TcStage::OutOg:
            return launch_out_og<DV>(s, static_cast<const bf16*>(f->q), static_cast<const bf16*>(f->k),
                                     static_cast<bf16*>(f->o), static_cast<const bf16*>(b->dO), w, st);
        case TcStage::Intra:
            return launch_intra<DV>(s, static_cast<const bf16*>(b->q), static_cast<const bf16*>(b->k),
                                    static_cast<const bf16*>(b->dO), w, st);
        case TcStage::ScanBwd: return launch_scan_bwd<DV, BETA>(s, *b, false, w, st);
        case TcStage::Grad: return launch_grad<DV, BETA>(s, *b, w, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool tc_supports(bool bf16_io, int dk, int dv, int Cc, bool) {
    return bf16_io && dk == DK && (dv == 64 || dv == 128) && Cc == C;
}

size_t tc_workspace_bytes(const SeqView& s, bool backward) { return tc_layout(s, backward, nullptr).total; }

size_t tc_keep_bytes(const SeqView& s) {
    size_t kb = 0, ob = 0;
    tc_parts(s, nullptr, nullptr, nullptr, &kb, &ob, nullptr);
    return kb + ob;
}

size_t tc_slot_bytes(const SeqView& s) {
    size_t sb = 0;
    tc_parts(s, nullptr, nullptr, nullptr, nullptr, nullptr, &sb);
    return sb;
}

cudaError_t tc_stage(TcStage stage, const SeqView& s, const FwdArgs* f, const BwdArgs* b, void* keep, void* slot,
                     cudaStream_t st) {
    if (s.dv == 128)
        return s.use_beta ? stage_impl<128, true>(stage, s, f, b, keep, slot, st)
                          : stage_impl<128, false>(stage, s, f, b, keep, slot, st);
    return s.use_beta ? stage_impl<64, true>(stage, s, f, b, keep, slot, st)
                      : stage_impl<64, false>(stage, s, f, b, keep, slot, st);
}

cudaError_t tc_fwd(const SeqView& s, const FwdArgs& a, void* ws, cudaStream_t st) {
    if (s.dv == 128) return s.use_beta ? fwd_impl<128, true>(s, a, ws, st) : fwd_impl<128, false>(s, a, ws, st);
    return s.use_beta ? fwd_impl<64, true>(s, a, ws, st) : fwd_impl<64, false>(s, a, ws, st);
}

cudaError_t tc_bwd(const SeqView& s, const BwdArgs& a, void* ws, cudaStream_t st) {
    if (s.dv == 128) return s.use_beta ? bwd_impl<128, true>(s, a, ws, st) : bwd_impl<128, false>(s, a, ws, st);
    return s.use_beta ? bwd_impl<64, true>(s, a, ws, st) : bwd_impl<64, false>(s, a, ws, st);
}

int tc_launches(bool backward) { return backward ? 4 : 3; }

cudaError_t tc_device_status(int* status, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(status, g_tc_status, sizeof(int));
    if (e != cudaSuccess || !clear || *status == 0) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
}

}  // namespace sf
