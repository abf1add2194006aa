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
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <string>

#include "tc_kernels.cuh"
#include "tc_mma.cuh"
#include "tc_umma.cuh"

namespace sf {
namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int C = 64;        // chunk length
constexpr int DK = 128;      // key head size
constexpr int LDK = DK + 8;  // shared row stride of [*][DK] tiles
constexpr int LDC = C + 8;   // shared row stride of [*][C] tiles
constexpr int LDF = 72;      // shared row stride of fp32 [C][C] tiles

// Offset of element (i, j) of the per-chunk fp32 L = (I + A)^{-1} as Pre
// stores it for the gradient kernels: row i, its 16-byte piece p at position
// p ^ (i % 8), so that the gradient kernel, which copies the tile linearly into
// shared memory, reads a column of it for eight rows without bank conflicts.
__host__ __device__ __forceinline__ int l_off(int i, int j) {
    return i * C + ((((j >> 2) ^ (i & 7))) << 2) + (j & 3);
}

// Set (bit 0) by a kernel that gave up waiting for one of its own bulk copies;
// read and cleared by sf_device_check().
__device__ int g_tc_status = 0;

struct TcWs {
    float* Gc;   // [BH][Tp]           chunk-local cumulative log-decay G
    float* Gm;   // [BH][Tp]           exp(G)
    bf16* W;     // [BH][Tp][DK]       -W (negated: the scans only ever subtract W products; canon per chunk)
    float* Lm;   // [BH][NC][C][C]     L = (I + A)^{-1} per chunk (delta path), for the gradient kernel
    bf16* Kh;    // [BH][Tp][DK]       K * exp(G_C - G) (canon per chunk)
    bf16* Ut;    // [BH][NC][DV][C]    U transposed per chunk, V^T without the beta path (canon)
    bf16* Vnt;   // [BH][NC][DV][C]    V_new transposed per chunk (canon, see tc_umma.cuh)
    bf16* S0t;   // [BH][NC][DV][DK]   state entering each chunk, transposed (canon)
    bf16* dVit;  // [BH][NC][DV][C]    intra-chunk part of dV_new, transposed (canon)
    bf16* dVnt;  // [BH][NC][DV][C]    dV_new transposed (canon)
    bf16* dSCt;  // [BH][NC][DV][DK]   gradient of the state leaving each chunk, transposed (canon)
    bf16* Dt;    // [BH][NC][DV][DK]   scale (gamma * dO)^T Q per chunk, transposed (canon)
    int* ticket;  // chunk counter of the persistent gradient kernel
    int* oticket;  // chunk counter of the persistent Out kernel
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
    w.oticket = reinterpret_cast<int*>(take(sizeof(int)));
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
    if (BETA)  // the blocks above the diagonal of L (block_inverse writes the others)
        for (int e = tid; e < C * C / 4; e += 256) {
            const int i = e >> 4, j = (e & 15) * 4;
            if (j >= 16 * ((i >> 4) + 1)) *reinterpret_cast<float4*>(Lf + i * LDF + j) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    cp_async_wait<0>();
    __syncthreads();

    for (int i = tid; i < C; i += 256) {
        const float e = __expf(Gs[i]);
        Gc[bh * Tp + t0 + i] = Gs[i];
        Gmo[bh * Tp + t0 + i] = e;
        BGs[i] = Bs[i] * e;
    }
    const float gC = Gs[C - 1];
    for (int e = tid; e < C * (DK / 8); e += 256) {  // canon tile, written in address order
        int r, cc;
        umma::canon_piece(e, DK, r, cc);
        const float d = __expf(gC - Gs[r]);
        uint4 x = *reinterpret_cast<const uint4*>(Ks + r * LDK + cc);
        x.x = scale2(x.x, d, d);
        x.y = scale2(x.y, d, d);
        x.z = scale2(x.z, d, d);
        x.w = scale2(x.w, d, d);
        reinterpret_cast<uint4*>(Kho + (bh * Tp + t0) * DK)[e] = x;
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
                for (int h = 0; h < 2; ++h) {
                    const int i = 16 * mw + gq + 8 * h, j = 32 * nw + 8 * nn + 2 * tq;
                    float2 a2;
                    a2.x = (j < i) ? Bs[i] * __expf(Gs[i] - Gs[j]) * acc[nn][2 * h] : 0.f;
                    a2.y = (j + 1 < i) ? Bs[i] * __expf(Gs[i] - Gs[j + 1]) * acc[nn][2 * h + 1] : 0.f;
                    *reinterpret_cast<float2*>(Af + i * LDF + j) = a2;
                }
        }
        __syncthreads();
        block_inverse(Af, LDF, Lf, LDF, Yb, tid, 256);
        float* Lg = Lmo + ((size_t)bh * s.NC + c) * C * C;
        for (int e = tid; e < C * C / 4; e += 256) {
            const int i = e >> 4, j = (e & 15) * 4;
            *reinterpret_cast<float4*>(Lg + l_off(i, j)) = *reinterpret_cast<const float4*>(Lf + i * LDF + j);
        }
        for (int e = tid; e < C * C / 8; e += 256) {  // A is dead: its region takes the T tiles
            const int i = e >> 3, j = (e & 7) * 8;
            float l[8], bg[8], b[8];
            *reinterpret_cast<float4*>(l) = *reinterpret_cast<const float4*>(Lf + i * LDF + j);
            *reinterpret_cast<float4*>(l + 4) = *reinterpret_cast<const float4*>(Lf + i * LDF + j + 4);
            *reinterpret_cast<float4*>(bg) = *reinterpret_cast<const float4*>(BGs + j);
            *reinterpret_cast<float4*>(bg + 4) = *reinterpret_cast<const float4*>(BGs + j + 4);
            *reinterpret_cast<float4*>(b) = *reinterpret_cast<const float4*>(Bs + j);
            *reinterpret_cast<float4*>(b + 4) = *reinterpret_cast<const float4*>(Bs + j + 4);
            uint32_t tw[4], tu[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                tw[h] = pack(l[2 * h] * bg[2 * h], l[2 * h + 1] * bg[2 * h + 1]);
                tu[h] = pack(l[2 * h] * b[2 * h], l[2 * h + 1] * b[2 * h + 1]);
            }
            *reinterpret_cast<uint4*>(Tw + i * LDC + j) = make_uint4(tw[0], tw[1], tw[2], tw[3]);
            *reinterpret_cast<uint4*>(Tu + i * LDC + j) = make_uint4(tu[0], tu[1], tu[2], tu[3]);
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
            // transposed by stmatrix: matrix m = (row half m % 2, n-tile nn + m / 2)
#pragma unroll
            for (int nn = 0; nn < DV / 16; nn += 2) {
                const uint32_t fr[4] = {pack(acc[nn][0], acc[nn][1]), pack(acc[nn][2], acc[nn][3]),
                                        pack(acc[nn + 1][0], acc[nn + 1][1]), pack(acc[nn + 1][2], acc[nn + 1][3])};
                const int m = lane >> 3;
                const int col = (DV / 2) * nw + 8 * (nn + (m >> 1)) + (lane & 7), i = 16 * mw + 8 * (m & 1);
                stsm_x4_t(Ust + col * LDC + i, fr);
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
        for (int e = tid; e < C * (DK / 8); e += 256) {  // canon, in address order
            int r, cc;
            umma::canon_piece(e, DK, r, cc);
            reinterpret_cast<uint4*>(Wo + (bh * Tp + t0) * DK)[e] = *reinterpret_cast<const uint4*>(Wst + r * LDK + cc);
        }
    } else {
        for (int e = tid; e < C * DV; e += 256) {
            const int i = e / DV, col = e % DV;
            Ust[col * LDC + i] = Vs[i * LDV + col];
        }
        __syncthreads();
    }
    bf16* Utg = Uto + ((size_t)bh * s.NC + c) * DV * C;
    for (int e = tid; e < DV * (C / 8); e += 256) {  // canon, in address order
        int r, cc;
        umma::canon_piece(e, C, r, cc);
        reinterpret_cast<uint4*>(Utg)[e] = *reinterpret_cast<const uint4*>(Ust + r * LDC + cc);
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
            *reinterpret_cast<uint32_t*>(dVi + umma::canon_el(r, j, C)) = pack(acc[nn][0], acc[nn][1]);
            *reinterpret_cast<uint32_t*>(dVi + umma::canon_el(r + 8, j, C)) = pack(acc[nn][2], acc[nn][3]);
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
                *reinterpret_cast<uint32_t*>(Dg + umma::canon_el(r, d, DK)) = pack(acc[nn][0], acc[nn][1]);
                *reinterpret_cast<uint32_t*>(Dg + umma::canon_el(r + 8, d, DK)) = pack(acc[nn][2], acc[nn][3]);
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

// Copy BYTES contiguous bytes global -> shared, 16 bytes per cp.async request.
template <int BYTES, int NT>
__device__ __forceinline__ void copy_linear(void* s, const void* g, int tid) {
    for (int e = tid; e < BYTES / 16; e += NT)
        cp_async16(static_cast<char*>(s) + 16 * e, static_cast<const char*>(g) + 16 * e, true);
}

// ------------------------------------------------------------ state scans ---
// The forward state scan (ST) and the reverse state-gradient scan (STB) run
// the same step on different operands.  With X, Y the two [C][DK] operand
// tiles of a chunk and R the running state (S^T or dS^T: d_v rows, d_k
// columns, fp32), one step is
//     Z^T = I^T + R X^T                 product 1: d_v x C, contraction over d_k
//     R  <- gamma_C R (+ E) + Z^T Y     product 2: d_v x d_k, contraction over C
// forward  (chunks in order):   X = -W, Y = Khat, I = U^T, Z = V_new;
//          per chunk the entering R (S0^T) and Z^T are written, R at the end is S_out^T;
// backward (chunks in reverse): X = Khat, Y = -W, I = dVi^T, E = D^T, Z = dV_new;
//          per chunk the entering R (dS_C^T) and Z^T, R at the end is dS_in^T.
// Without the beta path W is absent: the forward has no product 1 (V_new = V),
// the backward no product 2 (dS <- gamma_C dS + D).
//
// Work split (the pages' tiling of the state transition over d_v): a CTA owns
// NCG slices of 16 state columns, each carried by four warps.  In product 1
// warp q of a slice computes tokens 16q..16q+15 over all of d_k, in product 2
// state rows 32q..32q+31 of d_k over all C tokens; the bf16 left-operand
// fragments each warp needs from the other three (R for product 1, Z^T for
// product 2) pass through shared memory, with one 128-thread barrier per
// product.  The state never leaves the register file.  Operand tiles arrive by
// bulk copies (the TMA engine) into kStages buffers completing on mbarriers;
// the outputs are staged by stmatrix and written back by bulk stores.
constexpr uint32_t kTileK = C * DK * 2;   // a [C][DK] bf16 tile

template <int DV, bool BETA, bool BWD, int NCG>
struct Chain {
    static constexpr bool HAS_X = BWD || BETA;  // product 1 runs
    static constexpr bool HAS_Y = !BWD || BETA;  // product 2 runs
    static constexpr uint32_t kI = NCG * 16 * C * 2;                // I^T rows of this CTA
    static constexpr uint32_t kE = BWD ? NCG * 16 * DK * 2 : 0;     // E rows of this CTA
    static constexpr uint32_t kX = HAS_X ? kTileK : 0, kY = HAS_Y ? kTileK : 0;
    static constexpr uint32_t TX = kX + kY + kI + C * 4 + kE;       // bytes of one stage (all copied)
    static constexpr size_t OUT = (size_t)NCG * 16 * (DK + C) * 2;  // staged R and Z^T rows of one step
    static constexpr size_t XCH = (size_t)NCG * 12 * 32 * 16;       // 8 R + 4 Z^T fragments per slice
    // staged outputs of step i are flushed during step i+1 and must have been
    // read when step i + kOutBufs writes the buffer again
    static constexpr int kOutBufs = BWD ? 3 : 2;
    static constexpr size_t smem(int stages) { return stages * (size_t)TX + kOutBufs * OUT + XCH + 8 * stages; }
    // as many operand stages as fit (up to 6): a step's operands are requested
    // kStages - 1 steps ahead, which must cover the latency of the copies.  The
    // forward chain keeps 3 stages and 2 output buffers (145 KB at d_v = 128,
    // two slices) so that a Pre CTA (75.5 KB) fits beside it on its SM: the Pre
    // of later pieces then also runs on the chain's SMs (headline forward 1.49
    // instead of 1.54 ms, measured); the reverse chain runs beside the gradient
    // kernel, which leaves no room on an SM, and keeps as many stages as fit.
    static constexpr int kFit = smem(6) <= 227 * 1024 ? 6 : smem(5) <= 227 * 1024 ? 5
                              : smem(4) <= 227 * 1024 ? 4 : smem(3) <= 227 * 1024 ? 3 : 2;
    static constexpr int kStages = BWD ? kFit : (kFit < 3 ? kFit : 3);
    static constexpr size_t SMEM = smem(kStages);
};

__device__ __forceinline__ void put_frag(uint4* p, const uint32_t (&a)[4]) { *p = make_uint4(a[0], a[1], a[2], a[3]); }
__device__ __forceinline__ void get_frag(const uint4* p, uint32_t (&a)[4]) {
    const uint4 v = *p;
    a[0] = v.x;
    a[1] = v.y;
    a[2] = v.z;
    a[3] = v.w;
}
// Barrier of the four warps of slice g (named barriers 1..NCG).
__device__ __forceinline__ void slice_sync(int g) { asm volatile("bar.sync %0, 128;\n" ::"r"(g + 1) : "memory"); }

// Operands of one chain launch, for one direction.
struct ChainOps {
    const bf16* X;      // [BH][Tp][DK] canon per chunk: -W (forward) or Khat (backward)
    const bf16* Y;      // [BH][Tp][DK] canon per chunk: Khat (forward) or -W (backward)
    const bf16* I;      // [BH][NC][DV][C] canon: U^T or dVi^T
    const bf16* E;      // [BH][NC][DV][DK] canon: D^T (backward only)
    const float* Gm;    // [BH][Tp] exp(G)
    const float* R_in;  // [BH][DK][DV] S_in or dS_out (NULL = zeros)
    bf16* Rt;           // [BH][NC][DV][DK] canon: S0^T or dS_C^T per chunk (NULL = skip)
    bf16* Zt;           // [BH][NC][DV][C] canon: V_new^T or dV_new^T per chunk (NULL = skip)
    float* R_out;       // [BH][DK][DV] S_out or dS_in (NULL = skip)
};

template <int DV, bool BETA, bool BWD, int NCG>
__device__ __forceinline__ void chain_cta(const SeqView& s, int bh, int vb, const ChainOps& op, unsigned char* smem) {
    using CH = Chain<DV, BETA, BWD, NCG>;
    constexpr int NS = CH::kStages;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, gq = lane >> 2, tq = lane & 3;
    const int g = w >> 2, q = w & 3;        // slice of this warp, warp index inside the slice
    const int v0 = vb * 16 * NCG;           // first state column of the CTA
    const int vr = 16 * g;                  // first row of this slice in the CTA's tiles
    const size_t Tp = (size_t)s.NC * C;
    unsigned char* outs = smem + NS * (size_t)CH::TX;
    uint4* xch = reinterpret_cast<uint4*>(outs + CH::kOutBufs * CH::OUT) + g * 12 * 32 + lane;
    uint64_t* bars = reinterpret_cast<uint64_t*>(outs + CH::kOutBufs * CH::OUT + CH::XCH);
    bool failed = false;

    auto chunk_of = [&](int i) { return BWD ? s.NC - 1 - i : i; };
    struct Stage {
        bf16 *X, *Y, *I, *E;
        float* G;
    };
    auto stage = [&](int buf) {
        unsigned char* p = smem + buf * (size_t)CH::TX;
        Stage st;
        st.X = reinterpret_cast<bf16*>(p);
        st.Y = reinterpret_cast<bf16*>(p + CH::kX);
        st.I = reinterpret_cast<bf16*>(p + CH::kX + CH::kY);
        st.G = reinterpret_cast<float*>(p + CH::kX + CH::kY + CH::kI);
        st.E = reinterpret_cast<bf16*>(p + CH::kX + CH::kY + CH::kI + C * 4);
        return st;
    };
    auto load = [&](int i) {  // thread 0: bulk copies of step i's operands
        const int cc = chunk_of(i), buf = i % NS;
        const Stage st = stage(buf);
        const size_t row0 = (size_t)bh * Tp + (size_t)cc * C;
        const size_t blk = ((size_t)bh * s.NC + cc) * DV + v0;
        mbar_expect_tx(&bars[buf], CH::TX);
        if (CH::HAS_X) bulk_load(st.X, op.X + row0 * DK, kTileK, &bars[buf]);
        if (CH::HAS_Y) bulk_load(st.Y, op.Y + row0 * DK, kTileK, &bars[buf]);
        bulk_load(st.I, op.I + blk * C, CH::kI, &bars[buf]);
        bulk_load(st.G, op.Gm + row0, C * 4, &bars[buf]);
        if (BWD) bulk_load(st.E, op.E + blk * DK, CH::kE, &bars[buf]);
    };
    const bool outputs = op.Rt || op.Zt;
    auto flush = [&](int i) {  // thread 0: bulk-store the staged outputs of step i
        unsigned char* o = outs + (i % CH::kOutBufs) * CH::OUT;
        const size_t blk = ((size_t)bh * s.NC + chunk_of(i)) * DV + v0;
        if (op.Rt) bulk_store(op.Rt + blk * DK, o, NCG * 16 * DK * 2);
        if (op.Zt) bulk_store(op.Zt + blk * C, o + NCG * 16 * DK * 2, NCG * 16 * C * 2);
        bulk_commit();
    };

    // R: rows vr + gq (+8) of the slice, d_k columns 32q + 8j + 2tq (+1)
    float r[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int vv = v0 + vr + gq + 8 * (e >> 1), d = 32 * q + 8 * j + 2 * tq + (e & 1);
            r[j][e] = op.R_in ? op.R_in[((size_t)bh * DK + d) * DV + vv] : 0.f;
        }

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (tid == 0)
        for (int i = 0; i < NS - 1 && i < s.NC; ++i) load(i);
    for (int i = 0; i < s.NC; ++i) {
        if (tid == 0) {
            if (i + NS - 1 < s.NC) load(i + NS - 1);  // its buffer was released by the barrier ending step i-1
            if (outputs && i > 0) flush(i - 1);
        }
        const Stage st = stage(i % NS);
        bf16* Rs = reinterpret_cast<bf16*>(outs + (i % CH::kOutBufs) * CH::OUT);  // [16 NCG][DK]
        bf16* Zs = Rs + NCG * 16 * DK;                                        // [16 NCG][C]
        // the entering R as bf16 fragments of this warp's k-tiles 2q, 2q+1
        uint32_t sa[2][4];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            c2a(sa[jj], r[2 * jj], r[2 * jj + 1]);
            if (CH::HAS_X) put_frag(xch + (2 * q + jj) * 32, sa[jj]);
            if (op.Rt) umma::st_afrag_c(Rs, DK, vr, 16 * (2 * q + jj), sa[jj], lane);
        }
        if (CH::HAS_X) slice_sync(g);
        mbar_wait(&bars[i % NS], (i / NS) & 1, &g_tc_status, failed);
        const float gamC = st.G[C - 1];

        // product 1: Z^T (rows vr.., tokens 16q + 8n + 2tq ..) = I^T + R X^T
        float z[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const int tc0 = 16 * q + 8 * n + 2 * tq;
            const float2 u0 = unpack(*umma::canon_at<uint32_t>(st.I, vr + gq, tc0, C));
            const float2 u1 = unpack(*umma::canon_at<uint32_t>(st.I, vr + gq + 8, tc0, C));
            z[n][0] = u0.x;
            z[n][1] = u0.y;
            z[n][2] = u1.x;
            z[n][3] = u1.y;
        }
        if (CH::HAS_X) {
            uint32_t ra[8][4];  // all eight k-tiles of R (own ones from registers)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                if ((kk >> 1) == q) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) ra[kk][e] = sa[kk & 1][e];
                } else {
                    get_frag(xch + kk * 32, ra[kk]);
                }
            }
            float zq[2][4] = {};  // odd k-tiles: two shorter dependent chains
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t b[4];
                umma::ldBnk_c(b, st.X, DK, 16 * q, 16 * kk, lane);
                if (kk & 1) {
                    mma(zq[0], ra[kk], b[0], b[1]);
                    mma(zq[1], ra[kk], b[2], b[3]);
                } else {
                    mma(z[0], ra[kk], b[0], b[1]);
                    mma(z[1], ra[kk], b[2], b[3]);
                }
            }
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) z[n][e] += zq[n][e];
        }
        uint32_t za[4];
        c2a(za, z[0], z[1]);
        if (CH::HAS_Y) put_frag(xch + (8 + q) * 32, za);
        if (op.Zt) umma::st_afrag_c(Zs, C, vr, 16 * q, za, lane);

        // product 2: R <- gamma_C R (+ E) + Z^T Y
        if (BWD) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = 32 * q + 8 * j + 2 * tq;
                const float2 d0 = unpack(*umma::canon_at<uint32_t>(st.E, vr + gq, col, DK));
                const float2 d1 = unpack(*umma::canon_at<uint32_t>(st.E, vr + gq + 8, col, DK));
                r[j][0] = fmaf(r[j][0], gamC, d0.x);
                r[j][1] = fmaf(r[j][1], gamC, d0.y);
                r[j][2] = fmaf(r[j][2], gamC, d1.x);
                r[j][3] = fmaf(r[j][3], gamC, d1.y);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) r[j][e] *= gamC;
        }
        if (CH::HAS_Y) {
            slice_sync(g);
            uint32_t zf[4][4];
#pragma unroll
            for (int kt = 0; kt < 4; ++kt) {
                if (kt == q) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) zf[kt][e] = za[e];
                } else {
                    get_frag(xch + (8 + kt) * 32, zf[kt]);
                }
            }
#pragma unroll
            for (int kt = 0; kt < 4; ++kt)
#pragma unroll
                for (int n2 = 0; n2 < 2; ++n2) {
                    uint32_t b[4];
                    umma::ldBkn_c(b, st.Y, DK, 32 * q + 16 * n2, 16 * kt, lane);
                    mma(r[2 * n2], zf[kt], b[0], b[1]);
                    mma(r[2 * n2 + 1], zf[kt], b[2], b[3]);
                }
        }
        if (outputs) fence_proxy_async_smem();
        if (tid == 0 && outputs) bulk_wait_read<CH::kOutBufs - 2>();  // the buffer step i+1 writes is read out
        __syncthreads();
    }
    if (tid == 0) {
        if (outputs && s.NC > 0) flush(s.NC - 1);
        bulk_wait<0>();
    }
    if (op.R_out) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int vv = v0 + vr + gq + 8 * (e >> 1), d = 32 * q + 8 * j + 2 * tq + (e & 1);
                op.R_out[((size_t)bh * DK + d) * DV + vv] = r[j][e];
            }
    }
}

// Chain CTAs per head for NCG slices per CTA.
template <int DV, int NCG>
constexpr int chain_ctas_per_head() { return DV / (16 * NCG); }

template <int DV, bool BETA, int NCG>
__global__ void __launch_bounds__(128 * NCG, 1)
tc_scan_fwd_kernel(SeqView s, ChainOps op) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NB = chain_ctas_per_head<DV, NCG>();
    chain_cta<DV, BETA, false, NCG>(s, blockIdx.x / NB, blockIdx.x % NB, op, smem);
}

// Backward chains in one launch: with nsr > 0, blocks [0, nsr) recompute the
// forward states (V_new^T and the chunk-entry states, op_f) and the rest run
// the reverse state-gradient scan (op_b); the two groups share no data.
template <int DV, bool BETA, int NCG>
__global__ void __launch_bounds__(128 * NCG, 1)
tc_scan_bwd_dual_kernel(SeqView s, ChainOps op_f, ChainOps op_b, int nsr) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NB = chain_ctas_per_head<DV, NCG>();
    int id = blockIdx.x;
    if (id < nsr) {
        chain_cta<DV, BETA, false, NCG>(s, id / NB, id % NB, op_f, smem);
    } else {
        id -= nsr;
        chain_cta<DV, BETA, true, NCG>(s, id / NB, id % NB, op_b, smem);
    }
}

// ------------------------------------------------- state scans, tcgen05 ---
// The same step (see chain_cta) with the whole state of a head in one CTA, on
// the fifth-generation tensor cores (d_v = 128): R (S^T or dS^T, fp32) lives
// in TMEM, lane v = state row v, columns 0..127 = d_k; 8 warps, warp w's
// threads own lanes 32 (w % 4).. (thread = state row) and half of each row's
// columns (w / 4).  Per chunk:
//   every thread loads its row of R, writes it as bf16 into a canon [d_v][d_k]
//   tile (the A operand of product 1 and the chunk's R output) and stores
//   gamma_C R (+ E) back;
//   product 1: Z^T = R X^T, M = 128, N = C, K = d_k, into TMEM columns 128..;
//   every thread adds its row of I^T and writes Z^T as bf16 into a canon
//   [d_v][C] tile (the A operand of product 2 and the chunk's Z output);
//   product 2: R += Z^T Y, M = 128, N = d_k, K = C, accumulating on the
//   scaled R.
// One CTA per head instead of d_v / 32 CTAs of warp-level products: a quarter
// of the SMs and of the operand reads (each head's X and Y tiles are read
// once), the products at the full M = 128 rate.
template <bool BETA, bool BWD>
struct Chain5 {
    static constexpr bool HAS_X = BWD || BETA;
    static constexpr bool HAS_Y = !BWD || BETA;
    static constexpr uint32_t kI = 128 * C * 2;              // I^T, canon [d_v][C]
    static constexpr uint32_t kE = BWD ? 128 * DK * 2 : 0;   // E, canon [d_v][d_k]
    static constexpr uint32_t kX = HAS_X ? kTileK : 0, kY = HAS_Y ? kTileK : 0;
    static constexpr uint32_t TX = kX + kY + kI + C * 4 + kE;  // one stage, all copied
    static constexpr size_t kR = (size_t)128 * DK * 2;         // R as bf16, canon [d_v][d_k]
    static constexpr size_t kZ = (size_t)128 * C * 2;          // Z^T as bf16, canon [d_v][C]
    static constexpr size_t smem(int st) { return st * (size_t)TX + kR + kZ + 8 * (st + 2) + 16; }
    static constexpr int kStages = smem(4) <= 227 * 1024 ? 4 : smem(3) <= 227 * 1024 ? 3 : 2;
    static constexpr size_t SMEM = smem(kStages);
};

template <bool BETA, bool BWD>
__device__ __forceinline__ void chain5_cta(const SeqView& s, int bh, const ChainOps& op, unsigned char* smem) {
    using CH = Chain5<BETA, BWD>;
    constexpr int NS = CH::kStages;
    constexpr int DV = 128;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int v = 32 * (w & 3) + lane;  // this thread's state row = TMEM lane
    const int hf = w >> 2;              // the half of the row's columns this thread handles
    const size_t Tp = (size_t)s.NC * C;
    bf16* Rb = reinterpret_cast<bf16*>(smem + NS * (size_t)CH::TX);
    bf16* Zb = reinterpret_cast<bf16*>(smem + NS * (size_t)CH::TX + CH::kR);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NS * (size_t)CH::TX + CH::kR + CH::kZ);  // [NS]
    uint64_t* bM1 = bars + NS;
    uint64_t* bM2 = bars + NS + 1;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + NS + 2);
    bool failed = false;
    const bool outputs = op.Rt || op.Zt;

    auto chunk_of = [&](int i) { return BWD ? s.NC - 1 - i : i; };
    struct Stage {
        bf16 *X, *Y, *I, *E;
        float* G;
    };
    auto stage = [&](int buf) {
        unsigned char* p = smem + buf * (size_t)CH::TX;
        Stage st;
        st.X = reinterpret_cast<bf16*>(p);
        st.Y = reinterpret_cast<bf16*>(p + CH::kX);
        st.I = reinterpret_cast<bf16*>(p + CH::kX + CH::kY);
        st.G = reinterpret_cast<float*>(p + CH::kX + CH::kY + CH::kI);
        st.E = reinterpret_cast<bf16*>(p + CH::kX + CH::kY + CH::kI + C * 4);
        return st;
    };
    auto load = [&](int i) {  // thread 0: bulk copies of step i's operands
        const int cc = chunk_of(i), buf = i % NS;
        const Stage st = stage(buf);
        const size_t row0 = (size_t)bh * Tp + (size_t)cc * C;
        const size_t blk = ((size_t)bh * s.NC + cc) * DV;
        mbar_expect_tx(&bars[buf], CH::TX);
        if (CH::HAS_X) bulk_load(st.X, op.X + row0 * DK, kTileK, &bars[buf]);
        if (CH::HAS_Y) bulk_load(st.Y, op.Y + row0 * DK, kTileK, &bars[buf]);
        bulk_load(st.I, op.I + blk * C, CH::kI, &bars[buf]);
        bulk_load(st.G, op.Gm + row0, C * 4, &bars[buf]);
        if (BWD) bulk_load(st.E, op.E + blk * DK, CH::kE, &bars[buf]);
    };

    if (tid == 0) {
        for (int i = 0; i < NS + 2; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
    }
    if (w == 0) umma::alloc(tslot, 256);
    __syncthreads();
    umma::fence_after();
    const uint32_t tm = *tslot;
    const uint32_t trow = umma::taddr(tm, 32 * (w & 3), 0);
    const int rc0 = 64 * hf, zc0 = 32 * hf;  // first R and Z^T column of this thread
    constexpr uint32_t ZC = 128;  // TMEM column of Z^T
    if (tid == 0)
        for (int i = 0; i < NS - 1 && i < s.NC; ++i) load(i);
    // the entering state: R[v][d] = R_in[d][v]
#pragma unroll 1
    for (int g = 0; g < 2; ++g) {
        float x[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = op.R_in ? op.R_in[((size_t)bh * DK + rc0 + 32 * g + j) * DV + v] : 0.f;
        umma::st_row32(trow + rc0 + 32 * g, x);
    }
    umma::wait_st();

    constexpr uint32_t I1 = umma::idesc_bf16(128, C, false, false);
    constexpr uint32_t I2 = umma::idesc_bf16(128, DK, false, true);
    for (int i = 0; i < s.NC; ++i) {
        const Stage st = stage(i % NS);
        mbar_wait(&bars[i % NS], (i / NS) & 1, &g_tc_status, failed);
        if (CH::HAS_Y && i > 0) mbar_wait(bM2, (i - 1) & 1, &g_tc_status, failed);  // R updated
        umma::fence_after();
        float x[64];  // this thread's half row of R
#pragma unroll
        for (int g = 0; g < 2; ++g) umma::ld_row32(trow + rc0 + 32 * g, *reinterpret_cast<float(*)[32]>(x + 32 * g));
        if (tid == 0) {
            // step i-1's buffer is free (its products have completed)
            if (i + NS - 1 < s.NC) load(i + NS - 1);
            if (outputs && i > 0) bulk_wait_read<0>();  // step i-1's outputs have left Rb, Zb
        }
        umma::wait_ld();
        __syncthreads();  // Rb and Zb may be rewritten
        // R as bf16 into its canon row: product 1's A and the chunk's R output
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            uint4 o;
            o.x = pack(x[8 * p], x[8 * p + 1]);
            o.y = pack(x[8 * p + 2], x[8 * p + 3]);
            o.z = pack(x[8 * p + 4], x[8 * p + 5]);
            o.w = pack(x[8 * p + 6], x[8 * p + 7]);
            *umma::canon_at<uint4>(Rb, v, rc0 + 8 * p, DK) = o;
        }
        fence_proxy_async_smem();
        __syncthreads();  // Rb complete
        if (tid == 0) {
            umma::fence_after();
            if (CH::HAS_X) {
                umma::chain<DK / 16>(tm + ZC, I1, false, umma::op_k(Rb, DK), umma::op_k(st.X, DK));
                umma::commit(bM1);
            }
            if (op.Rt) bulk_store(op.Rt + ((size_t)bh * s.NC + chunk_of(i)) * DV * DK, Rb, (uint32_t)CH::kR);
        }
        // while product 1 runs: gamma_C R (+ E) back into TMEM, this thread's row of I^T
        const float gamC = st.G[C - 1];
        if (BWD) {
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const uint4 e = *umma::canon_at<uint4>(st.E, v, rc0 + 8 * p, DK);
                const uint32_t ev[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 f = unpack(ev[h]);
                    x[8 * p + 2 * h] = fmaf(x[8 * p + 2 * h], gamC, f.x);
                    x[8 * p + 2 * h + 1] = fmaf(x[8 * p + 2 * h + 1], gamC, f.y);
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) x[j] *= gamC;
        }
#pragma unroll
        for (int g = 0; g < 2; ++g)
            umma::st_row32(trow + rc0 + 32 * g, *reinterpret_cast<const float(*)[32]>(x + 32 * g));
        uint4 irow[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) irow[p] = *umma::canon_at<uint4>(st.I, v, zc0 + 8 * p, C);
        umma::wait_st();
        // Z^T = I^T (+ R X^T) as bf16 into its canon row: product 2's A and the chunk's Z output
        float z[32];
        if (CH::HAS_X) {
            mbar_wait(bM1, i & 1, &g_tc_status, failed);
            umma::fence_after();
            umma::ld_row32(trow + ZC + zc0, z);
            umma::wait_ld();
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) z[j] = 0.f;
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const uint32_t uv[4] = {irow[p].x, irow[p].y, irow[p].z, irow[p].w};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 f = unpack(uv[h]);
                o[h] = pack(f.x + z[8 * p + 2 * h], f.y + z[8 * p + 2 * h + 1]);
            }
            *umma::canon_at<uint4>(Zb, v, zc0 + 8 * p, C) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        umma::fence_before();
        __syncthreads();  // Zb complete, R scaled; I, E, G of this stage read
        if (tid == 0) {
            umma::fence_after();
            if (CH::HAS_Y) {
                umma::chain<C / 16>(tm, I2, true, umma::op_k(Zb, C), umma::op_mn(st.Y, DK));
                umma::commit(bM2);
            }
            if (op.Zt) bulk_store(op.Zt + ((size_t)bh * s.NC + chunk_of(i)) * DV * C, Zb, (uint32_t)CH::kZ);
            if (outputs) bulk_commit();
        }
    }
    if (CH::HAS_Y && s.NC > 0) mbar_wait(bM2, (s.NC - 1) & 1, &g_tc_status, failed);
    umma::fence_after();
    if (op.R_out) {
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
            float x[32];
            umma::ld_row32(trow + rc0 + 32 * g, x);
            umma::wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) op.R_out[((size_t)bh * DK + rc0 + 32 * g + j) * DV + v] = x[j];
        }
    }
    if (tid == 0 && outputs) bulk_wait<0>();
    umma::fence_before();
    __syncthreads();
    if (w == 0) {
        umma::fence_after();
        umma::dealloc(tm, 256);
    }
}

template <bool BETA>
__global__ void __launch_bounds__(256, 1) tc_chain5_fwd_kernel(SeqView s, ChainOps op) {
    extern __shared__ __align__(16) unsigned char smem[];
    chain5_cta<BETA, false>(s, blockIdx.x, op, smem);
}
// Blocks [0, nsr) recompute the forward states (op_f), the rest run the
// reverse state-gradient scan (op_b).
template <bool BETA>
__global__ void __launch_bounds__(256, 1) tc_chain5_bwd_kernel(SeqView s, ChainOps op_f, ChainOps op_b, int nsr) {
    extern __shared__ __align__(16) unsigned char smem[];
    if ((int)blockIdx.x < nsr)
        chain5_cta<BETA, false>(s, blockIdx.x, op_f, smem);
    else
        chain5_cta<BETA, true>(s, blockIdx.x - nsr, op_b, smem);
}

// ------------------------------------------------------------------- out ---
// Tensor maps of the token-major tiles a kernel copies by TMA (see canon_map):
// q, k and dO in canon layout; `on` is 0 when they could not be made, and
// chunks shorter than C always take per-thread cp.async.
struct TokMaps {
    CUtensorMap q, k, dO;
    int on;
};

template <int DV, bool OG>
struct O2 {
    static constexpr size_t kQ = (size_t)C * DK * 2;          // Q, K (canon [C][DK])
    static constexpr size_t kS = (size_t)DV * DK * 2;         // S0^T (canon [DV][DK])
    static constexpr size_t kVn = (size_t)DV * C * 2;         // V_new^T (canon [DV][C])
    static constexpr size_t kdO = OG ? (size_t)C * DV * 2 : 0;  // dO (canon [C][DV])
    static constexpr size_t kBuf = 2 * kQ + kS + kVn + kdO + C * 4;
    static constexpr size_t SMEM = 2 * kBuf + (size_t)C * C * 2 + 2 * 8 + 2 * 4;
};

// Intra-chunk backward products of one chunk from canon tiles, 8 warps:
// dVi^T = (P^T dO)^T and D^T = (scale (gamma * dO)^T Q)^T, each warp one
// 16-row tile of d_v (d_v = 128) or one tile and half the columns (d_v = 64).
template <int DV>
__device__ __forceinline__ void og_products8(const SeqView& s, const bf16* Qs, const bf16* dOs, const bf16* Ps,
                                             const float* Gs, bf16* dVi, bf16* Dg, int w, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    const int m0 = DV == 128 ? 16 * w : 16 * (w & 3);
    constexpr int NVI = DV == 128 ? 8 : 4;   // n-tiles of dVi^T per warp
    const int n0 = DV == 128 ? 0 : 32 * (w >> 2);
    {  // dVi^T[v][j] = sum_i dO[i][v] P[i][j]
        float acc[NVI][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t a[4];
            umma::ldAt_c(a, dOs, DV, m0, 16 * kk, lane);
#pragma unroll
            for (int nn = 0; nn < NVI; nn += 2) {
                uint32_t b[4];
                umma::ldBkn_c(b, Ps, C, n0 + 8 * nn, 16 * kk, lane);
                mma(acc[nn], a, b[0], b[1]);
                mma(acc[nn + 1], a, b[2], b[3]);
            }
        }
#pragma unroll
        for (int nn = 0; nn < NVI; ++nn) {
            const int r = m0 + gq, j = n0 + 8 * nn + 2 * tq;
            *reinterpret_cast<uint32_t*>(dVi + umma::canon_el(r, j, C)) = pack(acc[nn][0], acc[nn][1]);
            *reinterpret_cast<uint32_t*>(dVi + umma::canon_el(r + 8, j, C)) = pack(acc[nn][2], acc[nn][3]);
        }
    }
    // D^T[v][d] = sum_t scale gamma_t dO[t][v] Q[t][d]
    uint32_t a[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        umma::ldAt_c(a[kk], dOs, DV, m0, 16 * kk, lane);
        const int tk = 16 * kk + 2 * tq;
        const float g0 = s.scale * __expf(Gs[tk]), g1 = s.scale * __expf(Gs[tk + 1]);
        const float g2 = s.scale * __expf(Gs[tk + 8]), g3 = s.scale * __expf(Gs[tk + 9]);
        a[kk][0] = scale2(a[kk][0], g0, g1);
        a[kk][1] = scale2(a[kk][1], g0, g1);
        a[kk][2] = scale2(a[kk][2], g2, g3);
        a[kk][3] = scale2(a[kk][3], g2, g3);
    }
    constexpr int NH = DV == 128 ? 2 : 1;  // 64-column halves of D^T per warp
#pragma unroll 1
    for (int nh = 0; nh < NH; ++nh) {
        const int d0 = DV == 128 ? 64 * nh : 64 * (w >> 2);
        float acc[8][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int nn = 0; nn < 8; nn += 2) {
                uint32_t b[4];
                umma::ldBkn_c(b, Qs, DK, d0 + 8 * nn, 16 * kk, lane);
                mma(acc[nn], a[kk], b[0], b[1]);
                mma(acc[nn + 1], a[kk], b[2], b[3]);
            }
        }
#pragma unroll
        for (int nn = 0; nn < 8; ++nn) {
            const int r = m0 + gq, d = d0 + 8 * nn + 2 * tq;
            *reinterpret_cast<uint32_t*>(Dg + umma::canon_el(r, d, DK)) = pack(acc[nn][0], acc[nn][1]);
            *reinterpret_cast<uint32_t*>(Dg + umma::canon_el(r + 8, d, DK)) = pack(acc[nn][2], acc[nn][3]);
        }
    }
}

// O = scale (gamma * Q) S0 + (scale (Q K^T) * Gamma) V_new on warp-level MMAs
// (d_v = 64, and d_v = 128 when SF_GDN_OUT=warp; tc_out5_kernel below is the
// tcgen05 version).  Persistent: a CTA
// of 8 warps takes chunk tickets and copies the next chunk's tiles (Q, K, dO
// by tensor maps, S0^T, V_new^T, G by bulk copies) into the second of two
// buffers while it works on the current one.  Warp w computes rows
// 16 (w % 4).. of P = scale (Q K^T) * Gamma for columns 32 (w / 4).. and of O
// for half of d_v; P goes to shared memory, from where every warp reads the
// whole rows it needs for P V_new.  With OG (the forward of a segment whose
// backward follows) the same CTA also writes the intra-chunk backward products
// (og_products8), reusing Q and P.
template <int DV, bool OG>
__global__ void __launch_bounds__(256, 1)
tc_out2_kernel(SeqView s, const bf16* __restrict__ q, const bf16* __restrict__ k, const float* __restrict__ Gc,
               const bf16* __restrict__ Vnt, const bf16* __restrict__ S0t, bf16* __restrict__ o,
               const bf16* __restrict__ dO, bf16* __restrict__ dVito, bf16* __restrict__ Dto,
               int* __restrict__ ticket, const __grid_constant__ TokMaps maps) {
    using L = O2<DV, OG>;
    extern __shared__ __align__(16) unsigned char smem[];
    bf16* Ps = reinterpret_cast<bf16*>(smem + 2 * L::kBuf);                          // [C][C] canon
    uint64_t* bIn = reinterpret_cast<uint64_t*>(smem + 2 * L::kBuf + (size_t)C * C * 2);  // [2]
    int* tk = reinterpret_cast<int*>(bIn + 2);                                         // [2]
    auto Qb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf); };
    auto Kb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + L::kQ); };
    auto Sb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + 2 * L::kQ); };
    auto Vb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + 2 * L::kQ + L::kS); };
    auto dOb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + 2 * L::kQ + L::kS + L::kVn); };
    auto Gb = [&](int b) {
        return reinterpret_cast<float*>(smem + b * L::kBuf + 2 * L::kQ + L::kS + L::kVn + L::kdO);
    };
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3, mw = w & 3, nh = w >> 2;
    const int total = s.NC * s.BH;
    const size_t Tp = (size_t)s.NC * C;
    bool failed = false;
    auto where = [&](int j, int& c, int& bh) {
        bh = j / s.NC;
        c = j - bh * s.NC;
    };
    // every tile of chunk j into buffer b, completing on bIn[b] (cp.async
    // copies of a short chunk complete in the threads' FIFO groups)
    auto issue = [&](int j, int b) {
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        const size_t ci = (size_t)bh * s.NC + c;
        const bool tma = maps.on && nval == C;
        if (!tma) {
            umma::load_canon<C, DK, 256>(Qb(b), q + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
            umma::load_canon<C, DK, 256>(Kb(b), k + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
            if (OG) umma::load_canon<C, DV, 256>(dOb(b), dO + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
        }
        cp_async_commit();
        if (tid == 0) {
            mbar_expect_tx(&bIn[b], (uint32_t)(L::kS + L::kVn + C * 4 + (tma ? 2 * L::kQ + L::kdO : 0)));
            bulk_load(Sb(b), S0t + ci * DV * DK, (uint32_t)L::kS, &bIn[b]);
            bulk_load(Vb(b), Vnt + ci * DV * C, (uint32_t)L::kVn, &bIn[b]);
            bulk_load(Gb(b), Gc + bh * Tp + t0, C * 4, &bIn[b]);
            if (tma) {
                tma_load5(Qb(b), &maps.q, 0, t0 / 8, bh, &bIn[b]);
                tma_load5(Kb(b), &maps.k, 0, t0 / 8, bh, &bIn[b]);
                if (OG) tma_load5(dOb(b), &maps.dO, 0, t0 / 8, bh, &bIn[b]);
            }
        }
    };

    if (tid == 0) {
        mbar_init(&bIn[0], 1);
        mbar_init(&bIn[1], 1);
        mbar_init_fence();
        tk[0] = atomicAdd(ticket, 1);
        if (maps.on) {
            tma_prefetch_map(&maps.q);
            tma_prefetch_map(&maps.k);
            if (OG) tma_prefetch_map(&maps.dO);
        }
    }
    __syncthreads();
    int j = tk[0];
    if (j >= total) return;
    issue(j, 0);
    constexpr int NO = DV / 16;  // 8-column n-tiles of O per warp (half of d_v)
    for (int it = 0;; ++it) {
        const int buf = it & 1;
        if (tid == 0) tk[(it + 1) & 1] = atomicAdd(ticket, 1);
        cp_async_wait<0>();
        mbar_wait(&bIn[buf], (uint32_t)((it >> 1) & 1), &g_tc_status, failed);
        __syncthreads();  // this chunk's tiles are in; the other buffer is free
        const int jn = tk[(it + 1) & 1];
        const bool has_next = jn < total;
        if (has_next) issue(jn, buf ^ 1);

        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        const bf16* Qs = Qb(buf);
        const bf16* Ks = Kb(buf);
        const bf16* S0s = Sb(buf);
        const bf16* Vns = Vb(buf);
        const float* Gs = Gb(buf);
        const int pc0 = 32 * nh, oc0 = (DV / 2) * nh;
        float p[4][4] = {};
        float acc[NO][4] = {};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t a[4];
            umma::ldA_c(a, Qs, DK, 16 * mw, 16 * kk, lane);
#pragma unroll
            for (int nn = 0; nn < 4; nn += 2) {
                uint32_t b[4];
                umma::ldBnk_c(b, Ks, DK, pc0 + 8 * nn, 16 * kk, lane);
                mma(p[nn], a, b[0], b[1]);
                mma(p[nn + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nn = 0; nn < NO; nn += 2) {
                uint32_t b[4];
                umma::ldBnk_c(b, S0s, DK, oc0 + 8 * nn, 16 * kk, lane);
                mma(acc[nn], a, b[0], b[1]);
                mma(acc[nn + 1], a, b[2], b[3]);
            }
        }
        const int i0 = 16 * mw + gq, i1 = i0 + 8;
        const float G0 = Gs[i0], G1 = Gs[i1];
        const float sg0 = s.scale * __expf(G0), sg1 = s.scale * __expf(G1);
#pragma unroll
        for (int nn = 0; nn < NO; ++nn) {
            acc[nn][0] *= sg0;
            acc[nn][1] *= sg0;
            acc[nn][2] *= sg1;
            acc[nn][3] *= sg1;
        }
#pragma unroll
        for (int nn = 0; nn < 4; ++nn) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = (e >> 1) ? i1 : i0, jj = pc0 + 8 * nn + 2 * tq + (e & 1);
                p[nn][e] = (jj <= i) ? s.scale * __expf(((e >> 1) ? G1 : G0) - Gs[jj]) * p[nn][e] : 0.f;
            }
            const int jj = pc0 + 8 * nn + 2 * tq;
            *umma::canon_at<uint32_t>(Ps, i0, jj, C) = pack(p[nn][0], p[nn][1]);
            *umma::canon_at<uint32_t>(Ps, i1, jj, C) = pack(p[nn][2], p[nn][3]);
        }
        __syncthreads();  // P complete
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t a[4];
            umma::ldA_c(a, Ps, C, 16 * mw, 16 * kk, lane);
#pragma unroll
            for (int nn = 0; nn < NO; nn += 2) {
                uint32_t b[4];
                umma::ldBnk_c(b, Vns, C, oc0 + 8 * nn, 16 * kk, lane);
                mma(acc[nn], a, b[0], b[1]);
                mma(acc[nn + 1], a, b[2], b[3]);
            }
        }
        bf16* ob = o + bh * s.hs_v + (size_t)t0 * DV;
#pragma unroll
        for (int nn = 0; nn < NO; ++nn) {
            const int col = oc0 + 8 * nn + 2 * tq;
            if (i0 < nval) *reinterpret_cast<uint32_t*>(ob + (size_t)i0 * DV + col) = pack(acc[nn][0], acc[nn][1]);
            if (i1 < nval) *reinterpret_cast<uint32_t*>(ob + (size_t)i1 * DV + col) = pack(acc[nn][2], acc[nn][3]);
        }
        if (OG) {
            const size_t ci = (size_t)bh * s.NC + c;
            og_products8<DV>(s, Qs, dOb(buf), Ps, Gs, dVito + ci * DV * C, Dto + ci * DV * DK, w, lane);
        }
        __syncthreads();  // buffer `buf` and P are free
        if (!has_next) break;
        j = jn;
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
    bf16* Vns = dOs + C * LDV;   // [DV][C] canon V_new^T (sized [DV][LDC])
    bf16* dVns = Vns + DV * LDC;  // [DV][C] canon dV_new^T
    unsigned char* R = reinterpret_cast<unsigned char*>(dVns + DV * LDC);
    bf16* S0s = reinterpret_cast<bf16*>(R);       // [DV][DK] canon (phase S)
    bf16* dSs = S0s + DV * LDK;                   // [DV][DK] canon (phase S)
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
        copy_linear<DV * C * 2, GTH>(Vns, Vnt + ci * DV * C, tid);
    };
    auto copy_b1 = [&](int j) {  // V, dV_new
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        const size_t ci = (size_t)bh * s.NC + c;
        copy_linear<DV * C * 2, GTH>(dVns, dVnt + ci * DV * C, tid);
        load_tile<C, DV, GTH>(Vs, LDV, v + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
    };
    auto copy_b2 = [&](int j) {  // S0, dS_C
        int c, bh;
        where(j, c, bh);
        const size_t ci = (size_t)bh * s.NC + c;
        copy_linear<DV * DK * 2, GTH>(S0s, S0t + ci * DV * DK, tid);
        copy_linear<DV * DK * 2, GTH>(dSs, dSCt + ci * DV * DK, tid);
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
                umma::ldBkn_c(b, Vns, C, CW * nw + 8 * nn, 16 * kv, lane);
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
            umma::ldAt_c(aN, dVns, C, 16 * mw, 16 * kv, lane);
            umma::ldAt_c(aV, Vns, C, 16 * mw, 16 * kv, lane);
#pragma unroll
            for (int nn = 0; nn < DKW / 8; nn += 2) {
                uint32_t b[4];
                umma::ldBkn_c(b, S0s, DK, DKW * nw + 8 * nn, 16 * kv, lane);
                mma(accQ[nn], aO, b[0], b[1]);
                mma(accQ[nn + 1], aO, b[2], b[3]);
                mma(accW[nn], aN, b[0], b[1]);
                mma(accW[nn + 1], aN, b[2], b[3]);
                umma::ldBkn_c(b, dSs, DK, DKW * nw + 8 * nn, 16 * kv, lane);
                mma(accK[nn], aV, b[0], b[1]);
                mma(accK[nn + 1], aV, b[2], b[3]);
            }
        }
        float pd = 0.f;  // <S0, dS_C>
        for (int e = tid; e < DV * DK; e += GTH)  // both canon tiles: same element at the same offset
            pd += __bfloat162float(S0s[e]) * __bfloat162float(dSs[e]);
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
                cp_async16(Lf + i * LDF + j, Lg + l_off(i, j), true);
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
                    umma::ldBnk_c(b, dVns, C, (DV / GW) * nw + 8 * nn, 16 * kr, lane);
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
                dvb[(size_t)j * DV + col] = *umma::canon_at<bf16>(dVns, col, j, C);
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
            umma::ldAt_c(a, dVns, C, 16 * mw, 16 * kv, lane);
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

// ------------------------------------------------------- out on tcgen05 ---
// Out (+ OG) on tcgen05 (d_v = 128): the same products as tc_out2_kernel,
// issued by one thread into TMEM accumulators: P' = Q K^T and O1 = Q S0
// (M = 64 token rows), with OG D^T = (scale gamma * dO)^T Q (M = 128 d_v rows);
// then, from P (the masked, scaled bf16 tile the 8 warps build from P'),
// O2 = P V_new (M = 64) and with OG dVi^T = dO^T P (M = 128).  O = scale gamma O1
// + O2.  Persistent with two buffers of all input tiles (Q, K, dO by tensor
// maps, S0^T, V_new^T, G by bulk copies), like tc_out2_kernel.
// TMEM columns: P' [0, 64), O1 [64, 192), O2 [192, 320), dVi^T [320, 384),
// D^T [384, 512).
template <bool OG>
struct O5 {
    static constexpr int DV = 128;
    static constexpr size_t kQ = (size_t)C * DK * 2;
    static constexpr size_t kS = (size_t)DV * DK * 2;
    static constexpr size_t kVn = (size_t)DV * C * 2;
    static constexpr size_t kdO = OG ? (size_t)C * DV * 2 : 0;
    static constexpr size_t kBuf = 2 * kQ + kS + kVn + kdO + C * 4;
    static constexpr size_t SMEM = 2 * kBuf + (size_t)C * C * 2 + kdO + 4 * 8 + 16;
    static constexpr uint32_t TP = 0, TO1 = 64, TO2 = 192, TDVI = 320, TDT = 384;
};

template <bool OG>
__global__ void __launch_bounds__(256, 1)
tc_out5_kernel(SeqView s, const bf16* __restrict__ q, const bf16* __restrict__ k, const float* __restrict__ Gc,
               const bf16* __restrict__ Vnt, const bf16* __restrict__ S0t, bf16* __restrict__ o,
               const bf16* __restrict__ dO, bf16* __restrict__ dVito, bf16* __restrict__ Dto,
               int* __restrict__ ticket, const __grid_constant__ TokMaps maps) {
    using L = O5<OG>;
    constexpr int DV = L::DV;
    extern __shared__ __align__(16) unsigned char smem[];
    bf16* Ps = reinterpret_cast<bf16*>(smem + 2 * L::kBuf);                 // [C][C] canon
    bf16* dOg = reinterpret_cast<bf16*>(smem + 2 * L::kBuf + C * C * 2);     // [C][DV] canon, scale gamma dO
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * L::kBuf + C * C * 2 + L::kdO);
    uint64_t* bIn = bars;  // [2]
    uint64_t* bm1 = bars + 2;
    uint64_t* bm2 = bars + 3;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 4);
    int* tk = reinterpret_cast<int*>(bars + 4) + 1;  // [2]
    auto Qb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf); };
    auto Kb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + L::kQ); };
    auto Sb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + 2 * L::kQ); };
    auto Vb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + 2 * L::kQ + L::kS); };
    auto dOb = [&](int b) { return reinterpret_cast<bf16*>(smem + b * L::kBuf + 2 * L::kQ + L::kS + L::kVn); };
    auto Gb = [&](int b) {
        return reinterpret_cast<float*>(smem + b * L::kBuf + 2 * L::kQ + L::kS + L::kVn + L::kdO);
    };
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3, mw = w & 3, nh = w >> 2;
    const int total = s.NC * s.BH;
    const size_t Tp = (size_t)s.NC * C;
    bool failed = false;
    auto where = [&](int j, int& c, int& bh) {
        bh = j / s.NC;
        c = j - bh * s.NC;
    };
    auto issue = [&](int j, int b) {
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        const size_t ci = (size_t)bh * s.NC + c;
        const bool tma = maps.on && nval == C;
        if (!tma) {
            umma::load_canon<C, DK, 256>(Qb(b), q + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
            umma::load_canon<C, DK, 256>(Kb(b), k + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
            if (OG) umma::load_canon<C, DV, 256>(dOb(b), dO + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
        }
        cp_async_commit();
        if (tid == 0) {
            mbar_expect_tx(&bIn[b], (uint32_t)(L::kS + L::kVn + C * 4 + (tma ? 2 * L::kQ + L::kdO : 0)));
            bulk_load(Sb(b), S0t + ci * DV * DK, (uint32_t)L::kS, &bIn[b]);
            bulk_load(Vb(b), Vnt + ci * DV * C, (uint32_t)L::kVn, &bIn[b]);
            bulk_load(Gb(b), Gc + bh * Tp + t0, C * 4, &bIn[b]);
            if (tma) {
                tma_load5(Qb(b), &maps.q, 0, t0 / 8, bh, &bIn[b]);
                tma_load5(Kb(b), &maps.k, 0, t0 / 8, bh, &bIn[b]);
                if (OG) tma_load5(dOb(b), &maps.dO, 0, t0 / 8, bh, &bIn[b]);
            }
        }
    };

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
        tk[0] = atomicAdd(ticket, 1);
        if (maps.on) {
            tma_prefetch_map(&maps.q);
            tma_prefetch_map(&maps.k);
            if (OG) tma_prefetch_map(&maps.dO);
        }
    }
    if (w == 0) umma::alloc(tslot, 512);
    __syncthreads();
    umma::fence_after();
    const uint32_t tm = *tslot;
    const uint32_t trow = umma::taddr(tm, 32 * mw, 0);  // this warp's lane quarter
    int j = tk[0];
    if (j < total) issue(j, 0);
    constexpr uint32_t IP = umma::idesc_bf16(64, 64, false, false);
    constexpr uint32_t IO = umma::idesc_bf16(64, 128, false, false);
    constexpr uint32_t IDT = umma::idesc_bf16(128, 128, true, true);
    constexpr uint32_t IDVI = umma::idesc_bf16(128, 64, true, true);
    for (int it = 0; j < total; ++it) {
        const int buf = it & 1;
        const uint32_t par = (uint32_t)(it & 1);
        if (tid == 0) tk[(it + 1) & 1] = atomicAdd(ticket, 1);
        cp_async_wait<0>();
        mbar_wait(&bIn[buf], (uint32_t)((it >> 1) & 1), &g_tc_status, failed);
        __syncthreads();  // this chunk's tiles are in; the other buffer is free
        const int jn = tk[(it + 1) & 1];
        const bool has_next = jn < total;
        if (has_next) issue(jn, buf ^ 1);

        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        const bf16* Qs = Qb(buf);
        const float* Gs = Gb(buf);
        if (OG) {  // scale gamma_t dO[t][:], canon like dO (every thread 4 pieces)
            const uint4* src = reinterpret_cast<const uint4*>(dOb(buf));
            uint4* dst = reinterpret_cast<uint4*>(dOg);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = tid + 256 * u;
                int r, cc;
                umma::canon_piece(e, DV, r, cc);
                const float gs = s.scale * __expf(Gs[r]);
                uint4 x = src[e];
                x.x = scale2(x.x, gs, gs);
                x.y = scale2(x.y, gs, gs);
                x.z = scale2(x.z, gs, gs);
                x.w = scale2(x.w, gs, gs);
                dst[e] = x;
            }
            fence_proxy_async_smem();
            __syncthreads();
        }
        if (tid == 0) {  // P' = Q K^T, O1 = Q S0, D^T = (scale gamma dO)^T Q
            umma::fence_after();
            umma::chain<DK / 16>(tm + L::TP, IP, false, umma::op_k(Qs, DK), umma::op_k(Kb(buf), DK));
            umma::chain<DK / 16>(tm + L::TO1, IO, false, umma::op_k(Qs, DK), umma::op_k(Sb(buf), DK));
            if (OG) umma::chain<C / 16>(tm + L::TDT, IDT, false, umma::op_mn(dOg, DV), umma::op_mn(Qs, DK));
            umma::commit(bm1);
        }
        // P = scale (Q K^T) * Gamma (masked), bf16 canon; warp w: rows of its quarter, columns 32 (w / 4)..
        mbar_wait(bm1, par, &g_tc_status, failed);
        umma::fence_after();
        const int r0 = 16 * mw + gq, r1 = r0 + 8;
        {
            float pf[4][4];
            umma::ld32(trow + L::TP + 32 * nh, pf);
            umma::wait_ld();
            const float G0 = Gs[r0], G1 = Gs[r1];
#pragma unroll
            for (int jq = 0; jq < 4; ++jq) {
                const int col = 32 * nh + 8 * jq + 2 * tq;
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = (e >> 1) ? r1 : r0, jj = col + (e & 1);
                    v[e] = (jj <= i) ? s.scale * __expf(((e >> 1) ? G1 : G0) - Gs[jj]) * pf[jq][e] : 0.f;
                }
                *umma::canon_at<uint32_t>(Ps, r0, col, C) = pack(v[0], v[1]);
                *umma::canon_at<uint32_t>(Ps, r1, col, C) = pack(v[2], v[3]);
            }
        }
        fence_proxy_async_smem();
        umma::fence_before();
        __syncthreads();  // P complete
        if (tid == 0) {  // O2 = P V_new, dVi^T = dO^T P
            umma::fence_after();
            umma::chain<C / 16>(tm + L::TO2, IO, false, umma::op_k(Ps, C), umma::op_k(Vb(buf), C));
            if (OG) umma::chain<C / 16>(tm + L::TDVI, IDVI, false, umma::op_mn(dOb(buf), DV), umma::op_mn(Ps, C));
            umma::commit(bm2);
        }
        const size_t ci = (size_t)bh * s.NC + c;
        const int v = 32 * mw + lane;  // d_v row of the M = 128 accumulators this thread reads
        if (OG) {  // D^T out while the second products run: row v, columns 64 (w / 4)..
            bf16* Dg = Dto + ci * DV * DK;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float x[32];
                umma::ld_row32(trow + L::TDT + 64 * nh + 32 * g, x);
                umma::wait_ld();
#pragma unroll
                for (int p4 = 0; p4 < 4; ++p4) {
                    uint4 u;
                    u.x = pack(x[8 * p4], x[8 * p4 + 1]);
                    u.y = pack(x[8 * p4 + 2], x[8 * p4 + 3]);
                    u.z = pack(x[8 * p4 + 4], x[8 * p4 + 5]);
                    u.w = pack(x[8 * p4 + 6], x[8 * p4 + 7]);
                    *reinterpret_cast<uint4*>(Dg + umma::canon_el(v, 64 * nh + 32 * g + 8 * p4, DK)) = u;
                }
            }
        }
        mbar_wait(bm2, par, &g_tc_status, failed);
        umma::fence_after();
        {  // O = scale gamma O1 + O2: rows of this warp's quarter, columns 64 (w / 4)..
            bf16* ob = o + bh * s.hs_v + (size_t)t0 * DV;
            const float sg0 = s.scale * __expf(Gs[r0]), sg1 = s.scale * __expf(Gs[r1]);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float a[4][4], b[4][4];
                umma::ld32(trow + L::TO1 + 64 * nh + 32 * g, a);
                umma::ld32(trow + L::TO2 + 64 * nh + 32 * g, b);
                umma::wait_ld();
#pragma unroll
                for (int jq = 0; jq < 4; ++jq) {
                    const int col = 64 * nh + 32 * g + 8 * jq + 2 * tq;
                    if (r0 < nval)
                        *reinterpret_cast<uint32_t*>(ob + (size_t)r0 * DV + col) =
                            pack(fmaf(a[jq][0], sg0, b[jq][0]), fmaf(a[jq][1], sg0, b[jq][1]));
                    if (r1 < nval)
                        *reinterpret_cast<uint32_t*>(ob + (size_t)r1 * DV + col) =
                            pack(fmaf(a[jq][2], sg1, b[jq][2]), fmaf(a[jq][3], sg1, b[jq][3]));
                }
            }
        }
        if (OG) {  // dVi^T out: row v, columns 32 (w / 4)..
            float x[32];
            umma::ld_row32(trow + L::TDVI + 32 * nh, x);
            umma::wait_ld();
            bf16* dvi = dVito + ci * DV * C;
#pragma unroll
            for (int p4 = 0; p4 < 4; ++p4) {
                uint4 u;
                u.x = pack(x[8 * p4], x[8 * p4 + 1]);
                u.y = pack(x[8 * p4 + 2], x[8 * p4 + 3]);
                u.z = pack(x[8 * p4 + 4], x[8 * p4 + 5]);
                u.w = pack(x[8 * p4 + 6], x[8 * p4 + 7]);
                *reinterpret_cast<uint4*>(dvi + umma::canon_el(v, 32 * nh + 8 * p4, C)) = u;
            }
        }
        umma::fence_before();
        __syncthreads();  // buffer `buf`, P, dOg and TMEM are free
        j = jn;
    }
    umma::fence_before();
    __syncthreads();
    if (w == 0) {
        umma::fence_after();
        umma::dealloc(tm, 512);
    }
}

// ------------------------------------------------- grad on tcgen05 (PG) ---
// Every input gradient of a chunk with the products on the fifth-generation
// tensor cores: one thread issues each product as a chain of K = 16
// tcgen05.mma (M = 64 token rows, fp32 accumulators in TMEM, operands read
// from canon tiles in shared memory), and the 16 warps run the elementwise
// epilogues between them on the accumulators they load from TMEM (warp w
// owns rows 16 (w % 4).. and the column group w / 4).  With
//   P = scale (Q K^T) * Gamma,  M = scale (dO V_new^T) * Gamma,  T = L diag(beta),
//   dW = -dV_new S0^T,  dT = dW (gamma K)^T + dV_new V^T,  dL = dT diag(beta),
//   dA = -strictly-lower(L^T dL L^T),  Z = diag(beta) (dA * Gamma):
//   dq = scale gamma (dO S0^T) + M K
//   dk = dec (V_new dS_C^T) + gamma (T^T dW) + M^T Q + Z K + Z^T K
//   dv = T^T dV_new   (dv = dV_new without the beta path)
// and dG (hence dg, dbeta) from the row and column sums of the elementwise
// terms, reduced in a fixed order (bit-reproducible).
//
// Persistent: a CTA takes chunk tickets from a per-launch counter and copies
// the next chunk's tiles in while it works on the current one: Q, K, G into
// the second of two buffers at once; dO and V_new^T once the products reading
// them are done, then dV_new^T and V, then L; the state tiles as soon as the
// last product completes, into the region the epilogue tiles leave.  Q, K, dO,
// V arrive and dq, dk leave by tensor-map copies (whole chunks; a short last
// chunk takes per-thread copies), the rest by bulk copies.
//
// The term gamma (T^T dW) of dk accumulates in place; its share of dG,
// sum_k K_ik gamma_i (T^T dW)_ik = gamma_i beta_i sum_j L_ji (dW K^T)_ji, is a
// column sum of L * (dW K^T), taken where dT is formed.
//
// TMEM columns (512 allocated; M = 64 uses lanes 0-15 of each quarter):
//   [0,64) Q K^T -> [0,128) dk       [64,128) K K^T        [128,192) dP -> dT_b -> dA
//   [192,320) dq                     [320,448) dV_new S0^T -> dv
//   [448,512) dW K^T -> X
// Tensor maps of the gradient kernel's token-major tiles (q, k, v, dO in; dq,
// dk out), each a five-dimensional view of a [BH][T][D] bf16 tensor ordered
// (column within 8, row within 8, column block, row block, head), so that one
// box of (8, 8, D/8, C/8, 1) is a whole chunk tile and lands in shared memory
// (or is read from it) in the canonical core-matrix layout the tcgen05
// descriptors read.  `on` is 0 when the maps could not be made; the kernel
// then copies every tile with per-thread cp.async, as it always does for a
// chunk shorter than C (a box cannot stop at a row that is not a multiple of
// 8, so partial chunks never use the maps).
struct G5Maps {
    CUtensorMap q, k, v, dO, dq, dk;
    int on;
};

template <int DV>
struct G5 {
    // TMEM columns of the accumulators
    static constexpr uint32_t QK = 0, KK = 64, DP = 128, DQ = 192, DW = 320, DTA = 448;
    static constexpr uint32_t DKC = 0, DTB = 128, DVC = 320, XC = 448, DA = 128;
    static constexpr size_t kQK = (size_t)2 * C * 128 * 2;  // one buffer: Q then K
    static constexpr size_t kV = (size_t)C * DV * 2;        // V, dO, V_new^T, dV_new^T each
    static constexpr size_t kStateB = (size_t)DV * 128 * 2 * 2;
    static constexpr size_t kEpiB = (size_t)C * 128 * 2 + 6 * (size_t)C * C * 2;
    static constexpr size_t kB = kStateB > kEpiB ? kStateB : kEpiB;
    static constexpr size_t SMEM = 2 * kQK + 4 * kV + kB + (size_t)C * C * 4 + (size_t)C * C * 2 +
                                   (size_t)P_ROWS * C * 4 + 20 * 4 + 4 * C * 4 + 16 * 8 + 16;
};

template <int DV, bool BETA>
__global__ void __launch_bounds__(512, 1)
tc_grad5_kernel(SeqView s, const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                const float* __restrict__ beta, const bf16* __restrict__ dO, const float* __restrict__ Gc,
                const float* __restrict__ Lm, const bf16* __restrict__ Vnt, const bf16* __restrict__ dVnt,
                const bf16* __restrict__ S0t, const bf16* __restrict__ dSCt, bf16* __restrict__ dq,
                bf16* __restrict__ dk, bf16* __restrict__ dv, float* __restrict__ dg, float* __restrict__ dbeta,
                int* __restrict__ ticket, const __grid_constant__ G5Maps maps) {
    using L5 = G5<DV>;
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char* p = smem;
    unsigned char* QKb = p;                   p += 2 * L5::kQK;  // [2] x (Q [C][DK], K [C][DK])
    bf16* Vc = reinterpret_cast<bf16*>(p);   p += L5::kV;        // [C][DV]
    bf16* dOc = reinterpret_cast<bf16*>(p);  p += L5::kV;        // [C][DV]
    bf16* Vnc = reinterpret_cast<bf16*>(p);  p += L5::kV;        // [DV][C]  V_new^T
    bf16* dVnc = reinterpret_cast<bf16*>(p); p += L5::kV;        // [DV][C]  dV_new^T
    unsigned char* RB = p;                   p += L5::kB;
    bf16* S0c = reinterpret_cast<bf16*>(RB);           // [DV][DK]
    bf16* dSc = S0c + DV * 128;                        // [DV][DK]
    bf16* dWs = reinterpret_cast<bf16*>(RB);           // [C][DK]   (after the state products)
    bf16* Tpp = dWs + C * 128;                         // [C][C]    L diag(beta gamma)
    bf16* Ts = Tpp + C * C;                            // [C][C]    L diag(beta)
    bf16* Ls = Ts + C * C;                             // [C][C]    L
    bf16* dLs = Ls + C * C;                            // [C][C]
    bf16* Xs = dLs + C * C;                            // [C][C]
    bf16* Zs = Xs + C * C;                             // [C][C]
    float* Lf = reinterpret_cast<float*>(p);  p += C * C * 4;   // [C][C] fp32, row-major
    bf16* Ms = reinterpret_cast<bf16*>(p);    p += C * C * 2;   // [C][C]
    float* part = reinterpret_cast<float*>(p); p += P_ROWS * C * 4;
    float* red = reinterpret_cast<float*>(p);  p += 20 * 4;  // [16] per-warp <S0, dS_C>, [3] for the dG warps
    float* Gsb = reinterpret_cast<float*>(p);  p += 2 * C * 4;  // [2][C]
    float* Bsb = reinterpret_cast<float*>(p);  p += 2 * C * 4;  // [2][C]
    uint64_t* bars = reinterpret_cast<uint64_t*>(p);  p += 16 * 8;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(p);
    int* tk = reinterpret_cast<int*>(p + 4);  // [2] chunk tickets
    // mbarriers: copies (one phase per chunk) and product completions (one per chunk)
    uint64_t* bVn = &bars[0];
    uint64_t* bS = &bars[1];
    uint64_t* bdVn = &bars[2];
    uint64_t* bL = &bars[3];
    uint64_t* bm = &bars[4];  // [7]
    uint64_t* bQK = &bars[11];  // [2] Q, K, G of the chunk in buffer b
    uint64_t* bDO = &bars[13];
    uint64_t* bV = &bars[14];

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int mw = w & 3, nw = w >> 2;
    const size_t Tp = (size_t)s.NC * C;
    const int total = s.NC * s.BH;
    const int r0 = 16 * mw + gq, r1 = r0 + 8;  // the two rows this thread holds
    bool failed = false;

    auto where = [&](int j, int& c, int& bh) {
        bh = j / s.NC;
        c = j - bh * s.NC;
    };
    auto Qc_of = [&](int b) { return reinterpret_cast<bf16*>(QKb + b * L5::kQK); };
    auto Kc_of = [&](int b) { return reinterpret_cast<bf16*>(QKb + b * L5::kQK) + C * 128; };
    // copy groups (cp.async: per-thread FIFO groups; bulk: mbarriers, thread 0)
    // Q, K, G, dO and V complete on mbarriers: by tensor-map copies of thread 0
    // for whole chunks, else by cp.async (waited for in the threads' FIFO
    // groups) with a plain arrival of thread 0.
    auto copy_qkg = [&](int j, int b) {  // Q, K, G of chunk j into buffer b
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        if (maps.on && nval == C) {
            if (tid == 0) {
                mbar_expect_tx(&bQK[b], 2 * C * DK * 2 + C * 4);
                tma_load5(Qc_of(b), &maps.q, 0, t0 / 8, bh, &bQK[b]);
                tma_load5(Kc_of(b), &maps.k, 0, t0 / 8, bh, &bQK[b]);
                bulk_load(Gsb + b * C, Gc + bh * Tp + t0, C * 4, &bQK[b]);
            }
            return;
        }
        umma::load_canon<C, 128, 512>(Qc_of(b), q + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
        umma::load_canon<C, 128, 512>(Kc_of(b), k + bh * s.hs_k + (size_t)t0 * DK, DK, nval, tid);
        if (tid < C / 4) cp_async16(Gsb + b * C + 4 * tid, Gc + bh * Tp + t0 + 4 * tid, true);
        if (tid == 0) mbar_arrive(&bQK[b]);
    };
    auto copy_do = [&](int j) {
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        if (maps.on && nval == C) {
            if (tid == 0) {
                mbar_expect_tx(bDO, C * DV * 2);
                tma_load5(dOc, &maps.dO, 0, t0 / 8, bh, bDO);
            }
            return;
        }
        umma::load_canon<C, DV, 512>(dOc, dO + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
        if (tid == 0) mbar_arrive(bDO);
    };
    auto copy_v = [&](int j) {  // the delta path only: V is read by dV_new V^T alone
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        if (maps.on && nval == C) {
            if (tid == 0) {
                mbar_expect_tx(bV, C * DV * 2);
                tma_load5(Vc, &maps.v, 0, t0 / 8, bh, bV);
            }
            return;
        }
        umma::load_canon<C, DV, 512>(Vc, v + bh * s.hs_v + (size_t)t0 * DV, DV, nval, tid);
        if (tid == 0) mbar_arrive(bV);
    };
    auto bulk_vn = [&](int j) {  // thread 0
        int c, bh;
        where(j, c, bh);
        mbar_expect_tx(bVn, DV * C * 2);
        bulk_load(Vnc, Vnt + ((size_t)bh * s.NC + c) * DV * C, DV * C * 2, bVn);
    };
    auto bulk_state = [&](int j) {  // thread 0
        int c, bh;
        where(j, c, bh);
        const size_t ci = (size_t)bh * s.NC + c;
        mbar_expect_tx(bS, 2 * DV * 128 * 2);
        bulk_load(S0c, S0t + ci * DV * DK, DV * 128 * 2, bS);
        bulk_load(dSc, dSCt + ci * DV * DK, DV * 128 * 2, bS);
    };
    auto bulk_dvn = [&](int j) {  // thread 0
        int c, bh;
        where(j, c, bh);
        mbar_expect_tx(bdVn, DV * C * 2);
        bulk_load(dVnc, dVnt + ((size_t)bh * s.NC + c) * DV * C, DV * C * 2, bdVn);
    };
    auto bulk_l = [&](int j) {  // thread 0
        int c, bh;
        where(j, c, bh);
        mbar_expect_tx(bL, C * C * 4);
        bulk_load(Lf, Lm + ((size_t)bh * s.NC + c) * C * C, C * C * 4, bL);
    };
    auto beta_of = [&](int j) {
        int c, bh;
        where(j, c, bh);
        const int t0 = c * C, nval = min(C, s.T - t0);
        return (BETA && tid < nval) ? beta[bh * s.hs_g + t0 + tid] : 0.f;
    };

    if (tid == 0) {
        for (int i = 0; i < 15; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
        tk[0] = atomicAdd(ticket, 1);
        if (maps.on) {
            tma_prefetch_map(&maps.q);
            tma_prefetch_map(&maps.k);
            tma_prefetch_map(&maps.dO);
            if (BETA) tma_prefetch_map(&maps.v);
            tma_prefetch_map(&maps.dq);
            tma_prefetch_map(&maps.dk);
        }
    }
    __syncthreads();
    int j = tk[0];
    if (j >= total) return;
    if (w == 0) umma::alloc(tslot, 512);
    // first chunk: groups [Q K G dO] and [V]; bulk copies of its other tiles
    copy_qkg(j, 0);
    copy_do(j);
    cp_async_commit();
    if (BETA) copy_v(j);
    cp_async_commit();
    if (tid == 0) {
        bulk_vn(j);
        bulk_state(j);
        bulk_dvn(j);
        if (BETA) bulk_l(j);
    }
    if (tid < C) Bsb[tid] = beta_of(j);
    for (int e = tid; e < P_ROWS * C; e += 512) part[e] = 0.f;
    __syncthreads();  // TMEM allocated
    umma::fence_after();
    const uint32_t tm = *tslot;
    const uint32_t trow = umma::taddr(tm, 32 * mw, 0);  // this warp's lane quarter
    constexpr uint32_t I64kk = umma::idesc_bf16(64, 64, false, false);
    constexpr uint32_t I64km = umma::idesc_bf16(64, 64, false, true);
    constexpr uint32_t I64mk = umma::idesc_bf16(64, 64, true, false);
    constexpr uint32_t I64mm = umma::idesc_bf16(64, 64, true, true);
    constexpr uint32_t I128km = umma::idesc_bf16(64, 128, false, true);
    constexpr uint32_t I128mm = umma::idesc_bf16(64, 128, true, true);
    constexpr uint32_t IDVmk = umma::idesc_bf16(64, DV, true, false);
    auto sync_for_mma = [&]() {  // generic shared writes and TMEM accesses -> the next products
        fence_proxy_async_smem();
        umma::fence_before();
        __syncthreads();
    };

  for (int it = 0;; ++it) {
    const int buf = it & 1;
    const uint32_t par = (uint32_t)(it & 1);
    auto wait_bar = [&](uint64_t* b) {
        mbar_wait(b, par, &g_tc_status, failed);
        umma::fence_after();
    };
    int c, bh;
    where(j, c, bh);
    const int t0 = c * C;
    const int nval = min(C, s.T - t0);
    bf16* Qc = Qc_of(buf);
    bf16* Kc = Kc_of(buf);
    float* Gs = Gsb + buf * C;
    float* Bs = Bsb + buf * C;
    if (tid == 0) tk[(it + 1) & 1] = atomicAdd(ticket, 1);
    cp_async_wait<1>();  // Q, K, G, dO of this chunk (its V may still be landing)
    mbar_wait(&bQK[buf], (uint32_t)((it >> 1) & 1), &g_tc_status, failed);
    mbar_wait(bDO, par, &g_tc_status, failed);
    mbar_wait(bVn, par, &g_tc_status, failed);
    sync_for_mma();
    const int jn = tk[(it + 1) & 1];
    const bool has_next = jn < total;
    if (tid == 0) {  // Q K^T, K K^T, dP = dO V_new^T
        umma::fence_after();
        umma::chain<8>(tm + L5::QK, I64kk, false, umma::op_k(Qc, 128), umma::op_k(Kc, 128));
        if (BETA)
            umma::chain<8>(tm + L5::KK, I64kk, false, umma::op_k(Kc, 128), umma::op_k(Kc, 128));
        umma::chain<DV / 16>(tm + L5::DP, I64km, false, umma::op_k(dOc, DV), umma::op_mn(Vnc, C));
        umma::commit(&bm[0]);
    }
    if (has_next) copy_qkg(jn, buf ^ 1);  // the other buffer's chunk is done
    cp_async_commit();
    const float beta_next = has_next ? beta_of(jn) : 0.f;
    mbar_wait(bS, par, &g_tc_status, failed);
    mbar_wait(bdVn, par, &g_tc_status, failed);
    if (tid == 0) {  // dO S0^T, dV_new S0^T
        umma::fence_after();
        umma::chain<DV / 16>(tm + L5::DQ, I128km, false, umma::op_k(dOc, DV), umma::op_mn(S0c, 128));
        if (BETA)
            umma::chain<DV / 16>(tm + L5::DW, I128mm, false, umma::op_mn(dVnc, C), umma::op_mn(S0c, 128));
        umma::commit(&bm[1]);
    }

    const float gam0 = __expf(Gs[r0]), gam1 = __expf(Gs[r1]);
    const float gC = Gs[C - 1];
    const float dec0 = __expf(gC - Gs[r0]), dec1 = __expf(gC - Gs[r1]);

    // ---- E1: M = scale dP * Gamma (bf16 tile), row/column sums of M * QK; keep K K^T
    float kkr[2][4];
    float gmr[2][4];  // Gamma_ij = exp(G_i - G_j) (j <= i) of this thread's elements, for E6
    {
        wait_bar(&bm[0]);
        float qk[2][4], dp[2][4];
        umma::ld16(trow + L5::QK + 16 * nw, qk);
        if (BETA) umma::ld16(trow + L5::KK + 16 * nw, kkr);
        umma::ld16(trow + L5::DP + 16 * nw, dp);
        umma::wait_ld();
        float row0 = 0.f, row1 = 0.f;
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            float col[2] = {0.f, 0.f};
            float m[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = (e >> 1) ? r1 : r0, jj = 16 * nw + 8 * n + 2 * tq + (e & 1);
                const float gm = (jj <= i) ? __expf(Gs[i] - Gs[jj]) : 0.f;
                gmr[n][e] = gm;
                m[e] = s.scale * dp[n][e] * gm;
                const float zp = m[e] * qk[n][e];
                if (e >> 1) row1 += zp; else row0 += zp;
                col[e & 1] += zp;
            }
            const int jj = 16 * nw + 8 * n + 2 * tq;
            *umma::canon_at<uint32_t>(Ms, r0, jj, C) = pack(m[0], m[1]);
            *umma::canon_at<uint32_t>(Ms, r1, jj, C) = pack(m[2], m[3]);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                col[0] += __shfl_xor_sync(0xffffffffu, col[0], o);
                col[1] += __shfl_xor_sync(0xffffffffu, col[1], o);
            }
            if (gq == 0) {
                part[(P_COLP + mw) * C + jj] = col[0];
                part[(P_COLP + mw) * C + jj + 1] = col[1];
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
    sync_for_mma();
    if (tid == 0) {  // V_new dS_C^T
        umma::fence_after();
        umma::chain<DV / 16>(tm + L5::DKC, I128mm, false, umma::op_mn(Vnc, C), umma::op_mn(dSc, 128));
        umma::commit(&bm[2]);
    }

    // ---- E2a: dq <- scale gamma (dO S0^T) in place; sum_k Q dq; <S0, dS_C>
    {
        wait_bar(&bm[1]);
        float a[4][4];
        umma::ld32(trow + L5::DQ + 32 * nw, a);
        umma::wait_ld();
        const float sq0 = s.scale * gam0, sq1 = s.scale * gam1;
        float pi0 = 0.f, pi1 = 0.f;
#pragma unroll
        for (int jq = 0; jq < 4; ++jq) {
            const int col = 32 * nw + 8 * jq + 2 * tq;
            const float2 q0 = unpack(*umma::canon_at<uint32_t>(Qc, r0, col, 128));
            const float2 q1 = unpack(*umma::canon_at<uint32_t>(Qc, r1, col, 128));
            a[jq][0] *= sq0;
            a[jq][1] *= sq0;
            a[jq][2] *= sq1;
            a[jq][3] *= sq1;
            pi0 += q0.x * a[jq][0] + q0.y * a[jq][1];
            pi1 += q1.x * a[jq][2] + q1.y * a[jq][3];
        }
        umma::st32(trow + L5::DQ + 32 * nw, a);
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            pi0 += __shfl_xor_sync(0xffffffffu, pi0, o);
            pi1 += __shfl_xor_sync(0xffffffffu, pi1, o);
        }
        if (tq == 0) {
            part[(P_INTER + nw) * C + r0] = pi0;
            part[(P_INTER + nw) * C + r1] = pi1;
        }
        float pd = 0.f;  // both canon tiles: the same element at the same offset
        for (int e = tid; e < DV * 128 / 2; e += 512) {
            const float2 x = unpack(reinterpret_cast<const uint32_t*>(S0c)[e]);
            const float2 y = unpack(reinterpret_cast<const uint32_t*>(dSc)[e]);
            pd = fmaf(x.x, y.x, pd);
            pd = fmaf(x.y, y.y, pd);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pd += __shfl_xor_sync(0xffffffffu, pd, o);
        if (lane == 0) red[w] = pd;
        umma::wait_st();
    }
    sync_for_mma();
    if (tid == 0) {  // dq += M K
        umma::fence_after();
        umma::chain<C / 16>(tm + L5::DQ, I128km, true, umma::op_k(Ms, C), umma::op_mn(Kc, 128));
    }

    // ---- E2b: dk <- dec (V_new dS_C^T) in place, sum_k K dk; dW; T'', T, L tiles
    {
        wait_bar(&bm[2]);  // every earlier product too: dO, V_new^T and the state tiles are free
        if (has_next) copy_do(jn);
        cp_async_commit();
        if (tid == 0 && has_next) bulk_vn(jn);
        float a[4][4];
        umma::ld32(trow + L5::DKC + 32 * nw, a);
        umma::wait_ld();
        float pz0 = 0.f, pz1 = 0.f;
#pragma unroll
        for (int jq = 0; jq < 4; ++jq) {
            const int col = 32 * nw + 8 * jq + 2 * tq;
            const float2 k0 = unpack(*umma::canon_at<uint32_t>(Kc, r0, col, 128));
            const float2 k1 = unpack(*umma::canon_at<uint32_t>(Kc, r1, col, 128));
            a[jq][0] *= dec0;
            a[jq][1] *= dec0;
            a[jq][2] *= dec1;
            a[jq][3] *= dec1;
            pz0 += k0.x * a[jq][0] + k0.y * a[jq][1];
            pz1 += k1.x * a[jq][2] + k1.y * a[jq][3];
        }
        umma::st32(trow + L5::DKC + 32 * nw, a);
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            pz0 += __shfl_xor_sync(0xffffffffu, pz0, o);
            pz1 += __shfl_xor_sync(0xffffffffu, pz1, o);
        }
        if (tq == 0) {
            part[(P_Z + nw) * C + r0] = pz0;
            part[(P_Z + nw) * C + r1] = pz1;
        }
        if (BETA) {
            umma::ld32(trow + L5::DW + 32 * nw, a);
            umma::wait_ld();
#pragma unroll
            for (int jq = 0; jq < 4; ++jq) {
                const int col = 32 * nw + 8 * jq + 2 * tq;
                *umma::canon_at<uint32_t>(dWs, r0, col, 128) = pack(-a[jq][0], -a[jq][1]);
                *umma::canon_at<uint32_t>(dWs, r1, col, 128) = pack(-a[jq][2], -a[jq][3]);
            }
            mbar_wait(bL, par, &g_tc_status, failed);
            {  // T'' = L diag(beta gamma), T = L diag(beta), L: one 8-element row piece per thread
                const int i = tid >> 3, j0 = (tid & 7) * 8;
                uint32_t tpp[4], tt[4], ll[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int jj = j0 + 2 * h;
                    const float2 l = *reinterpret_cast<const float2*>(Lf + l_off(i, jj));
                    const float b0 = Bs[jj], b1 = Bs[jj + 1];
                    tpp[h] = pack(l.x * b0 * __expf(Gs[jj]), l.y * b1 * __expf(Gs[jj + 1]));
                    tt[h] = pack(l.x * b0, l.y * b1);
                    ll[h] = pack(l.x, l.y);
                }
                *umma::canon_at<uint4>(Tpp, i, j0, C) = make_uint4(tpp[0], tpp[1], tpp[2], tpp[3]);
                *umma::canon_at<uint4>(Ts, i, j0, C) = make_uint4(tt[0], tt[1], tt[2], tt[3]);
                *umma::canon_at<uint4>(Ls, i, j0, C) = make_uint4(ll[0], ll[1], ll[2], ll[3]);
            }
        }
        umma::wait_st();
    }
    if (BETA) {  // this chunk's V (the next chunk's Q, K, dO may still be landing)
        cp_async_wait<2>();
        mbar_wait(bV, par, &g_tc_status, failed);
    }
    sync_for_mma();
    if (tid == 0) {
        umma::fence_after();
        if (BETA) {  // dk += gamma T^T dW, dk += M^T Q, dW K^T, dV_new V^T, dv = T^T dV_new
            umma::chain<C / 16>(tm + L5::DKC, I128mm, true, umma::op_mn(Tpp, C), umma::op_mn(dWs, 128));
            umma::chain<C / 16>(tm + L5::DKC, I128mm, true, umma::op_mn(Ms, C), umma::op_mn(Qc, 128));
            umma::chain<8>(tm + L5::DTA, I64kk, false, umma::op_k(dWs, 128), umma::op_k(Kc, 128));
            umma::chain<DV / 16>(tm + L5::DTB, I64mk, false, umma::op_mn(dVnc, C), umma::op_k(Vc, DV));
            umma::chain<C / 16>(tm + L5::DVC, IDVmk, false, umma::op_mn(Ts, C), umma::op_k(dVnc, C));
        } else {  // dk += M^T Q
            umma::chain<C / 16>(tm + L5::DKC, I128mm, true, umma::op_mn(Ms, C), umma::op_mn(Qc, 128));
        }
        umma::commit(&bm[3]);
    }

    if (BETA) {
        // ---- E4: dT = dW (gamma K)^T + dV_new V^T, dL, dbeta (column part), the gamma T^T dW share of dG
        wait_bar(&bm[3]);  // V, dV_new^T are free
        if (has_next) copy_v(jn);
        cp_async_commit();
        if (tid == 0 && has_next) bulk_dvn(jn);
        {
            float ta[2][4], tb[2][4];
            umma::ld16(trow + L5::DTA + 16 * nw, ta);
            umma::ld16(trow + L5::DTB + 16 * nw, tb);
            umma::wait_ld();
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                float col[2] = {0.f, 0.f}, ckt[2] = {0.f, 0.f};
                float dl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = (e >> 1) ? r1 : r0, jj = 16 * nw + 8 * n + 2 * tq + (e & 1);
                    const float l = Lf[l_off(r, jj)];
                    const float dt = fmaf(ta[n][e], __expf(Gs[jj]), tb[n][e]);
                    col[e & 1] += dt * l;
                    ckt[e & 1] += ta[n][e] * l;
                    dl[e] = dt * Bs[jj];
                }
                const int jj = 16 * nw + 8 * n + 2 * tq;
                *umma::canon_at<uint32_t>(dLs, r0, jj, C) = pack(dl[0], dl[1]);
                *umma::canon_at<uint32_t>(dLs, r1, jj, C) = pack(dl[2], dl[3]);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    col[0] += __shfl_xor_sync(0xffffffffu, col[0], o);
                    col[1] += __shfl_xor_sync(0xffffffffu, col[1], o);
                    ckt[0] += __shfl_xor_sync(0xffffffffu, ckt[0], o);
                    ckt[1] += __shfl_xor_sync(0xffffffffu, ckt[1], o);
                }
                if (gq == 0) {
                    part[(P_DBC + mw) * C + jj] = col[0];
                    part[(P_DBC + mw) * C + jj + 1] = col[1];
                    part[(P_KT + mw) * C + jj] = ckt[0];
                    part[(P_KT + mw) * C + jj + 1] = ckt[1];
                }
            }
        }
        {  // dv out
            bf16* dvb = dv + bh * s.hs_v + (size_t)t0 * DV;
            if (DV == 128) {
                float a[4][4];
                umma::ld32(trow + L5::DVC + 32 * nw, a);
                umma::wait_ld();
#pragma unroll
                for (int jq = 0; jq < 4; ++jq) {
                    const int col = 32 * nw + 8 * jq + 2 * tq;
                    if (r0 < nval) *reinterpret_cast<uint32_t*>(dvb + (size_t)r0 * DV + col) = pack(a[jq][0], a[jq][1]);
                    if (r1 < nval) *reinterpret_cast<uint32_t*>(dvb + (size_t)r1 * DV + col) = pack(a[jq][2], a[jq][3]);
                }
            } else {
                float a[2][4];
                umma::ld16(trow + L5::DVC + 16 * nw, a);
                umma::wait_ld();
#pragma unroll
                for (int jq = 0; jq < 2; ++jq) {
                    const int col = 16 * nw + 8 * jq + 2 * tq;
                    if (r0 < nval) *reinterpret_cast<uint32_t*>(dvb + (size_t)r0 * DV + col) = pack(a[jq][0], a[jq][1]);
                    if (r1 < nval) *reinterpret_cast<uint32_t*>(dvb + (size_t)r1 * DV + col) = pack(a[jq][2], a[jq][3]);
                }
            }
        }
        sync_for_mma();  // L (fp32) is read for the last time above
        if (tid == 0) {  // X = L^T dL
            umma::fence_after();
            umma::chain<C / 16>(tm + L5::XC, I64mm, false, umma::op_mn(Ls, C), umma::op_mn(dLs, C));
            umma::commit(&bm[4]);
            if (has_next) bulk_l(jn);
        }
        // ---- E5: X (bf16 tile)
        wait_bar(&bm[4]);
        {
            float x[2][4];
            umma::ld16(trow + L5::XC + 16 * nw, x);
            umma::wait_ld();
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int jj = 16 * nw + 8 * n + 2 * tq;
                *umma::canon_at<uint32_t>(Xs, r0, jj, C) = pack(x[n][0], x[n][1]);
                *umma::canon_at<uint32_t>(Xs, r1, jj, C) = pack(x[n][2], x[n][3]);
            }
        }
        sync_for_mma();
        if (tid == 0) {  // dA' = X L^T
            umma::fence_after();
            umma::chain<C / 16>(tm + L5::DA, I64kk, false, umma::op_k(Xs, C), umma::op_k(Ls, C));
            umma::commit(&bm[5]);
        }
        // ---- E6: dA = strictly-lower(-X L^T); Z = dA beta_i Gamma; dbeta (row part); Z sums
        wait_bar(&bm[5]);
        {
            float da[2][4];
            umma::ld16(trow + L5::DA + 16 * nw, da);
            umma::wait_ld();
            float rz0 = 0.f, rz1 = 0.f, rb0 = 0.f, rb1 = 0.f;
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                float col[2] = {0.f, 0.f};
                float zz[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = (e >> 1) ? r1 : r0, jj = 16 * nw + 8 * n + 2 * tq + (e & 1);
                    float z = 0.f, bterm = 0.f;
                    if (jj < i) {
                        const float gm = gmr[n][e];
                        const float dav = -da[n][e];
                        bterm = dav * gm * kkr[n][e];
                        z = dav * Bs[i] * gm;
                    }
                    zz[e] = z;
                    const float za = z * kkr[n][e];
                    if (e >> 1) {
                        rz1 += za;
                        rb1 += bterm;
                    } else {
                        rz0 += za;
                        rb0 += bterm;
                    }
                    col[e & 1] += za;
                }
                const int jj = 16 * nw + 8 * n + 2 * tq;
                *umma::canon_at<uint32_t>(Zs, r0, jj, C) = pack(zz[0], zz[1]);
                *umma::canon_at<uint32_t>(Zs, r1, jj, C) = pack(zz[2], zz[3]);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    col[0] += __shfl_xor_sync(0xffffffffu, col[0], o);
                    col[1] += __shfl_xor_sync(0xffffffffu, col[1], o);
                }
                if (gq == 0) {
                    part[(P_COLA + mw) * C + jj] = col[0];
                    part[(P_COLA + mw) * C + jj + 1] = col[1];
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
        sync_for_mma();
        if (tid == 0) {  // dk += Z K + Z^T K
            umma::fence_after();
            umma::chain<C / 16>(tm + L5::DKC, I128km, true, umma::op_k(Zs, C), umma::op_mn(Kc, 128));
            umma::chain<C / 16>(tm + L5::DKC, I128mm, true, umma::op_mn(Zs, C), umma::op_mn(Kc, 128));
            umma::commit(&bm[6]);
        }
        wait_bar(&bm[6]);  // the last product: the state region is free
        if (tid == 0 && has_next) bulk_state(jn);
    } else {
        wait_bar(&bm[3]);  // the last product: the state region is free
        if (tid == 0 && has_next) bulk_state(jn);
        bf16* dvb = dv + bh * s.hs_v + (size_t)t0 * DV;
        for (int e = tid; e < nval * DV; e += 512) {
            const int jj = e / DV, col = e % DV;
            dvb[(size_t)jj * DV + col] = *umma::canon_at<bf16>(dVnc, col, jj, C);
        }
        __syncthreads();  // dV_new^T is free
        cp_async_commit();
        if (tid == 0 && has_next) bulk_dvn(jn);
    }

    // ---- E7: dq, dk staged as canon tiles in this chunk's Q and K buffer (no
    // product reads it any more), then written out 16 bytes per thread: piece e
    // of a canon [C][128] tile holds row 8 (e / 128) + e % 8, columns
    // 8 ((e / 8) % 16) + 0..7, so the shared reads are linear and a warp writes
    // whole 32-byte sectors of eight rows.
    {
        float a[4][4], b[4][4];
        umma::ld32(trow + L5::DQ + 32 * nw, a);
        umma::ld32(trow + L5::DKC + 32 * nw, b);
        umma::wait_ld();
#pragma unroll
        for (int jq = 0; jq < 4; ++jq) {
            const int col = 32 * nw + 8 * jq + 2 * tq;
            *umma::canon_at<uint32_t>(Qc, r0, col, 128) = pack(a[jq][0], a[jq][1]);
            *umma::canon_at<uint32_t>(Qc, r1, col, 128) = pack(a[jq][2], a[jq][3]);
            *umma::canon_at<uint32_t>(Kc, r0, col, 128) = pack(b[jq][0], b[jq][1]);
            *umma::canon_at<uint32_t>(Kc, r1, col, 128) = pack(b[jq][2], b[jq][3]);
        }
    }
    fence_proxy_async_smem();
    umma::fence_before();
    __syncthreads();  // staging written, partial sums written, TMEM reads done
    if (maps.on && nval == C) {
        if (tid == 0) {
            tma_store5(&maps.dq, 0, t0 / 8, bh, Qc);
            tma_store5(&maps.dk, 0, t0 / 8, bh, Kc);
            bulk_commit();
        }
    } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = tid + 512 * u, pe = e & 1023;
            const int r = ((pe >> 7) << 3) + (pe & 7), cb = (pe >> 3) & 15;
            if (r < nval) {
                const uint4 x = reinterpret_cast<const uint4*>(u < 2 ? Qc : Kc)[pe];
                bf16* dst = (u < 2 ? dq : dk) + bh * s.hs_k + (size_t)(t0 + r) * DK + 8 * cb;
                *reinterpret_cast<uint4*>(dst) = x;
            }
        }
    }
    if (w >= 14) {
        // ---- dG, dg (chunk-local reverse cumsum), dbeta; warps 14 and 15, one token per lane
        auto P = [&](int row, int n, int i) {
            float x = 0.f;
            for (int u = 0; u < n; ++u) x += part[(row + u) * C + i];
            return x;
        };
        const int half = w - 14, i = 32 * half + lane;
        float x = P(P_INTER, GW, i) + P(P_ROWP, GW, i) - P(P_COLP, 4, i) - P(P_Z, GW, i);
        float zs = P(P_Z, GW, i);
        if (BETA) {
            x += P(P_ROWA, GW, i) - P(P_COLA, 4, i) + __expf(Gs[i]) * Bs[i] * P(P_KT, 4, i);
            if (i < nval) dbeta[bh * s.hs_g + t0 + i] = P(P_DBC, 4, i) + P(P_DBR, GW, i);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        if (lane == 0) red[16 + half] = zs;
        asm volatile("bar.sync 1, 64;\n" ::: "memory");
        if (half == 1 && lane == 31) {  // the last token carries the state terms
            float sdot = 0.f;
            for (int u = 0; u < 16; ++u) sdot += red[u];
            x += __expf(gC) * sdot + (red[16] + red[17]);
        }
        float suf = x;  // sum over this warp's tokens from this one on
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += y;
        }
        if (half == 1 && lane == 0) red[18] = suf;
        asm volatile("bar.sync 1, 64;\n" ::: "memory");
        if (half == 0) suf += red[18];
        if (i < nval) dg[bh * s.hs_g + t0 + i] = suf;
    }
    if (tid == 0) bulk_wait_read<0>();  // the tensor-map stores have read the staging
    __syncthreads();  // partial sums consumed, the staging read out
    if (!has_next) break;
    for (int e = tid; e < P_ROWS * C; e += 512) part[e] = 0.f;
    if (tid < C) Bsb[(buf ^ 1) * C + tid] = beta_next;
    j = jn;
  }
    if (tid == 0) bulk_wait<0>();
    umma::fence_before();
    __syncthreads();
    if (w == 0) {
        umma::fence_after();
        umma::dealloc(tm, 512);
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

// Slices of 16 state columns per chain CTA: 1 (B*H*d_v/16 CTAs of 4 warps),
// 2 (half as many CTAs of 8 warps, the default) or 4.  Measured at B=1, H=16,
// T=65536, d=128 on B200, each launch alone: the forward chain takes 0.80,
// 0.96 and 1.60 ms for 1, 2 and 4 slices; the backward launch (forward
// recompute beside the reverse chain, twice the CTAs) 1.67, 1.02 and 1.68 ms.
// SF_GDN_CHAIN_SLICES overrides the default (read once).
int chain_slices() {
    static int n = 0;
    if (n == 0) {
        const char* e = std::getenv("SF_GDN_CHAIN_SLICES");
        n = e ? std::atoi(e) : 2;
        if (n != 1 && n != 4) n = 2;
    }
    return n;
}

ChainOps fwd_ops(const TcWs& w, const float* S_in, float* S_out) {
    return ChainOps{w.W, w.Kh, w.Ut, nullptr, w.Gm, S_in, w.S0t, w.Vnt, S_out};
}
ChainOps bwd_ops(const TcWs& w, const float* dS_out, float* dS_in) {
    return ChainOps{w.Kh, w.W, w.dVit, w.Dt, w.Gm, dS_out, w.dSCt, w.dVnt, dS_in};
}

template <int DV, bool BETA, int NCG>
cudaError_t launch_scan_fwd_n(const SeqView& s, const float* S_in, float* S_out, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = Chain<DV, BETA, false, NCG>::SMEM;
    TC_TRY(smem_attr(tc_scan_fwd_kernel<DV, BETA, NCG>, sm));
    SF_LAUNCH("tc_scan_fwd", st,
              tc_scan_fwd_kernel<DV, BETA, NCG><<<s.BH * chain_ctas_per_head<DV, NCG>(), 128 * NCG, sm, st>>>(
                  s, fwd_ops(w, S_in, S_out)));
    return cudaGetLastError();
}
// The state chains of d_v = 128 run on tcgen05 (one CTA per head) unless
// SF_GDN_CHAIN=warp selects the warp-level chains (read once); d_v = 64 always
// takes the warp-level chains.
bool chain_tcgen05() {
    static int v = -1;
    if (v < 0) {
        const char* e = std::getenv("SF_GDN_CHAIN");
        v = (e && std::string(e) == "tcgen05") ? 1 : 0;
    }
    return v == 1;
}

template <bool BETA>
cudaError_t launch_chain5_fwd(const SeqView& s, const float* S_in, float* S_out, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = Chain5<BETA, false>::SMEM;
    TC_TRY(smem_attr(tc_chain5_fwd_kernel<BETA>, sm));
    SF_LAUNCH("tc_scan_fwd", st, tc_chain5_fwd_kernel<BETA><<<s.BH, 256, sm, st>>>(s, fwd_ops(w, S_in, S_out)));
    return cudaGetLastError();
}
template <bool BETA>
cudaError_t launch_chain5_bwd(const SeqView& s, const BwdArgs& a, bool with_sr, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm_f = Chain5<BETA, false>::SMEM, sm_b = Chain5<BETA, true>::SMEM;
    constexpr size_t sm = sm_f > sm_b ? sm_f : sm_b;
    TC_TRY(smem_attr(tc_chain5_bwd_kernel<BETA>, sm));
    const int nsr = with_sr ? s.BH : 0;
    SF_LAUNCH("tc_scan_bwd", st,
              tc_chain5_bwd_kernel<BETA><<<nsr + s.BH, 256, sm, st>>>(
                  s, fwd_ops(w, a.S_in, nullptr), bwd_ops(w, a.dS_out, a.dS_in), nsr));
    return cudaGetLastError();
}

template <int DV, bool BETA>
cudaError_t launch_scan_fwd(const SeqView& s, const float* S_in, float* S_out, const TcWs& w, cudaStream_t st) {
    if (DV == 128 && chain_tcgen05()) return launch_chain5_fwd<BETA>(s, S_in, S_out, w, st);
    switch (chain_slices()) {
        case 4: return DV % 64 == 0 ? launch_scan_fwd_n<DV, BETA, 4>(s, S_in, S_out, w, st) : cudaErrorInvalidValue;
        case 2: return launch_scan_fwd_n<DV, BETA, 2>(s, S_in, S_out, w, st);
        default: return launch_scan_fwd_n<DV, BETA, 1>(s, S_in, S_out, w, st);
    }
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

// CTAs of a persistent kernel that takes chunk tickets: one per SM at most.
// (Measured at the headline segment chain: capping the chunks a CTA takes, so
// that the chain launches get SMs sooner, made the step slower at every cap.)
int persistent_grid(const SeqView& s) { return std::min(s.NC * s.BH, num_sms()); }

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library does not link the driver library); null if the driver lacks it.
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// The five-dimensional canon view of a [BH][T][D] bf16 tensor (head stride hs
// elements) described at G5Maps; false if it cannot be made (no driver entry
// point, a base not 16-byte aligned, fewer than C tokens).
bool canon_map(CUtensorMap* m, const void* base, int BH, int T, int D, long long hs) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = encode_tiled();
    if (!enc || T < C || BH < 1 || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
    const cuuint64_t dims[5] = {8, 8, (cuuint64_t)(D / 8), (cuuint64_t)(T / 8), (cuuint64_t)BH};
    const cuuint64_t strides[4] = {(cuuint64_t)D * 2, 16, (cuuint64_t)D * 16, (cuuint64_t)hs * 2};
    const cuuint32_t box[5] = {8, 8, (cuuint32_t)(D / 8), C / 8, 1};
    const cuuint32_t unit[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, unit,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Persistent Out: one CTA per SM at most, chunks from w.oticket.
template <int DV, bool OG>
cudaError_t launch_out2(const char* name, const SeqView& s, const bf16* q, const bf16* k, bf16* o, const bf16* dO,
                        const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = O2<DV, OG>::SMEM;
    TC_TRY(smem_attr(tc_out2_kernel<DV, OG>, sm));
    TC_TRY(cudaMemsetAsync(w.oticket, 0, sizeof(int), st));
    const int grid = persistent_grid(s);
    TokMaps maps;
    memset(&maps, 0, sizeof(maps));
    maps.on = canon_map(&maps.q, q, s.BH, s.T, DK, s.hs_k) && canon_map(&maps.k, k, s.BH, s.T, DK, s.hs_k) &&
              (!OG || canon_map(&maps.dO, dO, s.BH, s.T, DV, s.hs_v));
    SF_LAUNCH(name, st, tc_out2_kernel<DV, OG><<<grid, 256, sm, st>>>(
                            s, q, k, w.Gc, w.Vnt, w.S0t, o, dO, OG ? w.dVit : nullptr, OG ? w.Dt : nullptr,
                            w.oticket, maps));
    return cudaGetLastError();
}
// Out on tcgen05 (d_v = 128) unless SF_GDN_OUT=warp selects the warp-level
// kernel (read once); d_v = 64 always takes the warp-level kernel.
bool out_tcgen05() {
    static int v = -1;
    if (v < 0) {
        const char* e = std::getenv("SF_GDN_OUT");
        v = (e && std::string(e) == "warp") ? 0 : 1;
    }
    return v == 1;
}
template <bool OG>
cudaError_t launch_out5(const char* name, const SeqView& s, const bf16* q, const bf16* k, bf16* o, const bf16* dO,
                        const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = O5<OG>::SMEM;
    TC_TRY(smem_attr(tc_out5_kernel<OG>, sm));
    TC_TRY(cudaMemsetAsync(w.oticket, 0, sizeof(int), st));
    const int grid = persistent_grid(s);
    TokMaps maps;
    memset(&maps, 0, sizeof(maps));
    maps.on = canon_map(&maps.q, q, s.BH, s.T, DK, s.hs_k) && canon_map(&maps.k, k, s.BH, s.T, DK, s.hs_k) &&
              (!OG || canon_map(&maps.dO, dO, s.BH, s.T, 128, s.hs_v));
    SF_LAUNCH(name, st, tc_out5_kernel<OG><<<grid, 256, sm, st>>>(
                            s, q, k, w.Gc, w.Vnt, w.S0t, o, dO, OG ? w.dVit : nullptr, OG ? w.Dt : nullptr,
                            w.oticket, maps));
    return cudaGetLastError();
}
template <int DV>
cudaError_t launch_out(const SeqView& s, const bf16* q, const bf16* k, bf16* o, const TcWs& w, cudaStream_t st) {
    if (DV == 128 && out_tcgen05()) return launch_out5<false>("tc_out", s, q, k, o, nullptr, w, st);
    return launch_out2<DV, false>("tc_out", s, q, k, o, nullptr, w, st);
}
template <int DV>
cudaError_t launch_out_og(const SeqView& s, const bf16* q, const bf16* k, bf16* o, const bf16* dO, const TcWs& w,
                          cudaStream_t st) {
    if (DV == 128 && out_tcgen05()) return launch_out5<true>("tc_out_og", s, q, k, o, dO, w, st);
    return launch_out2<DV, true>("tc_out_og", s, q, k, o, dO, w, st);
}

template <int DV>
cudaError_t launch_intra(const SeqView& s, const bf16* q, const bf16* k, const bf16* dO, const TcWs& w,
                         cudaStream_t st) {
    constexpr size_t sm = intra_smem<DV>();
    TC_TRY(smem_attr(tc_intra_kernel<DV>, sm));
    SF_LAUNCH("tc_intra", st, tc_intra_kernel<DV><<<dim3(s.NC, s.BH), 128, sm, st>>>(s, q, k, dO, w.Gc, w.dVit, w.Dt));
    return cudaGetLastError();
}

template <int DV, bool BETA, int NCG>
cudaError_t launch_scan_bwd_n(const SeqView& s, const BwdArgs& a, bool with_sr, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm_f = Chain<DV, BETA, false, NCG>::SMEM, sm_b = Chain<DV, BETA, true, NCG>::SMEM;
    constexpr size_t sm = sm_f > sm_b ? sm_f : sm_b;
    TC_TRY(smem_attr(tc_scan_bwd_dual_kernel<DV, BETA, NCG>, sm));
    const int per = s.BH * chain_ctas_per_head<DV, NCG>();
    const int nsr = with_sr ? per : 0;
    SF_LAUNCH("tc_scan_bwd", st,
              tc_scan_bwd_dual_kernel<DV, BETA, NCG><<<nsr + per, 128 * NCG, sm, st>>>(
                  s, fwd_ops(w, a.S_in, nullptr), bwd_ops(w, a.dS_out, a.dS_in), nsr));
    return cudaGetLastError();
}
template <int DV, bool BETA>
cudaError_t launch_scan_bwd(const SeqView& s, const BwdArgs& a, bool with_sr, const TcWs& w, cudaStream_t st) {
    if (DV == 128 && chain_tcgen05()) return launch_chain5_bwd<BETA>(s, a, with_sr, w, st);
    switch (chain_slices()) {
        case 4: return launch_scan_bwd_n<DV, BETA, 4>(s, a, with_sr, w, st);
        case 2: return launch_scan_bwd_n<DV, BETA, 2>(s, a, with_sr, w, st);
        default: return launch_scan_bwd_n<DV, BETA, 1>(s, a, with_sr, w, st);
    }
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
cudaError_t launch_grad5(const SeqView& s, const BwdArgs& a, const TcWs& w, cudaStream_t st) {
    constexpr size_t sm = G5<DV>::SMEM;
    TC_TRY(smem_attr(tc_grad5_kernel<DV, BETA>, sm));
    TC_TRY(cudaMemsetAsync(w.ticket, 0, sizeof(int), st));
    const int grid = persistent_grid(s);
    G5Maps maps;
    memset(&maps, 0, sizeof(maps));
    maps.on = canon_map(&maps.q, a.q, s.BH, s.T, DK, s.hs_k) && canon_map(&maps.k, a.k, s.BH, s.T, DK, s.hs_k) &&
              canon_map(&maps.dO, a.dO, s.BH, s.T, DV, s.hs_v) &&
              (!BETA || canon_map(&maps.v, a.v, s.BH, s.T, DV, s.hs_v)) &&
              canon_map(&maps.dq, a.dq, s.BH, s.T, DK, s.hs_k) && canon_map(&maps.dk, a.dk, s.BH, s.T, DK, s.hs_k);
    SF_LAUNCH("tc_grad", st, tc_grad5_kernel<DV, BETA><<<grid, 512, sm, st>>>(
                                 s, static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k),
                                 static_cast<const bf16*>(a.v), a.beta, static_cast<const bf16*>(a.dO), w.Gc,
                                 w.Lm, w.Vnt, w.dVnt, w.S0t, w.dSCt, static_cast<bf16*>(a.dq), static_cast<bf16*>(a.dk),
                                 static_cast<bf16*>(a.dv), a.dg, a.dbeta, w.ticket, maps));
    return cudaGetLastError();
}

// Gradient kernel: the tcgen05 one (default) or the warp-level persistent one
// (SF_GDN_GRAD=warp), read once.
bool grad_tcgen05() {
    static int v = -1;
    if (v < 0) {
        const char* e = std::getenv("SF_GDN_GRAD");
        v = (e && std::string(e) == "warp") ? 0 : 1;
    }
    return v == 1;
}

template <int DV, bool BETA>
cudaError_t launch_grad_any(const SeqView& s, const BwdArgs& a, const TcWs& w, cudaStream_t st) {
    return grad_tcgen05() ? launch_grad5<DV, BETA>(s, a, w, st) : launch_grad<DV, BETA>(s, a, w, st);
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
    return launch_grad_any<DV, BETA>(s, a, w, st);
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
        case TcStage::Grad: return launch_grad_any<DV, BETA>(s, *b, w, st);
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
