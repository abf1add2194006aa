// Fifth-generation tensor cores (tcgen05, sm_100a): shared-memory operand
// descriptors, the kind::f16 instruction descriptor, tensor-memory (TMEM)
// allocation, single-thread MMA issue with completion on an mbarrier, and TMEM
// loads/stores in the register layout of the warp-level m16n8 accumulators.
//
// Operand tiles use the canonical layout without swizzle ("canon"): a
// [rows][rowlen] bf16 tile is cut into core matrices of 8 rows x 8 elements
// (16 bytes per row), each stored as 128 contiguous bytes (row i of the core
// matrix at byte 16 i); core matrix (a, b) (row block a, column block b) sits
// at byte a * 16 * rowlen + b * 128.  The same bytes serve as
//   a K-major operand  (rows = M or N, rowlen = K): the core matrices adjacent
//                      along K are 128 bytes apart (LBO), along M/N 16 rowlen (SBO);
//   an MN-major operand (rows = K, rowlen = M or N): adjacent along M/N are
//                      16 rowlen apart (LBO), along K 128 bytes (SBO).
// One MMA consumes K = 16 (two core matrices along K).  Any 8 x 8 block of a
// canon tile is 128 contiguous bytes, so ldmatrix/stmatrix and row-pair
// accesses of such tiles are free of bank conflicts.
//
// Accumulators are fp32 in TMEM.  For M = 64 (cta_group::1), row m of D is
// TMEM lane (m % 16) + 32 (m / 16) and column n is column base + n; a warp may
// only touch its own 32-lane quarter (warp index % 4), i.e. rows 16 (w % 4)
// .. 16 (w % 4) + 15, and the 16x256b loads below return them in the m16n8
// fragment layout: c[j] = {D[g][8j+2t], D[g][8j+2t+1], D[g+8][8j+2t],
// D[g+8][8j+2t+1]} with g = lane / 4, t = lane % 4.
#pragma once

#include <stdint.h>

#include "tc_mma.cuh"

namespace sf {
namespace umma {

using tc::smem_u32;

// Byte offset of element (r, c) of a canon [rows][rowlen] bf16 tile.
__host__ __device__ __forceinline__ uint32_t canon_off(int r, int c, int rowlen) {
    return (uint32_t)((r >> 3) * (16 * rowlen) + (c >> 3) * 128 + (r & 7) * 16 + (c & 7) * 2);
}
// Element offset of (r, c) in a canon bf16 tile.
__host__ __device__ __forceinline__ int canon_el(int r, int c, int rowlen) { return (int)(canon_off(r, c, rowlen) >> 1); }
// Row and column of the e-th 16-byte piece of a canon [rows][rowlen] tile
// (pieces in address order), for copies that write the tile linearly.
__host__ __device__ __forceinline__ void canon_piece(int e, int rowlen, int& r, int& c) {
    const int per_rb = rowlen;  // pieces in one 8-row block: 8 rows x rowlen / 8
    r = (e / per_rb) * 8 + (e & 7);
    c = ((e % per_rb) >> 3) * 8;
}
template <typename T>
__device__ __forceinline__ T* canon_at(void* base, int r, int c, int rowlen) {
    return reinterpret_cast<T*>(static_cast<char*>(base) + canon_off(r, c, rowlen));
}
template <typename T>
__device__ __forceinline__ const T* canon_at(const void* base, int r, int c, int rowlen) {
    return reinterpret_cast<const T*>(static_cast<const char*>(base) + canon_off(r, c, rowlen));
}

// Shared-memory matrix descriptor, no swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version of sm_100
    return d;                // base offset 0, swizzle none
}
// K = 16 slice `ks` of a K-major operand stored as a canon [R][K] tile.
__device__ __forceinline__ uint64_t desc_k(const void* base, int ks, int K) {
    return sdesc(smem_u32(base) + (uint32_t)ks * 256u, 128u, 16u * (uint32_t)K);
}
// K = 16 slice `ks` of an MN-major operand stored as a canon [K][R] tile.
__device__ __forceinline__ uint64_t desc_mn(const void* base, int ks, int R) {
    return sdesc(smem_u32(base) + (uint32_t)ks * 32u * (uint32_t)R, 16u * (uint32_t)R, 128u);
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32, dense, M x N,
// each operand K-major (false) or MN-major (true).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B, issued by one thread.
__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)accumulate));
}
// A K-sliced operand for a chain of MMAs: the descriptor of slice 0 and the
// step of its address field (byte address / 16) from one K = 16 slice to the
// next: 256 bytes in a K-major canon [R][K] tile, 32 R bytes in an MN-major
// canon [K][R] tile.  Shared addresses stay below 2^18 bytes, so adding to the
// field never carries into the next one.
struct Op {
    uint64_t d;
    uint32_t step;
};
__device__ __forceinline__ Op op_k(const void* base, int K) { return {desc_k(base, 0, K), 16u}; }
__device__ __forceinline__ Op op_mn(const void* base, int R) { return {desc_mn(base, 0, R), 2u * (uint32_t)R}; }
// D (+)= A B over NKS slices of K = 16, issued back to back by one thread:
// the descriptors are formed once and advanced by one addition per MMA, so the
// issue keeps ahead of the tensor core (forming each descriptor afresh costs
// about 100 cycles of dependent integer work per MMA, more than an M = 64 MMA
// takes to run).
template <int NKS>
__device__ __forceinline__ void chain(uint32_t d_tmem, uint32_t idesc, bool accumulate, Op a, Op b) {
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks)
        mma(d_tmem, a.d + (uint64_t)(ks * a.step), b.d + (uint64_t)(ks * b.step), idesc, accumulate || ks > 0);
}

// The mbarrier gets one arrival once every MMA this thread issued before has completed.
__device__ __forceinline__ void commit(void* mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_u32(mbar))
                 : "memory");
}

// TMEM allocation by one whole warp; the base address is written to *dst.
__device__ __forceinline__ void alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t taddr(uint32_t base, int lane, int col) {
    return base + ((uint32_t)lane << 16) + (uint32_t)col;
}

// 16 rows x 32 columns (four m16n8 accumulator fragments) at `ta`.
__device__ __forceinline__ void ld32(uint32_t ta, float (&c)[4][4]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
        "[%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta));
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[j][e] = __uint_as_float(r[4 * j + e]);
}
// 16 rows x 16 columns (two fragments) at `ta`.
__device__ __forceinline__ void ld16(uint32_t ta, float (&c)[2][4]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(ta));
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[j][e] = __uint_as_float(r[4 * j + e]);
}
// Store 16 rows x 32 columns back (the layout of ld32).
__device__ __forceinline__ void st32(uint32_t ta, const float (&c)[4][4]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
            ta),
        "r"(__float_as_uint(c[0][0])), "r"(__float_as_uint(c[0][1])), "r"(__float_as_uint(c[0][2])),
        "r"(__float_as_uint(c[0][3])), "r"(__float_as_uint(c[1][0])), "r"(__float_as_uint(c[1][1])),
        "r"(__float_as_uint(c[1][2])), "r"(__float_as_uint(c[1][3])), "r"(__float_as_uint(c[2][0])),
        "r"(__float_as_uint(c[2][1])), "r"(__float_as_uint(c[2][2])), "r"(__float_as_uint(c[2][3])),
        "r"(__float_as_uint(c[3][0])), "r"(__float_as_uint(c[3][1])), "r"(__float_as_uint(c[3][2])),
        "r"(__float_as_uint(c[3][3]))
        : "memory");
}
// 32 TMEM columns of this thread's lane (the 32x32b shape: warp w % 4 reads
// lanes 32 (w % 4).., thread t lane 32 (w % 4) + t; register j = column + j).
__device__ __forceinline__ void ld_row32(uint32_t ta, float (&c)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
        "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(ta));
#pragma unroll
    for (int j = 0; j < 32; ++j) c[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void st_row32(uint32_t ta, const float (&c)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(ta),
        "r"(__float_as_uint(c[0])), "r"(__float_as_uint(c[1])), "r"(__float_as_uint(c[2])), "r"(__float_as_uint(c[3])),
        "r"(__float_as_uint(c[4])), "r"(__float_as_uint(c[5])), "r"(__float_as_uint(c[6])), "r"(__float_as_uint(c[7])),
        "r"(__float_as_uint(c[8])), "r"(__float_as_uint(c[9])), "r"(__float_as_uint(c[10])), "r"(__float_as_uint(c[11])),
        "r"(__float_as_uint(c[12])), "r"(__float_as_uint(c[13])), "r"(__float_as_uint(c[14])),
        "r"(__float_as_uint(c[15])), "r"(__float_as_uint(c[16])), "r"(__float_as_uint(c[17])),
        "r"(__float_as_uint(c[18])), "r"(__float_as_uint(c[19])), "r"(__float_as_uint(c[20])),
        "r"(__float_as_uint(c[21])), "r"(__float_as_uint(c[22])), "r"(__float_as_uint(c[23])),
        "r"(__float_as_uint(c[24])), "r"(__float_as_uint(c[25])), "r"(__float_as_uint(c[26])),
        "r"(__float_as_uint(c[27])), "r"(__float_as_uint(c[28])), "r"(__float_as_uint(c[29])),
        "r"(__float_as_uint(c[30])), "r"(__float_as_uint(c[31]))
        : "memory");
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// ldmatrix fragments from canon tiles (lane roles as tc::ldA / ldAt / ldBnk / ldBkn).
// A (16 x 16 at [m0, k0]) from a tile [m][k].
__device__ __forceinline__ void ldA_c(uint32_t (&a)[4], const void* s, int rowlen, int m0, int k0, int lane) {
    tc::ldsm_x4(a, static_cast<const char*>(s) + canon_off(m0 + (lane & 15), k0 + ((lane >> 4) << 3), rowlen));
}
// A (16 x 16 at [m0, k0]) from a tile [k][m].
__device__ __forceinline__ void ldAt_c(uint32_t (&a)[4], const void* s, int rowlen, int m0, int k0, int lane) {
    tc::ldsm_x4_t(a, static_cast<const char*>(s) +
                         canon_off(k0 + (lane & 7) + ((lane >> 4) << 3), m0 + (((lane >> 3) & 1) << 3), rowlen));
}
// B for n-tiles n0, n0+8 over k0..k0+15 from a tile [n][k].
__device__ __forceinline__ void ldBnk_c(uint32_t (&b)[4], const void* s, int rowlen, int n0, int k0, int lane) {
    tc::ldsm_x4(b, static_cast<const char*>(s) +
                       canon_off(n0 + (lane & 7) + ((lane >> 4) << 3), k0 + (((lane >> 3) & 1) << 3), rowlen));
}
// B for n-tiles n0, n0+8 over k0..k0+15 from a tile [k][n].
__device__ __forceinline__ void ldBkn_c(uint32_t (&b)[4], const void* s, int rowlen, int n0, int k0, int lane) {
    tc::ldsm_x4_t(b, static_cast<const char*>(s) +
                         canon_off(k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n0 + ((lane >> 4) << 3), rowlen));
}
// stmatrix of a 16 x 16 bf16 A-fragment block into a canon tile at [r0, c0].
__device__ __forceinline__ void st_afrag_c(void* t, int rowlen, int r0, int c0, const uint32_t (&a)[4], int lane) {
    const int lr = (lane & 7) + (((lane >> 3) & 1) << 3), pb = lane >> 4;
    tc::stsm_x4(static_cast<char*>(t) + canon_off(r0 + lr, c0 + 8 * pb, rowlen), a);
}

// Copy a [ROWS][COLS] bf16 global tile (row stride gld elements; rows >= nrows
// zero-filled) into a canon shared tile.  Thread e fills the e-th 16-byte piece
// of the shared tile, so the shared writes are linear; a warp reads 8 rows x
// 64 bytes of global memory.
template <int ROWS, int COLS, int NT>
__device__ __forceinline__ void load_canon(void* s, const __nv_bfloat16* g, long long gld, int nrows, int tid) {
    constexpr int CPR = COLS / 8;
    for (int e = tid; e < ROWS * CPR; e += NT) {
        const int r = ((e >> 3) / CPR) * 8 + (e & 7), c = ((e >> 3) % CPR) * 8;
        const bool ok = r < nrows;
        tc::cp_async16(static_cast<char*>(s) + 16 * e, g + (ok ? (long long)r * gld : 0) + c, ok);
    }
}

}  // namespace umma
}  // namespace sf
