// Warp-level bf16 tensor-core fragments (m16n8k16, fp32 accumulate), shared
// memory fragment loads (ldmatrix) and asynchronous global->shared copies.
//
// Fragment layouts of mma.m16n8k16 (g = lane / 4, t = lane % 4):
//   A (16x16): a0 = A[g][2t..2t+1]   a1 = A[g+8][2t..]   a2 = A[g][2t+8..]   a3 = A[g+8][2t+8..]
//   B (16x8):  b0 = B[2t..2t+1][g]   b1 = B[2t+8..2t+9][g]
//   C (16x8):  c0 = C[g][2t]  c1 = C[g][2t+1]  c2 = C[g+8][2t]  c3 = C[g+8][2t+1]
// Shared tiles are row-major bf16 with a padded row stride (a multiple of 8
// elements that is not a multiple of 64), so the eight 16-byte rows one
// ldmatrix phase touches fall in distinct bank groups.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace sf {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous copy global -> shared; `valid == false` writes zeros
// (no global bytes are read, `src` only has to be a mapped address).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
}
__device__ __forceinline__ uint32_t scale2(uint32_t u, float s0, float s1) {
    const float2 f = unpack(u);
    return pack(f.x * s0, f.y * s1);
}

// A (16 x 16 at [m0, k0]) from a tile stored [m][k] (row-major A).
__device__ __forceinline__ void ldA(uint32_t (&a)[4], const __nv_bfloat16* s, int ld, int m0, int k0,
                                    int lane) {
    ldsm_x4(a, s + (m0 + (lane & 15)) * ld + k0 + ((lane >> 4) << 3));
}
// A (16 x 16 at [m0, k0]) from a tile stored [k][m] (A transposed in memory).
__device__ __forceinline__ void ldAt(uint32_t (&a)[4], const __nv_bfloat16* s, int ld, int m0, int k0,
                                     int lane) {
    ldsm_x4_t(a, s + (k0 + (lane & 7) + ((lane >> 4) << 3)) * ld + m0 + (((lane >> 3) & 1) << 3));
}
// B for two n-tiles (n0 and n0+8) over k0..k0+15, from a tile stored [n][k].
// b[0], b[1]: n-tile n0; b[2], b[3]: n-tile n0+8.
__device__ __forceinline__ void ldBnk(uint32_t (&b)[4], const __nv_bfloat16* s, int ld, int n0, int k0,
                                     int lane) {
    ldsm_x4(b, s + (n0 + (lane & 7) + ((lane >> 4) << 3)) * ld + k0 + (((lane >> 3) & 1) << 3));
}
// B for two n-tiles (n0 and n0+8) over k0..k0+15, from a tile stored [k][n].
__device__ __forceinline__ void ldBkn(uint32_t (&b)[4], const __nv_bfloat16* s, int ld, int n0, int k0,
                                     int lane) {
    ldsm_x4_t(b, s + (k0 + (lane & 7) + (((lane >> 3) & 1) << 3)) * ld + n0 + ((lane >> 4) << 3));
}

// A fragment for k-tile kk built from C fragments of n-tiles 2kk and 2kk+1
// (the accumulator of one product becomes the left operand of the next).
__device__ __forceinline__ void c2a(uint32_t (&a)[4], const float (&c0)[4], const float (&c1)[4]) {
    a[0] = pack(c0[0], c0[1]);
    a[1] = pack(c0[2], c0[3]);
    a[2] = pack(c1[0], c1[1]);
    a[3] = pack(c1[2], c1[3]);
}

// Bulk asynchronous shared -> global copy (one thread issues it; 16-byte
// aligned addresses, size a multiple of 16), its group commit and waits.
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n" ::"l"(gdst),
                 "r"(smem_u32(ssrc)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;\n" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;\n" ::"n"(N) : "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// stmatrix: store four 8x8 bf16 matrices held in fragment layout (the inverse of ldmatrix).
__device__ __forceinline__ void stsm_x4(void* p, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};\n" ::"r"(smem_u32(p)),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

// stmatrix with transpose: matrix m's row r (address from lane 8 m + r)
// receives column r of the fragment-layout 8x8 block held in register m.
__device__ __forceinline__ void stsm_x4_t(void* p, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};\n" ::"r"(smem_u32(p)),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

// mbarrier-tracked bulk asynchronous global -> shared copy (issued by one thread).
__device__ __forceinline__ void mbar_init(void* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(void* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_load(void* sdst, const void* gsrc, uint32_t bytes, void* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     smem_u32(sdst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// One arrival without a transaction count (a phase whose copies went another way).
__device__ __forceinline__ void mbar_arrive(void* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
// Tensor-map (TMA) copies of one box of a five-dimensional tensor map, issued
// by one thread: global -> shared completing on an mbarrier, shared -> global
// in the bulk group of the issuing thread.  `map` is the generic address of a
// __grid_constant__ CUtensorMap parameter; the innermost coordinate is 0.
__device__ __forceinline__ void tma_load5(void* sdst, const void* map, int c2, int c3, int c4, void* bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
        "%6}], [%7];\n" ::"r"(smem_u32(sdst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(0), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar))
        : "memory");
}
// Bring a tensor map (a __grid_constant__ parameter) into the TMA unit's
// descriptor cache ahead of its first copy.
__device__ __forceinline__ void tma_prefetch_map(const void* map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_store5(const void* map, int c2, int c3, int c4, const void* ssrc) {
    asm volatile("cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4, %5}], [%6];\n" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(0), "r"(0), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(ssrc))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(void* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for phase `parity` of an mbarrier, giving up after about 2^32 cycles
// (a couple of seconds): then `*status` gets bit 0 and `failed` is set, and
// later waits of this thread return at once, so the kernel always finishes.
__device__ __forceinline__ void mbar_wait(void* bar, uint32_t parity, int* status, bool& failed) {
    if (failed || mbar_try_wait(bar, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > (1ll << 32)) {
            atomicOr(status, 1);
            failed = true;
            return;
        }
    }
}

// Copy a [rows][cols] bf16 global tile (row stride gld elements) into shared
// memory (row stride sld), 16 bytes per request, rows >= nrows zero-filled.
template <int ROWS, int COLS, int NT>
__device__ __forceinline__ void load_tile(__nv_bfloat16* s, int sld, const __nv_bfloat16* g,
                                          long long gld, int nrows, int tid) {
    constexpr int CPR = COLS / 8;  // 16-byte pieces per row
    for (int e = tid; e < ROWS * CPR; e += NT) {
        const int r = e / CPR, c = (e % CPR) * 8;
        const bool ok = r < nrows;
        cp_async16(s + r * sld + c, g + (ok ? (long long)r * gld : 0) + c, ok);
    }
}

}  // namespace tc
}  // namespace sf
