// Blackwell (sm_100a) tensor-core building blocks, written as inline PTX:
// mbarriers with bounded waits, TMEM allocation, tcgen05.mma (kind::f16, BF16 in, FP32
// accumulate in TMEM), tcgen05.commit, TMEM <-> register moves, shared-memory matrix
// descriptors and the two 128-byte-swizzled BF16 layouts the descriptors describe.
//
// Layouts (bf16, 2 bytes per element; every tile base 1024-byte aligned):
//  K-major tile [R rows][Kc cols], Kc a multiple of 64: 8-row x 64-column atoms of 1024 B;
//    within an atom row r (r % 8) holds 128 B whose 16-byte chunks are permuted by
//    chunk ^ (r % 8). Atoms stack down the rows (stride 1024 B = SBO) and then across
//    64-column blocks (stride R * 128 B). One MMA K-step (16 columns, 32 B) is addressed
//    by advancing the descriptor start 32 B inside the atom row.
//  MN-major tile [Kx rows of K][MNx cols of M/N], MNx a multiple of 64: atoms of 8 K-rows x
//    64 MN-elements (1024 B), same chunk permutation by (k % 8); atoms stack along K with
//    stride 1024 B (SBO) and across 64-element MN blocks with stride Kx * 128 B (LBO). One
//    K-step (16 rows) is two atoms: the descriptor start advances 2048 B per step.
#pragma once

#include <stdint.h>

namespace kda {
namespace umma {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ layouts (byte offsets)

__device__ __forceinline__ uint32_t kmaj_off(int r, int c, int R) {
    return static_cast<uint32_t>((c >> 6) * (R * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                                 ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ uint32_t mnmaj_off(int mn, int k, int Kx) {
    return static_cast<uint32_t>((mn >> 6) * (Kx * 128) + (k >> 3) * 1024 + (k & 7) * 128 +
                                 ((((mn & 63) >> 3) ^ (k & 7)) << 4) + ((mn & 7) << 1));
}

// ------------------------------------------------------------------ descriptors

// Shared-memory matrix descriptor, SWIZZLE_128B, descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// K-step ks of a K-major tile with R rows starting at row0 (a multiple of 8).
__device__ __forceinline__ uint64_t kmaj_desc(uint32_t base, int R, int row0, int ks) {
    return sdesc(base + (ks >> 2) * (R * 128) + (row0 >> 3) * 1024 + (ks & 3) * 32, 16, 1024);
}

// K-step ks of an MN-major tile with Kx rows of K, starting at MN column mn0 (a multiple of 64).
__device__ __forceinline__ uint64_t mnmaj_desc(uint32_t base, int Kx, int mn0, int ks) {
    return sdesc(base + (mn0 >> 6) * (Kx * 128) + ks * 2048, Kx * 128, 1024);
}

// The descriptor of K-step ks minus that of K-step 0, for kmaj_desc (R rows) and mnmaj_desc: the
// start-address field counts 16-byte units, and a tile ends below 256 KB of shared memory, so the
// offset never carries into the other fields. An issuing thread keeps the K-step-0 descriptors
// and adds these constants (an unrolled K loop folds them into immediates).
__host__ __device__ constexpr uint64_t kmaj_step(int R, int ks) {
    return static_cast<uint64_t>(((ks >> 2) * (R * 128) + (ks & 3) * 32) >> 4);
}
__host__ __device__ constexpr uint64_t mnmaj_step(int ks) { return static_cast<uint64_t>((ks * 2048) >> 4); }

// Instruction descriptor, kind::f16: BF16 A and B, FP32 D, dense, no negation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One try: true once phase `parity` of the barrier has completed. The thread may be suspended
// inside the instruction until the phase completes or up to kSuspendNs nanoseconds pass, so a
// waiting warp does not spin and take issue slots from the warps that are working.
constexpr uint32_t kSuspendNs = 100000;
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return done;
}

// Bounded wait for phase `parity` of `bar`: true when it completed, false when
// `max_cycles` SM clocks passed first (the caller then records an error and bails out).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long max_cycles) {
    const uint32_t addr = smem_u32(bar);
    const long long t0 = clock64();
    while (!mbar_try_wait(addr, parity)) {
        if (clock64() - t0 > max_cycles) return false;
    }
    return true;
}

// ------------------------------------------------------------------ fences

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ------------------------------------------------------------------ TMEM allocation (one warp)

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ------------------------------------------------------------------ MMA (issued by one thread)

// D[tmem] (+)= A[smem] . B[smem]^T  (M x N x 16), BF16 inputs, FP32 accumulate.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ------------------------------------------------------------------ TMEM <-> registers (warp)

// Lane address of warp w's quarter: lanes 32*(w%4) .. +31.
__device__ __forceinline__ uint32_t tmem_lane_base(uint32_t taddr, int warp) {
    return taddr + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ BF16 split precision

// x = hi + lo + r with hi = bf16(x), lo = bf16(x - hi), |r| <= 2^-17 |x|: three BF16 MMAs
// (hi.hi + hi.lo + lo.hi) then carry a product to about 2^-16 relative accuracy.
__device__ __forceinline__ void split_bf16(float x, uint16_t &hi, uint16_t &lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const __nv_bfloat16 l = __float2bfloat16_rn(x - __bfloat162float(h));
    hi = *reinterpret_cast<const uint16_t *>(&h);
    lo = *reinterpret_cast<const uint16_t *>(&l);
}

// The same split for two values at once: hi and lo come back as packed BF16x2 words
// (first value in the low half), with one paired conversion for each.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

}  // namespace umma
}  // namespace kda
