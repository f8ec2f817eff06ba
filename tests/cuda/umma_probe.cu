// Test-only probe of the tcgen05 building blocks in umma.cuh: one CTA stages A [M][K] and
// B [N][K] (BF16-exact values) in the K-major or MN-major 128-byte-swizzled layout, issues
// K/16 MMAs into TMEM, commits to an mbarrier (bounded wait) and reads D = A.B^T back
// with tcgen05.ld. The host compares D with an exact product.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "umma.cuh"

using namespace kda::umma;

template <int M, int N, int K, bool AMN, bool BMN>
__global__ void __launch_bounds__(128) probe_kernel(const float *A, const float *Bt, float *D, int *status) {
    constexpr int MA = AMN ? ((M + 63) / 64) * 64 : M;
    constexpr int NB = BMN ? ((N + 63) / 64) * 64 : N;
    constexpr int A_BYTES = MA * K * 2, B_BYTES = NB * K * 2;
    constexpr uint32_t NCOLS = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base, *sB = base + A_BYTES;
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < (A_BYTES + B_BYTES) / 4; i += 128) reinterpret_cast<uint32_t *>(base)[i] = 0u;
    __syncthreads();
    for (int e = tid; e < M * K; e += 128) {
        const int m = e / K, k = e % K;
        const uint32_t off = AMN ? mnmaj_off(m, k, K) : kmaj_off(m, k, MA);
        *reinterpret_cast<__nv_bfloat16 *>(sA + off) = __float2bfloat16_rn(A[e]);
    }
    for (int e = tid; e < N * K; e += 128) {
        const int n = e / K, k = e % K;
        const uint32_t off = BMN ? mnmaj_off(n, k, K) : kmaj_off(n, k, NB);
        *reinterpret_cast<__nv_bfloat16 *>(sB + off) = __float2bfloat16_rn(Bt[e]);
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, NCOLS);
        tmem_relinquish();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t taddr = tmem_base;
    if (tid == 0) {
        constexpr uint32_t idesc = idesc_bf16(M, N, AMN, BMN);
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
        for (int ks = 0; ks < K / 16; ++ks) {
            const uint64_t ad = AMN ? mnmaj_desc(a0, K, 0, ks) : kmaj_desc(a0, MA, 0, ks);
            const uint64_t bd = BMN ? mnmaj_desc(b0, K, 0, ks) : kmaj_desc(b0, NB, 0, ks);
            mma_bf16(taddr, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0, 2000000000LL);
    tc_fence_after();
    if (!ok) {
        if ((tid & 31) == 0) atomicExch(status, 1);
    } else {
        const int lane_idx = 32 * warp + (tid & 31);
        int m = lane_idx;
        if (M == 64) m = ((tid & 31) < 16) ? 16 * warp + (tid & 31) : -1;
#pragma unroll 1
        for (int c0 = 0; c0 < N; c0 += 8) {
            float v[8];
            tmem_ld8(tmem_lane_base(taddr, warp) + c0, v);
            tmem_ld_wait();
            if (m >= 0)
#pragma unroll
                for (int j = 0; j < 8; ++j) D[m * N + c0 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(taddr, NCOLS);
}

template <int M, int N, int K, bool AMN, bool BMN>
static int run(const float *A, const float *B, float *D, int *status) {
    constexpr int MA = AMN ? ((M + 63) / 64) * 64 : M;
    constexpr int NB = BMN ? ((N + 63) / 64) * 64 : N;
    const int smem = (MA + NB) * K * 2 + 1024;
    auto k = probe_kernel<M, N, K, AMN, BMN>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -2;
    k<<<1, 128, smem>>>(A, B, D, status);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

struct Cfg { int M, N, K, amn, bmn; };
static const Cfg kCfgs[] = {
    {128, 16, 128, 0, 0}, {128, 32, 128, 0, 0}, {128, 64, 128, 0, 0}, {128, 128, 128, 0, 0}, {128, 256, 64, 0, 0},
    {128, 64, 64, 1, 0},  {128, 64, 128, 0, 1}, {128, 128, 64, 1, 1}, {64, 32, 128, 0, 0},   {64, 64, 64, 0, 0},
    {64, 16, 128, 0, 0},  {64, 64, 64, 1, 0},   {64, 128, 64, 0, 1},  {128, 32, 64, 0, 1},   {128, 256, 128, 1, 1},
};

extern "C" __attribute__((visibility("default"))) int probe_count() { return sizeof(kCfgs) / sizeof(kCfgs[0]); }

extern "C" __attribute__((visibility("default"))) int probe_shape(int i, int *out5) {
    if (i < 0 || i >= probe_count()) return -1;
    out5[0] = kCfgs[i].M; out5[1] = kCfgs[i].N; out5[2] = kCfgs[i].K; out5[3] = kCfgs[i].amn; out5[4] = kCfgs[i].bmn;
    return 0;
}

extern "C" __attribute__((visibility("default"))) int probe_run(int i, const float *A, const float *B, float *D,
                                                                int *status) {
    switch (i) {
        case 0: return run<128, 16, 128, false, false>(A, B, D, status);
        case 1: return run<128, 32, 128, false, false>(A, B, D, status);
        case 2: return run<128, 64, 128, false, false>(A, B, D, status);
        case 3: return run<128, 128, 128, false, false>(A, B, D, status);
        case 4: return run<128, 256, 64, false, false>(A, B, D, status);
        case 5: return run<128, 64, 64, true, false>(A, B, D, status);
        case 6: return run<128, 64, 128, false, true>(A, B, D, status);
        case 7: return run<128, 128, 64, true, true>(A, B, D, status);
        case 8: return run<64, 32, 128, false, false>(A, B, D, status);
        case 9: return run<64, 64, 64, false, false>(A, B, D, status);
        case 10: return run<64, 16, 128, false, false>(A, B, D, status);
        case 11: return run<64, 64, 64, true, false>(A, B, D, status);
        case 12: return run<64, 128, 64, false, true>(A, B, D, status);
        case 13: return run<128, 32, 64, false, true>(A, B, D, status);
        case 14: return run<128, 256, 128, true, true>(A, B, D, status);
        default: return -1;
    }
}

// A bounded wait that is never satisfied: nothing arrives on the barrier, so mbar_wait must
// give up after `cycles` SM clocks and the kernel records that in *status (1) and returns.
__global__ void timeout_kernel(int *status, long long cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0, cycles);
    if (threadIdx.x == 0) *status = ok ? 0 : 1;
}

extern "C" __attribute__((visibility("default"))) int probe_timeout(int *status, long long cycles) {
    timeout_kernel<<<1, 32>>>(status, cycles);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
