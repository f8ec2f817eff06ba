// BF16 projection GEMM on tcgen05: C[M x N] = A[M x K] . W[N x K]^T (torch Linear layout,
// Glm5NextKdaWeights: every projection is a [out, in] BF16 matrix), FP32 accumulation in
// TMEM, BF16 or FP32 output with a row stride (so q/k/v projections can write straight into
// the packed q|k|v rows of Glm5NextKdaWorkspace `qkv_proj`).
//
// Persistent, warp-specialised kernel (192 threads, one CTA per SM):
//   warp 0      TMA producer: 128 x 64 A tiles and BN x 64 W tiles, 128-byte swizzle, a ring of
//               4 to 10 shared-memory stages by tile width (full / empty mbarriers). No multicast.
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M = 128, N = BN, K = 16) into
//               one of two accumulators and commits to the stage's `empty` barrier.
//   warps 2..5  epilogue: tcgen05.ld the accumulator rows (TMEM lanes = rows), convert, store;
//               then release the accumulator so the MMAs of the next tile overlap this one.
// Every wait is bounded; a wait that gives up sets a shared abort flag so all roles leave
// their loops, records KDA_ERR_TIMEOUT in the device status word, and TMEM is freed.
#include <algorithm>

#include "common.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace kda {
namespace {

using namespace umma;

constexpr int BM = 128, BK = 64, kGemmThreads = 192;
constexpr long long kGemmWait = 4000000000LL;

template <int BN>
struct GemmCfg {
    static constexpr int A_STAGE = BM * BK * 2;
    static constexpr int B_STAGE = BN * BK * 2;
    static constexpr int STAGE = A_STAGE + B_STAGE;
    // as many stages as about 200 KB holds: narrow tiles (the small-M form, few CTAs) then keep
    // as many bytes in flight per SM as wide ones
    static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : (BN >= 64 ? 8 : 10));
    static constexpr int OFF_BARS = STAGES * STAGE;
    static_assert(OFF_BARS + 256 + 1024 <= 232448, "shared memory");
    static constexpr int bytes = OFF_BARS + 256 + 1024;
    static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;  // two accumulators
};

__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *tm, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Wait for a phase, giving up when another role aborted or the clock budget ran out.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort, int *status) {
    const uint32_t addr = smem_u32(bar);
    const long long t0 = clock64();
    while (!mbar_try_wait(addr, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > kGemmWait) {
            *abort = 1;
            atomicExch(status, KDA_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Up to six products in one launch, each its own A (M rows) and W (the shared N rows), its own
// output: a segment's tiles follow the previous segment's in the tile order. trans: element
// (m, n) of a product is stored at C[n ldc + m] (the small-M form below computes C^T).
constexpr int kMaxGemmSegs = 6;
struct GemmSeg {
    void *C;
    int ldc, M, out_f32, vec;
};
struct GemmArgs {
    CUtensorMap tmA[kMaxGemmSegs];
    CUtensorMap tmW[kMaxGemmSegs];
    GemmSeg seg[kMaxGemmSegs];
    int nseg, N, K, trans;
    // split-K (small-M form): each tile's K loop in ksplit consecutive parts, one work unit each;
    // a unit stores its FP32 sums to part[unit][BN][BM] and splitk_reduce_kernel adds the parts
    int ksplit;
    float *part;
};

// First k-block of a tile's K loop. In the small-M form every tile reads the same few input rows,
// so tiles that started together would read the same k-block of them from the same L2 lines at
// the same time; each tile starts its (wrapping) K loop at its own k-block instead.
__device__ __forceinline__ int k_start(const GemmArgs &g, int tile, int nk) {
    return g.trans && g.ksplit <= 1 ? static_cast<int>((static_cast<unsigned>(tile) * 37u) % static_cast<unsigned>(nk))
                                    : 0;
}

// The k-blocks [kb0, kb1) of work unit u (tile u / ks, part u % ks).
__device__ __forceinline__ void unit_k(int u, int ks, int nk, int &kb0, int &kb1) {
    const int kp = u % ks;
    kb0 = kp * nk / ks;
    kb1 = (kp + 1) * nk / ks;
}

// The segment and the tile origin of tile `t`.
template <int BN>
__device__ __forceinline__ int gemm_tile(const GemmArgs &g, int tiles_n, int t, int &m0, int &n0) {
    int s = 0;
    for (;;) {
        const int nt = (g.seg[s].M + BM - 1) / BM * tiles_n;
        if (t < nt || s + 1 == g.nseg) break;
        t -= nt;
        ++s;
    }
    m0 = (t / tiles_n) * BM;
    n0 = (t % tiles_n) * BN;
    return s;
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ GemmArgs g, int *__restrict__ status) {
    const int N = g.N, K = g.K;
    using G = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + G::OFF_BARS);
    uint64_t *empty = full + G::STAGES;
    uint64_t *accf = empty + G::STAGES;
    uint64_t *acce = accf + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acce + 2);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles_n = (N + BN - 1) / BN;
    int ntiles = 0;
    for (int i = 0; i < g.nseg; ++i) ntiles += (g.seg[i].M + BM - 1) / BM * tiles_n;
    const int nk = K / BK;
    const int ksp = g.ksplit > 1 ? g.ksplit : 1;
    const int nunits = ntiles * ksp;

    if (tid == 0) {
        for (int s = 0; s < G::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 4); }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, G::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {  // ---- TMA producer
            int it = 0;
            for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
                const int tile = u / ksp;
                int m0, n0, kb0, kb1;
                const int sg = gemm_tile<BN>(g, tiles_n, tile, m0, n0);
                unit_k(u, ksp, nk, kb0, kb1);
                const int k0 = k_start(g, tile, nk);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % G::STAGES;
                    const uint32_t ph = (it / G::STAGES) & 1;
                    if (!wait_or_abort(&empty[s], ph ^ 1, abort, status)) goto done;
                    uint8_t *sa = sm + s * G::STAGE;
                    const int kx = (k0 + kb < nk ? k0 + kb : k0 + kb - nk) * BK;
                    mbar_expect_tx(&full[s], G::STAGE);
                    tma_load_2d(sa, &g.tmA[sg], kx, m0, &full[s]);
                    tma_load_2d(sa + G::A_STAGE, &g.tmW[sg], kx, n0, &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ---- MMA issuer
            constexpr uint32_t id = idesc_bf16(BM, BN, false, false);
            int it = 0, tc = 0;
            for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++tc) {
                int kb0, kb1;
                unit_k(u, ksp, nk, kb0, kb1);
                const int acc = tc & 1;
                const uint32_t aph = (tc >> 1) & 1;
                if (!wait_or_abort(&acce[acc], aph ^ 1, abort, status)) goto done;
                tc_fence_after();
                const uint32_t dcol = tmem + acc * BN;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % G::STAGES;
                    const uint32_t ph = (it / G::STAGES) & 1;
                    if (!wait_or_abort(&full[s], ph, abort, status)) goto done;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sm + s * G::STAGE), b0 = a0 + G::A_STAGE;
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks)
                        mma_bf16(dcol, kmaj_desc(a0, BM, 0, ks), kmaj_desc(b0, BN, 0, ks), id,
                                 (kb > kb0 || ks > 0) ? 1u : 0u);
                    mma_commit(&empty[s]);
                }
                mma_commit(&accf[acc]);
            }
        }
    } else {  // ---- epilogue warps 2..5: TMEM lanes 32 (warp % 4) .. + 31
        const int quad = warp & 3;
        int tc = 0;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++tc) {
            const int tile = u / ksp;
            int m0, n0;
            const GemmSeg &sgm = g.seg[gemm_tile<BN>(g, tiles_n, tile, m0, n0)];
            void *const Cout = sgm.C;
            const int ldc = sgm.ldc, M = sgm.M, out_f32 = sgm.out_f32, vec = sgm.vec;
            const int acc = tc & 1;
            const uint32_t aph = (tc >> 1) & 1;
            if (!wait_or_abort(&accf[acc], aph, abort, status)) goto done;
            tc_fence_after();
            const int row = m0 + 32 * quad + lane;
            const uint32_t src = tmem_lane_base(tmem, warp) + acc * BN;
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                float x[16];
                tmem_ld16(src + c, x);
                tmem_ld_wait();
                if (ksp > 1) {  // this unit's FP32 sums: part[u][column][row], the warp's 32 rows contiguous
                    float *pu = g.part + static_cast<size_t>(u) * BN * BM + 32 * quad + lane;
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        if (n0 + c + v >= N) break;
                        pu[static_cast<size_t>(c + v) * BM] = x[v];
                    }
                } else if (g.trans) {  // C^T: for each column, the warp's 32 rows are 32 consecutive elements
                    if (row < M) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) {
                            if (n0 + c + u >= N) break;
                            const size_t o = static_cast<size_t>(n0 + c + u) * ldc + row;
                            if (out_f32) static_cast<float *>(Cout)[o] = x[u];
                            else static_cast<__nv_bfloat16 *>(Cout)[o] = __float2bfloat16_rn(x[u]);
                        }
                    }
                } else if (row < M && n0 + c < N && !(vec && n0 + c + 16 <= N)) {
                    // ragged column tail or unaligned rows: element stores
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        if (n0 + c + u >= N) break;
                        if (out_f32) static_cast<float *>(Cout)[static_cast<size_t>(row) * ldc + n0 + c + u] = x[u];
                        else static_cast<__nv_bfloat16 *>(Cout)[static_cast<size_t>(row) * ldc + n0 + c + u] = __float2bfloat16_rn(x[u]);
                    }
                } else if (row < M && n0 + c < N) {
                    if (out_f32) {
                        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(Cout) + static_cast<size_t>(row) * ldc + n0 + c);
#pragma unroll
                        for (int u = 0; u < 4; ++u) dst[u] = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
                    } else {
                        uint32_t w[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const __nv_bfloat162 p = __floats2bfloat162_rn(x[2 * u], x[2 * u + 1]);
                            w[u] = *reinterpret_cast<const uint32_t *>(&p);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(Cout) + static_cast<size_t>(row) * ldc + n0 + c);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[acc]);
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, G::TMEM_COLS);
}

// The parts of a split-K launch added in part order (a fixed order: the same bits on every
// call with the same split), each element stored as the unsplit epilogue stores it. Block
// (tile, group of 8 columns), one thread per 4 consecutive rows of a column (16-byte reads).
template <int BN>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const __grid_constant__ GemmArgs g) {
    const int tile = blockIdx.x, N = g.N, ksp = g.ksplit;
    const int tiles_n = (N + BN - 1) / BN;
    int m0, n0;
    const GemmSeg &sg = g.seg[gemm_tile<BN>(g, tiles_n, tile, m0, n0)];
    const int c = 8 * blockIdx.y + threadIdx.x / (BM / 4), r = 4 * (threadIdx.x % (BM / 4));
    if (n0 + c >= N || m0 + r >= sg.M) return;
    const float *p = g.part + static_cast<size_t>(tile) * ksp * BN * BM + static_cast<size_t>(c) * BM + r;
    float4 t = *reinterpret_cast<const float4 *>(p);
    for (int kp = 1; kp < ksp; ++kp) {
        const float4 v = *reinterpret_cast<const float4 *>(p + static_cast<size_t>(kp) * BN * BM);
        t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
    }
    const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (m0 + r + j >= sg.M) break;
        const size_t o = g.trans ? static_cast<size_t>(n0 + c) * sg.ldc + m0 + r + j
                                 : static_cast<size_t>(m0 + r + j) * sg.ldc + n0 + c;
        if (sg.out_f32) static_cast<float *>(sg.C)[o] = tv[j];
        else static_cast<__nv_bfloat16 *>(sg.C)[o] = __float2bfloat16_rn(tv[j]);
    }
}

// ------------------------------------------------------------------ host side

// 2-D BF16 tensor map over `rows` x `cols` (row stride ld elements), box 64 (K) x box_rows.
int make_map(CUtensorMap *tm, const void *base, int rows, int cols, int ld, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return KDA_ERR_CUDA;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KDA_OK : KDA_ERR_INVALID_ARG;
}

int sm_count() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

template <int BN>
int launch_gemm(GemmArgs &g, cudaStream_t s) {
    using G = GemmCfg<BN>;
    static std::atomic<unsigned long long> attr_done{0};
    KDA_TRY(smem_opt_in(gemm_kernel<BN>, G::bytes, attr_done));
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    long long ntiles = 0;
    for (int i = 0; i < g.nseg; ++i) ntiles += static_cast<long long>((g.seg[i].M + BM - 1) / BM) * ((g.N + BN - 1) / BN);
    if (ntiles == 0) return KDA_OK;
    const int grid = static_cast<int>(std::min<long long>(ntiles * std::max(g.ksplit, 1), sm_count()));
    gemm_kernel<BN><<<grid, kGemmThreads, G::bytes, s>>>(g, status);
    return launch_status();
}

template <int BN>
int gemm_one(const uint16_t *A, int lda, const uint16_t *W, int ldw, void *Cout, int ldc, int M, int N, int K,
             int out_f32, cudaStream_t s) {
    GemmArgs g{};
    KDA_TRY(make_map(&g.tmA[0], A, M, K, lda, BM));
    KDA_TRY(make_map(&g.tmW[0], W, N, K, ldw, BN));
    // 16-element vector stores need 16-byte aligned rows
    g.seg[0] = GemmSeg{Cout, ldc, M, out_f32, aligned16(Cout) && (ldc % (out_f32 ? 4 : 8)) == 0};
    g.nseg = 1;
    g.N = N;
    g.K = K;
    g.trans = 0;
    return launch_gemm<BN>(g, s);
}

// Several products of one width N and depth K in one launch: their tiles follow one another in the
// tile order, so the launch fills the machine where each alone would leave SMs idle or a ragged
// last wave. Each tile runs exactly as it would in its own launch.
template <int BN>
int gemm_multi(const GemmProd *prods, int n, cudaStream_t s) {
    GemmArgs g{};
    for (int i = 0; i < n; ++i) {
        const GemmProd &p = prods[i];
        KDA_TRY(make_map(&g.tmA[i], p.A, p.M, p.K, p.lda, BM));
        KDA_TRY(make_map(&g.tmW[i], p.W, p.N, p.K, p.ldw, BN));
        g.seg[i] = GemmSeg{p.C, p.ldc, p.M, p.out_f32, aligned16(p.C) && (p.ldc % (p.out_f32 ? 4 : 8)) == 0};
    }
    g.nseg = n;
    g.N = prods[0].N;
    g.K = prods[0].K;
    g.trans = 0;
    g.ksplit = 1;
    return launch_gemm<BN>(g, s);
}

// The small-M form: y_s[m][n] = x_s[m] . W_s[n] for a few rows m of each segment's input, as
// the transposed product W_s . x_s^T, so that the 128-row tiles run over the weights' output
// rows (every weight is read once, by many CTAs) and the few input rows are the N side.
// A CTA streams only so many bytes per second, so a launch with at most one tile per two SMs
// splits each tile's K loop over several CTAs, as many as one wave holds (at least 4 k-blocks
// each, at most 8 parts, as many as the part buffer holds), and adds the parts in a second, short
// launch. Launches with more tiles gain nothing from it: every tile re-reads all input rows, and
// that L2 traffic, not the CTA count, sets their time.
template <int BN>
int gemm_small_m(const GemmTSeg *segs, int nseg, int rows, int K, float *part, size_t part_bytes, cudaStream_t s) {
    GemmArgs g{};
    long long ntiles = 0;
    for (int i = 0; i < nseg; ++i) {
        const GemmTSeg &t = segs[i];
        KDA_TRY(make_map(&g.tmA[i], t.W, t.N, K, t.ldw, BM));
        KDA_TRY(make_map(&g.tmW[i], t.x, rows, K, t.ldx, BN));
        g.seg[i] = GemmSeg{t.y, t.ldy, t.N, t.out_f32, 0};
        ntiles += static_cast<long long>((t.N + BM - 1) / BM) * ((rows + BN - 1) / BN);
    }
    g.nseg = nseg;
    g.N = rows;
    g.K = K;
    g.trans = 1;
    g.ksplit = 1;
    const long long sms = sm_count();
    if (part && ntiles > 0 && 2 * ntiles <= sms) {
        long long ksp = std::min<long long>({sms / ntiles, 8, K / BK / 4});
        ksp = std::min<long long>(ksp, static_cast<long long>(part_bytes / (static_cast<size_t>(ntiles) * BN * BM * 4)));
        if (ksp >= 2) {
            g.ksplit = static_cast<int>(ksp);
            g.part = part;
        }
    }
    KDA_TRY(launch_gemm<BN>(g, s));
    if (g.ksplit == 1 || ntiles == 0) return KDA_OK;
    splitk_reduce_kernel<BN><<<dim3(static_cast<unsigned>(ntiles), BN / 8), 256, 0, s>>>(g);
    return launch_status();
}

}  // namespace

int gemm_bf16_multi(const GemmProd *prods, int n, cudaStream_t s) {
    if (n < 1 || n > kMaxGemmSegs) return KDA_ERR_INVALID_ARG;
    for (int i = 1; i < n; ++i)
        if (prods[i].N != prods[0].N || prods[i].K != prods[0].K) return KDA_ERR_INVALID_ARG;
    const int N = prods[0].N;
    if (N > 128) return gemm_multi<256>(prods, n, s);
    if (N > 64) return gemm_multi<128>(prods, n, s);
    if (N > 32) return gemm_multi<64>(prods, n, s);
    return gemm_multi<32>(prods, n, s);
}

int gemm_bf16(const uint16_t *A, int lda, const uint16_t *W, int ldw, void *Cout, int ldc, int M, int N, int K,
              int out_f32, cudaStream_t s) {
    if (N > 128) return gemm_one<256>(A, lda, W, ldw, Cout, ldc, M, N, K, out_f32, s);
    if (N > 64) return gemm_one<128>(A, lda, W, ldw, Cout, ldc, M, N, K, out_f32, s);
    if (N > 32) return gemm_one<64>(A, lda, W, ldw, Cout, ldc, M, N, K, out_f32, s);
    return gemm_one<32>(A, lda, W, ldw, Cout, ldc, M, N, K, out_f32, s);
}

size_t small_m_part_bytes(int rows) {
    const int bn = rows > 128 ? 256 : (rows > 64 ? 128 : (rows > 32 ? 64 : 32));
    return static_cast<size_t>(sm_count()) * bn * BM * 4;  // one wave of units
}

int gemm_bf16_small_m(const GemmTSeg *segs, int nseg, int rows, int K, cudaStream_t s, float *part,
                      size_t part_bytes) {
    if (nseg < 1 || nseg > kMaxGemmSegs || rows <= 0) return KDA_ERR_INVALID_ARG;
    if (rows > 128) return gemm_small_m<256>(segs, nseg, rows, K, part, part_bytes, s);
    if (rows > 64) return gemm_small_m<128>(segs, nseg, rows, K, part, part_bytes, s);
    if (rows > 32) return gemm_small_m<64>(segs, nseg, rows, K, part, part_bytes, s);
    return gemm_small_m<32>(segs, nseg, rows, K, part, part_bytes, s);
}

// ------------------------------------------------------------------ small-M matrix-vector products
//
// y[m][n] = sum_k x[m][k] W[n][k] for the M rows of a decode or verify step, W read once for
// (up to) kGemvRows rows at a time. The warp that owns column n gives lane l the k in
// {256 j + 8 l + e} (j, then e = 0..7 ascending, FP32 fma), then sums the 32 lanes by a fixed
// butterfly: every output's arithmetic depends on K and its own row only, never on M, so a
// row's result is the same bits in a call of one row and in a call of many (the identity the
// K-token verify needs). x rows are staged in shared memory; W streams with 16-byte loads.
// Segments may bring their own input rows (two products of one step that read different rows
// share a launch); their rows are staged side by side.
constexpr int kGemvRows = 8, kGemvWarps = 8, kGemvMaxK = 8192;

namespace {
template <int MB>
__global__ void __launch_bounds__(32 * kGemvWarps)
gemv_kernel(const uint16_t *__restrict__ x, int ldx, const GemvSegs segs, int M, int K) {
    // weight loads in flight per lane (U x 16 bytes): a whole 4096-wide row for one-row calls
    constexpr int U = MB == 1 ? 16 : 8;
    extern __shared__ __align__(16) uint16_t sx[];  // [set][mb][K]: this group's rows of each input
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m0 = blockIdx.y * MB;
    const int mb = min(MB, M - m0);
    const int nx = segs.s[0].x ? segs.count : 1;  // input sets: one per segment, or the call's x
    for (int q = 0; q < nx; ++q) {
        const uint16_t *xs = segs.s[0].x ? segs.s[q].x : x;
        for (int e = tid; e < mb * (K / 8); e += 32 * kGemvWarps) {
            const int r = e / (K / 8), c = 8 * (e % (K / 8));
            *reinterpret_cast<uint4 *>(sx + (q * mb + r) * K + c) =
                *reinterpret_cast<const uint4 *>(xs + static_cast<size_t>(m0 + r) * ldx + c);
        }
    }
    __syncthreads();
    for (int col = blockIdx.x * kGemvWarps + warp; col < segs.total; col += gridDim.x * kGemvWarps) {
        int si = 0, n = col;
        while (si + 1 < segs.count && n >= segs.s[si].N) { n -= segs.s[si].N; ++si; }
        const GemvSeg &sg = segs.s[si];
        const uint16_t *wr = sg.W + static_cast<size_t>(n) * sg.ldw;
        const uint16_t *sxs = sx + (nx > 1 ? si * mb * K : 0);  // this segment's input rows
        float acc[MB];
#pragma unroll
        for (int r = 0; r < MB; ++r) acc[r] = 0.f;
        // lane-strided K steps in ascending order (k = 8 lane + 256 j); the loads of U steps are
        // issued together, the products then accumulate in the same order as one step at a time
        for (int kb = 8 * lane; kb < K; kb += 256 * U) {
            uint4 wv[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                wv[u] = kb + 256 * u < K ? __ldcs(reinterpret_cast<const uint4 *>(wr + kb + 256 * u))
                                         : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = kb + 256 * u;
                if (k >= K) break;
                float w8[8];
                w8[0] = __uint_as_float(wv[u].x << 16); w8[1] = __uint_as_float(wv[u].x & 0xFFFF0000u);
                w8[2] = __uint_as_float(wv[u].y << 16); w8[3] = __uint_as_float(wv[u].y & 0xFFFF0000u);
                w8[4] = __uint_as_float(wv[u].z << 16); w8[5] = __uint_as_float(wv[u].z & 0xFFFF0000u);
                w8[6] = __uint_as_float(wv[u].w << 16); w8[7] = __uint_as_float(wv[u].w & 0xFFFF0000u);
#pragma unroll
                for (int r = 0; r < MB; ++r) {
                    if (r < mb) {
                        const uint4 xv = *reinterpret_cast<const uint4 *>(sxs + r * K + k);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.x << 16), w8[0], acc[r]);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.x & 0xFFFF0000u), w8[1], acc[r]);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.y << 16), w8[2], acc[r]);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.y & 0xFFFF0000u), w8[3], acc[r]);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.z << 16), w8[4], acc[r]);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.z & 0xFFFF0000u), w8[5], acc[r]);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.w << 16), w8[6], acc[r]);
                        acc[r] = __fmaf_rn(__uint_as_float(xv.w & 0xFFFF0000u), w8[7], acc[r]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < MB; ++r) {
            if (r < mb) {  // warp-uniform
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[r] = __fadd_rn(acc[r], __shfl_xor_sync(0xffffffffu, acc[r], o));
            }
        }
        if (lane < mb) {
            float v = acc[0];
#pragma unroll
            for (int r = 1; r < MB; ++r)
                if (lane == r) v = acc[r];
            const size_t o = static_cast<size_t>(m0 + lane) * sg.ldy + n;
            if (sg.out_f32) static_cast<float *>(sg.y)[o] = v;
            else static_cast<uint16_t *>(sg.y)[o] = f32_to_bf16(v);
        }
    }
}

}  // namespace

int gemv_segs(const uint16_t *x, int ldx, const GemvSegs &segs, int M, int K, cudaStream_t s) {
    const int nx = segs.s[0].x ? segs.count : 1;
    const int bytes = nx * std::min(M, kGemvRows) * K * 2;  // the rows of one group, per input
    if (bytes > (M == 1 ? 1 : kGemvRows) * kGemvMaxK * 2) {  // the inputs do not fit side by side: one launch each
        for (int i = 0; i < segs.count; ++i) {
            GemvSegs one{};
            one.s[0] = segs.s[i];
            one.s[0].x = nullptr;
            one.count = 1;
            one.total = segs.s[i].N;
            KDA_TRY(gemv_segs(segs.s[0].x ? segs.s[i].x : x, ldx, one, M, K, s));
        }
        return KDA_OK;
    }
    static std::atomic<unsigned long long> attr_done{0}, attr1_done{0};  // opted in once, at the largest K
    const int col_blocks = (segs.total + kGemvWarps - 1) / kGemvWarps;
    const int grid_x = std::min(col_blocks, 4 * sm_count());
    if (M == 1) {  // one row: the same per-output arithmetic without the other rows' registers
        KDA_TRY(smem_opt_in(gemv_kernel<1>, kGemvMaxK * 2, attr1_done));
        gemv_kernel<1><<<dim3(grid_x, 1), 32 * kGemvWarps, bytes, s>>>(x, ldx, segs, M, K);
        return launch_status();
    }
    KDA_TRY(smem_opt_in(gemv_kernel<kGemvRows>, kGemvRows * kGemvMaxK * 2, attr_done));
    gemv_kernel<kGemvRows><<<dim3(grid_x, (M + kGemvRows - 1) / kGemvRows), 32 * kGemvWarps, bytes, s>>>(x, ldx, segs,
                                                                                                      M, K);
    return launch_status();
}

int gemv_bf16(const uint16_t *x, int ldx, const uint16_t *W, int ldw, void *y, int ldy, int M, int N, int K,
              int out_f32, cudaStream_t s) {
    GemvSegs segs{};
    segs.s[0] = GemvSeg{W, y, N, ldw, ldy, out_f32};
    segs.count = 1;
    segs.total = N;
    return gemv_segs(x, ldx, segs, M, K, s);
}

}  // namespace kda

extern "C" int kda_gemm_bf16(const kda_bf16 *A, int lda, const kda_bf16 *W, int ldw, void *C, int ldc, int M, int N,
                             int K, int out_f32, void *stream) {
    if (!A || !W || !C || M < 0 || N < 0 || K < 0) return KDA_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return KDA_OK;
    if (K == 0 || K % 64 != 0) return KDA_ERR_UNSUPPORTED;
    if (lda < K || ldw < K || ldc < N) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(A) || !kda::aligned16(W) || (lda % 8) || (ldw % 8)) return KDA_ERR_MISALIGNED;
    return kda::gemm_bf16(A, lda, W, ldw, C, ldc, M, N, K, out_f32, static_cast<cudaStream_t>(stream));
}

extern "C" int kda_gemv_bf16(const kda_bf16 *x, int ldx, const kda_bf16 *W, int ldw, void *y, int ldy, int M, int N,
                             int K, int out_f32, void *stream) {
    if (!x || !W || !y || M < 0 || N < 0 || K < 0) return KDA_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return KDA_OK;
    if (K == 0 || K % 8 != 0 || K > kda::kGemvMaxK) return KDA_ERR_UNSUPPORTED;
    if (ldx < K || ldw < K || ldy < N) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(x) || !kda::aligned16(W) || (ldx % 8) || (ldw % 8)) return KDA_ERR_MISALIGNED;
    return kda::gemv_bf16(x, ldx, W, ldw, y, ldy, M, N, K, out_f32, static_cast<cudaStream_t>(stream));
}
