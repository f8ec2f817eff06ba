// Chunked KDA prefill with tcgen05 tensor cores (Glm5NextKdaLayer `prefill`, `kda_chunk_*`;
// Glm5NextKdaWorkspace q_f32/k_f32/v_f32/gate/beta -> core; Glm5NextLayer
// `prefill_gdn_full_batched`: B equal-length streams, a device array of state pointers).
//
// Per chunk of C = 64 tokens, Gamma the in-chunk inclusive cumulative log-decay per key
// channel (Gamma_C its last row), A = e^Gamma:
//   L[i][j] = beta_i sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc}  (i > j);  T = (I + L)^-1
//   M[i][j] =        sum_c q_ic k_jc e^{Gamma_ic - Gamma_jc}  (i >= j)
//   Tb = T diag(beta);  M' = M Tb
//   R = V - (K o A) S0;  U = Tb R;  O = scale ((Q o A) S0 + M' R)
//   S = diag(A_C) S0 + (K o e^{Gamma_C - Gamma})^T U
// which is the gated delta rule unrolled over the chunk (U = (I + L)^-1 diag(beta)(V - (K o A) S0)
// and M U = M' R).
//
// Two kernels:
//  intra (one CTA per chunk-head, all in parallel, CUDA cores): L, M, T, Tb, M'. The decay
//    factors come from a = e^g by running products inside 16-token blocks, and across blocks
//    as products of per-block factors, so every factor is <= 1 and nothing overflows. It writes
//    [Tb; M'] (128 x 64) as a BF16 hi/lo pair of 128-byte-swizzled K-major operand tiles.
//  state (one CTA per (stream, head, value slice), chunks in order): builds [K o A; Q o A] and
//    K o e^{Gamma_C - Gamma} from q, k, g, bulk-copies the [Tb; M'] tile, and runs three
//    tcgen05 MMAs per chunk, each in split-BF16 precision (x = hi + lo; hi.hi + hi.lo + lo.hi):
//      D1 = [K o A; Q o A] . S0        (M = 128, N = DVS, K = D)
//      D2 = [Tb; M'] . R               (M = 128, N = DVS, K = 64)  with R = V - D1[0:64]
//      D3 = (K o e^{Gamma_C-Gamma})^T . U  (M = D,  N = DVS, K = 64)  with U = D2[0:64]
//    O = scale (D1[64:128] + D2[64:128]);  S = A_C o S0 + D3 (FP32 master copy in registers).
// Rows >= T of the last chunk are loaded as zeros (k = q = v = 0, g = 0, beta = 0): the pad
// guard. They add nothing to L, M, R, U or the state, and their outputs are not written.
#include "common.cuh"
#include "umma.cuh"

namespace kda {
namespace {

using namespace umma;

constexpr int C = kChunk;          // 64
constexpr int kThreads = 256;
constexpr int kTileBytes = 16384;  // one 128 x 64 BF16 K-major tile
constexpr int kA2Bytes = 2 * kTileBytes;
constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at 1.9 GHz

// ================================================================ phase 1: intra-chunk

template <int D>
struct Intra {
    static constexpr int P = D + 8;   // fp32 row stride of [C][D] tiles (bank-spread, 16-B aligned)
    static constexpr int PC = C + 1;  // row stride of [C][C] tiles
    static constexpr int NZ = 48;     // rows of the block-local backward factors (blocks 0..2)
    static constexpr size_t floats = 3 * C * P + NZ * P + 3 * C * PC + 3 * D + C + 3 * 256;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
intra_kernel(const float *__restrict__ k, const float *__restrict__ q, const float *__restrict__ gate,
             const float *__restrict__ beta, uint8_t *__restrict__ scratch, int T, int T_pad, int H) {
    using I = Intra<D>;
    constexpr int P = I::P, PC = I::PC;
    extern __shared__ float smem[];
    float *sK = smem;              // k, then X (rows 16..63): k_i prod_{s=16a}^{i} a_s
    float *sQ = sK + C * P;        // q, then Y (rows 16..63): q_i prod_{s=16a}^{i} a_s
    float *sA = sQ + C * P;        // a = e^g
    float *sZ = sA + C * P;        // Z (rows 0..47): k_j prod_{s=j+1}^{16b+15} a_s
    float *sL = sZ + I::NZ * P;    // L' (unscaled), then M'
    float *sM = sL + C * PC;       // M
    float *sT = sM + C * PC;       // T, then Tb
    float *sSig = sT + C * PC;     // [3][D]: block-1 product, block-2 product, both
    float *sB = sSig + 3 * D;      // beta
    float *sTmp = sB + C;          // [3][256]

    const int tid = threadIdx.x;
    const int ch = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int n = min(C, T - ch * C);
    const size_t row0 = static_cast<size_t>(b) * T_pad + static_cast<size_t>(ch) * C;
    const size_t rs = static_cast<size_t>(H) * D;

    // ---- load k, q and a = e^g (pad guard: rows >= n are k = q = 0, a = 1)
    for (int e = tid; e < C * D / 4; e += kThreads) {
        const int i = e / (D / 4), c = 4 * (e % (D / 4));
        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), qv = kv, av = make_float4(1.f, 1.f, 1.f, 1.f);
        if (i < n) {
            const size_t off = (row0 + i) * rs + static_cast<size_t>(h) * D + c;
            kv = *reinterpret_cast<const float4 *>(k + off);
            qv = *reinterpret_cast<const float4 *>(q + off);
            const float4 g = *reinterpret_cast<const float4 *>(gate + off);
            av = make_float4(expf(g.x), expf(g.y), expf(g.z), expf(g.w));
        }
        *reinterpret_cast<float4 *>(sK + i * P + c) = kv;
        *reinterpret_cast<float4 *>(sQ + i * P + c) = qv;
        *reinterpret_cast<float4 *>(sA + i * P + c) = av;
    }
    if (tid < C) sB[tid] = tid < n ? beta[(row0 + tid) * H + h] : 0.f;
    __syncthreads();

    // ---- diagonal 16x16 blocks: thread (block a, j pair, channel group) walks i upward with
    //      the running product G = k_j prod_{s=j+1}^{i} a_s; the 8 channel groups of one j
    //      are 8 adjacent lanes and reduce with shuffles.
    {
        constexpr int CPT = D / 8;
        const int a = tid >> 6, jp = (tid >> 3) & 7, cg = tid & 7;
        const unsigned gmask = 0xFFu << (tid & 24);
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const int j = 16 * a + (pass == 0 ? jp : 15 - jp);
            float G[CPT];
#pragma unroll
            for (int cc = 0; cc < CPT; ++cc) G[cc] = sK[j * P + cg + 8 * cc];
#pragma unroll 1
            for (int i = j; i < 16 * a + 16; ++i) {
                float ls = 0.f, ms = 0.f;
#pragma unroll
                for (int cc = 0; cc < CPT; ++cc) {
                    const int c = cg + 8 * cc;
                    if (i > j) G[cc] *= sA[i * P + c];
                    ls = fmaf(sK[i * P + c], G[cc], ls);
                    ms = fmaf(sQ[i * P + c], G[cc], ms);
                }
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    ls += __shfl_xor_sync(gmask, ls, o);
                    ms += __shfl_xor_sync(gmask, ms, o);
                }
                if (cg == 0) {
                    sL[i * PC + j] = ls;
                    sM[i * PC + j] = ms;
                }
            }
        }
    }
    __syncthreads();

    // ---- block-local factors, one thread per channel: Z (backward, blocks 0..2), then X, Y
    //      (forward, blocks 1..3, in place over k and q) and the per-block decay products.
    if (tid < D) {
        const int c = tid;
#pragma unroll 1
        for (int bb = 0; bb < 3; ++bb) {
            float f = 1.f;
            for (int j = 16 * bb + 15; j >= 16 * bb; --j) {
                sZ[j * P + c] = sK[j * P + c] * f;
                f *= sA[j * P + c];
            }
        }
        float F[4];
#pragma unroll 1
        for (int aa = 0; aa < 4; ++aa) {
            float f = 1.f;
            for (int i = 16 * aa; i < 16 * aa + 16; ++i) {
                f *= sA[i * P + c];
                if (aa > 0) {
                    sK[i * P + c] *= f;
                    sQ[i * P + c] *= f;
                }
            }
            F[aa] = f;
        }
        sSig[c] = F[1];
        sSig[D + c] = F[2];
        sSig[2 * D + c] = F[1] * F[2];
    }
    __syncthreads();

    // ---- off-diagonal blocks (a > b): L'[i][j] = sum_c X_ic sigma_ab,c Z_jc (same with Y for M),
    //      sigma_ab = the decay of the whole blocks strictly between b and a (1 if adjacent).
    if (tid < 96) {
        const int p = tid >> 4;
        const int pa[6] = {1, 2, 2, 3, 3, 3}, pb[6] = {0, 0, 1, 0, 1, 2};
        const int a = pa[p], bb = pb[p];
        const int sig = (a == 2 && bb == 0) ? 0 : (a == 3 && bb == 1) ? 1 : (a == 3 && bb == 0) ? 2 : -1;
        const int i0 = 16 * a + 4 * ((tid & 15) >> 2), j0 = 16 * bb + 4 * (tid & 3);
        float l[4][4], m[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s = 0; s < 4; ++s) { l[r][s] = 0.f; m[r][s] = 0.f; }
#pragma unroll 2
        for (int c = 0; c < D; ++c) {
            const float sg = sig >= 0 ? sSig[sig * D + c] : 1.f;
            float z[4], x[4], y[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) z[s] = sZ[(j0 + s) * P + c] * sg;
#pragma unroll
            for (int r = 0; r < 4; ++r) { x[r] = sK[(i0 + r) * P + c]; y[r] = sQ[(i0 + r) * P + c]; }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    l[r][s] = fmaf(x[r], z[s], l[r][s]);
                    m[r][s] = fmaf(y[r], z[s], m[r][s]);
                }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                sL[(i0 + r) * PC + j0 + s] = l[r][s];
                sM[(i0 + r) * PC + j0 + s] = m[r][s];
            }
    }
    __syncthreads();

    // ---- L = diag(beta) L' (strict lower). T = (I + L)^-1: 16x16 diagonal blocks by
    //      substitution, then off-diagonal blocks T_ab = -T_aa sum_{b<=c<a} L_ac T_cb.
    for (int e = tid; e < C * C; e += kThreads) {
        const int i = e / C, j = e % C;
        if (i > j) sL[i * PC + j] *= sB[i];
    }
    __syncthreads();
    if (tid < 64) {
        const int a = tid / 16, j = tid % 16, base = 16 * a;
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float val = (i == j) ? 1.f : 0.f;
            if (i > j) {
                float acc = 0.f;
#pragma unroll
                for (int m2 = 0; m2 < 16; ++m2)
                    if (m2 >= j && m2 < i) acc = fmaf(sL[(base + i) * PC + base + m2], t[m2], acc);
                val = -acc;
            }
            t[i] = val;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) sT[(base + i) * PC + base + j] = t[i];
    }
    __syncthreads();
#pragma unroll 1
    for (int dist = 1; dist < 4; ++dist) {
        const int npairs = 4 - dist;
        for (int e = tid; e < npairs * 256; e += kThreads) {
            const int pr = e / 256, i = (e % 256) / 16, j = e % 16;
            const int bb = pr, aa = pr + dist;
            float acc = 0.f;
            for (int cb = bb; cb < aa; ++cb)
#pragma unroll
                for (int m2 = 0; m2 < 16; ++m2)
                    acc = fmaf(sL[(16 * aa + i) * PC + 16 * cb + m2], sT[(16 * cb + m2) * PC + 16 * bb + j], acc);
            sTmp[pr * 256 + i * 16 + j] = acc;
        }
        __syncthreads();
        for (int e = tid; e < npairs * 256; e += kThreads) {
            const int pr = e / 256, i = (e % 256) / 16, j = e % 16;
            const int bb = pr, aa = pr + dist;
            float acc = 0.f;
#pragma unroll
            for (int m2 = 0; m2 < 16; ++m2)
                acc = fmaf(sT[(16 * aa + i) * PC + 16 * aa + m2], sTmp[pr * 256 + m2 * 16 + j], acc);
            sT[(16 * aa + i) * PC + 16 * bb + j] = -acc;
        }
        __syncthreads();
    }
    // ---- Tb = T diag(beta) (lower incl. diagonal), then M' = M Tb (lower triangular) into sL
    for (int e = tid; e < C * C; e += kThreads) {
        const int i = e / C, j = e % C;
        if (j <= i) sT[i * PC + j] *= sB[j];
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kThreads) {
        const int i = e / C, l = e % C;
        float acc = 0.f;
        for (int j = l; j <= i; ++j) acc = fmaf(sM[i * PC + j], sT[j * PC + l], acc);
        sL[i * PC + l] = acc;  // zero when l > i (empty sum)
    }
    __syncthreads();
    // ---- write [Tb; M'] as BF16 hi and lo K-major swizzled tiles (128 rows x 64 columns)
    uint8_t *dst = scratch + ((static_cast<size_t>(b) * H + h) * (T_pad / C) + ch) * kA2Bytes;
    for (int e = tid; e < 128 * 8; e += kThreads) {
        const int row = e >> 3, c0 = 8 * (e & 7);
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float v2[2];
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const int col = c0 + 2 * u + w;
                float val;
                if (row < 64) val = col <= row ? sT[row * PC + col] : 0.f;
                else val = sL[(row - 64) * PC + col];
                v2[w] = val;
            }
            uint16_t h0, l0, h1, l1;
            split_bf16(v2[0], h0, l0);
            split_bf16(v2[1], h1, l1);
            hw[u] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
            lw[u] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
        }
        const uint32_t off = kmaj_off(row, c0, 128);
        *reinterpret_cast<uint4 *>(dst + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4 *>(dst + kTileBytes + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
}

// ================================================================ phase 2: state pass

template <int D, int DVS>
struct State {
    static constexpr int A1 = 2 * 128 * D * 2;  // [K o A; Q o A] hi + lo, K-major, K = D
    static constexpr int A2 = kA2Bytes;          // [Tb; M'] hi + lo
    static constexpr int A3 = 2 * C * D * 2;     // (K o e^{Gamma_C - Gamma}) hi + lo, MN-major
    static constexpr int B1 = 2 * DVS * D * 2;   // S0^T hi + lo, K-major (N = DVS, K = D)
    static constexpr int B2 = 2 * DVS * C * 2;   // R^T, then U^T: hi + lo, K-major (N = DVS, K = 64)
    static constexpr int OFF_A1 = 0, OFF_A2 = OFF_A1 + A1, OFF_A3 = OFF_A2 + A2, OFF_B1 = OFF_A3 + A3,
                         OFF_B2 = OFF_B1 + B1, OFF_MISC = OFF_B2 + B2;
    static constexpr int MISC = 4096;
    static constexpr int bytes = OFF_MISC + MISC + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = 3 * DVS <= 128 ? 128 : (3 * DVS <= 256 ? 256 : 512);
};

template <int D, int DVS>
__global__ void __launch_bounds__(kThreads, 1)
state_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
             const float *__restrict__ gate, const uint8_t *__restrict__ scratch, float *const *__restrict__ h_state,
             float *__restrict__ core, int T, int T_pad, int H, float scale, int *__restrict__ status) {
    using S = State<D, DVS>;
    constexpr int TPC = kThreads / D;   // threads per channel in the operand build (2 or 4)
    constexpr int TOK = C / TPC;        // tokens per thread (32 or 16)
    constexpr int HALF = DVS / 2;       // value columns per thread in the epilogues
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA1 = sm + S::OFF_A1, *sA2 = sm + S::OFF_A2, *sA3 = sm + S::OFF_A3, *sB1 = sm + S::OFF_B1,
            *sB2 = sm + S::OFF_B2;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::OFF_MISC);  // 0: A2 copy, 1..3: MMA groups
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::OFF_MISC + 64);
    float *sGseg = reinterpret_cast<float *>(sm + S::OFF_MISC + 128);  // [TPC][D] segment totals
    float *sAC = sGseg + 4 * D;                                        // [D] A_C = e^{Gamma_C}

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int c0 = slice * DVS;
    const size_t rs = static_cast<size_t>(H) * D;
    float *Sg = h_state[b] + static_cast<size_t>(h) * D * D;
    const int nch = T_pad / C;

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tD1 = tmem, tD2 = tmem + DVS, tD3 = tmem + 2 * DVS;
    bool ok = true;

    // Epilogue thread roles. For an M = 128 accumulator, warp w reads TMEM lanes 32(w%4)..+31
    // (rows), columns [ (w/4) * HALF, + HALF ). For D3 with D = 64 (M = 64) the rows are
    // 16 (w%4) + lane for lanes < 16.
    const int quad = warp & 3, colh = warp >> 2;
    const int erow = 32 * quad + lane;  // accumulator row of this thread (M = 128 layout)
    const int ccol = colh * HALF;       // first value column of this thread (within the slice)
    const int srow = (D == 128) ? erow : ((lane < 16) ? 16 * quad + lane : -1);  // key row of D3

    // FP32 master state slice: key row srow, columns [ccol, ccol + HALF)
    float st[HALF];
    if (srow >= 0) {
#pragma unroll
        for (int j = 0; j < HALF; j += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(Sg + static_cast<size_t>(srow) * D + c0 + ccol + j);
            st[j] = x.x; st[j + 1] = x.y; st[j + 2] = x.z; st[j + 3] = x.w;
        }
    }
    // S0^T into B1: element (n = value column, k = key row)
    auto write_state_operand = [&]() {
        if (srow >= 0) {
#pragma unroll
            for (int j = 0; j < HALF; ++j) {
                uint16_t hi, lo;
                split_bf16(st[j], hi, lo);
                const uint32_t off = kmaj_off(ccol + j, srow, DVS);
                *reinterpret_cast<uint16_t *>(sB1 + off) = hi;
                *reinterpret_cast<uint16_t *>(sB1 + S::B1 / 2 + off) = lo;
            }
        }
    };
    write_state_operand();

#pragma unroll 1
    for (int ch = 0; ch < nch; ++ch) {
        const int n = min(C, T - ch * C);
        const size_t row0 = static_cast<size_t>(b) * T_pad + static_cast<size_t>(ch) * C;
        const uint32_t par = ch & 1;
        // ---- bulk copy of this chunk's [Tb; M'] tile (the previous MMA2 finished reading A2)
        if (tid == 0) {
            const uint8_t *src = scratch + ((static_cast<size_t>(b) * H + h) * nch + ch) * kA2Bytes;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&bars[0])),
                         "r"(kA2Bytes)
                         : "memory");
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                    smem_u32(sA2)),
                "l"(src), "r"(kA2Bytes), "r"(smem_u32(&bars[0]))
                : "memory");
        }
        // ---- operands from q, k, g: thread (channel c, token segment sg)
        {
            const int c = tid % D, sg = tid / D, t0 = sg * TOK;
            float g[TOK];
#pragma unroll
            for (int t = 0; t < TOK; ++t) {
                const int i = t0 + t;
                g[t] = i < n ? gate[(row0 + i) * rs + static_cast<size_t>(h) * D + c] : 0.f;
            }
            // segment sums -> exclusive prefix over segments
            float tot = 0.f;
#pragma unroll
            for (int t = 0; t < TOK; ++t) tot += g[t];
            sGseg[sg * D + c] = tot;
            __syncthreads();
            float pre = 0.f, all = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < TPC; ++s2) {
                const float x = sGseg[s2 * D + c];
                if (s2 < sg) pre += x;
                all += x;
            }
            if (sg == 0) sAC[c] = expf(all);
            // e^{Gamma_i} by a forward running product (K o A, Q o A), then e^{Gamma_C - Gamma_i}
            // by a backward one (K o e^{Gamma_C - Gamma}); only a = e^g and k stay in registers.
            float av[TOK], kk[TOK];
            float f = expf(pre);
#pragma unroll
            for (int t = 0; t < TOK; ++t) {
                const int i = t0 + t;
                av[t] = expf(g[t]);
                f *= av[t];
                float kv = 0.f, qv = 0.f;
                if (i < n) {
                    const size_t off = (row0 + i) * rs + static_cast<size_t>(h) * D + c;
                    kv = k[off];
                    qv = q[off];
                }
                kk[t] = kv;
                uint16_t hi, lo;
                split_bf16(kv * f, hi, lo);
                uint32_t off = kmaj_off(i, c, 128);
                *reinterpret_cast<uint16_t *>(sA1 + off) = hi;
                *reinterpret_cast<uint16_t *>(sA1 + S::A1 / 2 + off) = lo;
                split_bf16(qv * f, hi, lo);
                off = kmaj_off(64 + i, c, 128);
                *reinterpret_cast<uint16_t *>(sA1 + off) = hi;
                *reinterpret_cast<uint16_t *>(sA1 + S::A1 / 2 + off) = lo;
            }
            // Gamma_C - Gamma_{t0+TOK-1} = the sum of the later segments
            float fb = expf(all - pre - tot);
#pragma unroll
            for (int t = TOK - 1; t >= 0; --t) {
                uint16_t hi, lo;
                split_bf16(kk[t] * fb, hi, lo);
                const uint32_t off = mnmaj_off(c, t0 + t, C);
                *reinterpret_cast<uint16_t *>(sA3 + off) = hi;
                *reinterpret_cast<uint16_t *>(sA3 + S::A3 / 2 + off) = lo;
                fb *= av[t];
            }
        }
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        tc_fence_after();
        // ---- MMA1: D1 = [K o A; Q o A] . S0
        if (tid == 0 && ok) {
            constexpr uint32_t id = idesc_bf16(128, DVS, false, false);
            const uint32_t a0 = smem_u32(sA1), b0 = smem_u32(sB1);
            int acc = 0;
#pragma unroll 1
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t ah = kmaj_desc(a0, 128, 0, ks), al = kmaj_desc(a0 + S::A1 / 2, 128, 0, ks);
                const uint64_t bh = kmaj_desc(b0, DVS, 0, ks), bl = kmaj_desc(b0 + S::B1 / 2, DVS, 0, ks);
                mma_bf16(tD1, ah, bh, id, acc); acc = 1;
                mma_bf16(tD1, ah, bl, id, 1);
                mma_bf16(tD1, al, bh, id, 1);
            }
            mma_commit(&bars[1]);
        }
        // e1: V rows of this thread for R (rows 0..63, quads 0 and 1), or the Q half of D1
        // kept for the output (rows 64..127, quads 2 and 3)
        float e1[HALF];
        if (quad < 2) {
            const int i = erow;
#pragma unroll
            for (int j = 0; j < HALF; j += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < n) x = *reinterpret_cast<const float4 *>(v + (row0 + i) * rs + static_cast<size_t>(h) * D + c0 + ccol + j);
                e1[j] = x.x; e1[j + 1] = x.y; e1[j + 2] = x.z; e1[j + 3] = x.w;
            }
        }
        ok = ok && mbar_wait(&bars[1], par, kWaitCycles);
        tc_fence_after();
        // ---- epilogue 1: R = V - D1[0:64] -> R^T into B2
#pragma unroll
        for (int j = 0; j < HALF; j += 8) {
            float x[8];
            tmem_ld8(tmem_lane_base(tD1, warp) + ccol + j, x);
            tmem_ld_wait();
            if (quad < 2) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint16_t hi, lo;
                    split_bf16(e1[j + u] - x[u], hi, lo);
                    const uint32_t off = kmaj_off(ccol + j + u, erow, DVS);
                    *reinterpret_cast<uint16_t *>(sB2 + off) = hi;
                    *reinterpret_cast<uint16_t *>(sB2 + S::B2 / 2 + off) = lo;
                }
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) e1[j + u] = x[u];
            }
        }
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        tc_fence_after();
        // ---- MMA2: D2 = [Tb; M'] . R  (after the bulk copy of the tile has landed)
        if (tid == 0 && ok) ok = mbar_wait(&bars[0], par, kWaitCycles);
        if (tid == 0 && ok) {
            constexpr uint32_t id = idesc_bf16(128, DVS, false, false);
            const uint32_t a0 = smem_u32(sA2), b0 = smem_u32(sB2);
            int acc = 0;
#pragma unroll 1
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t ah = kmaj_desc(a0, 128, 0, ks), al = kmaj_desc(a0 + kTileBytes, 128, 0, ks);
                const uint64_t bh = kmaj_desc(b0, DVS, 0, ks), bl = kmaj_desc(b0 + S::B2 / 2, DVS, 0, ks);
                mma_bf16(tD2, ah, bh, id, acc); acc = 1;
                mma_bf16(tD2, ah, bl, id, 1);
                mma_bf16(tD2, al, bh, id, 1);
            }
            mma_commit(&bars[2]);
        }
        ok = ok && mbar_wait(&bars[2], par, kWaitCycles);
        tc_fence_after();
        // ---- epilogue 2: U = D2[0:64] -> U^T into B2 (R^T is consumed); O = scale (D1q + D2q)
#pragma unroll
        for (int j = 0; j < HALF; j += 8) {
            float x[8];
            tmem_ld8(tmem_lane_base(tD2, warp) + ccol + j, x);
            tmem_ld_wait();
            if (quad < 2) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint16_t hi, lo;
                    split_bf16(x[u], hi, lo);
                    const uint32_t off = kmaj_off(ccol + j + u, erow, DVS);
                    *reinterpret_cast<uint16_t *>(sB2 + off) = hi;
                    *reinterpret_cast<uint16_t *>(sB2 + S::B2 / 2 + off) = lo;
                }
            } else {
                const int i = erow - 64;
                if (i < n) {
                    float *dst = core + (row0 + i) * rs + static_cast<size_t>(h) * D + c0 + ccol + j;
                    float4 o0 = make_float4(scale * (e1[j] + x[0]), scale * (e1[j + 1] + x[1]),
                                            scale * (e1[j + 2] + x[2]), scale * (e1[j + 3] + x[3]));
                    float4 o1 = make_float4(scale * (e1[j + 4] + x[4]), scale * (e1[j + 5] + x[5]),
                                            scale * (e1[j + 6] + x[6]), scale * (e1[j + 7] + x[7]));
                    *reinterpret_cast<float4 *>(dst) = o0;
                    *reinterpret_cast<float4 *>(dst + 4) = o1;
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        tc_fence_after();
        // ---- MMA3: D3 = (K o e^{Gamma_C - Gamma})^T . U
        if (tid == 0 && ok) {
            constexpr uint32_t id = idesc_bf16(D, DVS, true, false);
            const uint32_t a0 = smem_u32(sA3), b0 = smem_u32(sB2);
            int acc = 0;
#pragma unroll 1
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t ah = mnmaj_desc(a0, C, 0, ks), al = mnmaj_desc(a0 + S::A3 / 2, C, 0, ks);
                const uint64_t bh = kmaj_desc(b0, DVS, 0, ks), bl = kmaj_desc(b0 + S::B2 / 2, DVS, 0, ks);
                mma_bf16(tD3, ah, bh, id, acc); acc = 1;
                mma_bf16(tD3, ah, bl, id, 1);
                mma_bf16(tD3, al, bh, id, 1);
            }
            mma_commit(&bars[3]);
        }
        ok = ok && mbar_wait(&bars[3], par, kWaitCycles);
        tc_fence_after();
        // ---- epilogue 3: S = A_C o S0 + D3 (FP32 in registers), S^T split into B1
        {
            const float ac = srow >= 0 ? sAC[srow] : 0.f;
#pragma unroll
            for (int j = 0; j < HALF; j += 8) {
                float x[8];
                tmem_ld8(tmem_lane_base(tD3, warp) + ccol + j, x);
                tmem_ld_wait();
                if (srow >= 0) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) st[j + u] = fmaf(ac, st[j + u], x[u]);
                }
            }
        }
        write_state_operand();
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        tc_fence_after();
        if (!ok) break;  // block-uniform: every thread saw the same flag
    }
    if (!ok) {
        if (tid == 0) atomicExch(status, KDA_ERR_TIMEOUT);
    } else if (srow >= 0) {
#pragma unroll
        for (int j = 0; j < HALF; j += 4)
            *reinterpret_cast<float4 *>(Sg + static_cast<size_t>(srow) * D + c0 + ccol + j) =
                make_float4(st[j], st[j + 1], st[j + 2], st[j + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, S::TMEM_COLS);
}

template <typename K>
int set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
               ? KDA_OK
               : KDA_ERR_CUDA;
}

template <int D, int DVS>
int launch_tc(const float *q, const float *k, const float *v, const float *gate, const float *beta,
              float *const *h_state, float *core, int B, int T, int H, float scale, void *scratch, cudaStream_t s) {
    const int T_pad = static_cast<int>(kda_t_pad(static_cast<size_t>(T), C));
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    static bool attrs = false;
    if (!attrs) {
        KDA_TRY(set_smem(intra_kernel<D>, static_cast<int>(Intra<D>::bytes)));
        KDA_TRY(set_smem(state_kernel<D, DVS>, State<D, DVS>::bytes));
        attrs = true;
    }
    intra_kernel<D><<<dim3(T_pad / C, H, B), kThreads, Intra<D>::bytes, s>>>(
        k, q, gate, beta, static_cast<uint8_t *>(scratch), T, T_pad, H);
    KDA_TRY(launch_status());
    state_kernel<D, DVS><<<dim3(D / DVS, H, B), kThreads, State<D, DVS>::bytes, s>>>(
        q, k, v, gate, static_cast<const uint8_t *>(scratch), h_state, core, T, T_pad, H, scale, status);
    return launch_status();
}

}  // namespace

size_t chunk_prefill_scratch_bytes(int B, int T, int H) {
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    return static_cast<size_t>(B) * H * (kda_t_pad(static_cast<size_t>(T), C) / C) * kA2Bytes;
}

int chunk_prefill_tc(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                     float *const *h_state, float *core, int B, int T, const kda_dims *dims, void *scratch,
                     cudaStream_t s) {
    const int H = dims->heads;
    const float sc = dims->scale;
    if (dims->head_dim == 64) return launch_tc<64, 32>(q, k, v, gate, beta, h_state, core, B, T, H, sc, scratch, s);
    // value slice width: enough CTAs to cover the SMs (one CTA per SM fits in shared memory)
    const long long units = static_cast<long long>(B) * H;
    if (units >= 60) return launch_tc<128, 64>(q, k, v, gate, beta, h_state, core, B, T, H, sc, scratch, s);
    return launch_tc<128, 32>(q, k, v, gate, beta, h_state, core, B, T, H, sc, scratch, s);
}

}  // namespace kda
