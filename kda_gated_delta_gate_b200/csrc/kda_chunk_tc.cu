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
#include <algorithm>

#include "common.cuh"
#include "umma.cuh"

namespace kda {
namespace {

using namespace umma;

constexpr int C = kChunk;          // 64
constexpr int kThreads = 256;
constexpr int kTileBytes = 16384;  // one 128 x 64 BF16 K-major tile
constexpr int kA2Bytes = 2 * kTileBytes;

// Per (stream, head, chunk) the intra kernel writes one pack of state-independent operands,
// each a BF16 hi tile followed by its lo tile, laid out exactly as the state kernel's shared
// memory wants them (so a bulk copy moves each):
//   A1 [K o A; Q o A]           128 x D, K-major          (A = e^Gamma)
//   A2 [Tb; M']                 128 x 64, K-major
//   A3 K o e^{Gamma_C - Gamma}  D (M) x 64 (K), MN-major
//   AC e^{Gamma_C}              D FP32 (1 KB slot)
template <int D>
struct Pack {
    static constexpr int A1 = 2 * 128 * D * 2;
    static constexpr int A2 = kA2Bytes;
    static constexpr int A3 = 2 * C * D * 2;
    static constexpr int AC = 1024;
    static constexpr int OFF_A1 = 0, OFF_A2 = A1, OFF_A3 = A1 + A2, OFF_AC = A1 + A2 + A3;
    static constexpr int bytes = A1 + A2 + A3 + AC;
};
constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at 1.9 GHz

// Split 8 FP32 values into BF16 hi and lo, packed as two 16-byte chunks (paired conversions).
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) split_bf16x2(x[2 * u], x[2 * u + 1], h[u], l[u]);
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void st_pair(uint8_t *tile, int half_bytes, uint32_t off, const float (&x)[8]) {
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4 *>(tile + off) = hi;
    *reinterpret_cast<uint4 *>(tile + half_bytes + off) = lo;
}

// ================================================================ phase 1: intra-chunk

constexpr int kIntraThreads = 512;

template <int D>
struct Intra {
    static constexpr int P = D + 8;   // fp32 row stride of [C][D] tiles (bank-spread, 16-B aligned)
    static constexpr int PC = C + 1;  // row stride of [C][C] tiles
    static constexpr int NZ = 64;     // rows of the block-local backward factors
    static constexpr size_t floats = 3 * C * P + NZ * P + 3 * C * PC + 4 * D + C + 3 * 256;
    static constexpr size_t bytes = floats * sizeof(float);
};

// The exact CUDA-core intra-chunk computation of one (stream b, head h, chunk ch): every decay
// factor is a product of per-token factors <= 1, whatever g holds. It writes the whole operand
// pack. Used for the chunks whose in-block decay is too strong for the tensor-core path.
template <int D>
__device__ __forceinline__ void intra_simt_body(const float *__restrict__ k, const float *__restrict__ q,
                                                const float *__restrict__ gate, const float *__restrict__ beta,
                                                uint8_t *__restrict__ scratch, int T, int T_pad, int H, int b,
                                                int h, int ch, float *smem) {
    using I = Intra<D>;
    constexpr int P = I::P, PC = I::PC, NT = kIntraThreads;
    float *sK = smem;              // k, then X: k_i prod_{s=16a}^{i} a_s  (a = block of i)
    float *sQ = sK + C * P;        // q, then Y: q_i prod_{s=16a}^{i} a_s
    float *sA = sQ + C * P;        // a = e^g
    float *sZ = sA + C * P;        // Z: k_j prod_{s=j+1}^{16b+15} a_s
    float *sL = sZ + I::NZ * P;    // L' (unscaled), then M'
    float *sM = sL + C * PC;       // M
    float *sT = sM + C * PC;       // T, then Tb
    float *sF = sT + C * PC;       // [4][D]: whole-block decay products
    float *sB = sF + 4 * D;        // beta
    float *sTmp = sB + C;          // [3][256]

    const int tid = threadIdx.x;
    const int n = min(C, T - ch * C);
    const size_t row0 = static_cast<size_t>(b) * T_pad + static_cast<size_t>(ch) * C;
    const size_t rs = static_cast<size_t>(H) * D;

    // ---- load k, q and a = e^g (pad guard: rows >= n are k = q = 0, a = 1)
    for (int e = tid; e < C * D / 4; e += NT) {
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
    //      the running product G = k_j prod_{s=j+1}^{i} a_s over its channels; the 16 channel
    //      groups of one j are 16 adjacent lanes and reduce with shuffles. Channel group cg
    //      holds float4 columns cg, cg + 16, ... (conflict-free 16-byte loads).
    {
        constexpr int NV = D / 64;  // float4 per thread per row (2 for D = 128, 1 for D = 64)
        const int cg = tid & 15, jp = (tid >> 4) & 7, a = tid >> 7;
        const unsigned gmask = 0xFFFFu << (tid & 16);
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const int j = 16 * a + (pass == 0 ? jp : 15 - jp);
            float4 G[NV];
#pragma unroll
            for (int w = 0; w < NV; ++w) G[w] = *reinterpret_cast<const float4 *>(sK + j * P + 4 * (cg + 16 * w));
#pragma unroll 1
            for (int i = j; i < 16 * a + 16; ++i) {
                float ls = 0.f, ms = 0.f;
#pragma unroll
                for (int w = 0; w < NV; ++w) {
                    const int c = 4 * (cg + 16 * w);
                    if (i > j) {
                        const float4 av = *reinterpret_cast<const float4 *>(sA + i * P + c);
                        G[w].x *= av.x; G[w].y *= av.y; G[w].z *= av.z; G[w].w *= av.w;
                    }
                    const float4 kv = *reinterpret_cast<const float4 *>(sK + i * P + c);
                    const float4 qv = *reinterpret_cast<const float4 *>(sQ + i * P + c);
                    ls = fmaf(kv.x, G[w].x, fmaf(kv.y, G[w].y, fmaf(kv.z, G[w].z, fmaf(kv.w, G[w].w, ls))));
                    ms = fmaf(qv.x, G[w].x, fmaf(qv.y, G[w].y, fmaf(qv.z, G[w].z, fmaf(qv.w, G[w].w, ms))));
                }
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) {
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

    // ---- block-local factors, thread (channel c, block a): Z (backward within blocks 0..2),
    //      the whole-block products F, then X, Y (forward within blocks 1..3, in place).
    if (tid < 4 * D) {
        const int c = tid % D, a = tid / D;
        float f = 1.f;
        for (int j = 16 * a + 15; j >= 16 * a; --j) {
            sZ[j * P + c] = sK[j * P + c] * f;
            f *= sA[j * P + c];
        }
        sF[a * D + c] = f;
    }
    __syncthreads();
    if (tid < 4 * D) {
        const int c = tid % D, a = tid / D;
        float f = 1.f;
        for (int i = 16 * a; i < 16 * a + 16; ++i) {
            f *= sA[i * P + c];
            sK[i * P + c] *= f;
            sQ[i * P + c] *= f;
        }
    }
    __syncthreads();

    // ---- off-diagonal blocks (a > b): L'[i][j] = sum_c X_ic sigma_ab,c Z_jc (Y for M), with
    //      sigma_ab the decay of the whole blocks strictly between b and a (1 when adjacent).
    //      Thread = (4x4 tile, channel quarter); the 4 quarters are adjacent lanes.
    if (tid < 384) {
        const int qtr = tid & 3, tile = tid >> 2;
        const int p = tile >> 4;
        const int pa = p == 0 ? 1 : (p < 3 ? 2 : 3);
        const int pb = p == 0 ? 0 : (p == 1 ? 0 : (p == 2 ? 1 : p - 3));
        const int i0 = 16 * pa + 4 * ((tile & 15) >> 2), j0 = 16 * pb + 4 * (tile & 3);
        float l[4][4], m[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2) { l[r][s2] = 0.f; m[r][s2] = 0.f; }
#pragma unroll 2
        for (int cq = 0; cq < D / 16; ++cq) {
            const int c = 4 * (qtr + 4 * cq);
            float4 sg = make_float4(1.f, 1.f, 1.f, 1.f);
            if (pa - pb >= 2) {
                sg = *reinterpret_cast<const float4 *>(sF + 1 * D + c);
                if (pa - pb == 3) {
                    const float4 f2 = *reinterpret_cast<const float4 *>(sF + 2 * D + c);
                    sg.x *= f2.x; sg.y *= f2.y; sg.z *= f2.z; sg.w *= f2.w;
                } else if (pa == 3) {
                    sg = *reinterpret_cast<const float4 *>(sF + 2 * D + c);
                }
            }
            float4 z[4], x[4], y[4];
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2) {
                z[s2] = *reinterpret_cast<const float4 *>(sZ + (j0 + s2) * P + c);
                z[s2].x *= sg.x; z[s2].y *= sg.y; z[s2].z *= sg.z; z[s2].w *= sg.w;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                x[r] = *reinterpret_cast<const float4 *>(sK + (i0 + r) * P + c);
                y[r] = *reinterpret_cast<const float4 *>(sQ + (i0 + r) * P + c);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    l[r][s2] = fmaf(x[r].x, z[s2].x, fmaf(x[r].y, z[s2].y, fmaf(x[r].z, z[s2].z, fmaf(x[r].w, z[s2].w, l[r][s2]))));
                    m[r][s2] = fmaf(y[r].x, z[s2].x, fmaf(y[r].y, z[s2].y, fmaf(y[r].z, z[s2].z, fmaf(y[r].w, z[s2].w, m[r][s2]))));
                }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2) {
#pragma unroll
                for (int o = 1; o < 4; o <<= 1) {
                    l[r][s2] += __shfl_xor_sync(0xffffffffu, l[r][s2], o);
                    m[r][s2] += __shfl_xor_sync(0xffffffffu, m[r][s2], o);
                }
            }
        if (qtr == 0) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    sL[(i0 + r) * PC + j0 + s2] = l[r][s2];
                    sM[(i0 + r) * PC + j0 + s2] = m[r][s2];
                }
        }
    }
    __syncthreads();

    // ---- the state kernel's operands for this chunk: K o A = X P_a, Q o A = Y P_a and
    //      K o e^{Gamma_C - Gamma} = Z S_a, with P_a / S_a the decay of all blocks before / after
    //      block a; 16-byte chunks of 8 channels written straight into the pack.
    using PK = Pack<D>;
    uint8_t *pack = scratch + ((static_cast<size_t>(b) * H + h) * (T_pad / C) + ch) * PK::bytes;
    for (int e = tid; e < C * (D / 8); e += NT) {
        const int i = e / (D / 8), cb = 8 * (e % (D / 8)), a = i >> 4;
        float xk[8], xq[8], xb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = cb + u;
            float pre = 1.f, suf = 1.f;
            for (int bb = 0; bb < a; ++bb) pre *= sF[bb * D + c];
            for (int bb = a + 1; bb < 4; ++bb) suf *= sF[bb * D + c];
            xk[u] = sK[i * P + c] * pre;
            xq[u] = sQ[i * P + c] * pre;
            xb[u] = sZ[i * P + c] * suf;
        }
        uint4 hi, lo;
        split8(xk, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + kmaj_off(i, cb, 128)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + PK::A1 / 2 + kmaj_off(i, cb, 128)) = lo;
        split8(xq, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + kmaj_off(64 + i, cb, 128)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + PK::A1 / 2 + kmaj_off(64 + i, cb, 128)) = lo;
        split8(xb, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A3 + mnmaj_off(cb, i, C)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A3 + PK::A3 / 2 + mnmaj_off(cb, i, C)) = lo;
    }
    if (tid < D) {
        float acv = 1.f;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acv *= sF[bb * D + tid];
        reinterpret_cast<float *>(pack + PK::OFF_AC)[tid] = acv;
    }

    // ---- L = diag(beta) L' (strict lower). T = (I + L)^-1: 16x16 diagonal blocks by
    //      substitution, then off-diagonal blocks T_ab = -T_aa sum_{b<=c<a} L_ac T_cb.
    for (int e = tid; e < C * C; e += NT) {
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
        for (int e = tid; e < npairs * 256; e += NT) {
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
        for (int e = tid; e < npairs * 256; e += NT) {
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
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        if (j <= i) sT[i * PC + j] *= sB[j];
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, l = e % C;
        float acc = 0.f;
        for (int j = l; j <= i; ++j) acc = fmaf(sM[i * PC + j], sT[j * PC + l], acc);
        sL[i * PC + l] = acc;  // zero when l > i (empty sum)
    }
    __syncthreads();
    // ---- write [Tb; M'] as BF16 hi and lo K-major swizzled tiles (128 rows x 64 columns)
    uint8_t *dst = pack + PK::OFF_A2;
    for (int e = tid; e < 128 * 8; e += NT) {
        const int row = e >> 3, c0 = 8 * (e & 7);
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int col = c0 + u;
            x[u] = row < 64 ? (col <= row ? sT[row * PC + col] : 0.f) : sL[(row - 64) * PC + col];
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint16_t h0, l0, h1, l1;
            split_bf16(x[2 * u], h0, l0);
            split_bf16(x[2 * u + 1], h1, l1);
            hw[u] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
            lw[u] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
        }
        const uint32_t off = kmaj_off(row, c0, 128);
        *reinterpret_cast<uint4 *>(dst + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4 *>(dst + kTileBytes + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
}

// All chunks through the CUDA-core body (grid = chunks x heads x streams).
template <int D>
__global__ void __launch_bounds__(kIntraThreads, 1)
intra_simt_kernel(const float *__restrict__ k, const float *__restrict__ q, const float *__restrict__ gate,
                  const float *__restrict__ beta, uint8_t *__restrict__ scratch, int T, int T_pad, int H) {
    extern __shared__ float smem[];
    intra_simt_body<D>(k, q, gate, beta, scratch, T, T_pad, H, blockIdx.z, blockIdx.y, blockIdx.x, smem);
}

// Only the chunks the tensor-core kernel listed (count and packed (b, h, ch) entries in scratch).
template <int D>
__global__ void __launch_bounds__(kIntraThreads, 1)
intra_fix_kernel(const float *__restrict__ k, const float *__restrict__ q, const float *__restrict__ gate,
                 const float *__restrict__ beta, uint8_t *__restrict__ scratch, const int *__restrict__ list,
                 int T, int T_pad, int H) {
    extern __shared__ float smem[];
    const int count = list[0];
    const int nch = T_pad / C;
    for (int e = blockIdx.x; e < count; e += gridDim.x) {
        const int id = list[1 + e];
        const int ch = id % nch, h = (id / nch) % H, b = id / (nch * H);
        intra_simt_body<D>(k, q, gate, beta, scratch, T, T_pad, H, b, h, ch, smem);
        __syncthreads();
    }
}

// ---------------------------------------------------------------- intra-chunk on tensor cores
//
// L' and M for all pairs of the chunk in one tcgen05 MMA. Each 16-token block a gets the
// reference point m_a = 16a + 7 (its middle). With Gamma the in-chunk cumulative decay,
//   A rows  i (block a):      k_i e^{Gamma_i - Gamma_{m_a}}   (and q_i ... for rows 64 + i)
//   B rows  (a', j), j <= 16a'+15:  k_j e^{Gamma_{m_a'} - Gamma_j}
// so D[i][(a, j)] = sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc} = L'[i][j] exactly for every j <= i
// (the reference cancels). B holds the 16, 32, 48, 64 rows of a' = 0..3 at column offsets
// 0, 16, 48, 96 (160 rows). Factors above 1 come only from decay inside one block (at most
// 8 tokens); a chunk whose |Gamma_i - Gamma_{m_a}| exceeds kRefBound for some channel is
// handed to the CUDA-core body instead (listed in scratch, run by intra_fix_kernel).

constexpr float kRefBound = 80.0f;  // e^80 and e^-80 are comfortably inside BF16/FP32 range

template <int D>
struct IntraTC {
    static constexpr int NB = 160;                  // B rows
    static constexpr int A_BYTES = 2 * 128 * D * 2;  // A hi + lo (K-major, K = D)
    static constexpr int B_BYTES = 2 * NB * D * 2;   // B hi + lo
    static constexpr int GP = D + 4;                // Gamma row stride (floats)
    static constexpr int PC = C + 1;
    static constexpr int LMT = 3 * C * PC * 4;     // L, M, T (FP32); Gamma lives here first
    static constexpr int OFF_A = 0, OFF_B = A_BYTES, OFF_LMT = A_BYTES + B_BYTES, OFF_TAB = OFF_LMT + LMT;
    static constexpr int TAB = 14 * D * 4;          // per-channel reference factors
    static constexpr int OFF_MISC = OFF_TAB + TAB;  // beta[C], tmp[768], barrier, tmem slot, flags
    static constexpr int MISC = (C + 768) * 4 + 256;
    static constexpr int bytes = OFF_MISC + MISC + 1024;
};

template <int D>
__global__ void __launch_bounds__(kIntraThreads, 1)
intra_tc_kernel(const float *__restrict__ k, const float *__restrict__ q, const float *__restrict__ gate,
                const float *__restrict__ beta, uint8_t *__restrict__ scratch, int *__restrict__ list, int T,
                int T_pad, int H, int *__restrict__ status) {
    using I = IntraTC<D>;
    using PK = Pack<D>;
    constexpr int NT = kIntraThreads, GP = I::GP, PC = I::PC;
    constexpr int CG = D / 8;                 // 8-channel groups
    constexpr int UPT = C * CG / NT;          // (token, group) units per thread: 2 (D=128) or 1
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = sm + I::OFF_A, *sBt = sm + I::OFF_B;
    float *sG = reinterpret_cast<float *>(sm + I::OFF_LMT);  // Gamma [C][GP], before L/M/T
    float *sL = reinterpret_cast<float *>(sm + I::OFF_LMT);  // L' then M'
    float *sM = sL + C * PC;
    float *sT = sM + C * PC;
    float *sTab = reinterpret_cast<float *>(sm + I::OFF_TAB);
    float *sB = reinterpret_cast<float *>(sm + I::OFF_MISC);
    float *sTmp = sB + C;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + I::OFF_MISC + (C + 768) * 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
    // reference tables, [entry][D]: 0..3 e^{Gamma_{m_a}}, 4..7 e^{Gamma_C - Gamma_{m_a}},
    // 8..13 e^{Gamma_{m_a} - Gamma_{m_b}} for (a,b) = (1,0),(2,0),(2,1),(3,0),(3,1),(3,2)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ch = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int n = min(C, T - ch * C);
    const int nch = T_pad / C;
    const size_t row0 = static_cast<size_t>(b) * T_pad + static_cast<size_t>(ch) * C;
    const size_t rs = static_cast<size_t>(H) * D;
    uint8_t *pack = scratch + ((static_cast<size_t>(b) * H + h) * nch + ch) * PK::bytes;

    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    // ---- load: unit (token i, 8-channel group); g goes to shared memory for the scan
    float kk[UPT][8], qq[UPT][8];
#pragma unroll
    for (int u = 0; u < UPT; ++u) {
        const int e = tid + u * NT, i = e / CG, cb = 8 * (e % CG);
        float4 k0 = make_float4(0.f, 0.f, 0.f, 0.f), k1 = k0, q0 = k0, q1 = k0, g0 = k0, g1 = k0;
        if (i < n) {
            const size_t off = (row0 + i) * rs + static_cast<size_t>(h) * D + cb;
            k0 = *reinterpret_cast<const float4 *>(k + off);
            k1 = *reinterpret_cast<const float4 *>(k + off + 4);
            q0 = *reinterpret_cast<const float4 *>(q + off);
            q1 = *reinterpret_cast<const float4 *>(q + off + 4);
            g0 = *reinterpret_cast<const float4 *>(gate + off);
            g1 = *reinterpret_cast<const float4 *>(gate + off + 4);
        }
        kk[u][0] = k0.x; kk[u][1] = k0.y; kk[u][2] = k0.z; kk[u][3] = k0.w;
        kk[u][4] = k1.x; kk[u][5] = k1.y; kk[u][6] = k1.z; kk[u][7] = k1.w;
        qq[u][0] = q0.x; qq[u][1] = q0.y; qq[u][2] = q0.z; qq[u][3] = q0.w;
        qq[u][4] = q1.x; qq[u][5] = q1.y; qq[u][6] = q1.z; qq[u][7] = q1.w;
        *reinterpret_cast<float4 *>(sG + i * GP + cb) = g0;
        *reinterpret_cast<float4 *>(sG + i * GP + cb + 4) = g1;
    }
    if (tid < C) sB[tid] = tid < n ? beta[(row0 + tid) * H + h] : 0.f;
    __syncthreads();
    // ---- Gamma: inclusive cumulative sum over tokens, thread (channel, quarter of 16 tokens)
    {
        constexpr int QT = NT / D;  // 4 (D=128) or 8 (D=64) token ranges
        constexpr int TPQ = C / QT;
        const int c = tid % D, qr = tid / D;
        float acc = 0.f;
        for (int i = qr * TPQ; i < (qr + 1) * TPQ; ++i) { acc += sG[i * GP + c]; sG[i * GP + c] = acc; }
        sTmp[qr * D + c] = acc;
        __syncthreads();
        float pre = 0.f;
        for (int r = 0; r < qr; ++r) pre += sTmp[r * D + c];
        if (qr > 0)
            for (int i = qr * TPQ; i < (qr + 1) * TPQ; ++i) sG[i * GP + c] += pre;
        __syncthreads();
    }
    if (tid < D) {
        const int c = tid;
        const float gm[4] = {sG[7 * GP + c], sG[23 * GP + c], sG[39 * GP + c], sG[55 * GP + c]};
        const float gc = sG[63 * GP + c];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            sTab[a * D + c] = __expf(gm[a]);
            sTab[(4 + a) * D + c] = __expf(gc - gm[a]);
        }
        sTab[8 * D + c] = __expf(gm[1] - gm[0]);
        sTab[9 * D + c] = __expf(gm[2] - gm[0]);
        sTab[10 * D + c] = __expf(gm[2] - gm[1]);
        sTab[11 * D + c] = __expf(gm[3] - gm[0]);
        sTab[12 * D + c] = __expf(gm[3] - gm[1]);
        sTab[13 * D + c] = __expf(gm[3] - gm[2]);
    }
    __syncthreads();
    // ---- operands of the L/M MMA: A (mid-block reference) and B (all references), in shared memory
    bool safe = true;
    auto ld8 = [](const float *p, float (&x)[8]) {
        const float4 a0 = *reinterpret_cast<const float4 *>(p), a1 = *reinterpret_cast<const float4 *>(p + 4);
        x[0] = a0.x; x[1] = a0.y; x[2] = a0.z; x[3] = a0.w; x[4] = a1.x; x[5] = a1.y; x[6] = a1.z; x[7] = a1.w;
    };
#pragma unroll
    for (int u = 0; u < UPT; ++u) {
        const int e = tid + u * NT, i = e / CG, cb = 8 * (e % CG), a = i >> 4;
        float gi[8], gm[8], ef[8], ei[8], x[8];
        ld8(sG + i * GP + cb, gi);
        ld8(sG + (16 * a + 7) * GP + cb, gm);
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const float r = gi[w] - gm[w];
            safe = safe && fabsf(r) <= kRefBound;
            ef[w] = __expf(r);
            ei[w] = __expf(-r);
        }
#pragma unroll
        for (int w = 0; w < 8; ++w) x[w] = kk[u][w] * ef[w];
        st_pair(sA, I::A_BYTES / 2, kmaj_off(i, cb, 128), x);
#pragma unroll
        for (int w = 0; w < 8; ++w) x[w] = qq[u][w] * ef[w];
        st_pair(sA, I::A_BYTES / 2, kmaj_off(64 + i, cb, 128), x);
        // B rows for every reference block a2 >= a (column offsets 0, 16, 48, 96)
#pragma unroll
        for (int a2 = 0; a2 < 4; ++a2) {
            if (a2 < a) continue;
            const int off2 = 8 * a2 * (a2 + 1);
            if (a2 == a) {
#pragma unroll
                for (int w = 0; w < 8; ++w) x[w] = kk[u][w] * ei[w];
            } else {
                const int tix = a2 == 1 ? 8 : (a2 == 2 ? (a == 0 ? 9 : 10) : (a == 0 ? 11 : (a == 1 ? 12 : 13)));
                float tb[8];
                ld8(sTab + tix * D + cb, tb);
#pragma unroll
                for (int w = 0; w < 8; ++w) x[w] = kk[u][w] * ei[w] * tb[w];
            }
            st_pair(sBt, I::B_BYTES / 2, kmaj_off(off2 + i, cb, I::NB), x);
        }
    }
    fence_async_smem();
    tc_fence_before();
    safe = __syncthreads_and(safe) != 0;
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // ---- D[128 x 160] = A . B^T (L' in rows 0..63, M in rows 64..127), issued now so that the
    //      operand pack below is written while the tensor core works
    if (safe && tid == 0) {
        constexpr uint32_t id = idesc_bf16(128, I::NB, false, false);
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sBt);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t ah = kmaj_desc(a0, 128, 0, ks), al = kmaj_desc(a0 + I::A_BYTES / 2, 128, 0, ks);
            const uint64_t bh = kmaj_desc(b0, I::NB, 0, ks), bl = kmaj_desc(b0 + I::B_BYTES / 2, I::NB, 0, ks);
            mma_bf16(tmem, ah, bh, id, ks > 0 ? 1u : 0u);
            mma_bf16(tmem, ah, bl, id, 1);
            mma_bf16(tmem, al, bh, id, 1);
        }
        mma_commit(bar);
    }
    // ---- the state kernel's operands: K o e^Gamma, Q o e^Gamma, K o e^{Gamma_C - Gamma}
    //      (written for unsafe chunks too; the CUDA-core body then rewrites the whole pack)
#pragma unroll
    for (int u = 0; u < UPT; ++u) {
        const int e = tid + u * NT, i = e / CG, cb = 8 * (e % CG), a = i >> 4;
        float gi[8], gm[8], em[8], ecm[8], x[8];
        ld8(sG + i * GP + cb, gi);
        ld8(sG + (16 * a + 7) * GP + cb, gm);
        ld8(sTab + a * D + cb, em);
        ld8(sTab + (4 + a) * D + cb, ecm);
        float ef[8], ei[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            ef[w] = __expf(gi[w] - gm[w]) * em[w];    // e^{Gamma_i}
            ei[w] = __expf(gm[w] - gi[w]) * ecm[w];   // e^{Gamma_C - Gamma_i}
        }
        uint4 hi, lo;
#pragma unroll
        for (int w = 0; w < 8; ++w) x[w] = kk[u][w] * ef[w];
        split8(x, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + kmaj_off(i, cb, 128)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + PK::A1 / 2 + kmaj_off(i, cb, 128)) = lo;
#pragma unroll
        for (int w = 0; w < 8; ++w) x[w] = qq[u][w] * ef[w];
        split8(x, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + kmaj_off(64 + i, cb, 128)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + PK::A1 / 2 + kmaj_off(64 + i, cb, 128)) = lo;
#pragma unroll
        for (int w = 0; w < 8; ++w) x[w] = kk[u][w] * ei[w];
        split8(x, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A3 + mnmaj_off(cb, i, C)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A3 + PK::A3 / 2 + mnmaj_off(cb, i, C)) = lo;
    }
    if (tid < D) reinterpret_cast<float *>(pack + PK::OFF_AC)[tid] = sTab[3 * D + tid] * sTab[7 * D + tid];
    __syncthreads();  // every read of Gamma is done: L'/M are about to overwrite its space
    bool ok = true;
    if (safe) {
        ok = mbar_wait(bar, 0, kWaitCycles);
        tc_fence_after();
        // ---- read back: warp (quad, part); row r = 32 quad + lane (i = r % 64, block a = i / 16)
        //      needs columns [off_a, off_a + 16(a+1)); the quad's window is [0, 48) for rows in
        //      blocks 0-1 and [48, 160) for blocks 2-3, split over the 4 warps of the quad.
        {
            const int quad = warp & 3, part = warp >> 2;
            const int r = 32 * quad + lane, i = r & 63, a = i >> 4;
            const int off_a = 8 * a * (a + 1);
            const int w0 = (quad & 1) ? 48 : 0, wlen = (quad & 1) ? 112 : 48;
            float *dstm = r < 64 ? sL : sM;
            for (int c8 = part * 8; c8 < wlen; c8 += 32) {
                float x[8];
                tmem_ld8(tmem_lane_base(tmem, warp) + w0 + c8, x);
                tmem_ld_wait();
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    const int j = w0 + c8 + w - off_a;
                    if (j >= 0 && j <= i) dstm[i * PC + j] = x[w];
                }
            }
        }
        tc_fence_before();
    }
    ok = __syncthreads_and(ok) != 0;
    if (!safe || !ok) {
        // the CUDA-core body redoes this chunk (it rewrites the whole pack)
        if (tid == 0) {
            if (!ok) atomicExch(status, KDA_ERR_TIMEOUT);
            const int slot = atomicAdd(list, 1);
            list[1 + slot] = (b * H + h) * nch + ch;
        }
    } else {
        // ---- L = diag(beta) L' (strict lower). T = (I + L)^-1 as in the CUDA-core body.
        for (int e = tid; e < C * C; e += NT) {
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
            for (int e = tid; e < npairs * 256; e += NT) {
                const int pr = e / 256, i = (e % 256) / 16, j = e % 16;
                const int bb = pr, aa = pr + dist;
                float acc = 0.f;
                for (int cb2 = bb; cb2 < aa; ++cb2)
#pragma unroll
                    for (int m2 = 0; m2 < 16; ++m2)
                        acc = fmaf(sL[(16 * aa + i) * PC + 16 * cb2 + m2], sT[(16 * cb2 + m2) * PC + 16 * bb + j], acc);
                sTmp[pr * 256 + i * 16 + j] = acc;
            }
            __syncthreads();
            for (int e = tid; e < npairs * 256; e += NT) {
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
        for (int e = tid; e < C * C; e += NT) {
            const int i = e / C, j = e % C;
            if (j <= i) sT[i * PC + j] *= sB[j];
        }
        __syncthreads();
        // ---- M' = M Tb on the tensor cores (M = 64, N = 64, K = 64): A = M (K-major),
        //      B = Tb (MN-major: element (l, j) = Tb[j][l]); operands reuse the A region.
        uint8_t *sA2a = sA, *sA2b = sA + 16384;
        {
            const int r = tid >> 3, c0 = 8 * (tid & 7);  // one 8-column chunk of one row per thread
            float xm[8], xt[8];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const int c = c0 + w;
                xm[w] = c <= r ? sM[r * PC + c] : 0.f;
                xt[w] = c <= r ? sT[r * PC + c] : 0.f;
            }
            st_pair(sA2a, 8192, kmaj_off(r, c0, 64), xm);
            st_pair(sA2b, 8192, mnmaj_off(c0, r, 64), xt);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const uint32_t tM = tmem + I::NB;  // columns 160..223
        if (tid == 0) {
            constexpr uint32_t id = idesc_bf16(64, 64, false, true);
            const uint32_t a0 = smem_u32(sA2a), b0 = smem_u32(sA2b);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t ah = kmaj_desc(a0, 64, 0, ks), al = kmaj_desc(a0 + 8192, 64, 0, ks);
                const uint64_t bh = mnmaj_desc(b0, 64, 0, ks), bl = mnmaj_desc(b0 + 8192, 64, 0, ks);
                mma_bf16(tM, ah, bh, id, ks > 0 ? 1u : 0u);
                mma_bf16(tM, ah, bl, id, 1);
                mma_bf16(tM, al, bh, id, 1);
            }
            mma_commit(bar);
        }
        // rows 0..63 of [Tb; M']: Tb, written while M' is computed
        uint8_t *dst = pack + PK::OFF_A2;
        {
            const int row = tid >> 3, c0 = 8 * (tid & 7);
            float x[8];
#pragma unroll
            for (int w = 0; w < 8; ++w) x[w] = c0 + w <= row ? sT[row * PC + c0 + w] : 0.f;
            uint4 hi, lo;
            split8(x, hi, lo);
            const uint32_t off = kmaj_off(row, c0, 128);
            *reinterpret_cast<uint4 *>(dst + off) = hi;
            *reinterpret_cast<uint4 *>(dst + kTileBytes + off) = lo;
        }
        // rows 64..127: M' from TMEM (M = 64 layout: row 16 q + lane in lanes < 16 of quad q)
        const bool ok2 = mbar_wait(bar, 1, kWaitCycles);
        tc_fence_after();
        if (!ok2 && tid == 0) atomicExch(status, KDA_ERR_TIMEOUT);
        {
            const int quad = warp & 3, part = warp >> 2;
            const int row = 16 * quad + lane;
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                float x[8];
                tmem_ld8(tmem_lane_base(tM, warp) + 16 * part + 8 * h8, x);
                tmem_ld_wait();
                if (lane < 16 && ok2) {
                    uint4 hi, lo;
                    split8(x, hi, lo);
                    const uint32_t off = kmaj_off(64 + row, 16 * part + 8 * h8, 128);
                    *reinterpret_cast<uint4 *>(dst + off) = hi;
                    *reinterpret_cast<uint4 *>(dst + kTileBytes + off) = lo;
                }
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ================================================================ phase 2: state pass

template <int D, int DVS>
struct State {
    using PK = Pack<D>;
    static constexpr int NB = DVS < 64 ? 64 : DVS;  // MN-major B tiles span whole 64-wide atoms
    static constexpr int B1 = 2 * NB * D * 2;       // S0 hi + lo, MN-major (N = value columns, K = D keys)
    static constexpr int B2 = 2 * NB * C * 2;       // R, then U: hi + lo, MN-major (N = value columns, K = 64)
    static constexpr int VP = DVS + 4;              // V row stride (floats): 16-byte skew per row
    static constexpr int VS = C * VP * 4;           // V rows of the slice, FP32 (prefetched)
    // A1, A2, A3 at the front, in the pack's own order and sizes
    static constexpr int OFF_A1 = 0, OFF_A2 = PK::A1, OFF_A3 = PK::A1 + PK::A2, OFF_B1 = OFF_A3 + PK::A3,
                         OFF_B2 = OFF_B1 + B1, OFF_V = OFF_B2 + B2, OFF_MISC = OFF_V + VS;
    static constexpr int MISC = 1024;
    static constexpr int bytes = OFF_MISC + MISC + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = 3 * DVS <= 128 ? 128 : (3 * DVS <= 256 ? 256 : 512);
};

// 16-byte asynchronous global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Issue a bulk global -> shared copy of `bytes` (multiple of 16) completing on `bar`.
__device__ __forceinline__ void bulk_copy(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

template <int D, int DVS>
__global__ void __launch_bounds__(kThreads, 1)
state_kernel(const float *__restrict__ v, const uint8_t *__restrict__ scratch, float *const *__restrict__ h_state,
             float *__restrict__ core, int T, int T_pad, int H, float scale, int *__restrict__ status) {
    using S = State<D, DVS>;
    using PK = Pack<D>;
    constexpr int HALF = DVS / 2;  // value columns per thread in the epilogues
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA1 = sm + S::OFF_A1, *sA2 = sm + S::OFF_A2, *sA3 = sm + S::OFF_A3, *sB1 = sm + S::OFF_B1,
            *sB2 = sm + S::OFF_B2;
    float *sV = reinterpret_cast<float *>(sm + S::OFF_V);              // [C][VP]
    // barriers: 0/4/5 bulk copies of A1/A2/A3, 1..3 the three MMA groups
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::OFF_MISC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::OFF_MISC + 64);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int c0 = slice * DVS;
    const size_t rs = static_cast<size_t>(H) * D;
    float *Sg = h_state[b] + static_cast<size_t>(h) * D * D;
    const int nch = T_pad / C;
    const uint8_t *packs = scratch + (static_cast<size_t>(b) * H + h) * nch * PK::bytes;

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        bulk_copy(sA1, packs + PK::OFF_A1, PK::A1, &bars[0]);
        bulk_copy(sA2, packs + PK::OFF_A2, PK::A2, &bars[4]);
        bulk_copy(sA3, packs + PK::OFF_A3, PK::A3, &bars[5]);
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

    // Epilogue roles: for an M = 128 accumulator warp w reads TMEM lanes 32(w%4)..+31 (rows),
    // value columns [(w/4) HALF, + HALF). D3 with D = 64 (M = 64) has rows 16 (w%4) + lane, lane < 16.
    const int quad = warp & 3, colh = warp >> 2;
    const int erow = 32 * quad + lane;
    const int ccol = colh * HALF;
    const int srow = (D == 128) ? erow : ((lane < 16) ? 16 * quad + lane : -1);

    // V rows of the slice for epilogue 1, prefetched one chunk ahead into shared memory: the
    // thread that reads row erow, columns [ccol, ccol + HALF) is the thread that copies them.
    auto prefetch_v = [&](int chn) {
        if (quad < 2) {
            const int nn = min(C, T - chn * C);
            const size_t r0 = static_cast<size_t>(b) * T_pad + static_cast<size_t>(chn) * C;
            const float *src = v + (r0 + (erow < nn ? erow : 0)) * rs + static_cast<size_t>(h) * D + c0 + ccol;
#pragma unroll
            for (int j = 0; j < HALF; j += 4) cp_async16(sV + erow * S::VP + ccol + j, src + j, erow < nn ? 16u : 0u);
        }
        cp_async_commit();
    };

    // FP32 master state slice: key row srow, value columns [ccol, ccol + HALF)
    float st[HALF];
    if (srow >= 0) {
#pragma unroll
        for (int j = 0; j < HALF; j += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(Sg + static_cast<size_t>(srow) * D + c0 + ccol + j);
            st[j] = x.x; st[j + 1] = x.y; st[j + 2] = x.z; st[j + 3] = x.w;
        }
    }
    // S0 into B1 (MN-major: element (n = value column, k = key row)), 16-byte chunks
    auto write_state_operand = [&]() {
        if (srow >= 0) {
#pragma unroll
            for (int j = 0; j < HALF; j += 8) {
                float x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) x[u] = st[j + u];
                st_pair(sB1, S::B1 / 2, mnmaj_off(ccol + j, srow, D), x);
            }
        }
    };
    write_state_operand();
    prefetch_v(0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

#pragma unroll 1
    for (int ch = 0; ch < nch; ++ch) {
        const int n = min(C, T - ch * C);
        const size_t row0 = static_cast<size_t>(b) * T_pad + static_cast<size_t>(ch) * C;
        const uint32_t par = ch & 1;
        const uint8_t *next = packs + static_cast<size_t>(ch + 1) * PK::bytes;
        const bool more = ch + 1 < nch;
        // e^{Gamma_C} of this thread's key row, read early (used in epilogue 3)
        const float ac = srow >= 0 ? reinterpret_cast<const float *>(packs + static_cast<size_t>(ch) * PK::bytes +
                                                                    PK::OFF_AC)[srow]
                                   : 0.f;
        // ---- MMA1: D1 = [K o A; Q o A] . S0   (A1 copied for this chunk)
        if (tid == 0 && ok) ok = mbar_wait(&bars[0], par, kWaitCycles);
        if (tid == 0 && ok) {
            constexpr uint32_t id = idesc_bf16(128, DVS, false, true);
            const uint32_t a0 = smem_u32(sA1), b0 = smem_u32(sB1);
            int acc = 0;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t ah = kmaj_desc(a0, 128, 0, ks), al = kmaj_desc(a0 + PK::A1 / 2, 128, 0, ks);
                const uint64_t bh = mnmaj_desc(b0, D, 0, ks), bl = mnmaj_desc(b0 + S::B1 / 2, D, 0, ks);
                mma_bf16(tD1, ah, bh, id, acc); acc = 1;
                mma_bf16(tD1, ah, bl, id, 1);
                mma_bf16(tD1, al, bh, id, 1);
            }
            mma_commit(&bars[1]);
        }
        // e1: the Q half of D1 kept for the output (rows 64..127, quads 2 and 3)
        float e1[HALF];
        cp_async_wait_all();  // this thread's V rows of this chunk are in sV
        ok = ok && mbar_wait(&bars[1], par, kWaitCycles);
        tc_fence_after();
        if (tid == 0 && ok && more) bulk_copy(sA1, next + PK::OFF_A1, PK::A1, &bars[0]);  // A1 is free again
        // ---- epilogue 1: R = V - D1[0:64] -> B2 (MN-major: element (n = value column, k = token))
#pragma unroll
        for (int j = 0; j < HALF; j += 8) {
            float x[8];
            tmem_ld8(tmem_lane_base(tD1, warp) + ccol + j, x);
            tmem_ld_wait();
            if (quad < 2) {
                const float4 v0 = *reinterpret_cast<const float4 *>(sV + erow * S::VP + ccol + j);
                const float4 v1 = *reinterpret_cast<const float4 *>(sV + erow * S::VP + ccol + j + 4);
                const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int u = 0; u < 8; ++u) x[u] = vv[u] - x[u];
                st_pair(sB2, S::B2 / 2, mnmaj_off(ccol + j, erow, C), x);
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) e1[j + u] = x[u];
            }
        }
        if (more) prefetch_v(ch + 1);  // this thread is done with its V rows of this chunk
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        tc_fence_after();
        // ---- MMA2: D2 = [Tb; M'] . R
        if (tid == 0 && ok) ok = mbar_wait(&bars[4], par, kWaitCycles);
        if (tid == 0 && ok) {
            constexpr uint32_t id = idesc_bf16(128, DVS, false, true);
            const uint32_t a0 = smem_u32(sA2), b0 = smem_u32(sB2);
            int acc = 0;
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t ah = kmaj_desc(a0, 128, 0, ks), al = kmaj_desc(a0 + kTileBytes, 128, 0, ks);
                const uint64_t bh = mnmaj_desc(b0, C, 0, ks), bl = mnmaj_desc(b0 + S::B2 / 2, C, 0, ks);
                mma_bf16(tD2, ah, bh, id, acc); acc = 1;
                mma_bf16(tD2, ah, bl, id, 1);
                mma_bf16(tD2, al, bh, id, 1);
            }
            mma_commit(&bars[2]);
        }
        ok = ok && mbar_wait(&bars[2], par, kWaitCycles);
        tc_fence_after();
        if (tid == 0 && ok && more) bulk_copy(sA2, next + PK::OFF_A2, PK::A2, &bars[4]);  // A2 is free again
        // ---- epilogue 2: U = D2[0:64] -> B2 (R is consumed); O = scale (D1[64:] + D2[64:])
#pragma unroll
        for (int j = 0; j < HALF; j += 8) {
            float x[8];
            tmem_ld8(tmem_lane_base(tD2, warp) + ccol + j, x);
            tmem_ld_wait();
            if (quad < 2) {
                st_pair(sB2, S::B2 / 2, mnmaj_off(ccol + j, erow, C), x);
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
        if (tid == 0 && ok) ok = mbar_wait(&bars[5], par, kWaitCycles);
        if (tid == 0 && ok) {
            constexpr uint32_t id = idesc_bf16(D, DVS, true, true);
            const uint32_t a0 = smem_u32(sA3), b0 = smem_u32(sB2);
            int acc = 0;
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t ah = mnmaj_desc(a0, C, 0, ks), al = mnmaj_desc(a0 + PK::A3 / 2, C, 0, ks);
                const uint64_t bh = mnmaj_desc(b0, C, 0, ks), bl = mnmaj_desc(b0 + S::B2 / 2, C, 0, ks);
                mma_bf16(tD3, ah, bh, id, acc); acc = 1;
                mma_bf16(tD3, ah, bl, id, 1);
                mma_bf16(tD3, al, bh, id, 1);
            }
            mma_commit(&bars[3]);
        }
        ok = ok && mbar_wait(&bars[3], par, kWaitCycles);
        tc_fence_after();
        if (tid == 0 && ok && more) bulk_copy(sA3, next + PK::OFF_A3, PK::A3, &bars[5]);  // A3 is free again
        // ---- epilogue 3: S = A_C o S0 + D3 (FP32 in registers), S into B1
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

// Scratch layout: the operand packs, then a 256-byte slot with the count of chunks the
// tensor-core intra kernel handed to the CUDA-core body, then their (b, h, chunk) ids.
template <int D>
size_t packs_bytes(int B, int H, int nch) { return static_cast<size_t>(B) * H * nch * Pack<D>::bytes; }

template <int D, int DVS>
int launch_tc(const float *q, const float *k, const float *v, const float *gate, const float *beta,
              float *const *h_state, float *core, int B, int T, int H, float scale, void *scratch, cudaStream_t s) {
    const int T_pad = static_cast<int>(kda_t_pad(static_cast<size_t>(T), C));
    const int nch = T_pad / C;
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    static bool attrs = false;
    if (!attrs) {
        KDA_TRY(set_smem(intra_tc_kernel<D>, IntraTC<D>::bytes));
        KDA_TRY(set_smem(intra_fix_kernel<D>, static_cast<int>(Intra<D>::bytes)));
        KDA_TRY(set_smem(state_kernel<D, DVS>, State<D, DVS>::bytes));
        attrs = true;
    }
    uint8_t *sc = static_cast<uint8_t *>(scratch);
    int *list = reinterpret_cast<int *>(sc + packs_bytes<D>(B, H, nch));
    if (cudaMemsetAsync(list, 0, sizeof(int), s) != cudaSuccess) return KDA_ERR_CUDA;
    intra_tc_kernel<D><<<dim3(nch, H, B), kIntraThreads, IntraTC<D>::bytes, s>>>(k, q, gate, beta, sc, list, T, T_pad,
                                                                                 H, status);
    KDA_TRY(launch_status());
    int sms = 148;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int fix_grid = static_cast<int>(std::min<long long>(static_cast<long long>(B) * H * nch, sms));
    intra_fix_kernel<D><<<fix_grid, kIntraThreads, Intra<D>::bytes, s>>>(k, q, gate, beta, sc, list, T, T_pad, H);
    KDA_TRY(launch_status());
    state_kernel<D, DVS><<<dim3(D / DVS, H, B), kThreads, State<D, DVS>::bytes, s>>>(
        v, sc, h_state, core, T, T_pad, H, scale, status);
    return launch_status();
}

}  // namespace

size_t chunk_prefill_scratch_bytes(int B, int T, int H, int D) {
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    const int nch = static_cast<int>(kda_t_pad(static_cast<size_t>(T), C) / C);
    const size_t packs = D == 64 ? packs_bytes<64>(B, H, nch) : packs_bytes<128>(B, H, nch);
    const size_t list = (4 + 4 * static_cast<size_t>(B) * H * nch + 255) / 256 * 256;
    return packs + list;
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
