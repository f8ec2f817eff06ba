// Chunked KDA prefill on CUDA cores, FP32 (Glm5NextKdaLayer `prefill`, `kda_chunk_*`;
// Glm5NextKdaWorkspace fields q_f32/k_f32/v_f32/gate/beta -> core; Glm5NextLayer
// `prefill_gdn_full_batched` for B equal-length streams with a device state-pointer array).
//
// One CTA per (stream b, head h, value slice of DVS columns); it walks the chunks of its
// stream in order, carrying its [D x DVS] slice of the state in shared memory. Columns of
// the state evolve independently (the update S += k u^T and the read-out act column by
// column), so the value slices need no communication. Per chunk of C = 64 tokens, with
// Gamma the in-chunk inclusive cumulative log-decay per key channel:
//   L[i][j] = beta_i sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc}   (i > j)
//   M[i][j] =        sum_c q_ic k_jc e^{Gamma_ic - Gamma_jc}   (i >= j)
//   T = (I + L)^-1 (unit lower triangular; 16x16 diagonal blocks by substitution, then
//       the off-diagonal blocks T_ab = -T_aa sum_{b<=c<a} L_ac T_cb by block distance)
//   W = T diag(beta) (K o e^Gamma),  U~ = T diag(beta) V,  U = U~ - W S0
//   O = scale ((Q o e^Gamma) S0 + M U)
//   S = diag(e^{Gamma_C}) S0 + (K o e^{Gamma_C - Gamma})^T U
// Every exponent above is <= 0 (g <= 0, i >= j), so nothing overflows. Rows >= T of the
// last chunk are loaded as zeros (k = q = v = 0, g = 0, beta = 0): the pad guard; they
// then neither decay nor update the state, and their outputs are not written.
#include "common.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int C = kChunk;  // 64

template <int D, int DVS>
struct SimtSmem {
    static constexpr int P = D + 1;    // row stride of the [C][D] tiles
    static constexpr int PC = C + 1;   // row stride of the [C][C] tiles
    static constexpr size_t floats = 4 * C * P + 3 * C * PC + D * DVS + 2 * C * DVS + 3 * 256 + C + D;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int D, int DVS>
__global__ void __launch_bounds__(kThreads, 1)
chunk_simt_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
                  const float *__restrict__ gate, const float *__restrict__ beta, float *const *__restrict__ h_state,
                  float *__restrict__ core, int T, int T_pad, int H, float scale) {
    using SM = SimtSmem<D, DVS>;
    constexpr int P = SM::P, PC = SM::PC;
    extern __shared__ float smem[];
    float *sK = smem;              // k, later K o e^{Gamma_C - Gamma}
    float *sQ = sK + C * P;        // q, later Q o e^Gamma
    float *sG = sQ + C * P;        // g, then Gamma, then W
    float *sX = sG + C * P;        // beta K o e^Gamma
    float *sL = sX + C * P;        // L (strict lower, with beta)
    float *sM = sL + C * PC;       // M (lower incl. diagonal)
    float *sT = sM + C * PC;       // (I + L)^-1
    float *sS = sT + C * PC;       // state slice [D][DVS]
    float *sV = sS + D * DVS;      // beta V slice, later U~
    float *sU = sV + C * DVS;      // U
    float *sTmp = sU + C * DVS;    // 3 x 16x16 block products
    float *sB = sTmp + 3 * 256;    // beta [C]
    float *sAC = sB + C;           // e^{Gamma_C} [D]

    const int tid = threadIdx.x;
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int c0 = slice * DVS;
    float *Sg = h_state[b] + static_cast<size_t>(h) * D * D;
    const size_t rowstride = static_cast<size_t>(H) * D;

    for (int e = tid; e < D * DVS; e += kThreads) sS[e] = Sg[(e / DVS) * D + c0 + e % DVS];

    const int nchunks = T_pad / C;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int n = min(C, T - ch * C);  // valid rows in this chunk (>= 1)
        const size_t row0 = static_cast<size_t>(b) * T_pad + static_cast<size_t>(ch) * C;
        __syncthreads();
        // ---- load (pad guard: rows >= n are zero)
        for (int e = tid; e < C * D; e += kThreads) {
            const int i = e / D, c = e % D;
            float kv = 0.f, qv = 0.f, gv = 0.f;
            if (i < n) {
                const size_t off = (row0 + i) * rowstride + static_cast<size_t>(h) * D + c;
                kv = k[off]; qv = q[off]; gv = gate[off];
            }
            sK[i * P + c] = kv; sQ[i * P + c] = qv; sG[i * P + c] = gv;
        }
        for (int e = tid; e < C * DVS; e += kThreads) {
            const int i = e / DVS, cc = e % DVS;
            sV[i * DVS + cc] = i < n ? v[(row0 + i) * rowstride + static_cast<size_t>(h) * D + c0 + cc] : 0.f;
        }
        if (tid < C) sB[tid] = tid < n ? beta[(row0 + tid) * H + h] : 0.f;
        __syncthreads();
        // ---- Gamma: inclusive cumulative sum over the chunk, per key channel
        if (tid < D) {
            float acc = 0.f;
            for (int i = 0; i < C; ++i) { acc += sG[i * P + tid]; sG[i * P + tid] = acc; }
        }
        __syncthreads();
        // ---- L and M: 4x4 tiles (ti >= tj) of the 64x64 lower triangle, one per thread
        if (tid < 136) {
            int ti = 0, tj = tid;
            while (tj > ti) { tj -= ti + 1; ++ti; }
            float l[4][4], m[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s = 0; s < 4; ++s) { l[r][s] = 0.f; m[r][s] = 0.f; }
            for (int c = 0; c < D; ++c) {
                float gi[4], ki[4], qi[4], gj[4], kj[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    gi[r] = sG[(4 * ti + r) * P + c]; ki[r] = sK[(4 * ti + r) * P + c]; qi[r] = sQ[(4 * ti + r) * P + c];
                    gj[r] = sG[(4 * tj + r) * P + c]; kj[r] = sK[(4 * tj + r) * P + c];
                }
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        if (ti > tj || r >= s) {
                            const float ex = __expf(gi[r] - gj[s]);
                            l[r][s] = fmaf(ki[r] * kj[s], ex, l[r][s]);
                            m[r][s] = fmaf(qi[r] * kj[s], ex, m[r][s]);
                        }
                    }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const int i = 4 * ti + r, j = 4 * tj + s;
                    sL[i * PC + j] = i > j ? sB[i] * l[r][s] : 0.f;
                    sM[i * PC + j] = i >= j ? m[r][s] : 0.f;
                    if (ti != tj) { sL[j * PC + i] = 0.f; sM[j * PC + i] = 0.f; }
                }
        }
        __syncthreads();
        // ---- T = (I + L)^-1. Diagonal 16x16 blocks: column j of block a by substitution.
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
        // zero the strictly upper blocks of T
        for (int e = tid; e < C * C; e += kThreads) {
            const int i = e / C, j = e % C;
            if ((j / 16) > (i / 16)) sT[i * PC + j] = 0.f;
        }
        __syncthreads();
        // off-diagonal blocks by distance: X = sum_{b<=c<a} L_ac T_cb ; T_ab = -T_aa X
        for (int dist = 1; dist < 4; ++dist) {
            const int npairs = 4 - dist;
            for (int e = tid; e < npairs * 256; e += kThreads) {
                const int pr = e / 256, i = (e % 256) / 16, j = e % 16;
                const int bb = pr, aa = pr + dist;
                float acc = 0.f;
                for (int cb = bb; cb < aa; ++cb)
                    for (int m2 = 0; m2 < 16; ++m2)
                        acc = fmaf(sL[(16 * aa + i) * PC + 16 * cb + m2], sT[(16 * cb + m2) * PC + 16 * bb + j], acc);
                sTmp[pr * 256 + i * 16 + j] = acc;
            }
            __syncthreads();
            for (int e = tid; e < npairs * 256; e += kThreads) {
                const int pr = e / 256, i = (e % 256) / 16, j = e % 16;
                const int bb = pr, aa = pr + dist;
                float acc = 0.f;
                for (int m2 = 0; m2 < 16; ++m2)
                    acc = fmaf(sT[(16 * aa + i) * PC + 16 * aa + m2], sTmp[pr * 256 + m2 * 16 + j], acc);
                sT[(16 * aa + i) * PC + 16 * bb + j] = -acc;
            }
            __syncthreads();
        }
        // ---- decay-weighted operands
        if (tid < D) sAC[tid] = __expf(sG[(C - 1) * P + tid]);
        __syncthreads();
        for (int e = tid; e < C * D; e += kThreads) {
            const int i = e / D, c = e % D;
            const float gm = sG[i * P + c];
            const float kk = sK[i * P + c];
            const float eg = __expf(gm);
            sX[i * P + c] = sB[i] * kk * eg;
            sQ[i * P + c] *= eg;
            sK[i * P + c] = kk * __expf(sG[(C - 1) * P + c] - gm);
        }
        for (int e = tid; e < C * DVS; e += kThreads) sV[e] *= sB[e / DVS];
        __syncthreads();
        // ---- W = T X  (into sG) and U~ = T (beta V)  (into sU)
        {
            constexpr int G = kThreads / D;   // row groups
            constexpr int R = C / G;          // rows per thread
            const int c = tid % D, rg = tid / D;
            float acc[R];
#pragma unroll
            for (int r = 0; r < R; ++r) acc[r] = 0.f;
            for (int j = 0; j < C; ++j) {
                const float xv = sX[j * P + c];
#pragma unroll
                for (int r = 0; r < R; ++r) acc[r] = fmaf(sT[(rg + G * r) * PC + j], xv, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) sG[(rg + G * r) * P + c] = acc[r];
        }
        {
            constexpr int G = kThreads / DVS, R = C / G;
            const int cc = tid % DVS, rg = tid / DVS;
            float acc[R];
#pragma unroll
            for (int r = 0; r < R; ++r) acc[r] = 0.f;
            for (int j = 0; j < C; ++j) {
                const float vv = sV[j * DVS + cc];
#pragma unroll
                for (int r = 0; r < R; ++r) acc[r] = fmaf(sT[(rg + G * r) * PC + j], vv, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) sU[(rg + G * r) * DVS + cc] = acc[r];
        }
        __syncthreads();
        // ---- U = U~ - W S0 ; O = scale (Q^ S0 + M U)
        {
            constexpr int G = kThreads / DVS, R = C / G;
            const int cc = tid % DVS, rg = tid / DVS;
            float u[R], o[R];
#pragma unroll
            for (int r = 0; r < R; ++r) { u[r] = 0.f; o[r] = 0.f; }
            for (int c = 0; c < D; ++c) {
                const float sv = sS[c * DVS + cc];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    u[r] = fmaf(sG[(rg + G * r) * P + c], sv, u[r]);
                    o[r] = fmaf(sQ[(rg + G * r) * P + c], sv, o[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) u[r] = sU[(rg + G * r) * DVS + cc] - u[r];
            __syncthreads();
#pragma unroll
            for (int r = 0; r < R; ++r) sU[(rg + G * r) * DVS + cc] = u[r];
            __syncthreads();
            for (int j = 0; j < C; ++j) {
                const float uv = sU[j * DVS + cc];
#pragma unroll
                for (int r = 0; r < R; ++r) o[r] = fmaf(sM[(rg + G * r) * PC + j], uv, o[r]);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int i = rg + G * r;
                if (i < n) core[(row0 + i) * rowstride + static_cast<size_t>(h) * D + c0 + cc] = scale * o[r];
            }
        }
        // ---- S = diag(e^{Gamma_C}) S0 + Kbar^T U   (each thread updates its own entries)
        {
            constexpr int G = kThreads / DVS, R = D / G;
            const int cc = tid % DVS, rg = tid / DVS;
            float acc[R];
#pragma unroll
            for (int r = 0; r < R; ++r) acc[r] = 0.f;
            for (int j = 0; j < C; ++j) {
                const float uv = sU[j * DVS + cc];
#pragma unroll
                for (int r = 0; r < R; ++r) acc[r] = fmaf(sK[j * P + rg + G * r], uv, acc[r]);
            }
            __syncthreads();  // every read of S0 above (U, O) is done
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int c = rg + G * r;
                sS[c * DVS + cc] = fmaf(sAC[c], sS[c * DVS + cc], acc[r]);
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < D * DVS; e += kThreads) Sg[(e / DVS) * D + c0 + e % DVS] = sS[e];
}

template <int D, int DVS>
int launch_simt(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                float *const *h_state, float *core, int B, int T, int H, float scale, cudaStream_t s) {
    using SM = SimtSmem<D, DVS>;
    static std::atomic<unsigned long long> attr_done{0};
    KDA_TRY(smem_opt_in(chunk_simt_kernel<D, DVS>, static_cast<int>(SM::bytes), attr_done));
    const int T_pad = static_cast<int>(kda_t_pad(static_cast<size_t>(T), C));
    dim3 grid(D / DVS, H, B);
    chunk_simt_kernel<D, DVS><<<grid, kThreads, SM::bytes, s>>>(q, k, v, gate, beta, h_state, core, T, T_pad, H, scale);
    return launch_status();
}

}  // namespace

int chunk_prefill_check(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                        float *const *h_state, float *core, int B, int T, const kda_dims *dims) {
    KDA_TRY(check_dims(dims));
    if (!q || !k || !v || !gate || !beta || !h_state || !core || B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(core))
        return KDA_ERR_MISALIGNED;
    if (B > 65535 || dims->heads > 65535) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

int chunk_prefill_simt(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                       float *const *h_state, float *core, int B, int T, const kda_dims *dims, cudaStream_t s) {
    if (dims->head_dim == 128)
        return launch_simt<128, 32>(q, k, v, gate, beta, h_state, core, B, T, dims->heads, dims->scale, s);
    return launch_simt<64, 32>(q, k, v, gate, beta, h_state, core, B, T, dims->heads, dims->scale, s);
}

}  // namespace kda

extern "C" int kda_chunk_prefill_simt(const float *q, const float *k, const float *v, const float *gate,
                                      const float *beta, float *const *h_state, float *core, int B, int T,
                                      const kda_dims *dims, void *stream) {
    KDA_TRY(kda::chunk_prefill_check(q, k, v, gate, beta, h_state, core, B, T, dims));
    if (B == 0 || T == 0) return KDA_OK;
    return kda::chunk_prefill_simt(q, k, v, gate, beta, h_state, core, B, T, dims, static_cast<cudaStream_t>(stream));
}
