// KDA decode: one CTA per (sequence, head) streams that head's D x D FP32 state once in
// and once out (Glm5NextKdaLayer `decode`, `decode_k`; Glm5NextKdaWorkspace).
//
//   kda_recurrent_decode : the recurrence step alone, on pre-normalised F32 q/k/v/gate/beta.
//   kda_decode_fused     : the whole stateful row (conv + SiLU + L2, gate, beta, recurrence,
//                          sigmoid-gated RMSNorm) for N sequences, one token each.
//   kda_decode_k         : the same row K times for one sequence, state kept on chip,
//                          snapshots after each row but the last.
// decode_fused and decode_k launch the SAME kernel (N sequences x K rows), so every row
// executes identical device code; all arithmetic on the row uses explicitly rounded
// intrinsics (__fmul_rn / __fadd_rn / __fmaf_rn), which the compiler may not re-associate
// or contract differently — this is what makes decode_k bit-identical to K decodes.
//
// State thread layout (256 threads): D/4 threads per row, each holding a float4 column
// group; RG = 256/(D/4) row groups; thread (rg, c4) owns rows rg, rg+RG, ... (RPT rows).
// A warp therefore loads whole 512-byte (D=128) rows: coalesced 16-byte accesses.
#include "common.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;

template <int D>
struct Lay {
    static constexpr int TPR = D / 4;
    static constexpr int RG = kThreads / TPR;
    static constexpr int RPT = D / RG;
    static constexpr int NW = D / 32;  // warps spanned by threads 0..D-1
};

struct __align__(16) Smem {
    float q[128], k[128], v[128], a[128], u[128], o[128];
    float red[2][16][128];
    float wsum[2][8];
    float bcast[4];
};

// Sum of (x, y) over threads 0..D-1 in a fixed tree (same order on every call).
template <int D>
__device__ __forceinline__ float2 sum2_first_d(float x, float y, Smem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, o));
        y = __fadd_rn(y, __shfl_xor_sync(0xffffffffu, y, o));
    }
    if (lane == 0 && w < Lay<D>::NW) { sm.wsum[0][w] = x; sm.wsum[1][w] = y; }
    __syncthreads();
    float sx = sm.wsum[0][0], sy = sm.wsum[1][0];
#pragma unroll
    for (int i = 1; i < Lay<D>::NW; ++i) { sx = __fadd_rn(sx, sm.wsum[0][i]); sy = __fadd_rn(sy, sm.wsum[1][i]); }
    __syncthreads();
    return make_float2(sx, sy);
}

template <int D>
__device__ __forceinline__ void load_state(float4 (&st)[Lay<D>::RPT], const float *S) {
    const int rg = threadIdx.x / Lay<D>::TPR, c4 = threadIdx.x % Lay<D>::TPR;
#pragma unroll
    for (int r = 0; r < Lay<D>::RPT; ++r)
        st[r] = __ldcs(reinterpret_cast<const float4 *>(S + (rg + Lay<D>::RG * r) * D) + c4);
}

template <int D>
__device__ __forceinline__ void store_state(const float4 (&st)[Lay<D>::RPT], float *S, bool streaming) {
    const int rg = threadIdx.x / Lay<D>::TPR, c4 = threadIdx.x % Lay<D>::TPR;
#pragma unroll
    for (int r = 0; r < Lay<D>::RPT; ++r) {
        float4 *p = reinterpret_cast<float4 *>(S + (rg + Lay<D>::RG * r) * D) + c4;
        if (streaming) __stcs(p, st[r]); else *p = st[r];
    }
}

// One recurrence step on the register-resident state, with q,k,v,a(=exp g) in smem:
//   S' = diag(a) S;  y_k = S'^T k, y_q = S'^T q;  u = beta (v - y_k);  S = S' + k u^T;
//   o = scale (y_q + (k.q) u)   (= scale S^T q after the update).   o lands in sm.o.
template <int D>
__device__ __forceinline__ void state_step(float4 (&st)[Lay<D>::RPT], Smem &sm, float beta, float kq, float scale) {
    using L = Lay<D>;
    const int tid = threadIdx.x, rg = tid / L::TPR, c4 = tid % L::TPR;
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int r = 0; r < L::RPT; ++r) {
        const int row = rg + L::RG * r;
        const float a = sm.a[row], kr = sm.k[row], qr = sm.q[row];
        float4 s = st[r];
        s.x = __fmul_rn(s.x, a); s.y = __fmul_rn(s.y, a); s.z = __fmul_rn(s.z, a); s.w = __fmul_rn(s.w, a);
        st[r] = s;
        pk.x = __fmaf_rn(s.x, kr, pk.x); pk.y = __fmaf_rn(s.y, kr, pk.y);
        pk.z = __fmaf_rn(s.z, kr, pk.z); pk.w = __fmaf_rn(s.w, kr, pk.w);
        pq.x = __fmaf_rn(s.x, qr, pq.x); pq.y = __fmaf_rn(s.y, qr, pq.y);
        pq.z = __fmaf_rn(s.z, qr, pq.z); pq.w = __fmaf_rn(s.w, qr, pq.w);
    }
    *reinterpret_cast<float4 *>(&sm.red[0][rg][4 * c4]) = pk;
    *reinterpret_cast<float4 *>(&sm.red[1][rg][4 * c4]) = pq;
    __syncthreads();
    if (tid < D) {
        float yk = sm.red[0][0][tid], yq = sm.red[1][0][tid];
#pragma unroll
        for (int g = 1; g < L::RG; ++g) { yk = __fadd_rn(yk, sm.red[0][g][tid]); yq = __fadd_rn(yq, sm.red[1][g][tid]); }
        const float u = __fmul_rn(beta, __fsub_rn(sm.v[tid], yk));
        sm.u[tid] = u;
        sm.o[tid] = __fmul_rn(scale, __fmaf_rn(kq, u, yq));
    }
    __syncthreads();
    const float4 u4 = *reinterpret_cast<const float4 *>(&sm.u[4 * c4]);
#pragma unroll
    for (int r = 0; r < L::RPT; ++r) {
        const float kr = sm.k[rg + L::RG * r];
        float4 s = st[r];
        s.x = __fmaf_rn(kr, u4.x, s.x); s.y = __fmaf_rn(kr, u4.y, s.y);
        s.z = __fmaf_rn(kr, u4.z, s.z); s.w = __fmaf_rn(kr, u4.w, s.w);
        st[r] = s;
    }
}

__device__ __forceinline__ float sigmoid_rn(float x) {
    return __frcp_rn(__fadd_rn(1.0f, expf(-x)));
}

// ----------------------------------------------------------------------------- core-only decode

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
recurrent_decode_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
                        const float *__restrict__ gate, const float *__restrict__ beta,
                        float *const *__restrict__ h_state, float *__restrict__ o, int H, float scale) {
    __shared__ Smem sm;
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
    float *S = h_state[n] + static_cast<size_t>(h) * D * D;
    float4 st[Lay<D>::RPT];
    load_state<D>(st, S);
    const size_t row = (static_cast<size_t>(n) * H + h) * D;
    float qk = 0.f;
    if (tid < D) {
        const float qd = q[row + tid], kd = k[row + tid];
        sm.q[tid] = qd; sm.k[tid] = kd; sm.v[tid] = v[row + tid];
        sm.a[tid] = expf(gate[row + tid]);
        qk = __fmul_rn(qd, kd);
    }
    const float kq = sum2_first_d<D>(tid < D ? qk : 0.f, 0.f, sm).x;
    state_step<D>(st, sm, beta[static_cast<size_t>(n) * H + h], kq, scale);
    if (tid < D) o[row + tid] = sm.o[tid];
    store_state<D>(st, S, true);
}

// ----------------------------------------------------------------------------- fused stateful row

constexpr int kMaxSnap = 31;

struct RowParams {
    const uint16_t *x;          // [rows, 3*H*D]
    uint16_t *const *conv_arr;  // device array of N pointers, or null
    uint16_t *conv_one;         // single pointer (decode_k), or null
    const uint16_t *conv_w;     // [3*H*D, 4]
    const uint16_t *g_raw;      // [rows, H*D]
    const float *dt_bias, *a_log, *b_logit;
    float *const *h_arr;        // device array of N pointers, or null
    float *h_one;               // single pointer, or null
    const uint16_t *out_gate, *o_norm_w;
    uint16_t *o_norm_out, *conv_out;
    float *core;
    int H, K, n_snap;
    float scale, l2_eps, rms_eps;
    float *h_snap[kMaxSnap];
    uint16_t *conv_snap[kMaxSnap];
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2) decode_rows_kernel(const RowParams p) {
    __shared__ Smem sm;
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x, H = p.H;
    const int qkv = H * D;
    float *S = (p.h_one ? p.h_one : p.h_arr[n]) + static_cast<size_t>(h) * D * D;
    uint16_t *cst = p.conv_one ? p.conv_one : p.conv_arr[n];
    float4 st[Lay<D>::RPT];
    load_state<D>(st, S);

    // This thread's conv channels: q and k channel d (tid < D) or v channel d (D <= tid < 2D).
    const bool qk_thread = tid < D, v_thread = tid >= D && tid < 2 * D;
    const int d = qk_thread ? tid : tid - D;
    const int c0 = qk_thread ? h * D + d : 2 * qkv + h * D + d;  // q channel or v channel
    const int c1 = qkv + h * D + d;                              // k channel (qk threads)
    float w0[4] = {0, 0, 0, 0}, w1[4] = {0, 0, 0, 0}, s0[3] = {0, 0, 0}, s1[3] = {0, 0, 0};
    if (qk_thread || v_thread) {
#pragma unroll
        for (int j = 0; j < 4; ++j) w0[j] = bf16_to_f32(p.conv_w[c0 * 4 + j]);
#pragma unroll
        for (int j = 0; j < 3; ++j) s0[j] = bf16_to_f32(cst[c0 * 3 + j]);
        if (qk_thread) {
#pragma unroll
            for (int j = 0; j < 4; ++j) w1[j] = bf16_to_f32(p.conv_w[c1 * 4 + j]);
#pragma unroll
            for (int j = 0; j < 3; ++j) s1[j] = bf16_to_f32(cst[c1 * 3 + j]);
        }
    }
    const float nea = -expf(p.a_log[h]);
    const float dtb = qk_thread ? p.dt_bias[h * D + d] : 0.f;
    const float ow = qk_thread ? bf16_to_f32(p.o_norm_w[d]) : 0.f;

    for (int t = 0; t < p.K; ++t) {
        const size_t row = static_cast<size_t>(n) * p.K + t;
        // conv step + SiLU (fixed-order FP32), new conv state in registers
        float y0 = 0.f, y1 = 0.f;
        if (qk_thread || v_thread) {
            const float x0 = bf16_to_f32(p.x[row * 3 * qkv + c0]);
            y0 = __fmaf_rn(w0[3], x0, __fmaf_rn(w0[2], s0[2], __fmaf_rn(w0[1], s0[1], __fmul_rn(w0[0], s0[0]))));
            y0 = __fmul_rn(y0, sigmoid_rn(y0));
            s0[0] = s0[1]; s0[1] = s0[2]; s0[2] = x0;
            if (qk_thread) {
                const float x1 = bf16_to_f32(p.x[row * 3 * qkv + c1]);
                y1 = __fmaf_rn(w1[3], x1, __fmaf_rn(w1[2], s1[2], __fmaf_rn(w1[1], s1[1], __fmul_rn(w1[0], s1[0]))));
                y1 = __fmul_rn(y1, sigmoid_rn(y1));
                s1[0] = s1[1]; s1[1] = s1[2]; s1[2] = x1;
            }
        }
        // per-head L2 of q and k (one BF16 rounding after the norm), v rounded as is
        const float2 ss = sum2_first_d<D>(qk_thread ? __fmul_rn(y0, y0) : 0.f, qk_thread ? __fmul_rn(y1, y1) : 0.f, sm);
        float qv = 0.f, kv = 0.f;
        if (qk_thread) {
            const uint16_t qb = f32_to_bf16(__fmul_rn(y0, rsqrtf(__fadd_rn(ss.x, p.l2_eps))));
            const uint16_t kb = f32_to_bf16(__fmul_rn(y1, rsqrtf(__fadd_rn(ss.y, p.l2_eps))));
            qv = bf16_to_f32(qb); kv = bf16_to_f32(kb);
            sm.q[d] = qv; sm.k[d] = kv;
            if (p.conv_out) { p.conv_out[row * 3 * qkv + c0] = qb; p.conv_out[row * 3 * qkv + c1] = kb; }
            // gate for key channel d, and beta
            const float g = kda_gate_f32(bf16_to_f32(p.g_raw[row * qkv + h * D + d]), dtb, nea);
            sm.a[d] = expf(g);
        } else if (v_thread) {
            const uint16_t vb = f32_to_bf16(y0);
            sm.v[d] = bf16_to_f32(vb);
            if (p.conv_out) p.conv_out[row * 3 * qkv + c0] = vb;
        }
        const float beta = sigmoid_rn(p.b_logit[row * H + h]);
        const float kq = sum2_first_d<D>(qk_thread ? __fmul_rn(qv, kv) : 0.f, 0.f, sm).x;
        state_step<D>(st, sm, beta, kq, p.scale);
        // o_norm: sigmoid-gated RMSNorm over the head's D outputs
        const float ov = qk_thread ? sm.o[d] : 0.f;
        const float ms = sum2_first_d<D>(qk_thread ? __fmul_rn(ov, ov) : 0.f, 0.f, sm).x;
        if (qk_thread) {
            const float rs = rsqrtf(__fadd_rn(__fmul_rn(ms, 1.0f / D), p.rms_eps));
            const float og = bf16_to_f32(p.out_gate[row * qkv + h * D + d]);
            const float yv = __fmul_rn(__fmul_rn(__fmul_rn(ov, rs), ow), sigmoid_rn(og));
            p.o_norm_out[row * qkv + h * D + d] = f32_to_bf16(yv);
            if (p.core) p.core[row * qkv + h * D + d] = ov;
        }
        if (t < p.n_snap) {
            store_state<D>(st, p.h_snap[t] + static_cast<size_t>(h) * D * D, false);
            uint16_t *cs = p.conv_snap[t];
            if (qk_thread || v_thread) {
#pragma unroll
                for (int j = 0; j < 3; ++j) cs[c0 * 3 + j] = f32_to_bf16(s0[j]);
                if (qk_thread) {
#pragma unroll
                    for (int j = 0; j < 3; ++j) cs[c1 * 3 + j] = f32_to_bf16(s1[j]);
                }
            }
        }
        __syncthreads();  // smem rows are rewritten by the next row
    }
    store_state<D>(st, S, true);
    if (qk_thread || v_thread) {
#pragma unroll
        for (int j = 0; j < 3; ++j) cst[c0 * 3 + j] = f32_to_bf16(s0[j]);
        if (qk_thread) {
#pragma unroll
            for (int j = 0; j < 3; ++j) cst[c1 * 3 + j] = f32_to_bf16(s1[j]);
        }
    }
}

int launch_rows(const RowParams &p, int N, int D, cudaStream_t s) {
    dim3 grid(p.H, N);
    if (D == 128) decode_rows_kernel<128><<<grid, kThreads, 0, s>>>(p);
    else decode_rows_kernel<64><<<grid, kThreads, 0, s>>>(p);
    return launch_status();
}

}  // namespace
}  // namespace kda

extern "C" {

int kda_recurrent_decode(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                         float *const *h_state, float *o, int N, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!q || !k || !v || !gate || !beta || !h_state || !o || N < 0) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(q) || !kda::aligned16(k) || !kda::aligned16(v) || !kda::aligned16(gate) || !kda::aligned16(o))
        return KDA_ERR_MISALIGNED;
    if (N == 0) return KDA_OK;
    if (N > 65535) return KDA_ERR_UNSUPPORTED;
    dim3 grid(dims->heads, N);
    auto s = static_cast<cudaStream_t>(stream);
    if (dims->head_dim == 128)
        kda::recurrent_decode_kernel<128><<<grid, kda::kThreads, 0, s>>>(q, k, v, gate, beta, h_state, o, dims->heads, dims->scale);
    else
        kda::recurrent_decode_kernel<64><<<grid, kda::kThreads, 0, s>>>(q, k, v, gate, beta, h_state, o, dims->heads, dims->scale);
    return kda::launch_status();
}

static int fill_row_params(kda::RowParams &p, const kda_bf16 *x, const kda_bf16 *conv_w, const kda_bf16 *g_raw,
                           const float *dt_bias, const float *a_log, const float *b_logit, const kda_bf16 *out_gate,
                           const kda_bf16 *o_norm_w, kda_bf16 *o_norm_out, kda_bf16 *conv_out, float *core,
                           int rows, const kda_dims *dims) {
    KDA_TRY(kda::check_dims(dims));
    if (!x || !conv_w || !g_raw || !dt_bias || !a_log || !b_logit || !out_gate || !o_norm_w || !o_norm_out)
        return KDA_ERR_INVALID_ARG;
    const size_t qkv = static_cast<size_t>(dims->heads) * dims->head_dim;
    if (kda::overlaps(g_raw, rows * qkv * 2, out_gate, rows * qkv * 2)) return KDA_ERR_ALIAS;
    p = kda::RowParams{};
    p.x = x; p.conv_w = conv_w; p.g_raw = g_raw; p.dt_bias = dt_bias; p.a_log = a_log; p.b_logit = b_logit;
    p.out_gate = out_gate; p.o_norm_w = o_norm_w; p.o_norm_out = o_norm_out; p.conv_out = conv_out; p.core = core;
    p.H = dims->heads; p.scale = dims->scale; p.l2_eps = dims->l2_eps; p.rms_eps = dims->rms_eps;
    return KDA_OK;
}

int kda_decode_fused(const kda_bf16 *x, kda_bf16 *const *conv_state, const kda_bf16 *conv_w, const kda_bf16 *g_raw,
                     const float *dt_bias, const float *a_log, const float *b_logit, float *const *h_state,
                     const kda_bf16 *out_gate, const kda_bf16 *o_norm_w, kda_bf16 *o_norm_out, kda_bf16 *conv_out,
                     float *core, int N, const kda_dims *dims, void *stream) {
    if (N < 0 || !conv_state || !h_state) return KDA_ERR_INVALID_ARG;
    if (N > 65535) return KDA_ERR_UNSUPPORTED;
    kda::RowParams p;
    KDA_TRY(fill_row_params(p, x, conv_w, g_raw, dt_bias, a_log, b_logit, out_gate, o_norm_w, o_norm_out, conv_out,
                            core, N, dims));
    if (N == 0) return KDA_OK;
    p.conv_arr = conv_state; p.h_arr = h_state; p.K = 1; p.n_snap = 0;
    return kda::launch_rows(p, N, dims->head_dim, static_cast<cudaStream_t>(stream));
}

int kda_decode_k(const kda_bf16 *x, kda_bf16 *conv_state, const kda_bf16 *conv_w, const kda_bf16 *g_raw,
                 const float *dt_bias, const float *a_log, const float *b_logit, float *h_state,
                 const kda_bf16 *out_gate, const kda_bf16 *o_norm_w, kda_bf16 *o_norm_out, kda_bf16 *conv_out,
                 float *core, int K, float *const *h_snap, kda_bf16 *const *conv_snap, int n_snap,
                 const kda_dims *dims, void *stream) {
    if (K < 1 || !conv_state || !h_state) return KDA_ERR_INVALID_ARG;
    if (K > kda::kMaxSnap + 1) return KDA_ERR_UNSUPPORTED;
    if (n_snap != 0 && n_snap != K - 1) return KDA_ERR_INVALID_ARG;
    if (n_snap > 0 && (!h_snap || !conv_snap)) return KDA_ERR_INVALID_ARG;
    kda::RowParams p;
    KDA_TRY(fill_row_params(p, x, conv_w, g_raw, dt_bias, a_log, b_logit, out_gate, o_norm_w, o_norm_out, conv_out,
                            core, K, dims));
    if (!kda::aligned16(h_state)) return KDA_ERR_MISALIGNED;
    for (int t = 0; t < n_snap; ++t) {
        if (!h_snap[t] || !conv_snap[t]) return KDA_ERR_INVALID_ARG;
        if (!kda::aligned16(h_snap[t])) return KDA_ERR_MISALIGNED;
        p.h_snap[t] = h_snap[t];
        p.conv_snap[t] = conv_snap[t];
    }
    p.conv_one = conv_state; p.h_one = h_state; p.K = K; p.n_snap = n_snap;
    return kda::launch_rows(p, 1, dims->head_dim, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
