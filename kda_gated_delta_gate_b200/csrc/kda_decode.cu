// KDA decode: one CTA per (sequence, head) streams that head's D x D FP32 state once in
// and once out (Glm5NextKdaLayer `decode`, `decode_k`; Glm5NextKdaWorkspace).
//
//   kda_recurrent_decode : the recurrence step alone, on pre-normalised F32 q/k/v/gate/beta.
//   kda_decode_fused     : the whole stateful row (conv + SiLU + L2, gate, beta, recurrence,
//                          sigmoid-gated RMSNorm) for N sequences, one token each.
//   kda_decode_k         : the same row K times for one sequence, state kept on chip,
//                          snapshots after each row but the last (groups of up to 32 rows
//                          per launch, chained through the state in place).
// decode_fused and decode_k launch the SAME kernel (N sequences x K rows), so every row
// executes identical device code; all arithmetic on the row uses explicitly rounded
// intrinsics (__fmul_rn / __fadd_rn / __fmaf_rn), which the compiler may not re-associate
// or contract differently — this is what makes decode_k bit-identical to K decodes.
//
// The state comes in through shared memory: one bulk copy brings the head's 64 KB in (issued
// first, so the row's small inputs load under it). The updated state goes straight from
// registers to global memory (coalesced 128-byte rows), so a CTA's slot frees as soon as its
// stores are issued; only decode_k keeps the state in shared memory between its rows. Low
// register use lets three CTAs share an SM, so three heads' state streams overlap on every
// SM. Thread layout (256 threads): thread t owns value column j = t % D and the row group
// t / D (RG = 256 / D groups of D / RG consecutive key rows); a warp reads 32 consecutive
// floats of one row, so shared-memory accesses are conflict-free.
#include "common.cuh"
#include "umma.cuh"

namespace kda {
namespace {

using umma::fence_mbar_init;
using umma::mbar_init;
using umma::smem_u32;

constexpr int kThreads = 256;
constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at 1.9 GHz

template <int D>
struct Lay {
    static constexpr int RG = kThreads / D;  // row groups: 2 (D = 128) or 4 (D = 64)
    static constexpr int RPG = D / RG;       // rows per group
    static constexpr int NW = D / 32;        // warps spanned by threads 0..D-1
};

template <int D>
struct __align__(16) Smem {
    float S[D * D];  // the head's state, row i = key channel i
    float q[2][D], k[2][D], v[2][D], a[2][D], o[D];  // a row's vectors, in two slots (rows alternate)
    float red[2][Lay<D>::RG][D];
    float wsum[2][2][8];  // two buffers: consecutive sums alternate (see sum2_first_d)
    uint64_t bar;
};

// Sum of (x, y) over threads 0..D-1 in a fixed tree (same order on every call). Consecutive calls
// alternate between the two wsum buffers (the caller's parity `par`, flipped here), so one barrier
// per call suffices: a buffer is written again two calls later, and every thread has finished
// reading it before it arrives at the barrier of the call in between.
template <int D>
__device__ __forceinline__ float2 sum2_first_d(float x, float y, Smem<D> &sm, int &par) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, o));
        y = __fadd_rn(y, __shfl_xor_sync(0xffffffffu, y, o));
    }
    float(&ws)[2][8] = sm.wsum[par];
    par ^= 1;
    if (lane == 0 && w < Lay<D>::NW) { ws[0][w] = x; ws[1][w] = y; }
    __syncthreads();
    float sx = ws[0][0], sy = ws[1][0];
#pragma unroll
    for (int i = 1; i < Lay<D>::NW; ++i) { sx = __fadd_rn(sx, ws[0][i]); sy = __fadd_rn(sy, ws[1][i]); }
    return make_float2(sx, sy);
}

// L2 policy for data touched once (the state streams).
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// One thread: bulk-copy the state (D*D floats) from global memory into sm.S, completing on sm.bar.
template <int D>
__device__ __forceinline__ void state_load_issue(Smem<D> &sm, const float *S) {
    constexpr uint32_t bytes = D * D * 4;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&sm.bar)), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(sm.S)),
        "l"(S), "r"(bytes), "r"(smem_u32(&sm.bar)), "l"(evict_first_policy())
        : "memory");
}

// Every thread: wait (bounded) for the state copy; false on timeout.
template <int D>
__device__ __forceinline__ bool state_load_wait(Smem<D> &sm) {
    return umma::mbar_wait(&sm.bar, 0, kWaitCycles);
}

// One recurrence step on the shared-memory state, with q,k,v,a(=exp g) in shared memory:
//   S' = diag(a) S;  y_k = S'^T k, y_q = S'^T q;  u = beta (v - y_k);  S = S' + k u^T;
//   o = scale (y_q + (k.q) u)   (= scale S^T q after the update): thread j < D stores o[j] to sm.o[j].
// The decayed value S'[i][j] is formed twice (once per pass) by the same rounded product.
// Pass 2 writes the new state to shared memory (keep), to global memory (g, streaming), to
// a snapshot (snap, plain stores), in any combination.
template <int D>
__device__ __forceinline__ void state_step(Smem<D> &sm, float beta, float kq, float scale, bool keep, float *g,
                                           float *snap) {
    using L = Lay<D>;
    const int tid = threadIdx.x, j = tid % D, grp = tid / D, r0 = grp * L::RPG;
    float pk = 0.f, pq = 0.f;
#pragma unroll 16
    for (int r = 0; r < L::RPG; ++r) {
        const int i = r0 + r;
        const float s = __fmul_rn(sm.S[i * D + j], sm.a[0][i]);
        pk = __fmaf_rn(s, sm.k[0][i], pk);
        pq = __fmaf_rn(s, sm.q[0][i], pq);
    }
    sm.red[0][grp][j] = pk;
    sm.red[1][grp][j] = pq;
    __syncthreads();
    // every thread of column j forms u[j] itself, by the same fixed-order sums, so pass 2 needs no
    // second barrier; thread j < D also publishes o[j]
    float yk = sm.red[0][0][j], yq = sm.red[1][0][j];
#pragma unroll
    for (int gg = 1; gg < L::RG; ++gg) { yk = __fadd_rn(yk, sm.red[0][gg][j]); yq = __fadd_rn(yq, sm.red[1][gg][j]); }
    const float u = __fmul_rn(beta, __fsub_rn(sm.v[0][j], yk));
    if (tid < D) sm.o[tid] = __fmul_rn(scale, __fmaf_rn(kq, u, yq));
    if (!keep) {
#pragma unroll 16
        for (int r = 0; r < L::RPG; ++r) {
            const int i = r0 + r;
            __stcs(g + i * D + j, __fmaf_rn(sm.k[0][i], u, __fmul_rn(sm.S[i * D + j], sm.a[0][i])));
        }
    } else if (snap) {
#pragma unroll 16
        for (int r = 0; r < L::RPG; ++r) {
            const int i = r0 + r;
            const float x = __fmaf_rn(sm.k[0][i], u, __fmul_rn(sm.S[i * D + j], sm.a[0][i]));
            sm.S[i * D + j] = x;
            snap[i * D + j] = x;
        }
    } else {
#pragma unroll 16
        for (int r = 0; r < L::RPG; ++r) {
            const int i = r0 + r;
            sm.S[i * D + j] = __fmaf_rn(sm.k[0][i], u, __fmul_rn(sm.S[i * D + j], sm.a[0][i]));
        }
    }
}

// The stateful rows' two passes over the shared-memory state, with a row's q, k, v, a in slot b:
//   row_reduce   pass 1 of a row: y_k = S'^T k, y_q = S'^T q (S' = diag(a) S), then this thread's
//                column's u and, for thread j < D, o[j] (returned in o);
//   row_update   pass 2 of a row: S = S' + k u^T, to shared memory (keep; and snap), or streamed
//                to g; fused, when `next`, with pass 1 of the following row (slot nb) on the new
//                values, so a row reads the state once and writes it once.
// The same rounded operations, in the same order, as state_step: the bits do not depend on the
// fusion.
template <int D>
__device__ __forceinline__ float row_finish(Smem<D> &sm, int b, float pk, float pq, float beta, float kq, float scale,
                                            float &o) {
    using L = Lay<D>;
    const int tid = threadIdx.x, j = tid % D, grp = tid / D;
    sm.red[0][grp][j] = pk;
    sm.red[1][grp][j] = pq;
    __syncthreads();
    float yk = sm.red[0][0][j], yq = sm.red[1][0][j];
#pragma unroll
    for (int gg = 1; gg < L::RG; ++gg) { yk = __fadd_rn(yk, sm.red[0][gg][j]); yq = __fadd_rn(yq, sm.red[1][gg][j]); }
    const float u = __fmul_rn(beta, __fsub_rn(sm.v[b][j], yk));
    o = __fmul_rn(scale, __fmaf_rn(kq, u, yq));
    return u;
}

// Four consecutive entries of a row vector (every lane reads the same ones: one broadcast).
__device__ __forceinline__ void ld4(const float *p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}

template <int D>
__device__ __forceinline__ float row_reduce(Smem<D> &sm, int b, float beta, float kq, float scale, float &o) {
    using L = Lay<D>;
    const int tid = threadIdx.x, j = tid % D, r0 = (tid / D) * L::RPG;
    float pk = 0.f, pq = 0.f;
#pragma unroll 4
    for (int r = 0; r < L::RPG; r += 4) {
        float a4[4], k4[4], q4[4];
        ld4(&sm.a[b][r0 + r], a4);
        ld4(&sm.k[b][r0 + r], k4);
        ld4(&sm.q[b][r0 + r], q4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float s = __fmul_rn(sm.S[(r0 + r + e) * D + j], a4[e]);
            pk = __fmaf_rn(s, k4[e], pk);
            pq = __fmaf_rn(s, q4[e], pq);
        }
    }
    return row_finish<D>(sm, b, pk, pq, beta, kq, scale, o);
}

template <int D>
__device__ __forceinline__ float row_update(Smem<D> &sm, int b, float u, bool keep, float *g, float *snap, bool next,
                                            int nb, float beta_n, float kq_n, float scale, float &o_n) {
    using L = Lay<D>;
    const int tid = threadIdx.x, j = tid % D, r0 = (tid / D) * L::RPG;
    float pk = 0.f, pq = 0.f;
    if (!keep) {
#pragma unroll 4
        for (int r = 0; r < L::RPG; r += 4) {
            float a4[4], k4[4];
            ld4(&sm.a[b][r0 + r], a4);
            ld4(&sm.k[b][r0 + r], k4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = r0 + r + e;
                __stcs(g + i * D + j, __fmaf_rn(k4[e], u, __fmul_rn(sm.S[i * D + j], a4[e])));
            }
        }
        return 0.f;
    }
#pragma unroll 4
    for (int r = 0; r < L::RPG; r += 4) {
        float a4[4], k4[4], an[4], kn[4], qn[4];
        ld4(&sm.a[b][r0 + r], a4);
        ld4(&sm.k[b][r0 + r], k4);
        if (next) {
            ld4(&sm.a[nb][r0 + r], an);
            ld4(&sm.k[nb][r0 + r], kn);
            ld4(&sm.q[nb][r0 + r], qn);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = r0 + r + e;
            const float x = __fmaf_rn(k4[e], u, __fmul_rn(sm.S[i * D + j], a4[e]));
            sm.S[i * D + j] = x;
            if (snap) snap[i * D + j] = x;
            if (next) {
                const float s = __fmul_rn(x, an[e]);
                pk = __fmaf_rn(s, kn[e], pk);
                pq = __fmaf_rn(s, qn[e], pq);
            }
        }
    }
    return next ? row_finish<D>(sm, nb, pk, pq, beta_n, kq_n, scale, o_n) : 0.f;
}

__device__ __forceinline__ float sigmoid_rn(float x) {
    return __frcp_rn(__fadd_rn(1.0f, expf(-x)));
}

// Thread 0: initialise the copy barrier and start the state copy. The barrier's initialisation
// is made visible to the other threads by the first __syncthreads that follows.
template <int D>
__device__ __forceinline__ void state_begin(Smem<D> &sm, const float *S) {
    if (threadIdx.x == 0) {
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
        state_load_issue<D>(sm, S);
    }
}

// Every thread: wait for the state copy. On a timeout the status is latched, the copy is
// waited for once more (bounded), and false is returned to every thread of the block.
template <int D>
__device__ __forceinline__ bool state_ready(Smem<D> &sm, int *status) {
    bool ok = state_load_wait<D>(sm);
    ok = __syncthreads_and(ok) != 0;
    if (!ok) {
        if (threadIdx.x == 0) {
            atomicExch(status, KDA_ERR_TIMEOUT);
            state_load_wait<D>(sm);
        }
        __syncthreads();
    }
    return ok;
}

__device__ __forceinline__ bool misaligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// ----------------------------------------------------------------------------- core-only decode

template <int D>
__global__ void __launch_bounds__(kThreads, 3)
recurrent_decode_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
                        const float *__restrict__ gate, const float *__restrict__ beta,
                        float *const *__restrict__ h_state, float *__restrict__ o, int H, float scale,
                        int *__restrict__ status) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem<D> &sm = *reinterpret_cast<Smem<D> *>(smem_raw);
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
    float *S = h_state[n] + static_cast<size_t>(h) * D * D;
    if (misaligned16(S)) {  // the bulk copies need 16-byte alignment: skip this head
        if (tid == 0) atomicExch(status, KDA_ERR_MISALIGNED);
        return;
    }
    state_begin<D>(sm, S);
    const size_t row = (static_cast<size_t>(n) * H + h) * D;
    const float bt = beta[static_cast<size_t>(n) * H + h];
    float qk = 0.f;
    if (tid < D) {
        const float qd = q[row + tid], kd = k[row + tid];
        sm.q[0][tid] = qd; sm.k[0][tid] = kd; sm.v[0][tid] = v[row + tid];
        sm.a[0][tid] = expf(gate[row + tid]);
        qk = __fmul_rn(qd, kd);
    }
    int spar = 0;
    const float kq = sum2_first_d<D>(tid < D ? qk : 0.f, 0.f, sm, spar).x;
    if (!state_ready<D>(sm, status)) return;
    state_step<D>(sm, bt, kq, scale, false, S, nullptr);
    if (tid < D) o[row + tid] = sm.o[tid];
}

// ----------------------------------------------------------------------------- fused stateful row

constexpr int kMaxSnap = 31;
constexpr int kMaxPackedRows = 64;  // rows of one packed sequence (one chunk, as the chunked verify)

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
    int *status;
    int H, K, n_snap;
    float scale, l2_eps, rms_eps;
    float *h_snap[kMaxSnap];
    uint16_t *conv_snap[kMaxSnap];
    // packed rows (cu non-null): sequence n owns rows cu[n] .. cu[n+1]-1 of the call's total;
    // verify runs them all and writes neither state; with acc, only the first acc[n] rows run and
    // both states are advanced (outputs may then be null: the o_norm step is skipped)
    const int *cu, *acc;
    int total, verify;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 3) decode_rows_kernel(const RowParams p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem<D> &sm = *reinterpret_cast<Smem<D> *>(smem_raw);
    const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x, H = p.H;
    const int qkv = H * D;
    float *S = (p.h_one ? p.h_one : p.h_arr[n]) + static_cast<size_t>(h) * D * D;
    if (misaligned16(S)) {  // the bulk copies need 16-byte alignment: skip this head
        if (tid == 0) atomicExch(p.status, KDA_ERR_MISALIGNED);
        return;
    }
    // this CTA's rows: K rows from n K, or the packed sequence's (the first acc[n] of them)
    int nrows = p.K;
    size_t rbase = static_cast<size_t>(n) * p.K;
    if (p.cu) {
        const int s0 = p.cu[n], s1 = p.cu[n + 1];
        const int lim = p.acc ? p.acc[n] : s1 - s0;
        if (s0 < 0 || s1 < s0 || s1 > p.total || s1 - s0 > kMaxPackedRows || lim < 0 || lim > s1 - s0) {
            if (tid == 0 && h == 0) atomicExch(p.status, KDA_ERR_INVALID_ARG);  // this sequence is skipped
            return;
        }
        rbase = static_cast<size_t>(s0);
        nrows = lim;
    }
    if (nrows == 0) return;  // nothing to run: both states stay (no copy was issued)
    state_begin<D>(sm, S);
    uint16_t *cst = p.conv_one ? p.conv_one : p.conv_arr[n];

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
    const float ow = qk_thread && p.o_norm_w ? bf16_to_f32(p.o_norm_w[d]) : 0.f;
    bool ok = true;
    int spar = 0;  // wsum buffer parity of the next block sum

    // every global input of a row (none depends on the state): the next row's are requested while
    // the current one runs
    uint16_t nx0 = 0, nx1 = 0, ngr = 0, nog = 0;
    float nbl = 0.f;
    auto load_row = [&](size_t row) {
        if (qk_thread || v_thread) nx0 = p.x[row * 3 * qkv + c0];
        if (qk_thread) {
            nx1 = p.x[row * 3 * qkv + c1];
            ngr = p.g_raw[row * qkv + h * D + d];
            nog = p.out_gate[row * qkv + h * D + d];
        }
        nbl = p.b_logit[row * H + h];
    };
    load_row(rbase);
    // The front of a row (conv step, SiLU, q|k L2, gate, beta, k.q) into slot t & 1, its conv_out
    // and conv snapshot; returns the row's beta and k.q, and its output gate for the o_norm.
    float og_t = 0.f;
    auto front = [&](int t, float &beta, float &kq, float &og) {
        const size_t row = rbase + t;
        const int b = t & 1;
        const float x0 = bf16_to_f32(nx0), x1 = bf16_to_f32(nx1), graw = bf16_to_f32(ngr);
        og = bf16_to_f32(nog);
        const float blog = nbl;
        if (t + 1 < nrows) load_row(row + 1);
        // conv step + SiLU (fixed-order FP32), new conv state in registers
        float y0 = 0.f, y1 = 0.f;
        if (qk_thread || v_thread) {
            y0 = __fmaf_rn(w0[3], x0, __fmaf_rn(w0[2], s0[2], __fmaf_rn(w0[1], s0[1], __fmul_rn(w0[0], s0[0]))));
            y0 = __fmul_rn(y0, sigmoid_rn(y0));
            s0[0] = s0[1]; s0[1] = s0[2]; s0[2] = x0;
            if (qk_thread) {
                y1 = __fmaf_rn(w1[3], x1, __fmaf_rn(w1[2], s1[2], __fmaf_rn(w1[1], s1[1], __fmul_rn(w1[0], s1[0]))));
                y1 = __fmul_rn(y1, sigmoid_rn(y1));
                s1[0] = s1[1]; s1[1] = s1[2]; s1[2] = x1;
            }
        }
        // per-head L2 of q and k (one BF16 rounding after the norm), v rounded as is
        const float2 ss = sum2_first_d<D>(qk_thread ? __fmul_rn(y0, y0) : 0.f, qk_thread ? __fmul_rn(y1, y1) : 0.f, sm, spar);
        float qv = 0.f, kv = 0.f;
        if (qk_thread) {
            const uint16_t qb = f32_to_bf16(__fmul_rn(y0, rsqrtf(__fadd_rn(ss.x, p.l2_eps))));
            const uint16_t kb = f32_to_bf16(__fmul_rn(y1, rsqrtf(__fadd_rn(ss.y, p.l2_eps))));
            qv = bf16_to_f32(qb); kv = bf16_to_f32(kb);
            sm.q[b][d] = qv; sm.k[b][d] = kv;
            if (p.conv_out) { p.conv_out[row * 3 * qkv + c0] = qb; p.conv_out[row * 3 * qkv + c1] = kb; }
            // gate for key channel d
            sm.a[b][d] = expf(kda_gate_f32(graw, dtb, nea));
        } else if (v_thread) {
            const uint16_t vb = f32_to_bf16(y0);
            sm.v[b][d] = bf16_to_f32(vb);
            if (p.conv_out) p.conv_out[row * 3 * qkv + c0] = vb;
        }
        beta = sigmoid_rn(blog);
        kq = sum2_first_d<D>(qk_thread ? __fmul_rn(qv, kv) : 0.f, 0.f, sm, spar).x;
        if (t < p.n_snap) {
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
    };
    float beta_t, kq_t, o_t = 0.f;
    front(0, beta_t, kq_t, og_t);
    ok = state_ready<D>(sm, p.status);
    float u_t = 0.f;
    if (ok) u_t = row_reduce<D>(sm, 0, beta_t, kq_t, p.scale, o_t);
    for (int t = 0; t < nrows && ok; ++t) {
        const size_t row = rbase + t;
        const bool next = t + 1 < nrows;
        // the next row's front: its slot is free (the pass that last read it has finished)
        float beta_n = 0.f, kq_n = 0.f, og_n = 0.f;
        if (next) front(t + 1, beta_n, kq_n, og_n);
        // o_norm of this row: sigmoid-gated RMSNorm over the head's D outputs (skipped by a fold)
        const float ov = qk_thread ? o_t : 0.f;
        const float ms = p.o_norm_out ? sum2_first_d<D>(qk_thread ? __fmul_rn(ov, ov) : 0.f, 0.f, sm, spar).x : 0.f;
        if (qk_thread && p.o_norm_out) {
            const float rs = rsqrtf(__fadd_rn(__fmul_rn(ms, 1.0f / D), p.rms_eps));
            const float yv = __fmul_rn(__fmul_rn(__fmul_rn(ov, rs), ow), sigmoid_rn(og_t));
            p.o_norm_out[row * qkv + h * D + d] = f32_to_bf16(yv);
            if (p.core) p.core[row * qkv + h * D + d] = ov;
        }
        // this row's update, fused with the next row's first pass. The last row streams the state
        // out; earlier rows keep it (and write their snapshot); a verify leaves it (its last row
        // is not even applied)
        if (next || !p.verify) {
            float *snap = next && t < p.n_snap ? p.h_snap[t] + static_cast<size_t>(h) * D * D : nullptr;
            float o_n = 0.f;
            u_t = row_update<D>(sm, t & 1, u_t, next, S, snap, next, (t + 1) & 1, beta_n, kq_n, p.scale, o_n);
            o_t = o_n;
        }
        og_t = og_n;
    }
    if (!ok || p.verify) return;  // a verify leaves the conv state too
    if (qk_thread || v_thread) {
#pragma unroll
        for (int j = 0; j < 3; ++j) cst[c0 * 3 + j] = f32_to_bf16(s0[j]);
        if (qk_thread) {
#pragma unroll
            for (int j = 0; j < 3; ++j) cst[c1 * 3 + j] = f32_to_bf16(s1[j]);
        }
    }
}

template <int D>
int launch_rows_d(const RowParams &p, int N, cudaStream_t s) {
    static std::atomic<unsigned long long> attr_done{0};
    KDA_TRY(smem_opt_in(decode_rows_kernel<D>, static_cast<int>(sizeof(Smem<D>)), attr_done, true));
    decode_rows_kernel<D><<<dim3(p.H, N), kThreads, sizeof(Smem<D>), s>>>(p);
    return launch_status();
}

int launch_rows(RowParams &p, int N, int D, cudaStream_t s) {
    p.status = device_status_ptr();
    if (!p.status) return KDA_ERR_CUDA;
    return D == 128 ? launch_rows_d<128>(p, N, s) : launch_rows_d<64>(p, N, s);
}

template <int D>
int launch_recurrent(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                     float *const *h_state, float *o, int N, int H, float scale, cudaStream_t s) {
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    static std::atomic<unsigned long long> attr_done{0};
    KDA_TRY(smem_opt_in(recurrent_decode_kernel<D>, static_cast<int>(sizeof(Smem<D>)), attr_done, true));
    recurrent_decode_kernel<D><<<dim3(H, N), kThreads, sizeof(Smem<D>), s>>>(q, k, v, gate, beta, h_state, o, H,
                                                                               scale, status);
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
    auto s = static_cast<cudaStream_t>(stream);
    if (dims->head_dim == 128)
        return kda::launch_recurrent<128>(q, k, v, gate, beta, h_state, o, N, dims->heads, dims->scale, s);
    return kda::launch_recurrent<64>(q, k, v, gate, beta, h_state, o, N, dims->heads, dims->scale, s);
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
    if (n_snap != 0 && n_snap != K - 1) return KDA_ERR_INVALID_ARG;
    if (n_snap > 0 && (!h_snap || !conv_snap)) return KDA_ERR_INVALID_ARG;
    kda::RowParams p;
    KDA_TRY(fill_row_params(p, x, conv_w, g_raw, dt_bias, a_log, b_logit, out_gate, o_norm_w, o_norm_out, conv_out,
                            core, K, dims));
    if (!kda::aligned16(h_state)) return KDA_ERR_MISALIGNED;
    for (int t = 0; t < n_snap; ++t) {
        if (!h_snap[t] || !conv_snap[t]) return KDA_ERR_INVALID_ARG;
        if (!kda::aligned16(h_snap[t])) return KDA_ERR_MISALIGNED;
    }
    // One launch takes at most kMaxSnap + 1 rows (its snapshot pointers travel in the kernel
    // parameters). Longer calls run in groups, each continuing from the state the previous one
    // left in place: the FP32 state and the BF16 conv inputs round-trip exactly, so every row
    // sees the bits it would in one launch. A group that is not the last also snapshots its
    // own last row: the conv state from the kernel, the recurrent state (which the kernel
    // streams to h_state) by a copy.
    const size_t qkv = static_cast<size_t>(dims->heads) * dims->head_dim;
    const size_t h_bytes = qkv * dims->head_dim * sizeof(float);
    auto s = static_cast<cudaStream_t>(stream);
    const kda::RowParams base = p;
    for (int r0 = 0; r0 < K;) {
        const bool final_group = K - r0 <= kda::kMaxSnap + 1;
        const int rows = final_group ? K - r0 : (n_snap ? kda::kMaxSnap : kda::kMaxSnap + 1);
        p = base;
        p.x = base.x + r0 * 3 * qkv; p.g_raw = base.g_raw + r0 * qkv; p.b_logit = base.b_logit + r0 * dims->heads;
        p.out_gate = base.out_gate + r0 * qkv; p.o_norm_out = base.o_norm_out + r0 * qkv;
        if (base.conv_out) p.conv_out = base.conv_out + r0 * 3 * qkv;
        if (base.core) p.core = base.core + r0 * qkv;
        p.conv_one = conv_state; p.h_one = h_state; p.K = rows;
        p.n_snap = n_snap ? (final_group ? rows - 1 : rows) : 0;
        for (int t = 0; t < p.n_snap; ++t) {
            p.h_snap[t] = h_snap[r0 + t];
            p.conv_snap[t] = conv_snap[r0 + t];
        }
        KDA_TRY(kda::launch_rows(p, 1, dims->head_dim, s));
        if (n_snap && !final_group &&
            cudaMemcpyAsync(h_snap[r0 + rows - 1], h_state, h_bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return KDA_ERR_CUDA;
        r0 += rows;
    }
    return KDA_OK;
}

}  // extern "C"

namespace kda {

// The stateful row over packed sequences: rows cu[n] .. cu[n+1]-1 belong to sequence n (at most
// kMaxPackedRows). Without acc (a verify) every row runs and neither state is written; with acc
// (a fold) only each sequence's first acc[n] rows run, both states are advanced as decode_k's
// rows would advance them, and the outputs may be null.
int decode_rows_packed(const uint16_t *x, uint16_t *const *conv_state, const uint16_t *conv_w, const uint16_t *g_raw,
                       const float *dt_bias, const float *a_log, const float *b_logit, float *const *h_state,
                       const uint16_t *out_gate, const uint16_t *o_norm_w, uint16_t *o_norm_out, uint16_t *conv_out,
                       float *core, const int *cu, const int *acc, int B, int total, const kda_dims *dims,
                       cudaStream_t s) {
    KDA_TRY(check_dims(dims));
    if (!x || !conv_state || !conv_w || !g_raw || !dt_bias || !a_log || !b_logit || !h_state || !out_gate || !cu ||
        B < 0 || total < 0)
        return KDA_ERR_INVALID_ARG;
    if (!acc && (!o_norm_w || !o_norm_out)) return KDA_ERR_INVALID_ARG;
    if (B == 0) return KDA_OK;
    if (B > 65535) return KDA_ERR_UNSUPPORTED;
    RowParams p{};
    p.x = x; p.conv_arr = conv_state; p.conv_w = conv_w; p.g_raw = g_raw; p.dt_bias = dt_bias; p.a_log = a_log;
    p.b_logit = b_logit; p.h_arr = h_state; p.out_gate = out_gate; p.o_norm_w = o_norm_w;
    p.o_norm_out = acc ? nullptr : o_norm_out;
    p.conv_out = acc ? nullptr : conv_out;
    p.core = acc ? nullptr : core;
    p.H = dims->heads; p.scale = dims->scale; p.l2_eps = dims->l2_eps; p.rms_eps = dims->rms_eps;
    p.K = 0; p.n_snap = 0;
    p.cu = cu; p.acc = acc; p.total = total; p.verify = acc ? 0 : 1;
    return launch_rows(p, B, dims->head_dim, s);
}

}  // namespace kda
