// One KDA block prefill (Glm5NextKdaLayer `prefill` / `prefill_with_pad_fill`), stage by stage
// into the workspace buffers of Glm5NextKdaWorkspace, with the weights of Glm5NextKdaWeights:
//   q, k, v = h W^T           -> qkv_proj [T, 3*H*D] BF16 (three GEMMs writing the packed row)
//   conv + SiLU + q|k L2      -> conv_out [T, 3*H*D] BF16 (conv state carried in place)
//   g_raw = f_b(f_a(h))       -> g_raw [T, H*D] BF16
//   beta = sigmoid(b_proj(h)) (FP32 logits)
//   chunked core, fused-input mode: reads conv_out and g_raw directly (the gate is formed in
//   the kernel; rows past T are never read)  -> core [T_pad, H, D], recurrent state in place
//   out_gate = g_b(g_a(h));  o_norm_out = gated RMSNorm(core, out_gate);  final_out = o_proj
// The workspace is allocated once (kda_workspace_create) for at most max_tokens tokens (and, for
// packed calls, max_seqs sequences); the prefill call itself allocates nothing.
//
// Packed sequences (Glm5NextLayer batched prefill and its varlen form): the row-wise stages
// (projections, gate, beta, o_norm, o_proj) run once over all rows of all sequences; the conv
// takes each row's window from its own sequence and conv state, and the chunked core runs the
// packed-sequence (cu_seqlens) layout, so no stage mixes two sequences.
//
// Batched verify (Glm5NextLayer speculative verify; Glm5NextKdaLayer `decode_k`): the draft rows
// of N sequences, at most 64 each, through the same stages with every weight read once for all
// rows; the core runs in verify mode from each sequence's states, which stay as they were, and
// keeps the tables the fold needs. The fold then moves each sequence's recurrent state and conv
// state past its accepted rows without rerunning anything.
//
// Block decode (Glm5NextKdaLayer `decode`, `decode_k`): the same projections for the call's
// rows (N sequences x 1 token, or K rows of one sequence), each weight read once for all
// rows, then the fused stateful rows (kda_decode_fused / kda_decode_k: conv + SiLU + L2, gate,
// beta, recurrence, gated RMSNorm) and o_proj. decode_k's projections run the batched-M
// matrix-vector kernel (kda_gemv_bf16) on groups of up to 32 rows: its every output's
// arithmetic is fixed by K and its own row, so a row's projections are the same bits in a call
// of K rows and in a call of one, which the decode_k identity needs. Calls without that
// identity (N independent sequences, the batched verify) take the matrix-vector kernel up to 8
// rows (one pass over the weights), the small-M tensor-core form up to 256 rows (the weights'
// output rows as the 128-row tiles, so each weight is read once by many CTAs), and the GEMM
// beyond.
#include <algorithm>
#include <cstring>
#include <new>

#include "common.cuh"

namespace kda {
namespace {
// Writes the call's state pointer into the workspace's one-entry device pointer array (a kernel
// argument, so no host synchronisation is involved).
__global__ void store_ptr_kernel(float **slot, float *p) { *slot = p; }

// cu_seqlens of B sequences of T rows each: cu[b] = b T.
__global__ void equal_cu_kernel(int *cu, int B, int T) {
    for (int b = threadIdx.x; b <= B; b += blockDim.x) cu[b] = b * T;
}
}  // namespace
}

struct kda_workspace {
    kda_dims dims;
    int hidden, rank;
    size_t max_tokens, t_pad_max;
    int max_seqs;
    void *buf[KDA_BUF_COUNT];
    size_t bytes[KDA_BUF_COUNT];
    float **state_slot;  // device array holding the one state pointer of the call
    int *cu_equal;       // device [max_seqs + 1]: cu_seqlens of an equal-length batched call
    float *splitk;       // FP32 split-K partial sums of the small-M projections
    size_t splitk_bytes;
    // the weights of the last kda_block_verify that ran row by row: its fold re-runs the accepted
    // rows through the same stateful row, which needs the conv, gate and beta weights
    kda_block_weights verify_w;
    int verify_w_set;
};

namespace kda {
namespace {
constexpr int kRowsGemv = 32;   // exact calls: the matrix-vector kernel up to this many rows
constexpr int kRowsGemvFree = 8; // other calls: the matrix-vector kernel up to one row group
constexpr int kRowsSmallM = 256; // then the small-M tensor-core form, then the GEMM
// A batched verify of at most this many draft rows per sequence on average runs row by row in the
// stateful decode row (K steps per (sequence, head), the state in shared memory); longer drafts
// take the chunked verify. Its fold follows the same rule on the same (B, total_tokens).
constexpr int kVerifyRowsByRow = 16;
bool verify_by_rows(int B, int total) { return static_cast<long long>(total) <= static_cast<long long>(kVerifyRowsByRow) * B; }

// Which kernel takes M rows. `exact`: every row must get the bits it gets alone (decode_k's
// identity with serial one-row decodes), which only the matrix-vector kernel gives.
enum class ProjKind { Gemv, SmallM, Gemm };
ProjKind proj_kind(int M, bool exact) {
    if (M <= (exact ? kRowsGemv : kRowsGemvFree)) return ProjKind::Gemv;
    return M <= kRowsSmallM ? ProjKind::SmallM : ProjKind::Gemm;
}

// One projection of M rows.
int proj(const uint16_t *A, int lda, const uint16_t *W, int ldw, void *C, int ldc, int M, int N, int K, int out_f32,
         cudaStream_t s, bool exact, const kda_workspace *ws) {
    switch (proj_kind(M, exact)) {
    case ProjKind::Gemv: return gemv_bf16(A, lda, W, ldw, C, ldc, M, N, K, out_f32, s);
    case ProjKind::SmallM: {
        const GemmTSeg t{W, A, C, N, ldw, lda, ldc, out_f32};
        return gemm_bf16_small_m(&t, 1, M, K, s, ws->splitk, ws->splitk_bytes);
    }
    default: return gemm_bf16(A, lda, W, ldw, C, ldc, M, N, K, out_f32, s);
    }
}

// Projections of M rows of `hidden` into the workspace rows [r0, r0 + M): qkv_proj (q|k|v
// packed), g_raw, b_logit (FP32, in the BETA buffer), out_gate. For the matrix-vector path the
// weights that read the hidden rows share one launch ([q | k | v | f_a | g_a | b_proj]), then
// f_b and g_b share another.
int block_projections(const kda_block_weights *w, const kda_bf16 *hidden, int M, kda_workspace *ws, cudaStream_t s,
                      bool exact, int r0 = 0) {
    const kda_dims *d = &ws->dims;
    const int Hd = ws->hidden, R = ws->rank, H = d->heads, qkv = d->heads * d->head_dim, cd = 3 * qkv;
    const size_t o = static_cast<size_t>(r0);
    auto bf = [&](int i) { return static_cast<uint16_t *>(ws->buf[i]); };
    auto f32 = [&](int i) { return static_cast<float *>(ws->buf[i]); };
    uint16_t *qkv_p = bf(KDA_BUF_QKV_PROJ) + o * cd, *fa = bf(KDA_BUF_F_A_OUT) + o * R, *ga = bf(KDA_BUF_G_A_OUT) + o * R;
    uint16_t *graw = bf(KDA_BUF_G_RAW) + o * qkv, *og = bf(KDA_BUF_OUT_GATE) + o * qkv;
    float *blog = f32(KDA_BUF_BETA) + o * H;
    hidden += o * Hd;
    const ProjKind kind = proj_kind(M, exact);
    if (kind == ProjKind::SmallM) {  // two launches, each weight read once by many CTAs
        const GemmTSeg a[6] = {{w->q_proj, hidden, qkv_p, qkv, Hd, Hd, cd, 0},
                               {w->k_proj, hidden, qkv_p + qkv, qkv, Hd, Hd, cd, 0},
                               {w->v_proj, hidden, qkv_p + 2 * qkv, qkv, Hd, Hd, cd, 0},
                               {w->f_a, hidden, fa, R, Hd, Hd, R, 0},
                               {w->g_a, hidden, ga, R, Hd, Hd, R, 0},
                               {w->b_proj, hidden, blog, H, Hd, Hd, H, 1}};
        KDA_TRY(gemm_bf16_small_m(a, 6, M, Hd, s, ws->splitk, ws->splitk_bytes));
        const GemmTSeg c[2] = {{w->f_b, fa, graw, qkv, R, R, qkv, 0}, {w->g_b, ga, og, qkv, R, R, qkv, 0}};
        return gemm_bf16_small_m(c, 2, M, R, s, ws->splitk, ws->splitk_bytes);
    }
    if (kind == ProjKind::Gemv) {
        // every weight that reads the hidden rows: q, k, v, then the small f_a, g_a, b_proj
        // products ride in the tail of the same launch
        GemvSegs a{};
        a.s[0] = GemvSeg{w->q_proj, qkv_p, qkv, Hd, cd, 0};
        a.s[1] = GemvSeg{w->k_proj, qkv_p + qkv, qkv, Hd, cd, 0};
        a.s[2] = GemvSeg{w->v_proj, qkv_p + 2 * qkv, qkv, Hd, cd, 0};
        a.s[3] = GemvSeg{w->f_a, fa, R, Hd, R, 0};
        a.s[4] = GemvSeg{w->g_a, ga, R, Hd, R, 0};
        a.s[5] = GemvSeg{w->b_proj, blog, H, Hd, H, 1};
        a.count = 6;
        a.total = 3 * qkv + 2 * R + H;
        KDA_TRY(gemv_segs(hidden, Hd, a, M, Hd, s));
        // f_b and g_b read different rows (f_a_out, g_a_out) with one width: one launch
        GemvSegs c{};
        c.s[0] = GemvSeg{w->f_b, graw, qkv, R, qkv, 0, fa};
        c.s[1] = GemvSeg{w->g_b, og, qkv, R, qkv, 0, ga};
        c.count = 2;
        c.total = 2 * qkv;
        return gemv_segs(fa, R, c, M, R, s);
    }
    KDA_TRY(gemm_bf16(hidden, Hd, w->q_proj, Hd, qkv_p, cd, M, qkv, Hd, 0, s));
    KDA_TRY(gemm_bf16(hidden, Hd, w->k_proj, Hd, qkv_p + qkv, cd, M, qkv, Hd, 0, s));
    KDA_TRY(gemm_bf16(hidden, Hd, w->v_proj, Hd, qkv_p + 2 * qkv, cd, M, qkv, Hd, 0, s));
    KDA_TRY(gemm_bf16(hidden, Hd, w->f_a, Hd, fa, R, M, R, Hd, 0, s));
    KDA_TRY(gemm_bf16(fa, R, w->f_b, R, graw, qkv, M, qkv, R, 0, s));
    KDA_TRY(gemm_bf16(hidden, Hd, w->b_proj, Hd, blog, H, M, H, Hd, 1, s));
    KDA_TRY(gemm_bf16(hidden, Hd, w->g_a, Hd, ga, R, M, R, Hd, 0, s));
    return gemm_bf16(ga, R, w->g_b, R, og, qkv, M, qkv, R, 0, s);
}

// The prefill projections of T rows (always the tensor-core GEMM).
int prefill_projections(const kda_block_weights *w, const kda_bf16 *hidden, int T, kda_workspace *ws,
                        cudaStream_t s) {
    const kda_dims *d = &ws->dims;
    const int Hd = ws->hidden, R = ws->rank, H = d->heads, qkv = d->heads * d->head_dim, cd = 3 * qkv;
    auto bf = [&](int i) { return static_cast<uint16_t *>(ws->buf[i]); };
    auto f32 = [&](int i) { return static_cast<float *>(ws->buf[i]); };
    // q | k | v projections straight into the packed qkv_proj rows, one launch
    const GemmProd p_qkv[3] = {{hidden, Hd, w->q_proj, Hd, bf(KDA_BUF_QKV_PROJ), cd, T, qkv, Hd, 0},
                               {hidden, Hd, w->k_proj, Hd, bf(KDA_BUF_QKV_PROJ) + qkv, cd, T, qkv, Hd, 0},
                               {hidden, Hd, w->v_proj, Hd, bf(KDA_BUF_QKV_PROJ) + 2 * qkv, cd, T, qkv, Hd, 0}};
    KDA_TRY(gemm_bf16_multi(p_qkv, 3, s));
    // the two low-rank pairs: forget-gate input g_raw = f_b(f_a(h)) (the gate itself is formed
    // inside the chunked core) and the output gate g_b(g_a(h)), each stage of both in one launch
    const GemmProd p_a[2] = {{hidden, Hd, w->f_a, Hd, bf(KDA_BUF_F_A_OUT), R, T, R, Hd, 0},
                             {hidden, Hd, w->g_a, Hd, bf(KDA_BUF_G_A_OUT), R, T, R, Hd, 0}};
    KDA_TRY(gemm_bf16_multi(p_a, 2, s));
    const GemmProd p_b[2] = {{bf(KDA_BUF_F_A_OUT), R, w->f_b, R, bf(KDA_BUF_G_RAW), qkv, T, qkv, R, 0},
                             {bf(KDA_BUF_G_A_OUT), R, w->g_b, R, bf(KDA_BUF_OUT_GATE), qkv, T, qkv, R, 0}};
    KDA_TRY(gemm_bf16_multi(p_b, 2, s));
    // beta logits (FP32)
    return gemm_bf16(hidden, Hd, w->b_proj, Hd, f32(KDA_BUF_BETA), H, T, H, Hd, 1, s);
}

// gated RMSNorm of `rows` core rows, then o_proj (GEMM) unless the caller applies its own.
int prefill_back(const kda_block_weights *w, int rows, kda_workspace *ws, void *stream) {
    const kda_dims *d = &ws->dims;
    const int Hd = ws->hidden, qkv = d->heads * d->head_dim;
    auto bf = [&](int i) { return static_cast<uint16_t *>(ws->buf[i]); };
    KDA_TRY(kda_back_gated_rmsnorm(static_cast<float *>(ws->buf[KDA_BUF_CORE]), bf(KDA_BUF_OUT_GATE), w->o_norm,
                                   bf(KDA_BUF_O_NORM_OUT), rows, d, stream));
    if (!w->o_proj) return KDA_OK;  // the caller applies its own o_proj (a tensor-parallel slice)
    return gemm_bf16(bf(KDA_BUF_O_NORM_OUT), qkv, w->o_proj, qkv, bf(KDA_BUF_FINAL_OUT), Hd, rows, Hd, qkv, 0,
                     static_cast<cudaStream_t>(stream));
}

int check_block_args(const kda_block_weights *w, const kda_bf16 *hidden, const kda_workspace *ws) {
    if (!w || !hidden || !ws) return KDA_ERR_INVALID_ARG;
    if (w->hidden != ws->hidden || w->rank != ws->rank) return KDA_ERR_INVALID_ARG;
    if (!w->q_proj || !w->k_proj || !w->v_proj || !w->conv || !w->f_a || !w->f_b || !w->dt_bias || !w->a_log ||
        !w->b_proj || !w->g_a || !w->g_b || !w->o_norm)
        return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}
}  // namespace
}  // namespace kda

extern "C" {

int kda_workspace_create_batched(const kda_dims *dims, int hidden, int rank, size_t max_tokens, int max_seqs,
                                 kda_workspace **out) {
    if (!out) return KDA_ERR_INVALID_ARG;
    *out = nullptr;
    KDA_TRY(kda::check_dims(dims));
    if (hidden <= 0 || rank <= 0 || max_tokens == 0 || max_seqs <= 0) return KDA_ERR_INVALID_ARG;
    if (hidden % 64 || rank % 64 || (dims->heads * dims->head_dim) % 64) return KDA_ERR_UNSUPPORTED;
    if (max_tokens > 0x7fffffffULL || max_seqs > 65535) return KDA_ERR_UNSUPPORTED;
    kda_workspace *ws = new (std::nothrow) kda_workspace();
    if (!ws) return KDA_ERR_CUDA;
    ws->dims = *dims;
    ws->hidden = hidden;
    ws->rank = rank;
    ws->max_tokens = max_tokens;
    ws->max_seqs = max_seqs;
    ws->t_pad_max = kda_t_pad(max_tokens, dims->chunk);
    const size_t T = max_tokens, Tp = ws->t_pad_max;
    const size_t qkv = static_cast<size_t>(dims->heads) * dims->head_dim, H = dims->heads;
    const size_t sizes[KDA_BUF_COUNT] = {
        T * 3 * qkv * 2,   // QKV_PROJ
        T * 3 * qkv * 2,   // CONV_OUT
        0,                 // Q_F32 (the fused-input core does not widen q, k, v or the gate)
        0,                 // K_F32
        0,                 // V_F32
        0,                 // GATE
        Tp * H * 4,        // BETA
        Tp * qkv * 4,      // CORE
        T * qkv * 2,       // G_RAW
        T * qkv * 2,       // OUT_GATE
        T * qkv * 2,       // O_NORM_OUT
        T * hidden * 2,    // FINAL_OUT
        T * rank * 2,      // F_A_OUT
        T * rank * 2,      // G_A_OUT
        // PREFILL_SCRATCH: one sequence of T rows, or any packed call of max_seqs sequences and
        // T rows in all (the same size when max_seqs = 1)
        kda::chunk_prefill_packed_bytes(max_seqs, static_cast<int>(T), dims->heads, dims->head_dim),
    };
    for (int i = 0; i < KDA_BUF_COUNT; ++i) {
        ws->bytes[i] = sizes[i];
        if (cudaMalloc(&ws->buf[i], sizes[i] ? sizes[i] : 16) != cudaSuccess) {
            kda_workspace_destroy(ws);
            return KDA_ERR_CUDA;
        }
    }
    ws->splitk_bytes = kda::small_m_part_bytes(static_cast<int>(std::min<size_t>(T, 256)));
    if (cudaMalloc(reinterpret_cast<void **>(&ws->splitk), ws->splitk_bytes) != cudaSuccess) {
        kda_workspace_destroy(ws);
        return KDA_ERR_CUDA;
    }
    if (cudaMalloc(reinterpret_cast<void **>(&ws->state_slot), sizeof(float *)) != cudaSuccess ||
        cudaMalloc(reinterpret_cast<void **>(&ws->cu_equal), (static_cast<size_t>(max_seqs) + 1) * sizeof(int)) !=
            cudaSuccess) {
        kda_workspace_destroy(ws);
        return KDA_ERR_CUDA;
    }
    *out = ws;
    return KDA_OK;
}

int kda_workspace_create(const kda_dims *dims, int hidden, int rank, size_t max_tokens, kda_workspace **out) {
    return kda_workspace_create_batched(dims, hidden, rank, max_tokens, 1, out);
}

int kda_workspace_destroy(kda_workspace *ws) {
    if (!ws) return KDA_OK;
    for (int i = 0; i < KDA_BUF_COUNT; ++i)
        if (ws->buf[i]) cudaFree(ws->buf[i]);
    if (ws->state_slot) cudaFree(ws->state_slot);
    if (ws->splitk) cudaFree(ws->splitk);
    if (ws->cu_equal) cudaFree(ws->cu_equal);
    delete ws;
    return KDA_OK;
}

size_t kda_workspace_max_tokens(const kda_workspace *ws) { return ws ? ws->max_tokens : 0; }

int kda_workspace_max_seqs(const kda_workspace *ws) { return ws ? ws->max_seqs : 0; }

int kda_workspace_buffer(const kda_workspace *ws, int which, void **ptr, size_t *bytes) {
    if (!ws || !ptr || which < 0 || which >= KDA_BUF_COUNT) return KDA_ERR_INVALID_ARG;
    *ptr = ws->buf[which];
    if (bytes) *bytes = ws->bytes[which];
    return KDA_OK;
}

int kda_block_prefill(const kda_block_weights *w, const kda_bf16 *hidden, int T, float *h_state,
                      kda_bf16 *conv_state, float pad_fill, kda_workspace *ws, void *stream) {
    KDA_TRY(kda::check_block_args(w, hidden, ws));
    if (!h_state || !conv_state || T < 0) return KDA_ERR_INVALID_ARG;
    if (T == 0) return KDA_OK;
    if (static_cast<size_t>(T) > ws->max_tokens) return KDA_ERR_CAPACITY;
    const kda_dims *d = &ws->dims;
    auto s = static_cast<cudaStream_t>(stream);
    auto bf = [&](int i) { return static_cast<uint16_t *>(ws->buf[i]); };
    auto f32 = [&](int i) { return static_cast<float *>(ws->buf[i]); };
    KDA_TRY(kda::prefill_projections(w, hidden, T, ws, s));
    KDA_TRY(kda_front_conv_silu_l2(bf(KDA_BUF_QKV_PROJ), conv_state, w->conv, bf(KDA_BUF_CONV_OUT), nullptr, nullptr,
                                   nullptr, pad_fill, T, d, stream));
    KDA_TRY(kda_beta(f32(KDA_BUF_BETA), f32(KDA_BUF_BETA), T * d->heads, stream));
    // chunked core from the carried state, on the BF16 conv_out rows and g_raw
    kda::store_ptr_kernel<<<1, 1, 0, s>>>(ws->state_slot, h_state);
    KDA_TRY(kda::launch_status());
    KDA_TRY(kda_chunk_prefill_fused(bf(KDA_BUF_CONV_OUT), bf(KDA_BUF_G_RAW), w->dt_bias, w->a_log, f32(KDA_BUF_BETA),
                                    ws->state_slot, f32(KDA_BUF_CORE), 1, T, ws->buf[KDA_BUF_PREFILL_SCRATCH],
                                    ws->bytes[KDA_BUF_PREFILL_SCRATCH], d, stream));
    return kda::prefill_back(w, T, ws, stream);
}

int kda_block_prefill_varlen(const kda_block_weights *w, const kda_bf16 *hidden, const int *cu_seqlens, int B,
                             int max_num_chunks, int total_tokens, float *const *h_state,
                             kda_bf16 *const *conv_state, kda_workspace *ws, void *stream) {
    KDA_TRY(kda::check_block_args(w, hidden, ws));
    if (!cu_seqlens || !h_state || !conv_state || B < 0 || total_tokens < 0 || max_num_chunks < 0)
        return KDA_ERR_INVALID_ARG;
    if (B == 0 || total_tokens == 0) return KDA_OK;
    if (max_num_chunks == 0) return KDA_ERR_INVALID_ARG;
    if (static_cast<size_t>(total_tokens) > ws->max_tokens || B > ws->max_seqs) return KDA_ERR_CAPACITY;
    const kda_dims *d = &ws->dims;
    if (ws->bytes[KDA_BUF_PREFILL_SCRATCH] <
        kda::chunk_prefill_varlen_need_bytes(B, max_num_chunks, total_tokens, d->heads, d->head_dim))
        return KDA_ERR_CAPACITY;
    auto s = static_cast<cudaStream_t>(stream);
    auto bf = [&](int i) { return static_cast<uint16_t *>(ws->buf[i]); };
    auto f32 = [&](int i) { return static_cast<float *>(ws->buf[i]); };
    KDA_TRY(kda::prefill_projections(w, hidden, total_tokens, ws, s));
    KDA_TRY(kda::front_varlen(bf(KDA_BUF_QKV_PROJ), conv_state, w->conv, bf(KDA_BUF_CONV_OUT), cu_seqlens, B,
                              total_tokens, d, s));
    KDA_TRY(kda::conv_state_advance(bf(KDA_BUF_QKV_PROJ), conv_state, cu_seqlens, nullptr, B, total_tokens, d, s));
    KDA_TRY(kda_beta(f32(KDA_BUF_BETA), f32(KDA_BUF_BETA), total_tokens * d->heads, stream));
    KDA_TRY(kda::chunk_prefill_tc_fused_varlen(bf(KDA_BUF_CONV_OUT), bf(KDA_BUF_G_RAW), w->dt_bias, w->a_log,
                                               f32(KDA_BUF_BETA), cu_seqlens, B, max_num_chunks, total_tokens,
                                               h_state, f32(KDA_BUF_CORE), d, ws->buf[KDA_BUF_PREFILL_SCRATCH], s));
    return kda::prefill_back(w, total_tokens, ws, stream);
}

int kda_block_prefill_batched(const kda_block_weights *w, const kda_bf16 *hidden, int B, int T,
                              float *const *h_state, kda_bf16 *const *conv_state, kda_workspace *ws, void *stream) {
    KDA_TRY(kda::check_block_args(w, hidden, ws));
    if (!h_state || !conv_state || B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return KDA_OK;
    if (B > ws->max_seqs || static_cast<long long>(B) * T > static_cast<long long>(ws->max_tokens))
        return KDA_ERR_CAPACITY;
    auto s = static_cast<cudaStream_t>(stream);
    kda::equal_cu_kernel<<<1, 256, 0, s>>>(ws->cu_equal, B, T);
    KDA_TRY(kda::launch_status());
    const int nch = static_cast<int>(kda_t_pad(static_cast<size_t>(T), kda::kChunk) / kda::kChunk);
    return kda_block_prefill_varlen(w, hidden, ws->cu_equal, B, nch, B * T, h_state, conv_state, ws, stream);
}

int kda_block_decode(const kda_block_weights *w, const kda_bf16 *hidden, int N, float *const *h_state,
                     kda_bf16 *const *conv_state, kda_workspace *ws, void *stream) {
    KDA_TRY(kda::check_block_args(w, hidden, ws));
    if (!h_state || !conv_state || N < 0) return KDA_ERR_INVALID_ARG;
    if (N == 0) return KDA_OK;
    if (static_cast<size_t>(N) > ws->max_tokens) return KDA_ERR_CAPACITY;
    auto s = static_cast<cudaStream_t>(stream);
    const kda_dims *d = &ws->dims;
    const int qkv = d->heads * d->head_dim;
    auto bf = [&](int i) { return static_cast<kda_bf16 *>(ws->buf[i]); };
    auto f32 = [&](int i) { return static_cast<float *>(ws->buf[i]); };
    KDA_TRY(kda::block_projections(w, hidden, N, ws, s, false));
    KDA_TRY(kda_decode_fused(bf(KDA_BUF_QKV_PROJ), conv_state, w->conv, bf(KDA_BUF_G_RAW), w->dt_bias, w->a_log,
                             f32(KDA_BUF_BETA), h_state, bf(KDA_BUF_OUT_GATE), w->o_norm, bf(KDA_BUF_O_NORM_OUT),
                             bf(KDA_BUF_CONV_OUT), f32(KDA_BUF_CORE), N, d, stream));
    if (!w->o_proj) return KDA_OK;  // the caller applies its own o_proj (a tensor-parallel slice)
    return kda::proj(bf(KDA_BUF_O_NORM_OUT), qkv, w->o_proj, qkv, bf(KDA_BUF_FINAL_OUT), ws->hidden, N, ws->hidden, qkv,
                     0, s, false, ws);
}

int kda_block_decode_k(const kda_block_weights *w, const kda_bf16 *hidden, int K, float *h_state,
                       kda_bf16 *conv_state, float *const *h_snap, kda_bf16 *const *conv_snap, int n_snap,
                       kda_workspace *ws, void *stream) {
    KDA_TRY(kda::check_block_args(w, hidden, ws));
    if (!h_state || !conv_state || K < 1) return KDA_ERR_INVALID_ARG;
    if (static_cast<size_t>(K) > ws->max_tokens) return KDA_ERR_CAPACITY;
    auto s = static_cast<cudaStream_t>(stream);
    const kda_dims *d = &ws->dims;
    const int qkv = d->heads * d->head_dim, Hd = ws->hidden;
    auto bf = [&](int i) { return static_cast<kda_bf16 *>(ws->buf[i]); };
    auto f32 = [&](int i) { return static_cast<float *>(ws->buf[i]); };
    // projections and o_proj in groups of at most kRowsGemv rows: the matrix-vector kernel gives
    // each row the bits it gets alone, which the identity with serial decodes needs
    for (int r0 = 0; r0 < K; r0 += kda::kRowsGemv)
        KDA_TRY(kda::block_projections(w, hidden, std::min(kda::kRowsGemv, K - r0), ws, s, true, r0));
    KDA_TRY(kda_decode_k(bf(KDA_BUF_QKV_PROJ), conv_state, w->conv, bf(KDA_BUF_G_RAW), w->dt_bias, w->a_log,
                         f32(KDA_BUF_BETA), h_state, bf(KDA_BUF_OUT_GATE), w->o_norm, bf(KDA_BUF_O_NORM_OUT),
                         bf(KDA_BUF_CONV_OUT), f32(KDA_BUF_CORE), K, h_snap, conv_snap, n_snap, d, stream));
    if (!w->o_proj) return KDA_OK;
    for (int r0 = 0; r0 < K; r0 += kda::kRowsGemv) {
        const size_t o = static_cast<size_t>(r0);
        KDA_TRY(kda::proj(bf(KDA_BUF_O_NORM_OUT) + o * qkv, qkv, w->o_proj, qkv, bf(KDA_BUF_FINAL_OUT) + o * Hd, Hd,
                          std::min(kda::kRowsGemv, K - r0), Hd, qkv, 0, s, true, ws));
    }
    return KDA_OK;
}

int kda_block_verify(const kda_block_weights *w, const kda_bf16 *hidden, const int *cu_seqlens, int B,
                     int total_tokens, float *const *h_state, kda_bf16 *const *conv_state, float *tables,
                     size_t tables_bytes, kda_workspace *ws, void *stream) {
    KDA_TRY(kda::check_block_args(w, hidden, ws));
    if (!cu_seqlens || !h_state || !conv_state || !tables || B < 0 || total_tokens < 0) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(tables)) return KDA_ERR_MISALIGNED;
    if (B == 0 || total_tokens == 0) return KDA_OK;
    if (static_cast<size_t>(total_tokens) > ws->max_tokens || B > ws->max_seqs) return KDA_ERR_CAPACITY;
    const kda_dims *d = &ws->dims;
    if (tables_bytes < kda_chunk_verify_tables_bytes(B, d)) return KDA_ERR_CAPACITY;
    if (ws->bytes[KDA_BUF_PREFILL_SCRATCH] < kda::chunk_prefill_slots_scratch_bytes(B, 1, d->heads, d->head_dim))
        return KDA_ERR_CAPACITY;
    auto s = static_cast<cudaStream_t>(stream);
    const int qkv = d->heads * d->head_dim;
    auto bf = [&](int i) { return static_cast<uint16_t *>(ws->buf[i]); };
    auto f32 = [&](int i) { return static_cast<float *>(ws->buf[i]); };
    // every weight read once for all draft rows of all sequences
    KDA_TRY(kda::block_projections(w, hidden, total_tokens, ws, s, false));
    if (kda::verify_by_rows(B, total_tokens)) {
        // short drafts: each (sequence, head) runs its rows in the stateful decode row, with the
        // state in shared memory and written back nowhere (the beta buffer keeps its logits)
        ws->verify_w = *w;
        ws->verify_w_set = 1;
        KDA_TRY(kda::decode_rows_packed(bf(KDA_BUF_QKV_PROJ), conv_state, w->conv, bf(KDA_BUF_G_RAW), w->dt_bias,
                                        w->a_log, f32(KDA_BUF_BETA), h_state, bf(KDA_BUF_OUT_GATE), w->o_norm,
                                        bf(KDA_BUF_O_NORM_OUT), bf(KDA_BUF_CONV_OUT), f32(KDA_BUF_CORE), cu_seqlens,
                                        nullptr, B, total_tokens, d, s));
        if (!w->o_proj) return KDA_OK;
        return kda::proj(bf(KDA_BUF_O_NORM_OUT), qkv, w->o_proj, qkv, bf(KDA_BUF_FINAL_OUT), ws->hidden, total_tokens,
                         ws->hidden, qkv, 0, s, false, ws);
    }
    KDA_TRY(kda::front_varlen(bf(KDA_BUF_QKV_PROJ), conv_state, w->conv, bf(KDA_BUF_CONV_OUT), cu_seqlens, B,
                              total_tokens, d, s));
    KDA_TRY(kda_beta(f32(KDA_BUF_BETA), f32(KDA_BUF_BETA), total_tokens * d->heads, stream));
    KDA_TRY(kda::chunk_verify_tc_fused(bf(KDA_BUF_CONV_OUT), bf(KDA_BUF_G_RAW), w->dt_bias, w->a_log,
                                       f32(KDA_BUF_BETA), cu_seqlens, B, total_tokens, h_state, f32(KDA_BUF_CORE),
                                       tables, d, ws->buf[KDA_BUF_PREFILL_SCRATCH], s));
    KDA_TRY(kda_back_gated_rmsnorm(f32(KDA_BUF_CORE), bf(KDA_BUF_OUT_GATE), w->o_norm, bf(KDA_BUF_O_NORM_OUT),
                                   total_tokens, d, stream));
    if (!w->o_proj) return KDA_OK;
    return kda::proj(bf(KDA_BUF_O_NORM_OUT), qkv, w->o_proj, qkv, bf(KDA_BUF_FINAL_OUT), ws->hidden, total_tokens,
                     ws->hidden, qkv, 0, s, false, ws);
}

int kda_block_verify_fold(const int *cu_seqlens, const int *accepted, int B, int total_tokens, const float *tables,
                          float *const *h_state, kda_bf16 *const *conv_state, kda_workspace *ws, void *stream) {
    if (!ws || !cu_seqlens || !accepted || !tables || !h_state || !conv_state || B < 0 || total_tokens < 0)
        return KDA_ERR_INVALID_ARG;
    if (B == 0) return KDA_OK;
    if (static_cast<size_t>(total_tokens) > ws->max_tokens || B > ws->max_seqs) return KDA_ERR_CAPACITY;
    auto s = static_cast<cudaStream_t>(stream);
    const kda_dims *d = &ws->dims;
    const size_t qkv = static_cast<size_t>(d->heads) * d->head_dim;
    if (kda::verify_by_rows(B, total_tokens)) {
        // the verify ran row by row: the accepted rows run again through the same stateful row,
        // now advancing both states (bits as the verify computed them)
        if (!ws->verify_w_set) return KDA_ERR_INVALID_ARG;
        const kda_block_weights &vw = ws->verify_w;
        auto bfc = [&](int i) { return static_cast<const uint16_t *>(ws->buf[i]); };
        return kda::decode_rows_packed(bfc(KDA_BUF_QKV_PROJ), conv_state, vw.conv, bfc(KDA_BUF_G_RAW), vw.dt_bias,
                                       vw.a_log, static_cast<const float *>(ws->buf[KDA_BUF_BETA]), h_state,
                                       bfc(KDA_BUF_OUT_GATE), nullptr, nullptr, nullptr, nullptr, cu_seqlens, accepted, B,
                                       total_tokens, d, s);
    }
    const auto *conv_out = static_cast<const uint16_t *>(ws->buf[KDA_BUF_CONV_OUT]);
    // k: the BF16 k channels of the verify's conv_out rows (what its core read)
    KDA_TRY(kda::verify_fold(nullptr, conv_out + qkv, 3 * qkv, cu_seqlens, accepted, B, total_tokens, tables, h_state,
                             d, s));
    return kda::conv_state_advance(static_cast<const uint16_t *>(ws->buf[KDA_BUF_QKV_PROJ]), conv_state, cu_seqlens,
                                   accepted, B, total_tokens, d, s);
}

}  // extern "C"
