// Shared device/host helpers of libkda (sm_100a). Internal: not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "kda.h"

namespace kda {

constexpr int kChunk = 64;

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Round-to-nearest-even FP32 -> BF16 (the CUDA intrinsic; NaN stays NaN).
__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}

// softplus in the overflow-free form max(x,0) + log1p(y), y = e^{-|x|} in (0, 1], with y from
// the SFU exponential. log1p(y): for y < 1/8 the series 2 atanh(s) = 2 (s + s^3/3 + s^5/5 +
// s^7/7), s = y / (2 + y) <= 1/17, whose next term is below 1e-10 of the sum; otherwise
// ln(1 + y) from the SFU base-2 logarithm, 1 + y in [9/8, 2] so that its absolute error (about
// 1e-7) stays near 1e-6 of the value. Within 2e-6 of the exact softplus over the whole range.
__device__ __forceinline__ float softplus_f32(float x) {
    const float y = __expf(-fabsf(x));
    float l;
    if (y < 0.125f) {
        const float s = __fdividef(y, 2.0f + y), s2 = s * s;
        l = 2.0f * s * fmaf(s2, fmaf(s2, fmaf(s2, 1.0f / 7.0f, 1.0f / 5.0f), 1.0f / 3.0f), 1.0f);
    } else {
        l = __log2f(1.0f + y) * 0.69314718055994531f;
    }
    return fmaxf(x, 0.0f) + l;
}

// 1 / (1 + e^-x), the reciprocal correctly rounded (the same value an IEEE division gives).
__device__ __forceinline__ float sigmoid_f32(float x) {
    return __frcp_rn(1.0f + expf(-x));
}

// The bounded log-decay gate: -exp(a_log[h]) * softplus(g_raw + dt_bias).
__device__ __forceinline__ float kda_gate_f32(float g_raw, float dt_bias, float neg_exp_alog) {
    return neg_exp_alog * softplus_f32(g_raw + dt_bias);
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SMs of the current device (148 if the query fails).
inline int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

inline bool overlaps(const void *a, size_t abytes, const void *b, size_t bbytes) {
    const char *x = static_cast<const char *>(a), *y = static_cast<const char *>(b);
    return x < y + bbytes && y < x + abytes;
}

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// Basic validation shared by every entry point. Returns KDA_OK or an error code.
inline int check_dims(const kda_dims *d) {
    if (!d) return KDA_ERR_INVALID_ARG;
    if (d->heads < 1) return KDA_ERR_INVALID_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return KDA_ERR_UNSUPPORTED;
    if (d->chunk != kChunk) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// Opt a kernel in to `bytes` of dynamic shared memory, once per device (the attribute belongs
// to the device's context; `done` has one bit per device already set). With max_carveout the
// kernel also asks for the largest shared-memory carve-out, so that several of its CTAs fit.
template <typename K>
int smem_opt_in(K kernel, int bytes, std::atomic<unsigned long long> &done, bool max_carveout = false) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev > 63) return KDA_ERR_CUDA;
    const unsigned long long bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return KDA_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (max_carveout &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return KDA_ERR_CUDA;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return KDA_OK;
}

// Device address of this device's latched status word (kda_api.cu).
int *device_status_ptr();

// The calling thread's current CUDA context (the driver's cuCtxGetCurrent, reached through the
// runtime's entry-point query), or nullptr when there is none or the query fails. A device
// address cached per device is only valid for the context it was looked up in: after a
// cudaDeviceReset the device gets a new context and module-scope arrays new addresses.
void *current_context();

}  // namespace kda

#define KDA_TRY(expr)                        \
    do {                                     \
        int _kda_rc = (expr);                \
        if (_kda_rc != KDA_OK) return _kda_rc; \
    } while (0)

namespace kda {
// Chunked prefill implementations (kda_chunk_simt.cu, kda_chunk_tc.cu).
int chunk_prefill_check(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                        float *const *h_state, float *core, int B, int T, const kda_dims *dims);
int chunk_prefill_simt(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                       float *const *h_state, float *core, int B, int T, const kda_dims *dims, cudaStream_t s);
size_t chunk_prefill_scratch_bytes(int B, int T, int H, int D);
size_t chunk_prefill_slots_scratch_bytes(int B, int nch, int H, int D);  // B streams x nch chunk slots
// Scratch a packed (varlen) call of B streams, max_chunks chunks each at most, total rows needs.
size_t chunk_prefill_varlen_need_bytes(int B, int max_chunks, int total, int H, int D);
// Scratch enough for any packed call of at most max_seqs streams and max_total rows.
size_t chunk_prefill_packed_bytes(int max_seqs, int max_total, int H, int D);
int chunk_prefill_tc_fused_varlen(const uint16_t *qkv, const uint16_t *g_raw, const float *dt_bias, const float *a_log,
                                  const float *beta, const int *cu_seqlens, int B, int max_chunks, int total,
                                  float *const *h_state, float *core, const kda_dims *dims, void *scratch,
                                  cudaStream_t s);
int chunk_verify_tc_fused(const uint16_t *qkv, const uint16_t *g_raw, const float *dt_bias, const float *a_log,
                          const float *beta, const int *cu_seqlens, int B, int total, float *const *h_state,
                          float *core, float *tables, const kda_dims *dims, void *scratch, cudaStream_t s);
// Accepted-row folding (kda_verify.cu): k as FP32 rows [total, H*D] (kf) or BF16 rows of
// stride ldk elements (kb, pointing at head 0's channel 0 of row 0).
int verify_fold(const float *kf, const uint16_t *kb, size_t ldk, const int *cu_seqlens, const int *accepted, int B,
                int total, const float *tables, float *const *h_state, const kda_dims *dims, cudaStream_t s);
// Packed-sequence front end (kda_front.cu): conv + SiLU + q|k L2 of every row from its own
// sequence's conv state (read only), and the conv-state advance over each sequence's first
// `accepted[b]` rows (all rows if accepted is null).
int front_varlen(const uint16_t *x, uint16_t *const *conv_state, const uint16_t *conv_w, uint16_t *conv_out,
                 const int *cu_seqlens, int B, int total, const kda_dims *dims, cudaStream_t s);
int conv_state_advance(const uint16_t *x, uint16_t *const *conv_state, const int *cu_seqlens, const int *accepted,
                       int B, int total, const kda_dims *dims, cudaStream_t s);
int chunk_verify_tc(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                    const int *cu_seqlens, int B, int total, float *const *h_state, float *core, float *tables,
                    const kda_dims *dims, void *scratch, cudaStream_t s);
int chunk_prefill_tc_varlen(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                            const int *cu_seqlens, int B, int max_chunks, int total, float *const *h_state,
                            float *core, const kda_dims *dims, void *scratch, cudaStream_t s);
int chunk_prefill_tc(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                     float *const *h_state, float *core, int B, int T, const kda_dims *dims, void *scratch,
                     cudaStream_t s);
int chunk_prefill_tc_fused(const uint16_t *qkv, const uint16_t *g_raw, const float *dt_bias, const float *a_log,
                           const float *beta, float *const *h_state, float *core, int B, int T, const kda_dims *dims,
                           void *scratch, cudaStream_t s);
int chunk_prefill_tc_graw(const float *q, const float *k, const float *v, const uint16_t *g_raw,
                          const float *dt_bias, const float *a_log, const float *beta, float *const *h_state,
                          float *core, int B, int T, const kda_dims *dims, void *scratch, cudaStream_t s);
}  // namespace kda

namespace kda {
// Projection GEMM and the batched-M matrix-vector products (kda_gemm.cu). Up to three weights
// that read the same rows (q, k and v of one hidden row, say) go in one matrix-vector launch:
// the column index runs over the concatenated outputs.
// The stateful decode row over packed draft rows: a verify (acc null: every row, states kept) or
// a fold (each sequence's first acc[n] rows, states advanced). kda_decode.cu.
int decode_rows_packed(const uint16_t *x, uint16_t *const *conv_state, const uint16_t *conv_w, const uint16_t *g_raw,
                       const float *dt_bias, const float *a_log, const float *b_logit, float *const *h_state,
                       const uint16_t *out_gate, const uint16_t *o_norm_w, uint16_t *o_norm_out, uint16_t *conv_out,
                       float *core, const int *cu, const int *acc, int B, int total, const kda_dims *dims,
                       cudaStream_t s);

struct GemvSeg {
    const uint16_t *W;
    void *y;
    int N, ldw, ldy, out_f32;
    const uint16_t *x;  // this segment's input rows (same row stride), or null: the call's x
};
struct GemvSegs {
    GemvSeg s[6];
    int count, total;
};
int gemm_bf16(const uint16_t *A, int lda, const uint16_t *W, int ldw, void *Cout, int ldc, int M, int N, int K,
              int out_f32, cudaStream_t s);
// Up to six products C_i = A_i . W_i^T of one width N and depth K (M may differ) in one launch.
struct GemmProd {
    const uint16_t *A;
    int lda;
    const uint16_t *W;
    int ldw;
    void *C;
    int ldc, M, N, K, out_f32;
};
int gemm_bf16_multi(const GemmProd *prods, int n, cudaStream_t s);
// A few input rows (at most 256) against up to six weights in one launch, each weight read
// once: y[m][n] = x[m] . W[n] for m < rows, n < N (rows of y at stride ldy), on the tensor
// cores with the weights' rows as the 128-row tiles. Not the matrix-vector kernel's bits.
struct GemmTSeg {
    const uint16_t *W;  // [N, K], row stride ldw
    const uint16_t *x;  // [rows, K], row stride ldx
    void *y;
    int N, ldw, ldx, ldy, out_f32;
};
// part: FP32 buffer for split-K partial sums (null: no split); a launch splits only as far as
// part_bytes holds. small_m_part_bytes(rows) holds any split of a call of that many rows.
int gemm_bf16_small_m(const GemmTSeg *segs, int nseg, int rows, int K, cudaStream_t s, float *part = nullptr,
                      size_t part_bytes = 0);
size_t small_m_part_bytes(int rows);
int gemv_bf16(const uint16_t *x, int ldx, const uint16_t *W, int ldw, void *y, int ldy, int M, int N, int K,
              int out_f32, cudaStream_t s);
int gemv_segs(const uint16_t *x, int ldx, const GemvSegs &segs, int M, int K, cudaStream_t s);
}  // namespace kda
