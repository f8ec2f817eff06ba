/*
 * kda.h — C ABI of the B200 (sm_100a) KDA core library, libkda.so.
 *
 * The KDA core of a GLM-5.3-Next linear-attention block: per head and token, a
 * per-channel bounded log-decay gate, a sigmoid beta, a delta-rule update of a
 * head_dim x head_dim FP32 state and the read-out o = scale * S^T q; run as a chunked
 * prefill (64-token chunks, padded, guarded past T) or as a one-token / K-token decode.
 *
 * Sources (page title, section):
 *   Glm5NextKdaWorkspace — the stage buffers, their shapes and precisions;
 *   Glm5NextKdaLayer     — decode, decode_k (snapshots), prefill, prefill_with_pad_fill;
 *   Glm5NextLayer        — prefill_gdn_full_batched (equal-length streams, a device array
 *                          of one state pointer per stream);
 *   Glm5NextKdaWeights   — weight layouts: Linear [out, in] BF16, conv [conv_dim, 4],
 *                          dt_bias [heads*head_dim] F32 (per channel), a_log [heads] F32
 *                          (per head), o_norm [head_dim] BF16.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers owned by the caller unless a comment says "host".
 *     No compute call allocates device memory: the workspace is sized once, at creation,
 *     and scratch buffers are the caller's. The only other objects created are the graph
 *     kda_block_decode_graph returns and, on the first kda_chunk_prefill_host call on a
 *     device, that call's two copy streams and four events (kept for the process).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls are asynchronous: they enqueue kernels and return.
 *   - Return value: KDA_OK, or an error code from the list below. Argument errors are
 *     found on the host before anything is launched; on such an error nothing runs.
 *     KDA_ERR_CUDA reports a launch error (cudaGetLastError after the launch).
 *     Errors found on the device (a bounded wait that gave up) are latched into a
 *     device status word that kda_device_status() reads.
 *   - BF16 tensors are passed as their 16-bit patterns (kda_bf16).
 *   - Row-major layouts. "[T_pad, H, D]" means T_pad rows of H*D contiguous values.
 *   - Every FP32 / BF16 tensor pointer must be 16-byte aligned (vector loads/stores);
 *     otherwise KDA_ERR_MISALIGNED.
 *   - Dimensions: head_dim D in {64, 128}; chunk = 64; heads H >= 1.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null pointer, negative or zero size, bad count      */
    KDA_ERR_ALIAS = 2,        /* two buffers that must not overlap do (g_raw/out_gate) */
    KDA_ERR_CAPACITY = 3,     /* T beyond the workspace's max_tokens                  */
    KDA_ERR_UNSUPPORTED = 4,  /* head_dim not 64/128, chunk not 64, K too large        */
    KDA_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed                  */
    KDA_ERR_TIMEOUT = 6,      /* device-side bounded wait gave up (latched)            */
    KDA_ERR_MISALIGNED = 7    /* a tensor pointer is not 16-byte aligned               */
};

typedef uint16_t kda_bf16;

/* Model dimensions, passed by host pointer to every call. */
typedef struct kda_dims {
    int heads;      /* H                                                   */
    int head_dim;   /* D = dk = dv (64 or 128)                             */
    int chunk;      /* prefill chunk length; must be 64                    */
    float scale;    /* read-out scale: o = scale * S^T q (1.0 by default)  */
    float l2_eps;   /* q/k L2 norm: x / sqrt(sum x^2 + l2_eps)             */
    float rms_eps;  /* o_norm: x / sqrt(mean x^2 + rms_eps)                */
} kda_dims;

/* Library version (major*100 + minor). */
KDA_API int kda_version(void);

/* Short text for a status code (static storage, never NULL). */
KDA_API const char *kda_status_string(int status);

/* T rounded up to whole chunks: the row count of every prefill buffer ("T_pad",
 * Glm5NextKdaWorkspace: prefill buffers padded to a whole number of chunks). */
KDA_API size_t kda_t_pad(size_t T, int chunk);

/* Read (host *out) and optionally clear the current device's latched status word.
 * Synchronises the device. Returns KDA_OK or KDA_ERR_CUDA. */
KDA_API int kda_device_status(int *out, int clear);

/* ---------------------------------------------------------------------------------
 * kda_gate — the bounded log-decay gate (Glm5NextKdaWorkspace, field `gate`, from
 * field `g_raw`; Glm5NextKdaWeights, `dt_bias` per channel, `a_log` per head):
 *     gate[t, h, d] = -exp(a_log[h]) * softplus(g_raw[t, h*D + d] + dt_bias[h*D + d])
 *   g_raw   [n_rows, H*D] BF16
 *   dt_bias [H*D] F32,  a_log [H] F32
 *   gate    [n_rows, H, D] F32, written for rows 0..n_rows-1 only (a padded caller passes
 *           the valid row count; the tail is left as it is).
 */
KDA_API int kda_gate(const kda_bf16 *g_raw, const float *dt_bias, const float *a_log, float *gate,
             int n_rows, const kda_dims *dims, void *stream);

/* kda_beta — beta = sigmoid(b_logit), elementwise, n values (Glm5NextKdaWorkspace,
 * field `beta`: sigmoid(b_proj(h)) in FP32). b_logit and beta may be the same buffer. */
KDA_API int kda_beta(const float *b_logit, float *beta, int n, void *stream);

/* ---------------------------------------------------------------------------------
 * kda_chunk_prefill — the chunked KDA core over B equal-length streams of T tokens
 * (Glm5NextKdaLayer `prefill` / `prefill_with_pad_fill`; Glm5NextLayer
 * `prefill_gdn_full_batched`). Stream b occupies rows [b*T_pad, b*T_pad + T_pad) of
 * every token-major buffer, T_pad = kda_t_pad(T, 64); rows >= T of each stream are
 * padding: they are never read into the state or the valid outputs, whatever they hold
 * (the in-kernel guard that prefill_with_pad_fill's poison tail tests).
 *   q, k, v   [B*T_pad, H, D] F32; q and k are used as given (already L2-normalised)
 *   gate      [B*T_pad, H, D] F32 log-decay (kda_gate's output)
 *   beta      [B*T_pad, H]    F32 (kda_beta's output)
 *   h_state   DEVICE array of B device pointers, each to that stream's [H, D, D] F32
 *             state (row = key channel, column = value channel); read as the carried
 *             state and overwritten with the state after exactly T tokens.
 *   core      [B*T_pad, H, D] F32 output o = scale * S^T q for rows < T (pad rows are
 *             not written).
 *   scratch   caller-owned device scratch of at least kda_chunk_prefill_scratch_bytes(B, T,
 *             dims) bytes (149 KB per (stream, head, chunk) at head_dim 128), 16-byte aligned:
 *             the per-chunk operand tiles passed between the two kernels of the call; contents
 *             on entry do not matter. KDA_ERR_CAPACITY if scratch_bytes is too small.
 * Computed with tcgen05 tensor cores in split-BF16 precision (about 2^-16 relative per
 * product). The per-(stream, head) states must not overlap each other or any input.
 */
KDA_API int kda_chunk_prefill(const float *q, const float *k, const float *v, const float *gate,
                              const float *beta, float *const *h_state, float *core, int B, int T,
                              void *scratch, size_t scratch_bytes, const kda_dims *dims, void *stream);

/* Scratch bytes kda_chunk_prefill needs for B streams of T tokens (0 if B or T is 0). */
KDA_API size_t kda_chunk_prefill_scratch_bytes(int B, int T, const kda_dims *dims);

/* kda_chunk_prefill_varlen — kda_chunk_prefill over B sequences of UNEQUAL lengths packed back
 * to back (Glm5NextLayer varlen prefill: `cu_seqlens`, `max_num_chunks`): sequence b is rows
 * [cu_seqlens[b], cu_seqlens[b+1]) of every token-major buffer, chunked from its own first
 * row; the rows after a sequence's end (the next sequence's) never enter its chunks.
 *   q, k, v, gate [total_tokens, H, D] F32;  beta [total_tokens, H] F32;  core likewise
 *   cu_seqlens     DEVICE int32 [B + 1], cu_seqlens[0] = 0, non-decreasing, last = total_tokens
 *   max_num_chunks at least ceil(len_b / 64) for every sequence (the scratch has that many
 *                  chunk slots per sequence)
 *   h_state        DEVICE array of B state pointers, read and overwritten (an empty sequence
 *                  keeps its state)
 *   scratch        at least kda_chunk_prefill_varlen_scratch_bytes(B, max_num_chunks, dims), or
 *                  kda_chunk_prefill_packed_scratch_bytes(m, t, dims) for any m >= B, t >= total_tokens
 *                  (the call takes the smaller of the two chunk-slot layouts; KDA_ERR_CAPACITY if the
 *                  scratch holds neither)
 * A sequence whose bounds do not fit (negative, decreasing, past total_tokens, or longer than
 * max_num_chunks * 64) is skipped, its state untouched, and KDA_ERR_INVALID_ARG is latched in
 * kda_device_status. Each sequence's result equals kda_chunk_prefill on that sequence alone. */
KDA_API int kda_chunk_prefill_varlen(const float *q, const float *k, const float *v, const float *gate,
                                     const float *beta, const int *cu_seqlens, int B, int max_num_chunks,
                                     int total_tokens, float *const *h_state, float *core, void *scratch,
                                     size_t scratch_bytes, const kda_dims *dims, void *stream);

/* Scratch bytes kda_chunk_prefill_varlen needs (0 if B or max_num_chunks is 0): one operand
 * pack per (sequence, head, chunk slot). */
KDA_API size_t kda_chunk_prefill_varlen_scratch_bytes(int B, int max_num_chunks, const kda_dims *dims);

/* Scratch bytes enough for every kda_chunk_prefill_varlen call of at most max_seqs sequences and
 * max_total_tokens rows, whatever the mix of lengths (0 if either is 0): the compact layout, in
 * which sequence b's chunks take consecutive pack slots from floor(cu_seqlens[b] / 64) + b, so
 * a head needs ceil(max_total_tokens / 64) + max_seqs - 1 slots. */
KDA_API size_t kda_chunk_prefill_packed_scratch_bytes(int max_seqs, int max_total_tokens, const kda_dims *dims);

/* kda_chunk_verify — batched verify under the WY tables (Glm5NextLayer speculative verify):
 * the draft rows of B sequences, packed as for kda_chunk_prefill_varlen, each sequence at most
 * 64 rows (one chunk), go through the chunked kernels from each sequence's state, which is NOT
 * updated. Outputs `core` for every row (the same bits kda_chunk_prefill_varlen gives), and
 * keeps in `tables` (kda_chunk_verify_tables_bytes(B, dims) bytes, 16-byte aligned) per
 * (sequence, head): the rows' update vectors U [64][D] and the in-chunk cumulative log-decay
 * Gamma [64][D], both FP32, for kda_chunk_verify_fold. scratch as kda_chunk_prefill_varlen with
 * max_num_chunks = 1. A sequence longer than 64 rows is skipped and latches
 * KDA_ERR_INVALID_ARG. */
KDA_API int kda_chunk_verify(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                             const int *cu_seqlens, int B, int total_tokens, float *const *h_state, float *core,
                             float *tables, size_t tables_bytes, void *scratch, size_t scratch_bytes,
                             const kda_dims *dims, void *stream);

/* Bytes of the tables kda_chunk_verify keeps for B sequences (B * heads * 2 * 64 * D * 4). */
KDA_API size_t kda_chunk_verify_tables_bytes(int B, const kda_dims *dims);

/* kda_chunk_verify_fold — accepted-row folding: sequence b's state becomes the state after its
 * first accepted[b] verified rows (DEVICE int32 [B], 0 <= accepted[b] <= its row count):
 *   S_r = diag(e^{Gamma_{r-1}}) S + sum_{t<r} (k_t o e^{Gamma_{r-1} - Gamma_t}) u_t^T
 * from the verify tables and the same k rows; accepted[b] = 0 leaves the state. Run after
 * kda_chunk_verify on the same states, before anything else changes them. Bad bounds latch
 * KDA_ERR_INVALID_ARG and leave that state. */
KDA_API int kda_chunk_verify_fold(const float *k, const int *cu_seqlens, const int *accepted, int B,
                                  int total_tokens, const float *tables, float *const *h_state,
                                  const kda_dims *dims, void *stream);

/* kda_chunk_prefill_fused — kda_chunk_prefill reading the front end's BF16 output and the
 * raw gate directly (Glm5NextKdaWorkspace `conv_out` and `g_raw`: the fused-input mode, in
 * which the FP32 q/k/v/gate buffers are never written or read):
 *   qkv       [B*T_pad, 3*H*D] BF16 rows q | k | v after conv + SiLU + per-head L2 (the
 *             layout kda_front_conv_silu_l2 writes to conv_out); only rows < T are read
 *   g_raw     [B*T_pad, H*D] BF16; dt_bias [H*D] F32; a_log [H] F32: the gate
 *             g = -exp(a_log[h]) softplus(g_raw + dt_bias) (as kda_gate) is formed in the
 *             kernel; only rows < T are read
 *   beta      [B*T_pad, H] F32 (kda_beta's output)
 *   h_state, core, B, T, scratch, scratch_bytes, dims: as kda_chunk_prefill (same scratch size).
 * The result equals kda_chunk_prefill on the widened inputs and kda_gate's output. */
KDA_API int kda_chunk_prefill_fused(const kda_bf16 *qkv, const kda_bf16 *g_raw, const float *dt_bias,
                                    const float *a_log, const float *beta, float *const *h_state, float *core,
                                    int B, int T, void *scratch, size_t scratch_bytes, const kda_dims *dims,
                                    void *stream);

/* kda_chunk_prefill_graw — kda_chunk_prefill with the gate step folded in: FP32 q, k, v as
 * kda_chunk_prefill, and the raw gate projection instead of kda_gate's output
 * (Glm5NextKdaWorkspace `g_raw`; Glm5NextKdaWeights `dt_bias`, `a_log`):
 *   g_raw     [B*T_pad, H*D] BF16; dt_bias [H*D] F32; a_log [H] F32: the kernel forms
 *             g = -exp(a_log[h]) softplus(g_raw + dt_bias) exactly as kda_gate does; only rows
 *             < T are read (the FP32 gate buffer is never written or read)
 *   q, k, v, beta, h_state, core, B, T, scratch, scratch_bytes, dims: as kda_chunk_prefill
 *             (same scratch size).
 * Errors as kda_chunk_prefill (g_raw must be 16-byte aligned too). The result is bit-identical
 * to kda_gate followed by kda_chunk_prefill on the same inputs. */
KDA_API int kda_chunk_prefill_graw(const float *q, const float *k, const float *v, const kda_bf16 *g_raw,
                                   const float *dt_bias, const float *a_log, const float *beta,
                                   float *const *h_state, float *core, int B, int T, void *scratch,
                                   size_t scratch_bytes, const kda_dims *dims, void *stream);

/* kda_chunk_prefill_host — kda_beta + kda_chunk_prefill_fused for ONE sequence whose inputs
 * and outputs are in HOST memory (a deployment variant; the pages keep everything on the device):
 * the host->device copies, the kernels and the device->host copies of consecutive segments of
 * segment_tokens tokens overlap on three streams (two copy streams the library keeps per device,
 * and `stream`), so the call costs about the slower PCIe direction rather than the sum.
 *   qkv      HOST [T, 3*H*D] BF16 rows q | k | v (the layout kda_chunk_prefill_fused reads)
 *   g_raw    HOST [T, H*D] BF16;  b_logit HOST [T, H] F32 (beta = sigmoid(b_logit) is formed here)
 *   dt_bias  DEVICE [H*D] F32;  a_log DEVICE [H] F32
 *   h_state  HOST [H, D, D] F32: read as the carried state, overwritten with the state after T
 *   core     HOST [T, H, D] F32 output
 *   segment_tokens  a positive multiple of 64 (512 is a good size on PCIe 5)
 *   device_buffer   DEVICE, 16-byte aligned, at least kda_chunk_prefill_host_bytes(T,
 *                   segment_tokens, dims) bytes: the staging rows, beta, core, the state and one
 *                   segment's prefill scratch; contents on entry do not matter
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for the copies to
 * overlap; pageable ones work but serialise. The call only enqueues: host outputs are complete
 * once `stream` has completed (it waits for the last copy out). Calls from several host threads
 * are serialised while they enqueue. Because segments are whole chunks, core and the final state
 * are the same bits as kda_beta + kda_chunk_prefill_fused over all T rows on the device.
 * Errors: KDA_ERR_INVALID_ARG (NULL pointer, T < 0, bad segment_tokens), KDA_ERR_MISALIGNED,
 * KDA_ERR_CAPACITY (device_bytes too small), all found before anything is enqueued; KDA_ERR_CUDA
 * (a runtime call failed part-way: some copies or kernels may be in flight, so synchronise the
 * device before reading the outputs or reusing device_buffer). */
KDA_API int kda_chunk_prefill_host(const kda_bf16 *qkv, const kda_bf16 *g_raw, const float *b_logit,
                                   const float *dt_bias, const float *a_log, float *h_state, float *core, int T,
                                   int segment_tokens, void *device_buffer, size_t device_bytes,
                                   const kda_dims *dims, void *stream);

/* Device bytes kda_chunk_prefill_host needs (0 if T <= 0 or segment_tokens is not a positive
 * multiple of 64). */
KDA_API size_t kda_chunk_prefill_host_bytes(int T, int segment_tokens, const kda_dims *dims);

/* kda_chunk_prefill_host_f32 — the FP32-input form of kda_chunk_prefill_host: the device call it
 * stands for is kda_gate + kda_beta + kda_chunk_prefill on FP32 q, k, v (the workload of the
 * chunked-prefill benchmark), run segment by segment with the same three-stream overlap.
 *   q, k, v  HOST [T, H*D] F32 each;  g_raw HOST [T, H*D] BF16 (the gate is formed by kda_gate);
 *   b_logit, dt_bias, a_log, h_state, core, segment_tokens, stream: as kda_chunk_prefill_host
 *   device_buffer   at least kda_chunk_prefill_host_f32_bytes(T, segment_tokens, dims) bytes
 * core and the final state are the same bits as kda_gate + kda_beta + kda_chunk_prefill over all
 * T rows on the device. Errors as kda_chunk_prefill_host. */
KDA_API int kda_chunk_prefill_host_f32(const float *q, const float *k, const float *v, const kda_bf16 *g_raw,
                                       const float *b_logit, const float *dt_bias, const float *a_log,
                                       float *h_state, float *core, int T, int segment_tokens, void *device_buffer,
                                       size_t device_bytes, const kda_dims *dims, void *stream);

/* Device bytes kda_chunk_prefill_host_f32 needs (0 as kda_chunk_prefill_host_bytes). */
KDA_API size_t kda_chunk_prefill_host_f32_bytes(int T, int segment_tokens, const kda_dims *dims);

/* kda_chunk_prefill_noalloc — kda_chunk_prefill for callers that cannot allocate device
 * memory (the pages have no counterpart: this is a deployment variant). Some callers cannot
 * call cudaMalloc at all: an engine that hands all free HBM to its KV-cache / state pools at
 * start-up has no room left for a scratch buffer, and a plug-in inside a host framework that
 * owns the memory budget may not allocate behind its back. This entry point allocates
 * nothing and takes no scratch argument: it uses one file-scope device array of
 * kda_chunk_prefill_noalloc_max_scratch_bytes() bytes (32 MiB), which every GPU that loads
 * the library holds until the process exits.
 *   - Arguments, layouts and results are exactly those of kda_chunk_prefill.
 *   - Requests needing more scratch than that (kda_chunk_prefill_scratch_bytes(B, T, dims)
 *     above the maximum; for head_dim 128, B * heads * ceil(T / 64) > 219 chunks) are
 *     rejected with KDA_ERR_CAPACITY before anything runs.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before any stream capture. The lookup
 *     loads the array's module, which is when its 32 MiB are taken from the device (modules
 *     load lazily): a call with B == 0 or T == 0 does only this, so an engine that hands all
 *     free memory to its pools makes one such call per device first (or runs with
 *     CUDA_MODULE_LOADING=EAGER, which reserves the array when the library loads).
 *   - The address is cached per device together with the CUDA context it belongs to; after
 *     a cudaDeviceReset (a new context) the next call looks it up again.
 *   - Every call shares the one array and it keeps the last call's contents. Nothing in it
 *     needs to start at zero (each call writes every tile it later reads), but calls that
 *     overlap on the GPU (different streams, or different host threads) race on it:
 *     serialise them.
 */
KDA_API int kda_chunk_prefill_noalloc(const float *q, const float *k, const float *v, const float *gate,
                                      const float *beta, float *const *h_state, float *core, int B, int T,
                                      const kda_dims *dims, void *stream);

/* Size in bytes of the device array kda_chunk_prefill_noalloc uses (32 MiB). */
KDA_API size_t kda_chunk_prefill_noalloc_max_scratch_bytes(void);

/* kda_chunk_prefill_simt — the same contract as kda_chunk_prefill, computed by the
 * plain FP32 CUDA-core kernel (no tensor cores). Kept as a second implementation. */
KDA_API int kda_chunk_prefill_simt(const float *q, const float *k, const float *v, const float *gate,
                           const float *beta, float *const *h_state, float *core, int B, int T,
                           const kda_dims *dims, void *stream);

/* ---------------------------------------------------------------------------------
 * kda_recurrent_decode — one token for each of N independent sequences, from
 * pre-normalised q/k (Glm5NextKdaLayer `decode`: kda_recurrent takes q/k as given):
 *     S' = diag(exp(gate)) S;  u = beta (v - S'^T k);  S = S' + k u^T;  o = scale S^T q
 *   q, k, v, gate [N, H, D] F32;  beta [N, H] F32
 *   h_state   DEVICE array of N device pointers to [H, D, D] F32 states, updated in place;
 *             each 16-byte aligned (a misaligned one is skipped and latches
 *             KDA_ERR_MISALIGNED in kda_device_status)
 *   o         [N, H, D] F32
 */
KDA_API int kda_recurrent_decode(const float *q, const float *k, const float *v, const float *gate,
                         const float *beta, float *const *h_state, float *o, int N,
                         const kda_dims *dims, void *stream);

/* ---------------------------------------------------------------------------------
 * kda_decode_fused — the whole stateful row of the block decode for N sequences, one
 * token each, in one kernel per (sequence, head) (Glm5NextKdaLayer `decode`: the conv
 * fuses SiLU and L2, the recurrence reads the pre-normalised BF16 q/k, then o_norm):
 *   conv:  y[c] = sum_{j<3} w[c,j] * state[c,j] + w[c,3] * x[c]; SiLU; per-head L2 of the
 *          q and k channels (one BF16 rounding); state <- (state[c,1], state[c,2], x[c])
 *   gate:  as kda_gate;  beta = sigmoid(b_logit)
 *   core:  one recurrence step as kda_recurrent_decode
 *   o_norm: out = core / sqrt(mean_d core^2 + rms_eps) * w_o[d] * sigmoid(out_gate) (BF16)
 * Arguments:
 *   x          [N, 3*H*D] BF16: the q|k|v projection rows (before the conv)
 *   conv_state DEVICE array of N device pointers to [3*H*D, 3] BF16 (oldest -> newest),
 *              updated in place
 *   conv_w     [3*H*D, 4] BF16 (tap 3 multiplies the current token)
 *   g_raw      [N, H*D] BF16;  dt_bias [H*D] F32;  a_log [H] F32;  b_logit [N, H] F32
 *   h_state    DEVICE array of N device pointers to [H, D, D] F32 states, in place, each
 *              16-byte aligned (a misaligned one is skipped and latches KDA_ERR_MISALIGNED)
 *   out_gate   [N, H*D] BF16 (must not overlap g_raw: KDA_ERR_ALIAS)
 *   o_norm_w   [D] BF16
 *   o_norm_out [N, H*D] BF16 output
 *   conv_out   [N, 3*H*D] BF16 output of the front end, or NULL
 *   core       [N, H, D] F32 output before o_norm, or NULL
 */
KDA_API int kda_decode_fused(const kda_bf16 *x, kda_bf16 *const *conv_state, const kda_bf16 *conv_w,
                     const kda_bf16 *g_raw, const float *dt_bias, const float *a_log,
                     const float *b_logit, float *const *h_state, const kda_bf16 *out_gate,
                     const kda_bf16 *o_norm_w, kda_bf16 *o_norm_out, kda_bf16 *conv_out,
                     float *core, int N, const kda_dims *dims, void *stream);

/* kda_decode_k — K rows of ONE sequence (Glm5NextKdaLayer `decode_k`): the stateful
 * row of kda_decode_fused applied K times in order, the state kept in shared memory.
 * Bit-identical to K serial kda_decode_fused calls with N = 1 (the same device code
 * runs each row). Arguments as kda_decode_fused with N replaced by K rows of one
 * sequence, and conv_state / h_state single device pointers. Snapshots:
 *   n_snap     0 or K-1
 *   h_snap     HOST array of n_snap device pointers to [H, D, D] F32, or NULL if n_snap = 0
 *   conv_snap  HOST array of n_snap device pointers to [3*H*D, 3] BF16, or NULL
 * snapshot t receives the (recurrent, conv) state AFTER row t, t = 0..K-2.
 * K >= 1. One launch carries at most 32 rows; a longer call runs as launches of up to 32 rows,
 * each continuing from the state the previous one left in place (the FP32 state and the BF16
 * conv inputs round-trip exactly, so the result is still bit-identical to K serial decodes).
 */
KDA_API int kda_decode_k(const kda_bf16 *x, kda_bf16 *conv_state, const kda_bf16 *conv_w,
                 const kda_bf16 *g_raw, const float *dt_bias, const float *a_log,
                 const float *b_logit, float *h_state, const kda_bf16 *out_gate,
                 const kda_bf16 *o_norm_w, kda_bf16 *o_norm_out, kda_bf16 *conv_out, float *core,
                 int K, float *const *h_snap, kda_bf16 *const *conv_snap, int n_snap,
                 const kda_dims *dims, void *stream);

/* kda_front_conv_silu_l2_varlen — the front end of kda_front_conv_silu_l2 (the same per-row
 * arithmetic) over B sequences packed back to back (Glm5NextLayer varlen prefill): row t of
 * sequence b (rows [cu_seqlens[b], cu_seqlens[b+1])) takes its conv window from that sequence
 * only, reaching into sequence b's carried conv state before its first row.
 *   x           [total_tokens, 3*H*D] BF16 (qkv_proj rows);  conv_out likewise (output)
 *   conv_state  DEVICE array of B device pointers to [3*H*D, 3] BF16 conv states (16-byte aligned;
 *               a misaligned one latches KDA_ERR_MISALIGNED and its rows are skipped)
 *   cu_seqlens  DEVICE int32 [B + 1] as kda_chunk_prefill_varlen
 *   advance_state  0: the conv states are only read (a verify); else each is then replaced by
 *               the last three inputs of (state || its rows), as kda_front_conv_silu_l2 does
 * No FP32 widening (the packed block core reads conv_out). Bad cu_seqlens bounds latch
 * KDA_ERR_INVALID_ARG; the rows of the tile that met them are skipped. */
KDA_API int kda_front_conv_silu_l2_varlen(const kda_bf16 *x, kda_bf16 *const *conv_state, const kda_bf16 *conv_w,
                                          kda_bf16 *conv_out, const int *cu_seqlens, int B, int total_tokens,
                                          int advance_state, const kda_dims *dims, void *stream);

/* kda_conv_state_fold — the conv half of accepted-row folding (Glm5NextLayer `gdn_fold_accepted`):
 * sequence b's conv state becomes the last three inputs of (state || its first accepted[b] rows
 * of x), x the qkv_proj rows the verify's front end read; accepted = NULL takes every row.
 * accepted DEVICE int32 [B], 0 <= accepted[b] <= the sequence's rows (else KDA_ERR_INVALID_ARG is
 * latched and that state left); 0 leaves the state. Other arguments as
 * kda_front_conv_silu_l2_varlen. */
KDA_API int kda_conv_state_fold(const kda_bf16 *x, kda_bf16 *const *conv_state, const int *cu_seqlens,
                                const int *accepted, int B, int total_tokens, const kda_dims *dims, void *stream);

/* ---------------------------------------------------------------------------------
 * kda_front_conv_silu_l2 — prefill front end for one sequence of T tokens
 * (Glm5NextKdaWorkspace, fields `conv_out` and `q_f32`/`k_f32`/`v_f32`):
 *   conv (as kda_decode_fused, from the carried conv state) + SiLU -> BF16 conv_out;
 *   then l2_norm_bf16 in place on the q|k channels (per head, on the BF16 values);
 *   then, if the F32 pointers are not NULL, q/k/v widened to [T_pad, H*D] F32 with rows
 *   T..T_pad-1 set to pad_fill (Glm5NextKdaLayer `prefill_with_pad_fill`).
 *   x          [T, 3*H*D] BF16 (qkv_proj)
 *   conv_state [3*H*D, 3] BF16, carried: replaced by the last three inputs of (state || x)
 *   conv_w     [3*H*D, 4] BF16
 *   conv_out   [T, 3*H*D] BF16 output
 *   q_f32, k_f32, v_f32  [T_pad, H*D] F32 outputs, all three or none (NULL)
 */
KDA_API int kda_front_conv_silu_l2(const kda_bf16 *x, kda_bf16 *conv_state, const kda_bf16 *conv_w,
                           kda_bf16 *conv_out, float *q_f32, float *k_f32, float *v_f32,
                           float pad_fill, int T, const kda_dims *dims, void *stream);

/* kda_back_gated_rmsnorm — the sigmoid-gated RMSNorm over head_dim (Glm5NextKdaWorkspace,
 * field `o_norm_out`; Glm5NextKdaWeights, field `o_norm`):
 *     out[t, h*D+d] = core[t,h,d] / sqrt(mean_d core[t,h,:]^2 + rms_eps) * w[d]
 *                     * sigmoid(out_gate[t, h*D+d])                       -> BF16
 *   core [T, H, D] F32;  out_gate [T, H*D] BF16;  w [D] BF16;  out [T, H*D] BF16
 */
KDA_API int kda_back_gated_rmsnorm(const float *core, const kda_bf16 *out_gate, const kda_bf16 *w,
                           kda_bf16 *out, int T, const kda_dims *dims, void *stream);

/* ---------------------------------------------------------------------------------
 * kda_gemm_bf16 — C[M x N] = A[M x K] . W[N x K]^T with BF16 A and W (torch Linear
 * layout [out, in], Glm5NextKdaWeights) and FP32 accumulation on the tensor cores; C is
 * BF16 (out_f32 = 0) or FP32 (out_f32 = 1). Row strides lda, ldw, ldc in elements (ldc lets a
 * projection write into a column range of a wider row, e.g. the packed q|k|v rows).
 * K a multiple of 64; A and W 16-byte aligned with lda/ldw multiples of 8 (TMA tiles). M and N
 * are free (tiles are masked); C rows are written with 16-byte stores when C is 16-byte aligned
 * and ldc a multiple of 8 (BF16) / 4 (FP32), element by element otherwise.
 */
KDA_API int kda_gemm_bf16(const kda_bf16 *A, int lda, const kda_bf16 *W, int ldw, void *C, int ldc, int M, int N,
                          int K, int out_f32, void *stream);

/* kda_gemv_bf16 — y[m][n] = sum_k x[m][k] W[n][k] for a few rows (the decode / verify
 * projections; the batched-M matrix-vector product of Glm5NextKdaLayer `decode_k`): W [N, K]
 * BF16 (row stride ldw) is read once per group of 8 rows; FP32 accumulation; y BF16 (out_f32
 * = 0) or F32, row stride ldy. Each output's arithmetic is fixed by K and its own row (lane-
 * strided 8-element steps, then a fixed 32-lane butterfly), so a row gives the same bits
 * whatever M is. K % 8 == 0, K <= 8192 (else KDA_ERR_UNSUPPORTED); x, W 16-byte aligned with
 * ldx, ldw multiples of 8 (else KDA_ERR_MISALIGNED). */
KDA_API int kda_gemv_bf16(const kda_bf16 *x, int ldx, const kda_bf16 *W, int ldw, void *y, int ldy, int M, int N,
                          int K, int out_f32, void *stream);

/* ---------------------------------------------------------------------------------
 * Block prefill: one KDA block over T tokens of one sequence (Glm5NextKdaLayer `prefill` /
 * `prefill_with_pad_fill`), stage by stage into a workspace (Glm5NextKdaWorkspace) that is
 * allocated once for max_tokens. Weights are device pointers in the layouts of
 * Glm5NextKdaWeights; hidden, rank and H*D multiples of 64.
 */
typedef struct kda_block_weights {
    const kda_bf16 *q_proj, *k_proj, *v_proj; /* [H*D, hidden] each                     */
    const kda_bf16 *conv;                     /* [3*H*D, 4] depthwise conv (q|k|v)       */
    const kda_bf16 *f_a;                      /* [rank, hidden]                          */
    const kda_bf16 *f_b;                      /* [H*D, rank]                             */
    const float *dt_bias;                     /* [H*D] F32, per channel                  */
    const float *a_log;                       /* [H] F32, per head                       */
    const kda_bf16 *b_proj;                   /* [H, hidden]                             */
    const kda_bf16 *g_a;                      /* [rank, hidden]                          */
    const kda_bf16 *g_b;                      /* [H*D, rank]                             */
    const kda_bf16 *o_norm;                   /* [D]                                     */
    const kda_bf16 *o_proj;                   /* [hidden, H*D], or NULL: the block calls stop
                                                 after o_norm_out (a tensor-parallel caller
                                                 applies its o_proj slice and the all-reduce) */
    int hidden, rank;
} kda_block_weights;

/* Workspace stage buffers (kda_workspace_buffer): shapes for T tokens, T_pad = kda_t_pad(T, 64). */
enum {
    KDA_BUF_QKV_PROJ = 0,   /* [T, 3*H*D] BF16  q|k|v projections                  */
    KDA_BUF_CONV_OUT,       /* [T, 3*H*D] BF16  after conv + SiLU, q|k normalised  */
    KDA_BUF_Q_F32,          /* 0 bytes: the block's core reads conv_out directly   */
    KDA_BUF_K_F32,          /* 0 bytes (as above)                                  */
    KDA_BUF_V_F32,          /* 0 bytes (as above)                                  */
    KDA_BUF_GATE,           /* 0 bytes: the gate is formed inside the core         */
    KDA_BUF_BETA,           /* [T_pad, H] F32                                      */
    KDA_BUF_CORE,           /* [T_pad, H, D] F32 KDA output before o_norm          */
    KDA_BUF_G_RAW,          /* [T, H*D] BF16  f_b(f_a(h))                           */
    KDA_BUF_OUT_GATE,       /* [T, H*D] BF16  g_b(g_a(h))                           */
    KDA_BUF_O_NORM_OUT,     /* [T, H*D] BF16                                       */
    KDA_BUF_FINAL_OUT,      /* [T, hidden] BF16  block output                      */
    KDA_BUF_F_A_OUT,        /* [T, rank] BF16                                      */
    KDA_BUF_G_A_OUT,        /* [T, rank] BF16                                      */
    KDA_BUF_PREFILL_SCRATCH,/* chunked-prefill scratch                             */
    KDA_BUF_COUNT
};

typedef struct kda_workspace kda_workspace;

/* Allocate the workspace for up to max_tokens tokens (the only allocating call); single-sequence
 * calls and packed calls of one sequence. */
KDA_API int kda_workspace_create(const kda_dims *dims, int hidden, int rank, size_t max_tokens,
                                 kda_workspace **out);
/* The same for packed calls (kda_block_prefill_varlen / _batched, kda_block_verify) of up to
 * max_seqs sequences and max_tokens rows in all: the chunked-prefill scratch is sized by
 * kda_chunk_prefill_packed_scratch_bytes(max_seqs, max_tokens), which fits any mix of lengths.
 * max_seqs = 1 is kda_workspace_create. Besides the stage buffers, the workspace holds an FP32
 * buffer for the split-K partial sums of projections over at most 256 rows (one 128 x BN tile
 * per SM; BN the smallest of 32, 64, 128, 256 covering min(max_tokens, 256) rows: 19 MB on a
 * 148-SM GPU at BN 256). */
KDA_API int kda_workspace_create_batched(const kda_dims *dims, int hidden, int rank, size_t max_tokens,
                                         int max_seqs, kda_workspace **out);
KDA_API int kda_workspace_destroy(kda_workspace *ws);
KDA_API size_t kda_workspace_max_tokens(const kda_workspace *ws);
KDA_API int kda_workspace_max_seqs(const kda_workspace *ws);
/* Device pointer and size of one stage buffer (the buffers are public so each stage can be
 * compared on its own, as the workspace page intends). */
KDA_API int kda_workspace_buffer(const kda_workspace *ws, int which, void **ptr, size_t *bytes);

/* kda_block_prefill — hidden [T, hidden] BF16 (device); h_state [H, D, D] F32 and conv_state
 * [3*H*D, 3] BF16 are carried and updated in place. The chunked core runs in the fused-input
 * mode (kda_chunk_prefill_fused on conv_out and g_raw), which never reads a row past T, so
 * pad_fill (Glm5NextKdaLayer `prefill_with_pad_fill`; 0 for `prefill`) cannot change the
 * result; it is accepted for that signature. The block output lands in KDA_BUF_FINAL_OUT.
 * KDA_ERR_CAPACITY if T > max_tokens. Allocates nothing. */
KDA_API int kda_block_prefill(const kda_block_weights *w, const kda_bf16 *hidden, int T, float *h_state,
                              kda_bf16 *conv_state, float pad_fill, kda_workspace *ws, void *stream);

/* kda_block_prefill_varlen — B sequences packed back to back through one block call
 * (Glm5NextLayer `prefill_gdn_full_batched` in its varlen form): the projections, beta, o_norm
 * and o_proj run once over all total_tokens rows; the conv (kda_front_conv_silu_l2_varlen) and
 * the chunked core (the fused-input mode of kda_chunk_prefill_varlen) keep the sequences apart.
 *   hidden      [total_tokens, hidden] BF16 (device), sequence b = rows [cu_seqlens[b], cu_seqlens[b+1])
 *   cu_seqlens  DEVICE int32 [B + 1];  max_num_chunks >= ceil(len_b / 64) for every sequence
 *   h_state     DEVICE array of B pointers to [H, D, D] F32 states, carried and updated in place
 *   conv_state  DEVICE array of B pointers to [3*H*D, 3] BF16 conv states, likewise
 * Each sequence's rows and states equal kda_block_prefill on that sequence alone, up to the
 * projection GEMM (the same kernel on more rows). An empty sequence keeps its states.
 * Results in the workspace rows 0..total_tokens-1 (KDA_BUF_FINAL_OUT and the stage buffers).
 * KDA_ERR_CAPACITY if total_tokens > max_tokens or B > max_seqs. Allocates nothing. */
KDA_API int kda_block_prefill_varlen(const kda_block_weights *w, const kda_bf16 *hidden, const int *cu_seqlens, int B,
                                     int max_num_chunks, int total_tokens, float *const *h_state,
                                     kda_bf16 *const *conv_state, kda_workspace *ws, void *stream);

/* kda_block_prefill_batched — B sequences of T rows each (Glm5NextLayer
 * `prefill_gdn_full_batched`): hidden [B*T, hidden] BF16, sequence b = rows [b T, (b+1) T);
 * the call writes the cu_seqlens into the workspace and runs kda_block_prefill_varlen.
 * KDA_ERR_CAPACITY if B*T > max_tokens or B > max_seqs. */
KDA_API int kda_block_prefill_batched(const kda_block_weights *w, const kda_bf16 *hidden, int B, int T,
                                      float *const *h_state, kda_bf16 *const *conv_state, kda_workspace *ws,
                                      void *stream);

/* kda_block_decode — N independent sequences, one token each, through the whole block
 * (Glm5NextKdaLayer `decode`): the projections of the N hidden rows (each weight read once for
 * all rows), kda_decode_fused's stateful row, then o_proj.
 *   hidden      [N, hidden] BF16 (device)
 *   h_state     DEVICE array of N pointers to [H, D, D] F32 states (as kda_decode_fused)
 *   conv_state  DEVICE array of N pointers to [3*H*D, 3] BF16 conv states
 * Results: KDA_BUF_FINAL_OUT rows 0..N-1 (block output), and the stage buffers QKV_PROJ,
 * G_RAW, BETA (FP32 beta logits), OUT_GATE, CONV_OUT, CORE, O_NORM_OUT for those rows.
 * KDA_ERR_CAPACITY if N > max_tokens. Allocates nothing. */
KDA_API int kda_block_decode(const kda_block_weights *w, const kda_bf16 *hidden, int N, float *const *h_state,
                             kda_bf16 *const *conv_state, kda_workspace *ws, void *stream);

/* kda_block_decode_k — K rows of ONE sequence through the whole block (Glm5NextKdaLayer
 * `decode_k`: the K-token verify reads every weight once for all K rows). Projections of the
 * K rows in one pass, kda_decode_k's stateful rows with snapshots, then o_proj.
 * Bit-identical to K serial kda_block_decode calls with N = 1 on the same sequence (every
 * projection of a row computes the same bits whatever the number of rows in the call).
 *   hidden [K, hidden] BF16; h_state [H, D, D] F32 and conv_state [3*H*D, 3] BF16 (single
 *   device pointers, updated in place); h_snap, conv_snap, n_snap as kda_decode_k.
 * 1 <= K <= max_tokens (else KDA_ERR_CAPACITY). The projections and o_proj run on groups of
 * at most 32 rows (the matrix-vector kernel, whose per-row bits the identity needs), so a
 * call past 32 rows reads the weights once per group. */
KDA_API int kda_block_decode_k(const kda_block_weights *w, const kda_bf16 *hidden, int K, float *h_state,
                               kda_bf16 *conv_state, float *const *h_snap, kda_bf16 *const *conv_snap, int n_snap,
                               kda_workspace *ws, void *stream);

/* kda_block_verify — batched speculative verify through the whole block (Glm5NextLayer verify:
 * N sequences x K draft rows; Glm5NextKdaLayer `decode_k` at layer level): the projections of all
 * draft rows of all sequences in one pass (each weight read once for all rows), then one of two
 * routes, chosen from (B, total_tokens) alone:
 *   - short drafts (total_tokens <= 16 B): each (sequence, head) runs its rows in the stateful
 *     decode row (conv + SiLU + L2, gate, beta, recurrence, o_norm; the state in shared memory
 *     and written back nowhere), then o_proj. Every row's outputs are bit for bit what
 *     kda_decode_k gives on that sequence's stage rows. KDA_BUF_BETA then holds the beta LOGITS.
 *   - longer drafts: the packed conv from each conv state, the chunked core in verify mode
 *     (kda_chunk_verify, fused input) from each recurrent state, o_norm and o_proj; `tables`
 *     receives what the fold needs. Each row's output equals what kda_block_prefill_varlen on
 *     that sequence's first rows gives for it (the same core arithmetic), up to the projection
 *     kernel.
 * NO state changes on either route: the recurrent and conv states stay as they were. `tables`
 * (kda_chunk_verify_tables_bytes(B), 16-byte aligned) is required on both.
 *   hidden      [total_tokens, hidden] BF16, sequence b = rows [cu_seqlens[b], cu_seqlens[b+1]),
 *               at most 64 rows each (a longer one latches KDA_ERR_INVALID_ARG and is skipped)
 *   cu_seqlens  DEVICE int32 [B + 1];  h_state, conv_state: DEVICE pointer arrays as
 *               kda_block_prefill_varlen (read only here)
 * Projections: up to 8 rows in all the matrix-vector kernel, up to 256 the small-M tensor-core
 * form, beyond that the GEMM. The workspace keeps the rows' stage buffers (and, on the row route,
 * a copy of *w: the weights must stay valid until the fold) for the fold. KDA_ERR_CAPACITY if
 * total_tokens > max_tokens or B > max_seqs. */
KDA_API int kda_block_verify(const kda_block_weights *w, const kda_bf16 *hidden, const int *cu_seqlens, int B,
                             int total_tokens, float *const *h_state, kda_bf16 *const *conv_state, float *tables,
                             size_t tables_bytes, kda_workspace *ws, void *stream);

/* kda_block_verify_fold — accepted-row folding after kda_block_verify (Glm5NextLayer
 * `gdn_fold_accepted`): sequence b's recurrent state becomes its state after its first
 * accepted[b] verified rows and its conv state the last three inputs of (state || those rows'
 * qkv_proj). The route is the verify's (the same rule on B and total_tokens):
 *   - row route: the accepted rows run again through the stateful decode row with the verify's
 *     weights and stage buffers, now advancing both states: bit for bit the states kda_decode_k
 *     leaves after those rows (KDA_ERR_INVALID_ARG if no row-route verify ran on this workspace);
 *   - chunked route: kda_chunk_verify_fold's formula on the verify's tables and the BF16 k rows
 *     its core read.
 * accepted DEVICE int32 [B], 0 <= accepted[b] <= its rows; 0 leaves both states. Run on the same
 * workspace, cu_seqlens, tables and states right after kda_block_verify, before any other call
 * on that workspace. */
KDA_API int kda_block_verify_fold(const int *cu_seqlens, const int *accepted, int B, int total_tokens,
                                  const float *tables, float *const *h_state, kda_bf16 *const *conv_state,
                                  kda_workspace *ws, void *stream);

/* kda_block_decode_graph — kda_block_decode recorded once into a CUDA graph and instantiated,
 * for a serving loop that decodes the same N sequences from the same buffers every step: each
 * kda_graph_launch replays the call's kernels with one launch (the pages' engine has CUDA-graph
 * hooks; this is the block-level one). Recording runs nothing: no state changes. The graph
 * keeps the values the call would pass to its kernels: the pointers hidden, h_state,
 * conv_state, the weights in *w and the workspace buffers, and N. Each replay reads the
 * CURRENT contents of those buffers (new hidden rows, the advanced states), so they must stay
 * allocated and in place while the graph lives; the workspace must not be destroyed first.
 * Arguments and errors as kda_block_decode; KDA_ERR_CUDA if recording or instantiation fails.
 * *out receives the graph (NULL on error); release it with kda_graph_destroy. */
typedef struct kda_graph kda_graph;
KDA_API int kda_block_decode_graph(const kda_block_weights *w, const kda_bf16 *hidden, int N, float *const *h_state,
                                   kda_bf16 *const *conv_state, kda_workspace *ws, kda_graph **out);

/* Replay a recorded graph on `stream` (asynchronous, like the call it replaces). */
KDA_API int kda_graph_launch(kda_graph *g, void *stream);

/* Release a graph (NULL is a no-op). Do not destroy a graph whose replay may still run. */
KDA_API int kda_graph_destroy(kda_graph *g);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
