// Library-wide C-ABI entry points: version, status text, T_pad, latched device status.
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace kda {

// One status word per device (a __device__ variable exists once per device context).
// Kernels that run bounded waits write a KDA_ERR_* code here instead of trapping.
__device__ int g_device_status;

void *current_context() {
    typedef int (*GetCurrentFn)(void **);
    static std::atomic<GetCurrentFn> fn{nullptr};
    GetCurrentFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p)
            return nullptr;
        f = reinterpret_cast<GetCurrentFn>(p);
        fn.store(f, std::memory_order_release);
    }
    void *ctx = nullptr;
    return f(&ctx) == 0 ? ctx : nullptr;
}

int *device_status_ptr() {
    // per device: the context the address was looked up in, and the address (a per-thread copy
    // answers the common case without the lock)
    static std::mutex lock;
    static void *ctx_of[64] = {};
    static int *addr_of[64] = {};
    thread_local void *tl_ctx[64] = {};
    thread_local int *tl_addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    void *ctx = current_context();  // null before the runtime has made one current
    if (ctx && tl_addr[dev] && ctx == tl_ctx[dev]) return tl_addr[dev];
    std::lock_guard<std::mutex> g(lock);
    if (addr_of[dev] && ctx && ctx == ctx_of[dev]) {
        tl_ctx[dev] = ctx;
        tl_addr[dev] = addr_of[dev];
        return addr_of[dev];
    }
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess || !addr) return nullptr;
    ctx_of[dev] = current_context();  // the lookup made the device's context current
    addr_of[dev] = static_cast<int *>(addr);
    tl_ctx[dev] = ctx_of[dev];
    tl_addr[dev] = addr_of[dev];
    return addr_of[dev];
}

}  // namespace kda

extern "C" {

int kda_version(void) { return 100; }

const char *kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_ALIAS: return "buffers that must not overlap do";
        case KDA_ERR_CAPACITY: return "token count beyond the workspace capacity";
        case KDA_ERR_UNSUPPORTED: return "unsupported dimensions";
        case KDA_ERR_CUDA: return "CUDA runtime error";
        case KDA_ERR_TIMEOUT: return "device-side wait timed out";
        case KDA_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
        default: return "unknown status";
    }
}

size_t kda_t_pad(size_t T, int chunk) {
    if (chunk <= 0) return 0;
    const size_t c = static_cast<size_t>(chunk);
    return (T + c - 1) / c * c;
}

int kda_device_status(int *out, int clear) {
    if (!out) return KDA_ERR_INVALID_ARG;
    int *p = kda::device_status_ptr();
    if (!p) return KDA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemcpy(out, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

}  // extern "C"

extern "C" size_t kda_chunk_prefill_scratch_bytes(int B, int T, const kda_dims *dims) {
    if (kda::check_dims(dims) != KDA_OK) return 0;
    return kda::chunk_prefill_scratch_bytes(B, T, dims->heads, dims->head_dim);
}

extern "C" int kda_chunk_prefill(const float *q, const float *k, const float *v, const float *gate,
                                 const float *beta, float *const *h_state, float *core, int B, int T, void *scratch,
                                 size_t scratch_bytes, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::chunk_prefill_check(q, k, v, gate, beta, h_state, core, B, T, dims));
    if (B == 0 || T == 0) return KDA_OK;
    if (!scratch) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(scratch)) return KDA_ERR_MISALIGNED;
    if (scratch_bytes < kda::chunk_prefill_scratch_bytes(B, T, dims->heads, dims->head_dim)) return KDA_ERR_CAPACITY;
    return kda::chunk_prefill_tc(q, k, v, gate, beta, h_state, core, B, T, dims, scratch,
                                 static_cast<cudaStream_t>(stream));
}

extern "C" int kda_chunk_prefill_fused(const kda_bf16 *qkv, const kda_bf16 *g_raw, const float *dt_bias,
                                       const float *a_log, const float *beta, float *const *h_state, float *core, int B,
                                       int T, void *scratch, size_t scratch_bytes, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!qkv || !g_raw || !dt_bias || !a_log || !beta || !h_state || !core || B < 0 || T < 0)
        return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(qkv) || !kda::aligned16(g_raw) || !kda::aligned16(core)) return KDA_ERR_MISALIGNED;
    if (B > 65535 || dims->heads > 65535) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0) return KDA_OK;
    if (!scratch) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(scratch)) return KDA_ERR_MISALIGNED;
    if (scratch_bytes < kda::chunk_prefill_scratch_bytes(B, T, dims->heads, dims->head_dim)) return KDA_ERR_CAPACITY;
    return kda::chunk_prefill_tc_fused(qkv, g_raw, dt_bias, a_log, beta, h_state, core, B, T, dims, scratch,
                                       static_cast<cudaStream_t>(stream));
}

extern "C" int kda_chunk_prefill_graw(const float *q, const float *k, const float *v, const kda_bf16 *g_raw,
                                      const float *dt_bias, const float *a_log, const float *beta,
                                      float *const *h_state, float *core, int B, int T, void *scratch,
                                      size_t scratch_bytes, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!q || !k || !v || !g_raw || !dt_bias || !a_log || !beta || !h_state || !core || B < 0 || T < 0)
        return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(q) || !kda::aligned16(k) || !kda::aligned16(v) || !kda::aligned16(g_raw) ||
        !kda::aligned16(core))
        return KDA_ERR_MISALIGNED;
    if (B > 65535 || dims->heads > 65535) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0) return KDA_OK;
    if (!scratch) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(scratch)) return KDA_ERR_MISALIGNED;
    if (scratch_bytes < kda::chunk_prefill_scratch_bytes(B, T, dims->heads, dims->head_dim)) return KDA_ERR_CAPACITY;
    return kda::chunk_prefill_tc_graw(q, k, v, g_raw, dt_bias, a_log, beta, h_state, core, B, T, dims, scratch,
                                      static_cast<cudaStream_t>(stream));
}

extern "C" size_t kda_chunk_prefill_varlen_scratch_bytes(int B, int max_num_chunks, const kda_dims *dims) {
    if (!dims || kda::check_dims(dims) != KDA_OK) return 0;
    return kda::chunk_prefill_slots_scratch_bytes(B, max_num_chunks, dims->heads, dims->head_dim);
}

extern "C" size_t kda_chunk_prefill_packed_scratch_bytes(int max_seqs, int max_total_tokens, const kda_dims *dims) {
    if (!dims || kda::check_dims(dims) != KDA_OK) return 0;
    return kda::chunk_prefill_packed_bytes(max_seqs, max_total_tokens, dims->heads, dims->head_dim);
}

extern "C" int kda_chunk_prefill_varlen(const float *q, const float *k, const float *v, const float *gate,
                                        const float *beta, const int *cu_seqlens, int B, int max_num_chunks,
                                        int total_tokens, float *const *h_state, float *core, void *scratch,
                                        size_t scratch_bytes, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!q || !k || !v || !gate || !beta || !cu_seqlens || !h_state || !core || B < 0 || max_num_chunks < 0 ||
        total_tokens < 0)
        return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(q) || !kda::aligned16(k) || !kda::aligned16(v) || !kda::aligned16(gate) ||
        !kda::aligned16(core))
        return KDA_ERR_MISALIGNED;
    if (B > 65535 || dims->heads > 65535) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || total_tokens == 0) return KDA_OK;  // every stream is empty: the states stay as they are
    if (max_num_chunks == 0) return KDA_ERR_INVALID_ARG;
    if (!scratch) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(scratch)) return KDA_ERR_MISALIGNED;
    if (scratch_bytes <
        kda::chunk_prefill_varlen_need_bytes(B, max_num_chunks, total_tokens, dims->heads, dims->head_dim))
        return KDA_ERR_CAPACITY;
    return kda::chunk_prefill_tc_varlen(q, k, v, gate, beta, cu_seqlens, B, max_num_chunks, total_tokens, h_state,
                                        core, dims, scratch, static_cast<cudaStream_t>(stream));
}
