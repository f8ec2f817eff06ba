// kda_chunk_prefill_noalloc: the tensor-core chunked prefill for callers that must not
// allocate device memory. Some callers cannot call cudaMalloc (or any allocator): a serving
// engine that carves all free HBM into its KV-cache / state pools at start-up has no
// headroom left for a late allocation, and a plug-in called from a host framework that owns
// the device memory budget may be forbidden from allocating behind that framework's back.
// This entry point takes no scratch argument: its scratch is a file-scope __device__ array
// of kNoAllocScratchBytes (32 MiB), which every GPU that loads the library holds until the
// process exits. The array is reserved when its module loads, which (modules load lazily) is
// the first call on the device: a call with B == 0 or T == 0 reserves it and runs nothing, so
// an engine makes one such call per device before its pools claim the free memory (or sets
// CUDA_MODULE_LOADING=EAGER). The computation is exactly that of kda_chunk_prefill.
#include <mutex>

#include "common.cuh"

namespace kda {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

// One per device context. In host code this name is only a host-side stand-in for the
// device array: its device address must come from cudaGetSymbolAddress (set-up below).
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_lock;
void *g_scratch_ctx[kMaxDevices] = {};   // the context each address was looked up in
void *g_scratch_addr[kMaxDevices] = {};

// Device address of this device's scratch array, looked up (cudaGetSymbolAddress, with the
// device current) on the first call in each context of the device: once per device, and again
// after a cudaDeviceReset has given the device a new context. The lookup is also what loads
// the array's module, and so what reserves its 32 MiB on the device (modules load lazily).
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    void *ctx = current_context();  // null before the runtime has made one current
    std::lock_guard<std::mutex> lock(g_setup_lock);
    if (!g_scratch_addr[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return KDA_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
        g_scratch_ctx[dev] = current_context();  // the lookup made the device's context current
    }
    *out = g_scratch_addr[dev];
    return KDA_OK;
}

}  // namespace
}  // namespace kda

extern "C" size_t kda_chunk_prefill_noalloc_max_scratch_bytes(void) { return kda::kNoAllocScratchBytes; }

extern "C" int kda_chunk_prefill_noalloc(const float *q, const float *k, const float *v, const float *gate,
                                         const float *beta, float *const *h_state, float *core, int B, int T,
                                         const kda_dims *dims, void *stream) {
    KDA_TRY(kda::chunk_prefill_check(q, k, v, gate, beta, h_state, core, B, T, dims));
    if (kda::chunk_prefill_scratch_bytes(B, T, dims->heads, dims->head_dim) > kda::kNoAllocScratchBytes)
        return KDA_ERR_CAPACITY;
    // the address (and with it the array's reservation) before anything else, so that a call
    // with B == 0 or T == 0 reserves the array without running anything
    void *scratch = nullptr;
    KDA_TRY(kda::scratch_address(&scratch));
    if (B == 0 || T == 0) return KDA_OK;
    return kda::chunk_prefill_tc(q, k, v, gate, beta, h_state, core, B, T, dims, scratch,
                                 static_cast<cudaStream_t>(stream));
}
