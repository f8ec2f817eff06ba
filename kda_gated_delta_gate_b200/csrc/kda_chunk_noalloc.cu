// kda_chunk_prefill_noalloc: the tensor-core chunked prefill for callers that must not
// allocate device memory. Some callers cannot call cudaMalloc (or any allocator): a serving
// engine that carves all free HBM into its KV-cache / state pools at start-up has no
// headroom left for a late allocation, and a plug-in called from a host framework that owns
// the device memory budget may be forbidden from allocating behind that framework's back.
// This entry point takes no scratch argument: its scratch is a file-scope __device__ array
// of kNoAllocScratchBytes (32 MiB), which every GPU that loads the library holds until the
// process exits. The computation is exactly that of kda_chunk_prefill.
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
void *g_scratch_addr[kMaxDevices] = {};

// Device address of this device's scratch array; fetched once per device with that device
// current (the first call on a device does it).
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_lock);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return KDA_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
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
    if (B == 0 || T == 0) return KDA_OK;
    if (kda::chunk_prefill_scratch_bytes(B, T, dims->heads, dims->head_dim) > kda::kNoAllocScratchBytes)
        return KDA_ERR_CAPACITY;
    void *scratch = nullptr;
    KDA_TRY(kda::scratch_address(&scratch));
    return kda::chunk_prefill_tc(q, k, v, gate, beta, h_state, core, B, T, dims, scratch,
                                 static_cast<cudaStream_t>(stream));
}
