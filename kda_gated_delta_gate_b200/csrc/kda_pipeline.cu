// Host-resident prefill (kda_chunk_prefill_host): kda_beta + kda_chunk_prefill_fused for inputs
// and outputs that live in host memory. The sequence is cut into segments of whole chunks; the
// host->device copies of segment i+1, the kernels of segment i and the device->host copy of
// segment i-1 run at once on three streams (copy-in, the caller's stream, copy-out), so the
// call costs about the larger of the two PCIe directions instead of their sum plus the compute.
// The state is carried from segment to segment in device memory; because segments are whole
// chunks, the chunking is the one a single call over all T tokens makes and the results are
// the same bits.
#include <mutex>

#include "common.cuh"

namespace kda {
namespace {

__global__ void set_state_slot_kernel(float **slot, float *p) { *slot = p; }

// Per device: the two copy streams and the events that order them against the caller's stream.
// Created on first use and kept for the life of the process.
struct Lanes {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, landed = nullptr, computed = nullptr, drained = nullptr;
};

std::mutex g_lanes_mu;  // also serialises the enqueueing of calls (they share the events)
Lanes g_lanes[64];

int lanes(Lanes *&out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KDA_ERR_CUDA;
    Lanes &l = g_lanes[dev];
    if (!l.in) {
        const unsigned ef = cudaEventDisableTiming;
        Lanes n;
        if (cudaStreamCreateWithFlags(&n.in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&n.out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&n.start, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&n.landed, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&n.computed, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&n.drained, ef) != cudaSuccess) {
            for (cudaEvent_t e : {n.start, n.landed, n.computed, n.drained})
                if (e) cudaEventDestroy(e);
            if (n.in) cudaStreamDestroy(n.in);
            if (n.out) cudaStreamDestroy(n.out);
            return KDA_ERR_CUDA;
        }
        l = n;
    }
    out = &l;
    return KDA_OK;
}

constexpr size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Device buffer layout of one call (each piece 256-byte aligned).
struct HostLayout {
    size_t qkv, g_raw, beta, core, state, slot, scratch, total;
};

HostLayout host_layout(int T, int seg, int H, int D) {
    const size_t Tp = kda_t_pad(static_cast<size_t>(T), kChunk), hd = static_cast<size_t>(H) * D;
    HostLayout L{};
    size_t o = 0;
    L.qkv = o;     o += round256(Tp * 3 * hd * 2);
    L.g_raw = o;   o += round256(Tp * hd * 2);
    L.beta = o;    o += round256(Tp * H * 4);
    L.core = o;    o += round256(Tp * hd * 4);
    L.state = o;   o += round256(hd * D * 4);
    L.slot = o;    o += 256;
    L.scratch = o; o += round256(chunk_prefill_scratch_bytes(1, seg < T ? seg : T, H, D));
    L.total = o;
    return L;
}

}  // namespace
}  // namespace kda

extern "C" size_t kda_chunk_prefill_host_bytes(int T, int segment_tokens, const kda_dims *dims) {
    if (kda::check_dims(dims) != KDA_OK || T <= 0 || segment_tokens <= 0 || segment_tokens % kda::kChunk) return 0;
    return kda::host_layout(T, segment_tokens, dims->heads, dims->head_dim).total;
}

extern "C" int kda_chunk_prefill_host(const kda_bf16 *qkv, const kda_bf16 *g_raw, const float *b_logit,
                                      const float *dt_bias, const float *a_log, float *h_state, float *core, int T,
                                      int segment_tokens, void *device_buffer, size_t device_bytes,
                                      const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!qkv || !g_raw || !b_logit || !dt_bias || !a_log || !h_state || !core || T < 0) return KDA_ERR_INVALID_ARG;
    if (segment_tokens <= 0 || segment_tokens % kda::kChunk) return KDA_ERR_INVALID_ARG;
    if (T == 0) return KDA_OK;
    if (!device_buffer) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(device_buffer)) return KDA_ERR_MISALIGNED;
    const int H = dims->heads, D = dims->head_dim;
    if (H > 65535) return KDA_ERR_UNSUPPORTED;
    const kda::HostLayout L = kda::host_layout(T, segment_tokens, H, D);
    if (device_bytes < L.total) return KDA_ERR_CAPACITY;

    uint8_t *base = static_cast<uint8_t *>(device_buffer);
    auto *qkv_d = reinterpret_cast<kda_bf16 *>(base + L.qkv);
    auto *g_d = reinterpret_cast<kda_bf16 *>(base + L.g_raw);
    auto *beta_d = reinterpret_cast<float *>(base + L.beta);
    auto *core_d = reinterpret_cast<float *>(base + L.core);
    auto *state_d = reinterpret_cast<float *>(base + L.state);
    auto **slot_d = reinterpret_cast<float **>(base + L.slot);
    void *scratch = base + L.scratch;
    const size_t scratch_bytes = L.total - L.scratch;
    const size_t hd = static_cast<size_t>(H) * D, row_qkv = 3 * hd * 2, row_g = hd * 2, row_b = H * 4,
                 row_core = hd * 4, state_bytes = hd * D * 4;

    std::lock_guard<std::mutex> lock(kda::g_lanes_mu);
    kda::Lanes *ln = nullptr;
    KDA_TRY(kda::lanes(ln));
    auto cs = static_cast<cudaStream_t>(stream);
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    // the copy-in stream starts after everything already queued on the caller's stream (an
    // earlier call may still read these device buffers)
    if (!ok(cudaEventRecord(ln->start, cs)) || !ok(cudaStreamWaitEvent(ln->in, ln->start, 0))) return KDA_ERR_CUDA;
    if (!ok(cudaMemcpyAsync(state_d, h_state, state_bytes, cudaMemcpyHostToDevice, ln->in))) return KDA_ERR_CUDA;
    kda::set_state_slot_kernel<<<1, 1, 0, cs>>>(slot_d, state_d);
    KDA_TRY(kda::launch_status());
    for (int t0 = 0; t0 < T; t0 += segment_tokens) {
        const int n = T - t0 < segment_tokens ? T - t0 : segment_tokens;
        const size_t r = static_cast<size_t>(t0);
        // in: this segment's rows
        if (!ok(cudaMemcpyAsync(reinterpret_cast<uint8_t *>(qkv_d) + r * row_qkv,
                                reinterpret_cast<const uint8_t *>(qkv) + r * row_qkv, n * row_qkv,
                                cudaMemcpyHostToDevice, ln->in)) ||
            !ok(cudaMemcpyAsync(reinterpret_cast<uint8_t *>(g_d) + r * row_g,
                                reinterpret_cast<const uint8_t *>(g_raw) + r * row_g, n * row_g,
                                cudaMemcpyHostToDevice, ln->in)) ||
            !ok(cudaMemcpyAsync(reinterpret_cast<uint8_t *>(beta_d) + r * row_b,
                                reinterpret_cast<const uint8_t *>(b_logit) + r * row_b, n * row_b,
                                cudaMemcpyHostToDevice, ln->in)) ||
            !ok(cudaEventRecord(ln->landed, ln->in)) || !ok(cudaStreamWaitEvent(cs, ln->landed, 0)))
            return KDA_ERR_CUDA;
        // compute: beta in place, then the chunked core from the carried state
        KDA_TRY(kda_beta(beta_d + r * H, beta_d + r * H, n * H, stream));
        KDA_TRY(kda_chunk_prefill_fused(qkv_d + r * 3 * hd, g_d + r * hd, dt_bias, a_log, beta_d + r * H, slot_d,
                                        core_d + r * hd, 1, n, scratch, scratch_bytes, dims, stream));
        // out: this segment's core rows (and the state after the last one)
        if (!ok(cudaEventRecord(ln->computed, cs)) || !ok(cudaStreamWaitEvent(ln->out, ln->computed, 0)) ||
            !ok(cudaMemcpyAsync(reinterpret_cast<uint8_t *>(core) + r * row_core,
                                reinterpret_cast<const uint8_t *>(core_d) + r * row_core, n * row_core,
                                cudaMemcpyDeviceToHost, ln->out)))
            return KDA_ERR_CUDA;
    }
    if (!ok(cudaMemcpyAsync(h_state, state_d, state_bytes, cudaMemcpyDeviceToHost, ln->out)) ||
        !ok(cudaEventRecord(ln->drained, ln->out)) || !ok(cudaStreamWaitEvent(cs, ln->drained, 0)))
        return KDA_ERR_CUDA;
    return KDA_OK;
}
