// Host-resident prefill (kda_chunk_prefill_host: kda_beta + kda_chunk_prefill_fused;
// kda_chunk_prefill_host_f32: kda_gate + kda_beta + kda_chunk_prefill) for inputs and outputs
// that live in host memory. The sequence is cut into segments of whole chunks; the
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

// The host inputs of one call: BF16 q|k|v rows (the fused-input mode), or FP32 q, k, v rows
// (the FP32 mode: kda_gate + kda_beta + kda_chunk_prefill, the device call's own kernels).
struct HostIn {
    const kda_bf16 *qkv;
    const float *q, *k, *v;
    const kda_bf16 *g_raw;
    const float *b_logit;
    bool f32() const { return q != nullptr; }
};

// Device buffer layout of one call (each piece 256-byte aligned). FP32 mode: q, k, v at
// qkv + {0, 1, 2} x the q size, and an FP32 gate buffer.
struct HostLayout {
    size_t qkv, qsize, gate, g_raw, beta, core, state, slot, scratch, total;
};

HostLayout host_layout(int T, int seg, int H, int D, bool f32) {
    const size_t Tp = kda_t_pad(static_cast<size_t>(T), kChunk), hd = static_cast<size_t>(H) * D;
    HostLayout L{};
    size_t o = 0;
    L.qkv = o;
    L.qsize = round256(Tp * hd * 4);
    o += f32 ? 3 * L.qsize : round256(Tp * 3 * hd * 2);
    L.gate = o;    o += f32 ? round256(Tp * hd * 4) : 0;
    L.g_raw = o;   o += round256(Tp * hd * 2);
    L.beta = o;    o += round256(Tp * H * 4);
    L.core = o;    o += round256(Tp * hd * 4);
    L.state = o;   o += round256(hd * D * 4);
    L.slot = o;    o += 256;
    L.scratch = o; o += round256(chunk_prefill_scratch_bytes(1, seg < T ? seg : T, H, D));
    L.total = o;
    return L;
}

int host_prefill(const HostIn &in, const float *dt_bias, const float *a_log, float *h_state, float *core, int T,
                 int segment_tokens, void *device_buffer, size_t device_bytes, const kda_dims *dims, void *stream) {
    KDA_TRY(check_dims(dims));
    if (!in.g_raw || !in.b_logit || !dt_bias || !a_log || !h_state || !core || T < 0) return KDA_ERR_INVALID_ARG;
    if (segment_tokens <= 0 || segment_tokens % kChunk) return KDA_ERR_INVALID_ARG;
    if (T == 0) return KDA_OK;
    if (!device_buffer) return KDA_ERR_INVALID_ARG;
    if (!aligned16(device_buffer)) return KDA_ERR_MISALIGNED;
    const int H = dims->heads, D = dims->head_dim;
    if (H > 65535) return KDA_ERR_UNSUPPORTED;
    const bool f32 = in.f32();
    const HostLayout L = host_layout(T, segment_tokens, H, D, f32);
    if (device_bytes < L.total) return KDA_ERR_CAPACITY;

    uint8_t *base = static_cast<uint8_t *>(device_buffer);
    auto *qkv_d = reinterpret_cast<kda_bf16 *>(base + L.qkv);
    float *q_d[3] = {reinterpret_cast<float *>(base + L.qkv), reinterpret_cast<float *>(base + L.qkv + L.qsize),
                     reinterpret_cast<float *>(base + L.qkv + 2 * L.qsize)};
    auto *gate_d = reinterpret_cast<float *>(base + L.gate);
    auto *g_d = reinterpret_cast<kda_bf16 *>(base + L.g_raw);
    auto *beta_d = reinterpret_cast<float *>(base + L.beta);
    auto *core_d = reinterpret_cast<float *>(base + L.core);
    auto *state_d = reinterpret_cast<float *>(base + L.state);
    auto **slot_d = reinterpret_cast<float **>(base + L.slot);
    void *scratch = base + L.scratch;
    const size_t scratch_bytes = L.total - L.scratch;
    const size_t hd = static_cast<size_t>(H) * D, row_qkv = 3 * hd * 2, row_q = hd * 4, row_g = hd * 2,
                 row_b = H * 4, row_core = hd * 4, state_bytes = hd * D * 4;
    const float *q_h[3] = {in.q, in.k, in.v};

    std::lock_guard<std::mutex> lock(g_lanes_mu);
    Lanes *ln = nullptr;
    KDA_TRY(lanes(ln));
    auto cs = static_cast<cudaStream_t>(stream);
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    auto h2d = [&](void *dst, const void *src, size_t row, size_t r, int n) {
        return ok(cudaMemcpyAsync(static_cast<uint8_t *>(dst) + r * row, static_cast<const uint8_t *>(src) + r * row,
                                  n * row, cudaMemcpyHostToDevice, ln->in));
    };
    // the copy-in stream starts after everything already queued on the caller's stream (an
    // earlier call may still read these device buffers)
    if (!ok(cudaEventRecord(ln->start, cs)) || !ok(cudaStreamWaitEvent(ln->in, ln->start, 0))) return KDA_ERR_CUDA;
    if (!ok(cudaMemcpyAsync(state_d, h_state, state_bytes, cudaMemcpyHostToDevice, ln->in))) return KDA_ERR_CUDA;
    set_state_slot_kernel<<<1, 1, 0, cs>>>(slot_d, state_d);
    KDA_TRY(launch_status());
    for (int t0 = 0; t0 < T; t0 += segment_tokens) {
        const int n = T - t0 < segment_tokens ? T - t0 : segment_tokens;
        const size_t r = static_cast<size_t>(t0);
        // in: this segment's rows
        bool good = true;
        if (f32) {
            for (int i = 0; i < 3; ++i) good = good && h2d(q_d[i], q_h[i], row_q, r, n);
        } else {
            good = h2d(qkv_d, in.qkv, row_qkv, r, n);
        }
        if (!good || !h2d(g_d, in.g_raw, row_g, r, n) || !h2d(beta_d, in.b_logit, row_b, r, n) ||
            !ok(cudaEventRecord(ln->landed, ln->in)) || !ok(cudaStreamWaitEvent(cs, ln->landed, 0)))
            return KDA_ERR_CUDA;
        // compute: beta in place, then the chunked core from the carried state
        KDA_TRY(kda_beta(beta_d + r * H, beta_d + r * H, n * H, stream));
        if (f32) {
            KDA_TRY(kda_gate(g_d + r * hd, dt_bias, a_log, gate_d + r * hd, n, dims, stream));
            KDA_TRY(kda_chunk_prefill(q_d[0] + r * hd, q_d[1] + r * hd, q_d[2] + r * hd, gate_d + r * hd,
                                      beta_d + r * H, slot_d, core_d + r * hd, 1, n, scratch, scratch_bytes, dims,
                                      stream));
        } else {
            KDA_TRY(kda_chunk_prefill_fused(qkv_d + r * 3 * hd, g_d + r * hd, dt_bias, a_log, beta_d + r * H, slot_d,
                                            core_d + r * hd, 1, n, scratch, scratch_bytes, dims, stream));
        }
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

}  // namespace
}  // namespace kda

extern "C" size_t kda_chunk_prefill_host_bytes(int T, int segment_tokens, const kda_dims *dims) {
    if (kda::check_dims(dims) != KDA_OK || T <= 0 || segment_tokens <= 0 || segment_tokens % kda::kChunk) return 0;
    return kda::host_layout(T, segment_tokens, dims->heads, dims->head_dim, false).total;
}

extern "C" size_t kda_chunk_prefill_host_f32_bytes(int T, int segment_tokens, const kda_dims *dims) {
    if (kda::check_dims(dims) != KDA_OK || T <= 0 || segment_tokens <= 0 || segment_tokens % kda::kChunk) return 0;
    return kda::host_layout(T, segment_tokens, dims->heads, dims->head_dim, true).total;
}

extern "C" int kda_chunk_prefill_host(const kda_bf16 *qkv, const kda_bf16 *g_raw, const float *b_logit,
                                      const float *dt_bias, const float *a_log, float *h_state, float *core, int T,
                                      int segment_tokens, void *device_buffer, size_t device_bytes,
                                      const kda_dims *dims, void *stream) {
    if (!qkv) return KDA_ERR_INVALID_ARG;
    const kda::HostIn in{qkv, nullptr, nullptr, nullptr, g_raw, b_logit};
    return kda::host_prefill(in, dt_bias, a_log, h_state, core, T, segment_tokens, device_buffer, device_bytes, dims,
                             stream);
}

extern "C" int kda_chunk_prefill_host_f32(const float *q, const float *k, const float *v, const kda_bf16 *g_raw,
                                          const float *b_logit, const float *dt_bias, const float *a_log,
                                          float *h_state, float *core, int T, int segment_tokens,
                                          void *device_buffer, size_t device_bytes, const kda_dims *dims,
                                          void *stream) {
    if (!q || !k || !v) return KDA_ERR_INVALID_ARG;
    const kda::HostIn in{nullptr, q, k, v, g_raw, b_logit};
    return kda::host_prefill(in, dt_bias, a_log, h_state, core, T, segment_tokens, device_buffer, device_bytes, dims,
                             stream);
}
