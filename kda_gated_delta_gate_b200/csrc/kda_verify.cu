// Batched verify under the WY tables, and accepted-row folding (Glm5NextLayer speculative
// verify: K draft rows of many sequences checked at once, then each sequence keeps the rows the
// target accepted).
//
// kda_chunk_verify runs every sequence's rows (at most one 64-row chunk each) through the
// chunked kernels from the sequence's state, which stays as it was, and keeps per (sequence,
// head) the rows' update vectors U = T diag(beta) (V - (K o A) S0) (U[t] is exactly the u_t of
// the token recurrence) and the in-chunk cumulative log-decay Gamma. Folding r accepted rows
// then needs no recurrence:
//   S_r = diag(e^{Gamma_{r-1}}) S0 + sum_{t<r} (k_t o e^{Gamma_{r-1} - Gamma_t}) u_t^T
// (every exponent <= 0), one CTA per (sequence, head) here.
#include "common.cuh"

namespace kda {
namespace {

// k rows: FP32 [total, H*D] (kf), or BF16 rows of ldk elements (kb: the block's conv_out, whose
// k channels the verify read the same way, widened exactly).
template <int D>
__global__ void __launch_bounds__(256)
fold_kernel(const float *__restrict__ kf, const uint16_t *__restrict__ kb, size_t ldk, const int *__restrict__ cu,
            const int *__restrict__ accepted, const float *__restrict__ tables, float *const *__restrict__ h_state,
            int H, int total, int *__restrict__ status) {
    extern __shared__ __align__(16) float fs[];
    float *w = fs;               // [64][D]: k_t o e^{Gamma_{r-1} - Gamma_t}
    float *u = fs + kChunk * D;  // [64][D]: u_t
    float *dcy = u + kChunk * D; // [D]: e^{Gamma_{r-1}}
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int s0 = cu[b], s1 = cu[b + 1], r = accepted[b];
    if (s0 < 0 || s1 < s0 || s1 > total || s1 - s0 > kChunk || r < 0 || r > s1 - s0) {
        if (tid == 0 && h == 0) atomicExch(status, KDA_ERR_INVALID_ARG);
        return;
    }
    if (r == 0) return;  // nothing accepted: the state stays
    const float *U = tables + (static_cast<size_t>(b) * H + h) * 2 * kChunk * D;
    const float *G = U + kChunk * D;
    for (int e = tid; e < r * D; e += 256) {
        const int t = e / D, i = e % D;
        const size_t at = (static_cast<size_t>(s0) + t) * ldk + static_cast<size_t>(h) * D + i;
        const float kv = kf ? kf[at] : bf16_to_f32(kb[at]);
        w[e] = kv * expf(G[(r - 1) * D + i] - G[t * D + i]);
        u[e] = U[e];
    }
    for (int i = tid; i < D; i += 256) dcy[i] = expf(G[(r - 1) * D + i]);
    __syncthreads();
    constexpr int RG = 256 / D, RPG = D / RG;  // thread: value column j, a group of RPG key rows
    const int j = tid % D, g = tid / D;
    float *S = h_state[b] + static_cast<size_t>(h) * D * D;
    for (int ii = 0; ii < RPG; ++ii) {
        const int i = g * RPG + ii;
        float acc = dcy[i] * S[i * D + j];
        for (int t = 0; t < r; ++t) acc = fmaf(w[t * D + i], u[t * D + j], acc);
        S[i * D + j] = acc;
    }
}

}  // namespace

int verify_fold(const float *kf, const uint16_t *kb, size_t ldk, const int *cu_seqlens, const int *accepted, int B,
                int total, const float *tables, float *const *h_state, const kda_dims *dims, cudaStream_t s) {
    if (B == 0) return KDA_OK;
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    const int D = dims->head_dim;
    const int bytes = (2 * kChunk * D + D) * static_cast<int>(sizeof(float));
    dim3 grid(dims->heads, B);
    if (D == 128) {
        static std::atomic<unsigned long long> attr{0};
        KDA_TRY(smem_opt_in(fold_kernel<128>, bytes, attr));
        fold_kernel<128><<<grid, 256, bytes, s>>>(kf, kb, ldk, cu_seqlens, accepted, tables, h_state, dims->heads,
                                                   total, status);
    } else {
        static std::atomic<unsigned long long> attr{0};
        KDA_TRY(smem_opt_in(fold_kernel<64>, bytes, attr));
        fold_kernel<64><<<grid, 256, bytes, s>>>(kf, kb, ldk, cu_seqlens, accepted, tables, h_state, dims->heads,
                                                  total, status);
    }
    return launch_status();
}

}  // namespace kda

extern "C" {

size_t kda_chunk_verify_tables_bytes(int B, const kda_dims *dims) {
    if (B <= 0 || !dims || kda::check_dims(dims) != KDA_OK) return 0;
    return static_cast<size_t>(B) * dims->heads * 2 * kda::kChunk * dims->head_dim * sizeof(float);
}

int kda_chunk_verify(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                     const int *cu_seqlens, int B, int total_tokens, float *const *h_state, float *core,
                     float *tables, size_t tables_bytes, void *scratch, size_t scratch_bytes, const kda_dims *dims,
                     void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!q || !k || !v || !gate || !beta || !cu_seqlens || !h_state || !core || !tables || B < 0 ||
        total_tokens < 0)
        return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(q) || !kda::aligned16(k) || !kda::aligned16(v) || !kda::aligned16(gate) ||
        !kda::aligned16(core) || !kda::aligned16(tables))
        return KDA_ERR_MISALIGNED;
    if (B > 65535 || dims->heads > 65535) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || total_tokens == 0) return KDA_OK;
    if (tables_bytes < kda_chunk_verify_tables_bytes(B, dims)) return KDA_ERR_CAPACITY;
    if (!scratch) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(scratch)) return KDA_ERR_MISALIGNED;
    if (scratch_bytes < kda::chunk_prefill_slots_scratch_bytes(B, 1, dims->heads, dims->head_dim))
        return KDA_ERR_CAPACITY;
    return kda::chunk_verify_tc(q, k, v, gate, beta, cu_seqlens, B, total_tokens, h_state, core, tables, dims, scratch,
                                static_cast<cudaStream_t>(stream));
}

int kda_chunk_verify_fold(const float *k, const int *cu_seqlens, const int *accepted, int B, int total_tokens,
                          const float *tables, float *const *h_state, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!k || !cu_seqlens || !accepted || !tables || !h_state || B < 0 || total_tokens < 0) return KDA_ERR_INVALID_ARG;
    if (B > 65535 || dims->heads > 65535) return KDA_ERR_UNSUPPORTED;
    return kda::verify_fold(k, nullptr, static_cast<size_t>(dims->heads) * dims->head_dim, cu_seqlens, accepted, B,
                            total_tokens, tables, h_state, dims, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
