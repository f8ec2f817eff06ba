// HBM-bound elementwise stages of the KDA block:
//   kda_gate               (Glm5NextKdaWorkspace, field `gate` from field `g_raw`)
//   kda_beta               (Glm5NextKdaWorkspace, field `beta`)
//   kda_back_gated_rmsnorm (Glm5NextKdaWorkspace, field `o_norm_out`; Glm5NextKdaWeights `o_norm`)
// Each thread moves 16-byte vectors; grids are sized in multiples of the SM count and
// walk the tensor with a grid-stride loop.
#include <algorithm>

#include "common.cuh"

namespace kda {
namespace {

int grid_for(long long work_items, int threads) {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    long long blocks = (work_items + threads - 1) / threads;
    long long cap = static_cast<long long>(sms) * 16;
    if (blocks > cap) blocks = cap;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

// 8 gate values per thread: one 16-byte BF16 load of g_raw, two float4 of dt_bias, two
// float4 stores. groups = n_rows * H*D / 8; hd8 = H*D/8; d8 = D/8 (all 8 in one head).
// Thread (x) owns one 8-channel group of the H*D columns and walks rows (y): its dt_bias and
// -exp(a_log) are loaded once; each row is one 16-byte load and two 16-byte stores, four rows'
// loads in flight at a time.
__global__ void __launch_bounds__(256) gate_kernel(const uint4 *__restrict__ g_raw,
                                                   const float4 *__restrict__ dt_bias,
                                                   const float *__restrict__ a_log,
                                                   float4 *__restrict__ gate, int rows, int hd8, int d8) {
    const int c8 = blockIdx.x * blockDim.x + threadIdx.x;
    if (c8 >= hd8) return;
    const float nea = -expf(__ldg(a_log + c8 / d8));
    const float4 b0 = __ldg(dt_bias + 2 * c8), b1 = __ldg(dt_bias + 2 * c8 + 1);
    const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    // kRows rows per step, their loads issued together (bytes in flight, not issue, bound this)
    constexpr int kRows = 4;
    for (int r0 = blockIdx.y; r0 < rows; r0 += kRows * gridDim.y) {
        uint4 raw[kRows];
#pragma unroll
        for (int q = 0; q < kRows; ++q) {
            const int r = r0 + q * gridDim.y;
            raw[q] = r < rows ? g_raw[static_cast<size_t>(r) * hd8 + c8] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < kRows; ++q) {
            const int r = r0 + q * gridDim.y;
            if (r >= rows) break;
            const size_t i = static_cast<size_t>(r) * hd8 + c8;
            const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
            float g[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint16_t bits = static_cast<uint16_t>((e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xffffu));
                g[e] = kda_gate_f32(bf16_to_f32(bits), bb[e], nea);
            }
            gate[2 * i] = make_float4(g[0], g[1], g[2], g[3]);
            gate[2 * i + 1] = make_float4(g[4], g[5], g[6], g[7]);
        }
    }
}

__global__ void __launch_bounds__(256) beta_kernel(const float *__restrict__ x, float *__restrict__ y, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        y[i] = sigmoid_f32(x[i]);
}

// One warp per (token, head): D/32 consecutive channels per lane, warp-shuffle sum of
// squares, then the gated, weighted, normalised value rounded to BF16.
template <int D>
__global__ void __launch_bounds__(256) gated_rmsnorm_kernel(const float *__restrict__ core,
                                                            const uint16_t *__restrict__ out_gate,
                                                            const uint16_t *__restrict__ w,
                                                            uint16_t *__restrict__ out, long long rows,
                                                            float eps) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    float wv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) wv[e] = bf16_to_f32(w[lane * E + e]);
    for (long long r = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
        const size_t base = static_cast<size_t>(r) * D + lane * E;
        float x[E], gt[E];
        if constexpr (E == 4) {
            const float4 c = *reinterpret_cast<const float4 *>(core + base);
            x[0] = c.x; x[1] = c.y; x[2] = c.z; x[3] = c.w;
            const uint2 gg = *reinterpret_cast<const uint2 *>(out_gate + base);
            gt[0] = bf16_to_f32(gg.x & 0xffffu); gt[1] = bf16_to_f32(gg.x >> 16);
            gt[2] = bf16_to_f32(gg.y & 0xffffu); gt[3] = bf16_to_f32(gg.y >> 16);
        } else {
            const float2 c = *reinterpret_cast<const float2 *>(core + base);
            x[0] = c.x; x[1] = c.y;
            const uint32_t gg = *reinterpret_cast<const uint32_t *>(out_gate + base);
            gt[0] = bf16_to_f32(gg & 0xffffu); gt[1] = bf16_to_f32(gg >> 16);
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss += x[e] * x[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rs = rsqrtf(ss * (1.0f / D) + eps);
        uint32_t packed[E / 2];
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const float y0 = x[e] * rs * wv[e] * sigmoid_f32(gt[e]);
            const float y1 = x[e + 1] * rs * wv[e + 1] * sigmoid_f32(gt[e + 1]);
            packed[e / 2] = static_cast<uint32_t>(f32_to_bf16(y0)) | (static_cast<uint32_t>(f32_to_bf16(y1)) << 16);
        }
        if constexpr (E == 4) *reinterpret_cast<uint2 *>(out + base) = make_uint2(packed[0], packed[1]);
        else *reinterpret_cast<uint32_t *>(out + base) = packed[0];
    }
}

}  // namespace
}  // namespace kda

extern "C" {

int kda_gate(const kda_bf16 *g_raw, const float *dt_bias, const float *a_log, float *gate, int n_rows,
             const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!g_raw || !dt_bias || !a_log || !gate || n_rows < 0) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(g_raw) || !kda::aligned16(dt_bias) || !kda::aligned16(gate)) return KDA_ERR_MISALIGNED;
    if (n_rows == 0) return KDA_OK;
    const int hd8 = dims->heads * dims->head_dim / 8;
    const int gx = (hd8 + 255) / 256;
    // one wave of 256-thread blocks (8 per SM), each walking rows four at a time
    const int gy = static_cast<int>(std::min<long long>((n_rows + 3) / 4, std::max(1, 8 * kda::num_sms() / gx)));
    kda::gate_kernel<<<dim3(gx, gy), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(g_raw), reinterpret_cast<const float4 *>(dt_bias), a_log,
        reinterpret_cast<float4 *>(gate), n_rows, hd8, dims->head_dim / 8);
    return kda::launch_status();
}

int kda_beta(const float *b_logit, float *beta, int n, void *stream) {
    if (!b_logit || !beta || n < 0) return KDA_ERR_INVALID_ARG;
    if (n == 0) return KDA_OK;
    kda::beta_kernel<<<kda::grid_for(n, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(b_logit, beta, n);
    return kda::launch_status();
}

int kda_back_gated_rmsnorm(const float *core, const kda_bf16 *out_gate, const kda_bf16 *w, kda_bf16 *out, int T,
                           const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!core || !out_gate || !w || !out || T < 0) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(core) || !kda::aligned16(out_gate) || !kda::aligned16(w) || !kda::aligned16(out))
        return KDA_ERR_MISALIGNED;
    if (T == 0) return KDA_OK;
    const long long rows = static_cast<long long>(T) * dims->heads;
    const int grid = kda::grid_for(rows * 32, 256);
    auto s = static_cast<cudaStream_t>(stream);
    if (dims->head_dim == 128)
        kda::gated_rmsnorm_kernel<128><<<grid, 256, 0, s>>>(core, out_gate, w, out, rows, dims->rms_eps);
    else
        kda::gated_rmsnorm_kernel<64><<<grid, 256, 0, s>>>(core, out_gate, w, out, rows, dims->rms_eps);
    return kda::launch_status();
}

}  // extern "C"
