// Prefill front end (Glm5NextKdaWorkspace, fields `qkv_proj` -> `conv_out` -> `q_f32`,
// `k_f32`, `v_f32`; Glm5NextKdaWeights, field `conv`; Glm5NextKdaLayer,
// `prefill_with_pad_fill`): one kernel does the depthwise causal conv (kernel 4) from the
// carried conv state, SiLU, the BF16 conv_out write, the in-place per-head L2 of q|k on
// those BF16 values (a second BF16 rounding, as l2_norm_bf16 does on prefill), and the
// widening to FP32 with the pad rows set to pad_fill.
//
// Grid: (T_pad / 16 token tiles, heads). Block: D threads; thread d owns the head's three
// channels q_d, k_d, v_d. The tile-0 block is the only reader of the carried conv state
// and, after its reads, the only writer of the new one (the last three inputs).
#include "common.cuh"

namespace kda {
namespace {

constexpr int kTile = 16;

template <int D>
__global__ void __launch_bounds__(D) front_kernel(const uint16_t *__restrict__ x, uint16_t *__restrict__ conv_state,
                                                  const uint16_t *__restrict__ conv_w, uint16_t *__restrict__ conv_out,
                                                  float *__restrict__ qf, float *__restrict__ kf, float *__restrict__ vf,
                                                  float pad_fill, int T, int H, float eps) {
    constexpr int NW = D / 32;
    __shared__ float wsum[2][kTile][NW];
    const int d = threadIdx.x, lane = d & 31, w = d >> 5;
    const int h = blockIdx.y, t0 = blockIdx.x * kTile;
    const int qkv = H * D, cd = 3 * qkv;
    const int ch[3] = {h * D + d, qkv + h * D + d, 2 * qkv + h * D + d};

    float wt[3][4];
    float xx[3][kTile + 3];
#pragma unroll
    for (int m = 0; m < 3; ++m) {
#pragma unroll
        for (int j = 0; j < 4; ++j) wt[m][j] = bf16_to_f32(conv_w[ch[m] * 4 + j]);
#pragma unroll
        for (int j = 0; j < kTile + 3; ++j) {
            const int t = t0 - 3 + j;  // token index of xx[j]
            float val = 0.f;
            if (t < 0) val = bf16_to_f32(conv_state[ch[m] * 3 + (t + 3)]);
            else if (t < T) val = bf16_to_f32(x[static_cast<size_t>(t) * cd + ch[m]]);
            xx[m][j] = val;
        }
    }
    // conv + SiLU, rounded to BF16 (conv_out before the in-place L2)
    float c[3][kTile];
    float ssq[2][kTile];
#pragma unroll
    for (int i = 0; i < kTile; ++i) {
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            float y = wt[m][0] * xx[m][i];
            y = fmaf(wt[m][1], xx[m][i + 1], y);
            y = fmaf(wt[m][2], xx[m][i + 2], y);
            y = fmaf(wt[m][3], xx[m][i + 3], y);
            y = y * sigmoid_f32(y);
            c[m][i] = bf16_to_f32(f32_to_bf16(y));
        }
        ssq[0][i] = c[0][i] * c[0][i];
        ssq[1][i] = c[1][i] * c[1][i];
    }
#pragma unroll
    for (int i = 0; i < kTile; ++i) {
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            float s = ssq[m][i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) wsum[m][i][w] = s;
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kTile; ++i) {
        const int t = t0 + i;
        const size_t prow = static_cast<size_t>(t) * qkv + h * D + d;
        if (t < T) {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int j = 0; j < NW; ++j) { s0 += wsum[0][i][j]; s1 += wsum[1][i][j]; }
            const uint16_t qb = f32_to_bf16(c[0][i] * rsqrtf(s0 + eps));
            const uint16_t kb = f32_to_bf16(c[1][i] * rsqrtf(s1 + eps));
            const uint16_t vb = f32_to_bf16(c[2][i]);
            uint16_t *orow = conv_out + static_cast<size_t>(t) * cd;
            orow[ch[0]] = qb; orow[ch[1]] = kb; orow[ch[2]] = vb;
            if (qf) { qf[prow] = bf16_to_f32(qb); kf[prow] = bf16_to_f32(kb); vf[prow] = bf16_to_f32(vb); }
        } else if (qf) {
            qf[prow] = pad_fill; kf[prow] = pad_fill; vf[prow] = pad_fill;
        }
    }
    if (blockIdx.x == 0) {
        // new state = the last three inputs of (old state || x); only this block read the old state
        float ns[3][3];
#pragma unroll
        for (int m = 0; m < 3; ++m)
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const int idx = T + j;  // index into (state[0..2], x[0..T-1])
                ns[m][j] = idx < 3 ? bf16_to_f32(conv_state[ch[m] * 3 + idx])
                                   : bf16_to_f32(x[static_cast<size_t>(idx - 3) * cd + ch[m]]);
            }
#pragma unroll
        for (int m = 0; m < 3; ++m)
#pragma unroll
            for (int j = 0; j < 3; ++j) conv_state[ch[m] * 3 + j] = f32_to_bf16(ns[m][j]);
    }
}

}  // namespace
}  // namespace kda

extern "C" int kda_front_conv_silu_l2(const kda_bf16 *x, kda_bf16 *conv_state, const kda_bf16 *conv_w,
                                      kda_bf16 *conv_out, float *q_f32, float *k_f32, float *v_f32, float pad_fill,
                                      int T, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!x || !conv_state || !conv_w || !conv_out || T < 0) return KDA_ERR_INVALID_ARG;
    const bool any_f = q_f32 || k_f32 || v_f32, all_f = q_f32 && k_f32 && v_f32;
    if (any_f && !all_f) return KDA_ERR_INVALID_ARG;
    if (T == 0) return KDA_OK;
    const int T_pad = static_cast<int>(kda_t_pad(static_cast<size_t>(T), kda::kChunk));
    dim3 grid(T_pad / kda::kTile, dims->heads);
    auto s = static_cast<cudaStream_t>(stream);
    if (dims->head_dim == 128)
        kda::front_kernel<128><<<grid, 128, 0, s>>>(x, conv_state, conv_w, conv_out, q_f32, k_f32, v_f32, pad_fill, T,
                                                    dims->heads, dims->l2_eps);
    else
        kda::front_kernel<64><<<grid, 64, 0, s>>>(x, conv_state, conv_w, conv_out, q_f32, k_f32, v_f32, pad_fill, T,
                                                  dims->heads, dims->l2_eps);
    return kda::launch_status();
}
