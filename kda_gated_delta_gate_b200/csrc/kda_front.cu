// Prefill front end (Glm5NextKdaWorkspace, fields `qkv_proj` -> `conv_out` -> `q_f32`,
// `k_f32`, `v_f32`; Glm5NextKdaWeights, field `conv`; Glm5NextKdaLayer,
// `prefill_with_pad_fill`): one kernel does the depthwise causal conv (kernel 4) from the
// carried conv state, SiLU, the BF16 conv_out write, the in-place per-head L2 of q|k on
// those BF16 values (a second BF16 rounding, as l2_norm_bf16 does on prefill), and the
// widening to FP32 with the pad rows set to pad_fill.
//
// Grid: (ceil(T_pad / 16) token tiles, column blocks of 256 x 8 channels). Thread j of
// column block c owns the 8 consecutive channels [8 g, 8 g + 8), g = 256 c + j, of the
// q|k|v row (16-byte loads and stores) and walks the tile's 16 tokens with a sliding
// window of the 3 previous inputs. Short tiles and three CTAs per SM keep enough rows in
// flight: the kernel is bound by latency and issue, not by the 2 x 16 bytes it moves per
// token and thread. The D/8 threads of one head's q (or k) are adjacent
// lanes and reduce the per-token sum of squares with shuffles. The tile-0 block of each
// column block is the only reader of those channels' carried conv state and, after its
// reads, the only writer of the new one (the last three inputs).
#include <algorithm>

#include "common.cuh"

namespace kda {
namespace {

constexpr int kFrontThreads = 256, kTT = 16;

__device__ __forceinline__ void unpack8(const uint4 u, float (&x)[8]) {
    x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xFFFF0000u);
    x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xFFFF0000u);
    x[4] = __uint_as_float(u.z << 16); x[5] = __uint_as_float(u.z & 0xFFFF0000u);
    x[6] = __uint_as_float(u.w << 16); x[7] = __uint_as_float(u.w & 0xFFFF0000u);
}
// SiLU y / (1 + e^-y) from the SFU exponential and the fast divide (a few ulp of FP32; the
// result is rounded to BF16 next). For y << 0 the denominator overflows to inf and the result
// is -0, as the exact value rounds.
__device__ __forceinline__ float silu_fast(float y) { return __fdividef(y, 1.0f + __expf(-y)); }

__device__ __forceinline__ uint32_t pack2(uint16_t lo, uint16_t hi) {
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <int D>
__global__ void __launch_bounds__(kFrontThreads, 3) front_kernel(const uint16_t *__restrict__ x, uint16_t *__restrict__ conv_state,
                                                              const uint16_t *__restrict__ conv_w,
                                                              uint16_t *__restrict__ conv_out, float *__restrict__ qf,
                                                              float *__restrict__ kf, float *__restrict__ vf,
                                                              float pad_fill, int T, int T_pad, int H, float eps) {
    constexpr int LG = D / 8;  // lanes per head part (q, k or v of one head)
    const int qkv = H * D, cd = 3 * qkv;
    const int g = blockIdx.y * kFrontThreads + threadIdx.x;
    const bool valid = 8 * g < cd;  // whole head groups are in or out (cd is a multiple of D)
    const int c0 = valid ? 8 * g : 0;
    const int part = c0 / qkv, pc = c0 - part * qkv;  // 0 = q, 1 = k, 2 = v; channel within the part
    const int t0 = blockIdx.x * kTT;
    float *wide = part == 0 ? qf : (part == 1 ? kf : vf);

    float w[4][8];  // w[tap][channel]
    {
        float wr[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float tmp[8];
            unpack8(reinterpret_cast<const uint4 *>(conv_w + static_cast<size_t>(c0) * 4)[q4], tmp);
#pragma unroll
            for (int e = 0; e < 8; ++e) wr[8 * q4 + e] = tmp[e];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j][e] = wr[4 * e + j];
    }
    // window: xm[0] = x_{t-3}, xm[1] = x_{t-2}, xm[2] = x_{t-1} (tiles at or past T read no x)
    float xm[3][8];
    if (t0 >= T) {
#pragma unroll
        for (int j = 0; j < 3; ++j)
#pragma unroll
            for (int e = 0; e < 8; ++e) xm[j][e] = 0.f;
    } else if (t0 == 0) {
        float st[24];
#pragma unroll
        for (int q3 = 0; q3 < 3; ++q3) {
            float tmp[8];
            unpack8(reinterpret_cast<const uint4 *>(conv_state + static_cast<size_t>(c0) * 3)[q3], tmp);
#pragma unroll
            for (int e = 0; e < 8; ++e) st[8 * q3 + e] = tmp[e];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int j = 0; j < 3; ++j) xm[j][e] = st[3 * e + j];
    } else {
#pragma unroll
        for (int j = 0; j < 3; ++j)
            unpack8(*reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t0 - 3 + j) * cd + c0), xm[j]);
    }
    const int tend = min(t0 + kTT, T);
#pragma unroll 4
    for (int t = t0; t < tend; ++t) {
        float xc[8], c[8];
        unpack8(*reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t) * cd + c0), xc);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float y = w[0][e] * xm[0][e];
            y = fmaf(w[1][e], xm[1][e], y);
            y = fmaf(w[2][e], xm[2][e], y);
            y = fmaf(w[3][e], xc[e], y);
            y = silu_fast(y);
            c[e] = bf16_to_f32(f32_to_bf16(y));  // conv_out before the in-place L2
            ss = fmaf(c[e], c[e], ss);
            xm[0][e] = xm[1][e]; xm[1][e] = xm[2][e]; xm[2][e] = xc[e];
        }
#pragma unroll
        for (int o = 1; o < LG; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rs = part < 2 ? rsqrtf(ss + eps) : 1.f;
        uint16_t ob[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ob[e] = f32_to_bf16(part < 2 ? c[e] * rs : c[e]);
        if (valid) {
            *reinterpret_cast<uint4 *>(conv_out + static_cast<size_t>(t) * cd + c0) =
                make_uint4(pack2(ob[0], ob[1]), pack2(ob[2], ob[3]), pack2(ob[4], ob[5]), pack2(ob[6], ob[7]));
            if (qf) {
                float *dst = wide + static_cast<size_t>(t) * qkv + pc;
                *reinterpret_cast<float4 *>(dst) =
                    make_float4(bf16_to_f32(ob[0]), bf16_to_f32(ob[1]), bf16_to_f32(ob[2]), bf16_to_f32(ob[3]));
                *reinterpret_cast<float4 *>(dst + 4) =
                    make_float4(bf16_to_f32(ob[4]), bf16_to_f32(ob[5]), bf16_to_f32(ob[6]), bf16_to_f32(ob[7]));
            }
        }
    }
    if (qf && valid) {  // pad rows of the widened copies
        for (int t = max(t0, T); t < min(t0 + kTT, T_pad); ++t) {
            float *dst = wide + static_cast<size_t>(t) * qkv + pc;
            *reinterpret_cast<float4 *>(dst) = make_float4(pad_fill, pad_fill, pad_fill, pad_fill);
            *reinterpret_cast<float4 *>(dst + 4) = make_float4(pad_fill, pad_fill, pad_fill, pad_fill);
        }
    }
    if (blockIdx.x == 0 && valid) {
        // new state = the last three inputs of (old state || x); only this block read the old state
        uint16_t ns[24];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int idx = T + j;  // index into (state[0..2], x[0..T-1])
            float v8[8];
            if (idx < 3) {
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = bf16_to_f32(conv_state[static_cast<size_t>(c0 + e) * 3 + idx]);
            } else {
                unpack8(*reinterpret_cast<const uint4 *>(x + static_cast<size_t>(idx - 3) * cd + c0), v8);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) ns[3 * e + j] = f32_to_bf16(v8[e]);
        }
        // only this thread reads or writes these 8 channels' state, and its reads come first
        uint4 *dst = reinterpret_cast<uint4 *>(conv_state + static_cast<size_t>(c0) * 3);
#pragma unroll
        for (int q3 = 0; q3 < 3; ++q3)
            dst[q3] = make_uint4(pack2(ns[8 * q3], ns[8 * q3 + 1]), pack2(ns[8 * q3 + 2], ns[8 * q3 + 3]),
                                 pack2(ns[8 * q3 + 4], ns[8 * q3 + 5]), pack2(ns[8 * q3 + 6], ns[8 * q3 + 7]));
    }
}

// ---- packed sequences (cu_seqlens): the same per-row arithmetic as front_kernel, each row's
// window taken from its own sequence (the carried conv state before the sequence's first row).
// A token tile may hold the end of one sequence and the start of the next; the window is
// rebuilt at each sequence start. The conv states are only read here: conv_advance_kernel
// moves them on afterwards, so no reader of a state can race its writer.

// Row r of sequence [s0, s1) (r < s0 reaches into the carried state, 3 inputs deep); st holds
// the state's 8 channels x 3 inputs once loaded.
__device__ __forceinline__ void window_input(const uint16_t *x, const float (&st)[24], int r, int s0, int cd,
                                             int c0, float (&out)[8]) {
    if (r >= s0) {
        unpack8(*reinterpret_cast<const uint4 *>(x + static_cast<size_t>(r) * cd + c0), out);
    } else {
        const int m = r - s0 + 3;  // 0..2: oldest .. newest carried input
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = m == 0 ? st[3 * e] : (m == 1 ? st[3 * e + 1] : st[3 * e + 2]);
    }
}

__device__ __forceinline__ void load_state8(const uint16_t *cst, int c0, float (&st)[24]) {
#pragma unroll
    for (int q3 = 0; q3 < 3; ++q3) {
        float tmp[8];
        unpack8(reinterpret_cast<const uint4 *>(cst + static_cast<size_t>(c0) * 3)[q3], tmp);
#pragma unroll
        for (int e = 0; e < 8; ++e) st[8 * q3 + e] = tmp[e];
    }
}

// Sequence bounds [s0, s1) of stream b, false (and the error latched) when they do not fit.
__device__ __forceinline__ bool seq_bounds(const int *cu, int b, int total, int &s0, int &s1, int *status) {
    s0 = cu[b];
    s1 = cu[b + 1];
    if (s0 < 0 || s1 < s0 || s1 > total) {
        atomicExch(status, KDA_ERR_INVALID_ARG);
        return false;
    }
    return true;
}

// Row t starts (or resumes) sequence b: its bounds, and the window x_{t-3} .. x_{t-1} from its
// rows and carried state. False (the error latched) if t is not in the sequence or the state
// pointer is misaligned. Every thread of a block reads the same cu entries: block-uniform.
__device__ __forceinline__ bool enter_seq(const uint16_t *x, uint16_t *const *conv_state, const int *cu, int b, int t,
                                          int total, int cd, int c0, int &s0, int &s1, float (&xm)[3][8],
                                          int *status) {
    if (!seq_bounds(cu, b, total, s0, s1, status) || t < s0 || t >= s1) {
        atomicExch(status, KDA_ERR_INVALID_ARG);
        return false;
    }
    const uint16_t *cst = conv_state[b];
    if (reinterpret_cast<uintptr_t>(cst) & 15) {
        atomicExch(status, KDA_ERR_MISALIGNED);
        return false;
    }
    float st[24];
    if (t - s0 < 3) load_state8(cst, c0, st);
#pragma unroll
    for (int j = 0; j < 3; ++j) window_input(x, st, t - 3 + j, s0, cd, c0, xm[j]);
    return true;
}

template <int D>
__global__ void __launch_bounds__(kFrontThreads, 2)
front_varlen_kernel(const uint16_t *__restrict__ x, uint16_t *const *__restrict__ conv_state,
                    const uint16_t *__restrict__ conv_w, uint16_t *__restrict__ conv_out, const int *__restrict__ cu,
                    int B, int total, int tt, int H, float eps, int *__restrict__ status) {
    constexpr int LG = D / 8;
    const int qkv = H * D, cd = 3 * qkv;
    const int g = blockIdx.y * kFrontThreads + threadIdx.x;
    const bool valid = 8 * g < cd;
    const int c0 = valid ? 8 * g : 0;
    const int part = c0 / qkv;
    const int t0 = blockIdx.x * tt, tend = min(t0 + tt, total);
    float w[4][8];
    {
        float wr[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float tmp[8];
            unpack8(reinterpret_cast<const uint4 *>(conv_w + static_cast<size_t>(c0) * 4)[q4], tmp);
#pragma unroll
            for (int e = 0; e < 8; ++e) wr[8 * q4 + e] = tmp[e];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j][e] = wr[4 * e + j];
    }
    // the sequence holding row t0: the last b with cu[b] <= t0 (empty sequences are passed over)
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t0) lo = mid;
        else hi = mid - 1;
    }
    int b = lo, s0 = 0, s1 = 0;
    float xm[3][8];
    if (t0 >= tend || !enter_seq(x, conv_state, cu, b, t0, total, cd, c0, s0, s1, xm, status)) return;
    // rows four at a time: their loads go out together (the sequence switch inside would keep
    // the compiler from hoisting them)
    for (int t4 = t0; t4 < tend; t4 += 4) {
      uint4 raw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
          raw[q] = t4 + q < tend ? *reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t4 + q) * cd + c0)
                                 : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = t4 + q;
        if (t >= tend) break;
        if (t == s1) {  // the next non-empty sequence starts here
            while (b < B - 1 && cu[b + 1] <= t) ++b;
            if (!enter_seq(x, conv_state, cu, b, t, total, cd, c0, s0, s1, xm, status)) return;
        }
        float xc[8], c[8];
        unpack8(raw[q], xc);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float y = w[0][e] * xm[0][e];
            y = fmaf(w[1][e], xm[1][e], y);
            y = fmaf(w[2][e], xm[2][e], y);
            y = fmaf(w[3][e], xc[e], y);
            y = silu_fast(y);
            c[e] = bf16_to_f32(f32_to_bf16(y));
            ss = fmaf(c[e], c[e], ss);
            xm[0][e] = xm[1][e]; xm[1][e] = xm[2][e]; xm[2][e] = xc[e];
        }
#pragma unroll
        for (int o = 1; o < LG; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rs = part < 2 ? rsqrtf(ss + eps) : 1.f;
        uint16_t ob[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ob[e] = f32_to_bf16(part < 2 ? c[e] * rs : c[e]);
        if (valid)
            *reinterpret_cast<uint4 *>(conv_out + static_cast<size_t>(t) * cd + c0) =
                make_uint4(pack2(ob[0], ob[1]), pack2(ob[2], ob[3]), pack2(ob[4], ob[5]), pack2(ob[6], ob[7]));
      }
    }
}

// Conv state of sequence b after its first r rows (r = accepted[b], or all of them): the last
// three inputs of (state || x rows s0 .. s0 + r - 1). One thread per 8 channels of a sequence
// reads its state before it writes it.
__global__ void __launch_bounds__(kFrontThreads)
conv_advance_kernel(const uint16_t *__restrict__ x, uint16_t *const *__restrict__ conv_state,
                    const int *__restrict__ cu, const int *__restrict__ accepted, int total, int cd,
                    int *__restrict__ status) {
    const int b = blockIdx.x, g = blockIdx.y * kFrontThreads + threadIdx.x;
    if (8 * g >= cd) return;
    const int c0 = 8 * g;
    int s0, s1;
    if (!seq_bounds(cu, b, total, s0, s1, status)) return;
    const int r = accepted ? accepted[b] : s1 - s0;
    if (r < 0 || r > s1 - s0) {
        atomicExch(status, KDA_ERR_INVALID_ARG);
        return;
    }
    if (r == 0) return;  // nothing taken: the state stays
    uint16_t *cst = conv_state[b];
    if (reinterpret_cast<uintptr_t>(cst) & 15) {
        atomicExch(status, KDA_ERR_MISALIGNED);
        return;
    }
    float st[24];
    load_state8(cst, c0, st);
    uint16_t ns[24];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        float v8[8];
        window_input(x, st, s0 + r - 3 + j, s0, cd, c0, v8);  // input r + j of (state || x)
#pragma unroll
        for (int e = 0; e < 8; ++e) ns[3 * e + j] = f32_to_bf16(v8[e]);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(cst + static_cast<size_t>(c0) * 3);
#pragma unroll
    for (int q3 = 0; q3 < 3; ++q3)
        dst[q3] = make_uint4(pack2(ns[8 * q3], ns[8 * q3 + 1]), pack2(ns[8 * q3 + 2], ns[8 * q3 + 3]),
                             pack2(ns[8 * q3 + 4], ns[8 * q3 + 5]), pack2(ns[8 * q3 + 6], ns[8 * q3 + 7]));
}

}  // namespace

int front_varlen(const uint16_t *x, uint16_t *const *conv_state, const uint16_t *conv_w, uint16_t *conv_out,
                 const int *cu_seqlens, int B, int total, const kda_dims *dims, cudaStream_t s) {
    if (B == 0 || total == 0) return KDA_OK;
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    const int cd = 3 * dims->heads * dims->head_dim;
    const int colb = (cd / 8 + kFrontThreads - 1) / kFrontThreads;
    // token tiles of up to 16 rows, shorter when the call has too few rows for two blocks per SM
    const int tt = std::max(1, std::min(kTT, total / std::max(1, 2 * num_sms() / colb)));
    dim3 grid((total + tt - 1) / tt, colb);
    if (dims->head_dim == 128)
        front_varlen_kernel<128><<<grid, kFrontThreads, 0, s>>>(x, conv_state, conv_w, conv_out, cu_seqlens, B, total,
                                                                tt, dims->heads, dims->l2_eps, status);
    else
        front_varlen_kernel<64><<<grid, kFrontThreads, 0, s>>>(x, conv_state, conv_w, conv_out, cu_seqlens, B, total,
                                                               tt, dims->heads, dims->l2_eps, status);
    return launch_status();
}

int conv_state_advance(const uint16_t *x, uint16_t *const *conv_state, const int *cu_seqlens, const int *accepted,
                       int B, int total, const kda_dims *dims, cudaStream_t s) {
    if (B == 0) return KDA_OK;
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    const int cd = 3 * dims->heads * dims->head_dim;
    dim3 grid(B, (cd / 8 + kFrontThreads - 1) / kFrontThreads);
    conv_advance_kernel<<<grid, kFrontThreads, 0, s>>>(x, conv_state, cu_seqlens, accepted, total, cd, status);
    return launch_status();
}

}  // namespace kda

extern "C" int kda_front_conv_silu_l2(const kda_bf16 *x, kda_bf16 *conv_state, const kda_bf16 *conv_w,
                                      kda_bf16 *conv_out, float *q_f32, float *k_f32, float *v_f32, float pad_fill,
                                      int T, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!x || !conv_state || !conv_w || !conv_out || T < 0) return KDA_ERR_INVALID_ARG;
    const bool any_f = q_f32 || k_f32 || v_f32, all_f = q_f32 && k_f32 && v_f32;
    if (any_f && !all_f) return KDA_ERR_INVALID_ARG;
    if (T == 0) return KDA_OK;
    if (!kda::aligned16(x) || !kda::aligned16(conv_state) || !kda::aligned16(conv_w) || !kda::aligned16(conv_out) ||
        (any_f && (!kda::aligned16(q_f32) || !kda::aligned16(k_f32) || !kda::aligned16(v_f32))))
        return KDA_ERR_MISALIGNED;
    const int T_pad = static_cast<int>(kda_t_pad(static_cast<size_t>(T), kda::kChunk));
    const int cd = 3 * dims->heads * dims->head_dim;
    dim3 grid((T_pad + kda::kTT - 1) / kda::kTT, (cd / 8 + kda::kFrontThreads - 1) / kda::kFrontThreads);
    auto s = static_cast<cudaStream_t>(stream);
    if (dims->head_dim == 128)
        kda::front_kernel<128><<<grid, kda::kFrontThreads, 0, s>>>(x, conv_state, conv_w, conv_out, q_f32, k_f32, v_f32,
                                                                   pad_fill, T, T_pad, dims->heads, dims->l2_eps);
    else
        kda::front_kernel<64><<<grid, kda::kFrontThreads, 0, s>>>(x, conv_state, conv_w, conv_out, q_f32, k_f32, v_f32,
                                                                  pad_fill, T, T_pad, dims->heads, dims->l2_eps);
    return kda::launch_status();
}

extern "C" int kda_front_conv_silu_l2_varlen(const kda_bf16 *x, kda_bf16 *const *conv_state, const kda_bf16 *conv_w,
                                             kda_bf16 *conv_out, const int *cu_seqlens, int B, int total_tokens,
                                             int advance_state, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!x || !conv_state || !conv_w || !conv_out || !cu_seqlens || B < 0 || total_tokens < 0)
        return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(x) || !kda::aligned16(conv_w) || !kda::aligned16(conv_out)) return KDA_ERR_MISALIGNED;
    if (B > 65535) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || total_tokens == 0) return KDA_OK;
    auto s = static_cast<cudaStream_t>(stream);
    KDA_TRY(kda::front_varlen(x, conv_state, conv_w, conv_out, cu_seqlens, B, total_tokens, dims, s));
    if (!advance_state) return KDA_OK;
    return kda::conv_state_advance(x, conv_state, cu_seqlens, nullptr, B, total_tokens, dims, s);
}

extern "C" int kda_conv_state_fold(const kda_bf16 *x, kda_bf16 *const *conv_state, const int *cu_seqlens,
                                   const int *accepted, int B, int total_tokens, const kda_dims *dims, void *stream) {
    KDA_TRY(kda::check_dims(dims));
    if (!x || !conv_state || !cu_seqlens || B < 0 || total_tokens < 0) return KDA_ERR_INVALID_ARG;
    if (!kda::aligned16(x)) return KDA_ERR_MISALIGNED;
    if (B > 65535) return KDA_ERR_UNSUPPORTED;
    return kda::conv_state_advance(x, conv_state, cu_seqlens, accepted, B, total_tokens, dims,
                                   static_cast<cudaStream_t>(stream));
}
