// Chunked KDA prefill with tcgen05 tensor cores (Glm5NextKdaLayer `prefill`, `kda_chunk_*`;
// Glm5NextKdaWorkspace q_f32/k_f32/v_f32/gate/beta -> core; Glm5NextLayer
// `prefill_gdn_full_batched`: B equal-length streams, a device array of state pointers).
//
// Per chunk of C = 64 tokens, Gamma the in-chunk inclusive cumulative log-decay per key
// channel (Gamma_C its last row), A = e^Gamma:
//   L[i][j] = beta_i sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc}  (i > j);  T = (I + L)^-1
//   M[i][j] =        sum_c q_ic k_jc e^{Gamma_ic - Gamma_jc}  (i >= j)
//   W = T diag(beta) (K o A);  U~ = T diag(beta) V              (the WY / UT form)
//   U = U~ - W S0;  O = scale ((Q o A) S0 + M U)
//   S = diag(A_C) S0 + (K o e^{Gamma_C - Gamma})^T U
// which is the gated delta rule unrolled over the chunk (U = (I + L)^-1 diag(beta)(V - (K o A) S0)).
//
// Two kernels:
//  intra (one CTA per chunk-head, all in parallel): L and M in one tcgen05 MMA, T on CUDA
//    cores, then W | U~ in a second MMA. It writes a pack of state-independent operands,
//    laid out as the state kernel's shared memory wants them (so one bulk copy moves each).
//  state (one CTA per (stream, head, value slice), chunks in order): two dependent tcgen05
//    MMA groups per chunk, each in split-BF16 precision (x = hi + lo; hi.hi + hi.lo + lo.hi):
//      D1  = [W; Q o A] . S0                 (M = 128, N = DVS, K = D)
//      U   = U~ - D1[0:64]                   (epilogue, into shared memory)
//      D3  = (K o e^{Gamma_C - Gamma})^T . U (M = D, N = DVS, K = 64)
//      D1 += [0; M] . U                      (so D1[64:128] = (Q o A) S0 + M U)
//    O = scale D1[64:128];  S = A_C o S0 + D3 (FP32 master copy in registers).
// Rows >= T of the last chunk are loaded as zeros (k = q = v = 0, g = 0, beta = 0): the pad
// guard. They add nothing to L, M, W, U~ or the state, and their outputs are not written.
#include <algorithm>

#include "common.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace kda {
namespace {

using namespace umma;

constexpr int C = kChunk;          // 64
constexpr int kTileBytes = 16384;  // one 128 x 64 BF16 K-major tile

// Per (stream, head, chunk) the intra kernel writes one pack of state-independent operands,
// each BF16 operand as a hi tile followed by its lo tile, laid out exactly as the state
// kernel's shared memory wants them (so a bulk copy moves each):
//   A1 [W; Q o A]                 128 x D, K-major          (A = e^Gamma)
//   AM M (lower, with diagonal)   64 x 64, K-major          (rows 64..127 of the [0; M] tile)
//   A3 K o e^{Gamma_C - Gamma}    D (M) x 64 (K), MN-major
//   UT U~ in FP32, D/32 groups of 32 value columns, [group][64 rows][UP] (UP = 36: a 16-byte
//      skew per row, so the state kernel's per-row 16-byte reads are conflict-free)
//   AC e^{Gamma_C}                D FP32 (1 KB slot)
template <int D>
struct Pack {
    static constexpr int A1 = 2 * 128 * D * 2;
    static constexpr int AM = 2 * C * C * 2;
    static constexpr int A3 = 2 * C * D * 2;
    static constexpr int UP = 36;
    static constexpr int UG_BYTES = C * UP * 4;
    static constexpr int UT = (D / 32) * UG_BYTES;
    static constexpr int AC = 1024;
    static constexpr int OFF_A1 = 0, OFF_AM = A1, OFF_A3 = OFF_AM + AM, OFF_UT = OFF_A3 + A3, OFF_AC = OFF_UT + UT;
    static constexpr int bytes = OFF_AC + AC;
};
// The chunked path's inputs. FP32 mode: q, k, v, gate [B*T_pad, H, D]. Fused mode: qkv, the
// BF16 conv_out rows [B*T_pad, 3*H*D] (q | k | v after conv + SiLU + L2), and the BF16 g_raw
// rows [B*T_pad, H*D] with dt_bias and a_log: the gate is formed in the kernel. beta
// [B*T_pad, H] FP32 in both.
struct PrefillIn {
    const float *q, *k, *v, *gate;
    const uint16_t *qkv, *g_raw;
    const float *dt_bias, *a_log, *beta;
    float *tables;  // verify mode: per (stream, head) U [64][D] then Gamma [64][D] (FP32); else null
    int stream_pack;  // the call's operand packs overflow L2: store them evict-first
};

// Programmatic dependent launch: the kernels of a call run back to back with the next one
// launched as soon as every CTA of the current one has started (pdl_release at the start), so
// its launch and its set-up that reads nothing the current one writes overlap the current
// one's tail; pdl_acquire waits until the previous kernel has completed and its memory is
// visible. A kernel launched without the attribute passes both at once.
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_acquire() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// L2 eviction policies (createpolicy): evict-first for data read or written for the last time
// in this pass, so that the inputs prefetched for the coming items keep their place in L2.
__device__ __forceinline__ uint64_t l2_policy(bool evict_first) {
    uint64_t p;
    if (evict_first) asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    else asm("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint4 ld16_hint(const void *p, uint64_t pol) {
    uint4 r;
    asm("ld.global.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p), "l"(pol));
    return r;
}
__device__ __forceinline__ void st16_hint(void *p, const uint4 &v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w), "l"(pol)
                 : "memory");
}

// Input modes of the chunked kernels: where q, k, v and the log-decay come from.
//   kInF32   FP32 q, k, v and FP32 gate (kda_gate's output)
//   kInFused BF16 q|k|v rows (the front end's conv_out) and BF16 g_raw; the gate is formed in-kernel
//   kInGraw  FP32 q, k, v and BF16 g_raw; the gate is formed in-kernel
constexpr int kInF32 = 0, kInFused = 1, kInGraw = 2;
template <int MODE> constexpr bool kQkv16 = MODE == kInFused;  // q|k|v in BF16 rows
template <int MODE> constexpr bool kGraw = MODE != kInF32;      // gate formed from BF16 g_raw

__device__ __forceinline__ void bf16x2_to_f32(uint32_t u, float &lo, float &hi) {
    lo = __uint_as_float(u << 16);
    hi = __uint_as_float(u & 0xFFFF0000u);
}

// Channels [c, c + 8) of global token row `row`, head h: q (part 0), k (1) or v (2), as FP32.
template <int D, bool QKV16>
// last: the kernel's last read of these values (loaded evict-first with policy `pol`).
__device__ __forceinline__ void load8_in(const PrefillIn &in, int part, size_t row, int H, int h, int c,
                                         float (&x)[8], bool last = false, uint64_t pol = 0) {
    if constexpr (QKV16) {
        const uint16_t *p = in.qkv + row * (3 * static_cast<size_t>(H) * D) + static_cast<size_t>(part * H + h) * D + c;
        const uint4 u = last ? ld16_hint(p, pol) : *reinterpret_cast<const uint4 *>(p);
        bf16x2_to_f32(u.x, x[0], x[1]); bf16x2_to_f32(u.y, x[2], x[3]);
        bf16x2_to_f32(u.z, x[4], x[5]); bf16x2_to_f32(u.w, x[6], x[7]);
    } else {
        const float *p = (part == 0 ? in.q : (part == 1 ? in.k : in.v)) + row * (static_cast<size_t>(H) * D) +
                         static_cast<size_t>(h) * D + c;
        uint4 a, b;
        if (last) {
            a = ld16_hint(p, pol);
            b = ld16_hint(p + 4, pol);
        } else {
            a = *reinterpret_cast<const uint4 *>(p);
            b = *reinterpret_cast<const uint4 *>(p + 4);
        }
        x[0] = __uint_as_float(a.x); x[1] = __uint_as_float(a.y); x[2] = __uint_as_float(a.z);
        x[3] = __uint_as_float(a.w); x[4] = __uint_as_float(b.x); x[5] = __uint_as_float(b.y);
        x[6] = __uint_as_float(b.z); x[7] = __uint_as_float(b.w);
    }
}

// Channels [c, c + 4): q / k / v as above, or the log-decay g (part 3; formed from g_raw when
// the mode says so).
template <int D, int MODE>
__device__ __forceinline__ float4 load4_in(const PrefillIn &in, int part, size_t row, int H, int h, int c) {
    if constexpr (kGraw<MODE>) {
        if (part == 3) {
            const uint2 u = *reinterpret_cast<const uint2 *>(in.g_raw + row * (static_cast<size_t>(H) * D) +
                                                             static_cast<size_t>(h) * D + c);
            const float nea = -expf(in.a_log[h]);
            const float *dt = in.dt_bias + static_cast<size_t>(h) * D + c;
            float r0, r1, r2, r3;
            bf16x2_to_f32(u.x, r0, r1);
            bf16x2_to_f32(u.y, r2, r3);
            return make_float4(kda_gate_f32(r0, dt[0], nea), kda_gate_f32(r1, dt[1], nea),
                               kda_gate_f32(r2, dt[2], nea), kda_gate_f32(r3, dt[3], nea));
        }
    }
    if constexpr (kQkv16<MODE>) {
        const uint2 u = *reinterpret_cast<const uint2 *>(in.qkv + row * (3 * static_cast<size_t>(H) * D) +
                                                         static_cast<size_t>(part * H + h) * D + c);
        float4 r;
        bf16x2_to_f32(u.x, r.x, r.y);
        bf16x2_to_f32(u.y, r.z, r.w);
        return r;
    } else {
        const float *p = (part == 0 ? in.q : (part == 1 ? in.k : (part == 2 ? in.v : in.gate))) +
                         row * (static_cast<size_t>(H) * D) + static_cast<size_t>(h) * D + c;
        return *reinterpret_cast<const float4 *>(p);
    }
}

// Where the chunks of stream b live. Equal-length mode (cu == nullptr): B streams of T tokens
// at a stride of T_pad rows (Glm5NextLayer `prefill_gdn_full_batched`). Varlen mode: stream b
// is rows [cu[b], cu[b+1]) of the packed buffers (`cu_seqlens`, with `max_num_chunks` chunk
// slots per stream); the rows after a stream's end belong to the next stream, and the chunk
// guard keeps them out exactly as it keeps out the padding of equal-length streams.
struct Seqs {
    const int *cu;  // device [B + 1], or nullptr
    int T, T_pad;   // equal-length mode
    int nch;        // chunks a stream may have: T_pad / C, or max_num_chunks
    int total;      // varlen mode: rows of the packed buffers
    int slots;      // varlen mode, compact pack layout: pack slots per head; 0 = one slot per
                    // (stream, head, chunk)
};

// The operand pack of chunk c of stream b, head h (row0: the chunk's first row, from seq_chunk).
// Rectangular layout: slot (b H + h) nch + c. Compact layout (varlen mode, sq.slots > 0): head h
// owns slots [h slots, (h + 1) slots) and stream b's chunks take the consecutive slots from
// floor(cu[b] / C) + b. Consecutive streams cannot collide: the next stream starts at
// floor(cu[b+1] / C) + b + 1, at least this one's start plus its ceil(len / C) chunks. The last
// slot any stream with 0 <= cu[b] <= cu[b+1] <= total uses is below ceil(total / C) + B - 1,
// the per-head slot count the host sizes the scratch for.
__device__ __forceinline__ size_t pack_slot(const Seqs &sq, int b, int h, int c, size_t row0, int H) {
    if (sq.slots)
        return static_cast<size_t>(h) * sq.slots + (row0 - static_cast<size_t>(c) * C) / C + b + c;
    return (static_cast<size_t>(b) * H + h) * sq.nch + c;
}

// Rows of chunk c of stream b: first row (row0) and count (n). False for an empty slot or (in
// varlen mode) a stream whose bounds are not inside the buffers, which also latches
// KDA_ERR_INVALID_ARG: nothing is addressed from a bad cu_seqlens entry.
__device__ __forceinline__ bool seq_chunk(const Seqs &sq, int b, int c, size_t &row0, int &n, int *status) {
    if (!sq.cu) {
        row0 = static_cast<size_t>(b) * sq.T_pad + static_cast<size_t>(c) * C;
        n = min(C, sq.T - c * C);
        return n > 0;
    }
    const int s0 = sq.cu[b], s1 = sq.cu[b + 1];
    if (s0 < 0 || s1 < s0 || s1 > sq.total || s1 - s0 > sq.nch * C) {
        if (status) atomicExch(status, KDA_ERR_INVALID_ARG);
        n = 0;
        return false;
    }
    row0 = static_cast<size_t>(s0) + static_cast<size_t>(c) * C;
    n = min(C, s1 - s0 - c * C);
    return n > 0;
}

constexpr long long kWaitCycles = 4000000000LL;  // about 2 s at 1.9 GHz

// Split 8 FP32 values into BF16 hi and lo, packed as two 16-byte chunks (paired conversions).
__device__ __forceinline__ void split8(const float (&x)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) split_bf16x2(x[2 * u], x[2 * u + 1], h[u], l[u]);
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void st_pair(uint8_t *tile, int half_bytes, uint32_t off, const float (&x)[8]) {
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4 *>(tile + off) = hi;
    *reinterpret_cast<uint4 *>(tile + half_bytes + off) = lo;
}

// ================================================================ phase 1: intra-chunk

constexpr int kIntraThreads = 512;
constexpr int kLPC = C + 1;  // row stride of the FP32 [C][C] tiles L and M (conflict-free column writes)
constexpr int kTPC = C + 4;  // row stride of T (16-byte aligned rows for vector reads)

// T = (I + L)^-1 for the strictly lower 64 x 64 L in sL (row stride kLPC; only i > j is read);
// T's lower triangle and diagonal land in sT (row stride kTPC), together with zeros in the
// blocks above the diagonal that the combination steps read. Blocked, each step parallel:
//   16 x 16 diagonal blocks by substitution (one thread per column);
//   32 x 32 halves:  T_21 = -T_22 (L_21 T_11)  from their 16 x 16 blocks;
//   the whole:       T_21 = -T_22 (L_21 T_11)  from the two 32 x 32 halves.
// The products run 4 columns per thread (16-byte reads of the right operand). All NT (>= 256)
// threads of the block call it; sTmp holds 1024 floats (16-byte aligned).
template <int NT>
__device__ __forceinline__ void invert_unit_lower64(const float *__restrict__ sL, float *__restrict__ sT,
                                                    float *__restrict__ sTmp) {
    static_assert(NT >= 256, "the 32 x 32 products take 256 threads");
    constexpr int PC = kLPC, PT = kTPC;
    const int tid = threadIdx.x;
    auto fma4 = [](float a, const float4 &b, float4 &acc) {
        acc.x = fmaf(a, b.x, acc.x); acc.y = fmaf(a, b.y, acc.y); acc.z = fmaf(a, b.z, acc.z); acc.w = fmaf(a, b.w, acc.w);
    };
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < 64) {
        const int base = 16 * (tid >> 4), j = tid & 15;
        float t[16];  // column j of the block's inverse; t[m] = 0 above the diagonal
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < i; ++m) acc = fmaf(sL[(base + i) * PC + base + m], t[m], acc);
            t[i] = i == j ? 1.f : (i < j ? 0.f : -acc);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) sT[(base + i) * PT + base + j] = t[i];
    }
    __syncthreads();
    if (tid < 128) {  // X_h = L_{2h+1,2h} T_{2h,2h}, row i, columns 4c..4c+3
        const int hh = tid >> 6, i = (tid >> 2) & 15, c4 = 4 * (tid & 3), b0 = 32 * hh;
        float4 x = zero4;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            fma4(sL[(b0 + 16 + i) * PC + b0 + m], *reinterpret_cast<const float4 *>(sT + (b0 + m) * PT + b0 + c4), x);
        *reinterpret_cast<float4 *>(sTmp + hh * 256 + i * 16 + c4) = x;
        *reinterpret_cast<float4 *>(sT + (b0 + i) * PT + b0 + 16 + c4) = zero4;  // block above the diagonal
    }
    __syncthreads();
    if (tid < 128) {  // T_{2h+1,2h} = -T_{2h+1,2h+1} X_h
        const int hh = tid >> 6, i = (tid >> 2) & 15, c4 = 4 * (tid & 3), b0 = 32 * hh;
        float4 x = zero4;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            fma4(sT[(b0 + 16 + i) * PT + b0 + 16 + m], *reinterpret_cast<const float4 *>(sTmp + hh * 256 + m * 16 + c4), x);
        *reinterpret_cast<float4 *>(sT + (b0 + 16 + i) * PT + b0 + c4) = make_float4(-x.x, -x.y, -x.z, -x.w);
    } else {  // the upper-right 32 x 32 block
        for (int e = tid - 128; e < 256; e += NT - 128)
            *reinterpret_cast<float4 *>(sT + (e >> 3) * PT + 32 + 4 * (e & 7)) = zero4;
    }
    __syncthreads();
    if (tid < 256) {  // Y = L_LU T_UU, row i, columns 4c..4c+3
        const int i = tid >> 3, c4 = 4 * (tid & 7);
        float4 y = zero4;
#pragma unroll
        for (int m = 0; m < 32; ++m) fma4(sL[(32 + i) * PC + m], *reinterpret_cast<const float4 *>(sT + m * PT + c4), y);
        *reinterpret_cast<float4 *>(sTmp + i * 32 + c4) = y;
    }
    __syncthreads();
    if (tid < 256) {  // T_LU = -T_LL Y
        const int i = tid >> 3, c4 = 4 * (tid & 7);
        float4 y = zero4;
#pragma unroll
        for (int m = 0; m < 32; ++m)
            fma4(sT[(32 + i) * PT + 32 + m], *reinterpret_cast<const float4 *>(sTmp + m * 32 + c4), y);
        *reinterpret_cast<float4 *>(sT + (32 + i) * PT + c4) = make_float4(-y.x, -y.y, -y.z, -y.w);
    }
    __syncthreads();
}

template <int D>
struct Intra {
    static constexpr int P = D + 8;   // fp32 row stride of [C][D] tiles (bank-spread, 16-B aligned)
    static constexpr int PC = kLPC;   // row stride of [C][C] tiles
    static constexpr int NZ = 64;     // rows of the block-local backward factors
    static constexpr int PT = kTPC;   // row stride of T
    static constexpr size_t floats = 3 * C * P + NZ * P + 2 * C * PC + C * PT + 4 * D + C + 1024;
    static constexpr size_t bytes = floats * sizeof(float);
};

// The exact CUDA-core intra-chunk computation of one (stream b, head h, chunk ch): every decay
// factor is a product of per-token factors <= 1, whatever g holds. It writes the whole operand
// pack. Used for the chunks whose in-block decay is too strong for the tensor-core path.
template <int D, int MODE>
__device__ __forceinline__ void intra_simt_body(const PrefillIn &in, uint8_t *__restrict__ scratch, const Seqs &sq,
                                                int H, int b, int h, int ch, float *smem) {
    using I = Intra<D>;
    constexpr int P = I::P, PC = I::PC, NT = kIntraThreads;
    float *sK = smem;              // k, then X: k_i prod_{s=16a}^{i} a_s  (a = block of i)
    float *sQ = sK + C * P;        // q, then Y: q_i prod_{s=16a}^{i} a_s
    float *sA = sQ + C * P;        // a = e^g, then v
    float *sZ = sA + C * P;        // Z: k_j prod_{s=j+1}^{16b+15} a_s
    float *sL = sZ + I::NZ * P;    // L' (unscaled), then M'
    float *sM = sL + C * PC;       // M
    float *sT = sM + C * PC;       // T, then Tb (row stride PT)
    float *sF = sT + C * I::PT;    // [4][D]: whole-block decay products
    float *sB = sF + 4 * D;        // beta
    float *sTmp = sB + C;          // [1024]

    const int tid = threadIdx.x;
    int n = 0;
    size_t row0 = 0;
    seq_chunk(sq, b, ch, row0, n, nullptr);  // listed chunks are non-empty and in bounds

    // ---- load k, q and a = e^g (pad guard: rows >= n are k = q = 0, a = 1)
    for (int e = tid; e < C * D / 4; e += NT) {
        const int i = e / (D / 4), c = 4 * (e % (D / 4));
        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), qv = kv, av = make_float4(1.f, 1.f, 1.f, 1.f);
        if (i < n) {
            kv = load4_in<D, MODE>(in, 1, row0 + i, H, h, c);
            qv = load4_in<D, MODE>(in, 0, row0 + i, H, h, c);
            const float4 g = load4_in<D, MODE>(in, 3, row0 + i, H, h, c);
            av = make_float4(expf(g.x), expf(g.y), expf(g.z), expf(g.w));
        }
        *reinterpret_cast<float4 *>(sK + i * P + c) = kv;
        *reinterpret_cast<float4 *>(sQ + i * P + c) = qv;
        *reinterpret_cast<float4 *>(sA + i * P + c) = av;
    }
    if (tid < C) sB[tid] = tid < n ? in.beta[(row0 + tid) * H + h] : 0.f;
    __syncthreads();

    // ---- diagonal 16x16 blocks: thread (block a, j pair, channel group) walks i upward with
    //      the running product G = k_j prod_{s=j+1}^{i} a_s over its channels; the 16 channel
    //      groups of one j are 16 adjacent lanes and reduce with shuffles. Channel group cg
    //      holds float4 columns cg, cg + 16, ... (conflict-free 16-byte loads).
    {
        constexpr int NV = D / 64;  // float4 per thread per row (2 for D = 128, 1 for D = 64)
        const int cg = tid & 15, jp = (tid >> 4) & 7, a = tid >> 7;
        const unsigned gmask = 0xFFFFu << (tid & 16);
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const int j = 16 * a + (pass == 0 ? jp : 15 - jp);
            float4 G[NV];
#pragma unroll
            for (int w = 0; w < NV; ++w) G[w] = *reinterpret_cast<const float4 *>(sK + j * P + 4 * (cg + 16 * w));
#pragma unroll 1
            for (int i = j; i < 16 * a + 16; ++i) {
                float ls = 0.f, ms = 0.f;
#pragma unroll
                for (int w = 0; w < NV; ++w) {
                    const int c = 4 * (cg + 16 * w);
                    if (i > j) {
                        const float4 av = *reinterpret_cast<const float4 *>(sA + i * P + c);
                        G[w].x *= av.x; G[w].y *= av.y; G[w].z *= av.z; G[w].w *= av.w;
                    }
                    const float4 kv = *reinterpret_cast<const float4 *>(sK + i * P + c);
                    const float4 qv = *reinterpret_cast<const float4 *>(sQ + i * P + c);
                    ls = fmaf(kv.x, G[w].x, fmaf(kv.y, G[w].y, fmaf(kv.z, G[w].z, fmaf(kv.w, G[w].w, ls))));
                    ms = fmaf(qv.x, G[w].x, fmaf(qv.y, G[w].y, fmaf(qv.z, G[w].z, fmaf(qv.w, G[w].w, ms))));
                }
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) {
                    ls += __shfl_xor_sync(gmask, ls, o);
                    ms += __shfl_xor_sync(gmask, ms, o);
                }
                if (cg == 0) {
                    sL[i * PC + j] = ls;
                    sM[i * PC + j] = ms;
                }
            }
        }
    }
    __syncthreads();

    // ---- block-local factors, thread (channel c, block a): Z (backward within blocks 0..2),
    //      the whole-block products F, then X, Y (forward within blocks 1..3, in place).
    if (tid < 4 * D) {
        const int c = tid % D, a = tid / D;
        float f = 1.f;
        for (int j = 16 * a + 15; j >= 16 * a; --j) {
            sZ[j * P + c] = sK[j * P + c] * f;
            f *= sA[j * P + c];
        }
        sF[a * D + c] = f;
    }
    __syncthreads();
    if (tid < 4 * D) {
        const int c = tid % D, a = tid / D;
        float f = 1.f;
        for (int i = 16 * a; i < 16 * a + 16; ++i) {
            f *= sA[i * P + c];
            sK[i * P + c] *= f;
            sQ[i * P + c] *= f;
        }
    }
    __syncthreads();

    // ---- off-diagonal blocks (a > b): L'[i][j] = sum_c X_ic sigma_ab,c Z_jc (Y for M), with
    //      sigma_ab the decay of the whole blocks strictly between b and a (1 when adjacent).
    //      Thread = (4x4 tile, channel quarter); the 4 quarters are adjacent lanes.
    if (tid < 384) {
        const int qtr = tid & 3, tile = tid >> 2;
        const int p = tile >> 4;
        const int pa = p == 0 ? 1 : (p < 3 ? 2 : 3);
        const int pb = p == 0 ? 0 : (p == 1 ? 0 : (p == 2 ? 1 : p - 3));
        const int i0 = 16 * pa + 4 * ((tile & 15) >> 2), j0 = 16 * pb + 4 * (tile & 3);
        float l[4][4], m[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2) { l[r][s2] = 0.f; m[r][s2] = 0.f; }
#pragma unroll 2
        for (int cq = 0; cq < D / 16; ++cq) {
            const int c = 4 * (qtr + 4 * cq);
            float4 sg = make_float4(1.f, 1.f, 1.f, 1.f);
            if (pa - pb >= 2) {
                sg = *reinterpret_cast<const float4 *>(sF + 1 * D + c);
                if (pa - pb == 3) {
                    const float4 f2 = *reinterpret_cast<const float4 *>(sF + 2 * D + c);
                    sg.x *= f2.x; sg.y *= f2.y; sg.z *= f2.z; sg.w *= f2.w;
                } else if (pa == 3) {
                    sg = *reinterpret_cast<const float4 *>(sF + 2 * D + c);
                }
            }
            float4 z[4], x[4], y[4];
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2) {
                z[s2] = *reinterpret_cast<const float4 *>(sZ + (j0 + s2) * P + c);
                z[s2].x *= sg.x; z[s2].y *= sg.y; z[s2].z *= sg.z; z[s2].w *= sg.w;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                x[r] = *reinterpret_cast<const float4 *>(sK + (i0 + r) * P + c);
                y[r] = *reinterpret_cast<const float4 *>(sQ + (i0 + r) * P + c);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    l[r][s2] = fmaf(x[r].x, z[s2].x, fmaf(x[r].y, z[s2].y, fmaf(x[r].z, z[s2].z, fmaf(x[r].w, z[s2].w, l[r][s2]))));
                    m[r][s2] = fmaf(y[r].x, z[s2].x, fmaf(y[r].y, z[s2].y, fmaf(y[r].z, z[s2].z, fmaf(y[r].w, z[s2].w, m[r][s2]))));
                }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2) {
#pragma unroll
                for (int o = 1; o < 4; o <<= 1) {
                    l[r][s2] += __shfl_xor_sync(0xffffffffu, l[r][s2], o);
                    m[r][s2] += __shfl_xor_sync(0xffffffffu, m[r][s2], o);
                }
            }
        if (qtr == 0) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    sL[(i0 + r) * PC + j0 + s2] = l[r][s2];
                    sM[(i0 + r) * PC + j0 + s2] = m[r][s2];
                }
        }
    }
    __syncthreads();

    // ---- the chunk's operands: K o A = X P_a (kept in sK for W), Q o A = Y P_a (pack), and
    //      K o e^{Gamma_C - Gamma} = Z S_a (pack), with P_a / S_a the decay of all blocks before /
    //      after block a; 16-byte chunks of 8 channels. v replaces a = e^g in sA (pad rows 0).
    using PK = Pack<D>;
    uint8_t *pack = scratch + pack_slot(sq, b, h, ch, row0, H) * PK::bytes;
    for (int e = tid; e < C * (D / 8); e += NT) {
        const int i = e / (D / 8), cb = 8 * (e % (D / 8)), a = i >> 4;
        float xq[8], xb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = cb + u;
            float pre = 1.f, suf = 1.f;
            for (int bb = 0; bb < a; ++bb) pre *= sF[bb * D + c];
            for (int bb = a + 1; bb < 4; ++bb) suf *= sF[bb * D + c];
            sK[i * P + c] *= pre;
            xq[u] = sQ[i * P + c] * pre;
            xb[u] = sZ[i * P + c] * suf;
        }
        uint4 hi, lo;
        split8(xq, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + kmaj_off(64 + i, cb, 128)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + PK::A1 / 2 + kmaj_off(64 + i, cb, 128)) = lo;
        split8(xb, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A3 + mnmaj_off(cb, i, C)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_A3 + PK::A3 / 2 + mnmaj_off(cb, i, C)) = lo;
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
        if (i < n) {
            v0 = load4_in<D, MODE>(in, 2, row0 + i, H, h, cb);
            v1 = load4_in<D, MODE>(in, 2, row0 + i, H, h, cb + 4);
        }
        *reinterpret_cast<float4 *>(sA + i * P + cb) = v0;
        *reinterpret_cast<float4 *>(sA + i * P + cb + 4) = v1;
    }
    if (tid < D) {
        float acv = 1.f;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acv *= sF[bb * D + tid];
        reinterpret_cast<float *>(pack + PK::OFF_AC)[tid] = acv;
    }
    // ---- M into the pack (64 x 64 K-major, zero above the diagonal); L = diag(beta) L'
    {
        const int r = tid >> 3, c0 = 8 * (tid & 7);
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = c0 + u <= r ? sM[r * PC + c0 + u] : 0.f;
        uint4 hi, lo;
        split8(x, hi, lo);
        *reinterpret_cast<uint4 *>(pack + PK::OFF_AM + kmaj_off(r, c0, 64)) = hi;
        *reinterpret_cast<uint4 *>(pack + PK::OFF_AM + PK::AM / 2 + kmaj_off(r, c0, 64)) = lo;
    }
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        if (i > j) sL[i * PC + j] *= sB[i];
    }
    __syncthreads();
    invert_unit_lower64<NT>(sL, sT, sTmp);
    // ---- Tb = T diag(beta) in place (lower triangle and diagonal)
    for (int e = tid; e < C * C; e += NT) {
        const int i = e / C, j = e % C;
        if (j <= i) sT[i * I::PT + j] *= sB[j];
    }
    __syncthreads();
    // ---- W = Tb (K o A) -> A1 rows 0..63 (BF16 hi/lo);  U~ = Tb V -> UT (FP32)
    for (int e = tid; e < 2 * C * (D / 8); e += NT) {
        const int wv = e / (C * (D / 8)), r = e % (C * (D / 8));
        const int i = r / (D / 8), cb = 8 * (r % (D / 8));
        const float *src = wv == 0 ? sK : sA;
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j <= i; ++j) {
            const float t = sT[i * I::PT + j];
            const float4 s0 = *reinterpret_cast<const float4 *>(src + j * P + cb);
            const float4 s1 = *reinterpret_cast<const float4 *>(src + j * P + cb + 4);
            x[0] = fmaf(t, s0.x, x[0]); x[1] = fmaf(t, s0.y, x[1]); x[2] = fmaf(t, s0.z, x[2]); x[3] = fmaf(t, s0.w, x[3]);
            x[4] = fmaf(t, s1.x, x[4]); x[5] = fmaf(t, s1.y, x[5]); x[6] = fmaf(t, s1.z, x[6]); x[7] = fmaf(t, s1.w, x[7]);
        }
        if (wv == 0) {
            uint4 hi, lo;
            split8(x, hi, lo);
            *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + kmaj_off(i, cb, 128)) = hi;
            *reinterpret_cast<uint4 *>(pack + PK::OFF_A1 + PK::A1 / 2 + kmaj_off(i, cb, 128)) = lo;
        } else {
            float *dst = reinterpret_cast<float *>(pack + PK::OFF_UT + (cb >> 5) * PK::UG_BYTES) + i * PK::UP + (cb & 31);
            *reinterpret_cast<float4 *>(dst) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4 *>(dst + 4) = make_float4(x[4], x[5], x[6], x[7]);
        }
    }
    if (in.tables && tid < D) {  // verify mode: Gamma (in-chunk cumulative log-decay) for the fold
        float *gt = in.tables + ((static_cast<size_t>(b) * H + h) * 2 + 1) * C * D;
        float acc = 0.f;
        for (int i = 0; i < C; ++i) {
            if (i < n) {
                const float4 g4 = load4_in<D, MODE>(in, 3, row0 + i, H, h, tid & ~3);
                acc += (tid & 3) == 0 ? g4.x : ((tid & 3) == 1 ? g4.y : ((tid & 3) == 2 ? g4.z : g4.w));
            }
            gt[i * D + tid] = acc;
        }
    }
}

// Only the chunks the tensor-core kernel listed (count and packed (b, h, ch) entries in scratch).
template <int D, int MODE>
__global__ void __launch_bounds__(kIntraThreads, 1)
intra_fix_kernel(const PrefillIn in, uint8_t *__restrict__ scratch, const int *__restrict__ list, const Seqs sq,
                 int H) {
    extern __shared__ float smem[];
    pdl_release();
    pdl_acquire();  // the tensor-core pass has listed its chunks
    const int count = list[0];
    const int nch = sq.nch;
    for (int e = blockIdx.x; e < count; e += gridDim.x) {
        const int id = list[1 + e];
        const int ch = id % nch, h = (id / nch) % H, b = id / (nch * H);
        intra_simt_body<D, MODE>(in, scratch, sq, H, b, h, ch, smem);
        __syncthreads();
    }
}

// ---------------------------------------------------------------- intra-chunk on tensor cores
//
// L' and M for all pairs of the chunk in one tcgen05 contraction. Each 16-token block a gets
// the reference point m_a = 16a + 7 (its middle). With Gamma the in-chunk cumulative decay,
//   A rows  i (block a):      k_i e^{Gamma_i - Gamma_{m_a}}   (and q_i ... for rows 64 + i)
//   B rows  (a', j), j <= 16a'+15:  k_j e^{Gamma_{m_a'} - Gamma_j}
// so D[i][(a, j)] = sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc} = L'[i][j] exactly for every j <= i
// (the reference cancels). B holds the 16, 32, 48, 64 rows of a' = 0..3 at column offsets
// 0, 16, 48, 96 (160 rows). Factors above 1 come only from decay inside one block (at most
// 8 tokens); a chunk whose |Gamma_i - Gamma_{m_a}| exceeds kRefBound for some channel is
// handed to the CUDA-core body instead (listed in scratch, run by intra_fix_kernel).
//
// Two 256-thread CTAs share an SM (113 KB of shared memory and 256 TMEM columns each), so one
// CTA's MMA, barrier and load latencies run under the other's CUDA-core work. The L/M operands
// are built and contracted 64 channels at a time through one 72 KB buffer; q, k and v come
// straight from global memory, read evict-first where an item reads them for the last time (an
// L2 prefetch of the next item's rows measured slower: it competes with the current item's
// misses); W and U~ leave TMEM straight for the pack.

constexpr float kRefBound = 80.0f;  // e^80 and e^-80 are comfortably inside BF16/FP32 range
constexpr int kTcThreads = 256;

template <int D>
struct IntraTC {
    static constexpr int NH = D / 64;             // 64-channel parts of the L/M contraction
    static constexpr int NB = 160;                // B rows of the L/M MMA
    static constexpr int A_H = 2 * 128 * 64 * 2;  // L/M A part: 128 rows x 64 channels, hi + lo
    static constexpr int B_H = 2 * NB * 64 * 2;   // L/M B part: 160 rows x 64 channels, hi + lo
    static constexpr int R1 = A_H + B_H;          // 72 KB
    static constexpr int R2 = C * D * 4;          // g / Gamma [C][D] FP32, then the V part of the W|U~ B operand
    static constexpr int KA = 2 * C * D * 2;      // one [C tokens][D channels] MN-major operand, hi + lo
    static constexpr int TAB = 14 * D * 4;        // per-channel reference factors
    static constexpr int OFF_R2 = R1, OFF_TAB = OFF_R2 + R2, OFF_MISC = OFF_TAB + TAB;
    static constexpr int MISC = C * 4 + 64;       // beta[C], two barriers, TMEM slot
    static constexpr int bytes = OFF_MISC + MISC + 1024;
    // R1 once the L/M MMA has completed: L, T (FP32), scratch of the inverse, Tb (K-major hi + lo);
    // then the K o A part of the W|U~ B operand at offset 0 (over the dead L and T)
    static constexpr int OFF_L = 0, OFF_T = C * kLPC * 4, OFF_TMP = OFF_T + C * kTPC * 4;
    static constexpr int OFF_TB = (OFF_TMP + 4096 + 1023) / 1024 * 1024;
    static_assert(OFF_TB + 16384 <= R1, "R1 holds L, T, the inverse's scratch and Tb");
    static_assert(KA <= OFF_TB, "the K o A operand part must not overlap Tb");
    static_assert(KA == R2, "the V operand part fills R2");
    static constexpr int W_STAGE = 2 * C * D * 2;  // W rows 0..63 of A1 (hi + lo), staged in R1 for the bulk stores
    static_assert(W_STAGE + Pack<D>::UT <= R1, "the staged W and U~ fit in R1");
    static_assert(2 * (bytes + 1024) <= 233472, "two CTAs per SM");
};

__device__ __forceinline__ void ld8f(const float *p, float (&x)[8]) {
    const float4 a0 = *reinterpret_cast<const float4 *>(p), a1 = *reinterpret_cast<const float4 *>(p + 4);
    x[0] = a0.x; x[1] = a0.y; x[2] = a0.z; x[3] = a0.w; x[4] = a1.x; x[5] = a1.y; x[6] = a1.z; x[7] = a1.w;
}

// 16 BF16 hi + lo bytes of 8 values at `off` of a split tile in global memory (hi at dst, lo at dst + half)
__device__ __forceinline__ void st_pair_g(uint8_t *dst, int half_bytes, uint32_t off, const float (&x)[8],
                                          uint64_t pol) {
    uint4 hi, lo;
    split8(x, hi, lo);
    st16_hint(dst + off, hi, pol);
    st16_hint(dst + half_bytes + off, lo, pol);
}

// One thread: bulk shared -> global copy (bytes a multiple of 16), in this thread's bulk group.
__device__ __forceinline__ void bulk_store(void *gdst, const void *smem_src, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(gdst),
                 "r"(smem_u32(smem_src)), "r"(bytes), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// The map over the rows of the log-decay input (3-D: columns, row in stream, stream): the g box
// (FP32 gate, or BF16 g_raw) of an item is loaded through it.
struct InMaps {
    CUtensorMap g;
};

template <int D, int MODE>
__global__ void __launch_bounds__(kTcThreads, 2)
intra_tc_kernel(const __grid_constant__ InMaps maps, const PrefillIn in, uint8_t *__restrict__ scratch,
                int *__restrict__ list, int B, const Seqs sq, int H, int *__restrict__ status) {
    const CUtensorMap &tmG = maps.g;
    using I = IntraTC<D>;
    using PK = Pack<D>;
    constexpr int NT = kTcThreads, PC = kLPC, PT = kTPC, NH = I::NH;
    constexpr int UB = C * (D / 8) / NT;  // (token, 8-channel group) units per thread over all D channels
    constexpr bool QKV16 = kQkv16<MODE>, GRAW = kGraw<MODE>;
    extern __shared__ uint8_t smem_raw[];
    pdl_release();  // the fix-up pass may launch (it waits for this pass to complete)
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = sm, *sBt = sm + I::A_H, *sR2 = sm + I::OFF_R2, *sTb = sm + I::OFF_TB, *sKA = sm;
    float *sG = reinterpret_cast<float *>(sR2);
    float *sL = reinterpret_cast<float *>(sm + I::OFF_L);
    float *sT = reinterpret_cast<float *>(sm + I::OFF_T);
    float *sTmp = reinterpret_cast<float *>(sm + I::OFF_TMP);
    float *sTab = reinterpret_cast<float *>(sm + I::OFF_TAB);
    float *sB = reinterpret_cast<float *>(sm + I::OFF_MISC);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + I::OFF_MISC + C * 4);  // MMA commits
    uint64_t *gbar = bar + 1;                                                // the g box
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 2);
    // reference tables, [entry][D]: 0..3 e^{Gamma_{m_a}}, 4..7 e^{Gamma_C - Gamma_{m_a}},
    // 8..13 e^{Gamma_{m_a} - Gamma_{m_b}} for (a,b) = (1,0),(2,0),(2,1),(3,0),(3,1),(3,2)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nch = sq.nch;
    const int total = B * H * nch;
    const uint64_t pol_first = l2_policy(true), pol_pack = l2_policy(in.stream_pack != 0);
    constexpr uint32_t kGBox = C * D * (GRAW ? 2 : 4);
    // g's box: FP32 g at the start of R2, or BF16 g_raw in its upper half (the gate is then
    // formed in place, FP32, dense)
    void *gdst = sR2 + (GRAW ? C * D * 2 : 0);

    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(gbar, 1);
        fence_mbar_init();
    }
    // this CTA's items are blockIdx.x + j gridDim.x; empty chunk slots (varlen) are skipped
    auto next_item = [&](int it) {
        size_t r0;
        int nn;
        for (; it < total; it += gridDim.x) {
            const int c = it % nch, bb = it / (nch * H);
            if (seq_chunk(sq, bb, c, r0, nn, (it % (nch * H)) < nch && c == 0 ? status : nullptr)) break;
        }
        return it;
    };
    // TMA coordinates of a chunk's rows: (stream, row in stream) on the 3-D map, or the packed row
    auto box_yz = [&](int ch, int b, size_t row0, int &y, int &z) {
        if (sq.cu) { y = static_cast<int>(row0); z = 0; }
        else { y = ch * C; z = b; }
    };
    // an item's g box into R2 (thread 0; the caller made R2 free) and its beta (threads < C)
    float bnext = 0.f;
    auto fetch_g = [&](int it) {
        const int ch = it % nch, h = (it / nch) % H, b = it / (nch * H);
        int n;
        size_t row0;
        seq_chunk(sq, b, ch, row0, n, nullptr);
        if (tid == 0) {
            int y, z;
            box_yz(ch, b, row0, y, z);
            mbar_expect_tx(gbar, kGBox);
            tma_load_3d(gdst, &tmG, h * D, y, z, gbar);
        }
        if (tid < C) bnext = tid < n ? in.beta[(row0 + tid) * H + h] : 0.f;
    };
    tc_fence_before();
    __syncthreads();  // barriers initialised, TMEM allocated
    tc_fence_after();
    const int first = next_item(blockIdx.x);
    if (first < total) fetch_g(first);
    const uint32_t tmem = *tmem_slot;
    bool dead = false;   // a wait timed out: hand every remaining item to the CUDA-core body
    uint32_t iter = 0;   // items started by this CTA: the parity of the g box
    uint32_t mph = 0;    // MMA commits waited for: the parity of `bar`
    // a wait on `b` (phase `par`) gave up: latch the error, give the operation one more bounded
    // wait (nothing may still write shared memory), list the item for the CUDA-core body
    auto give_up = [&](uint64_t *b, uint32_t par, int it) {
        if (tid == 0) {
            atomicExch(status, KDA_ERR_TIMEOUT);
            mbar_wait(b, par, kWaitCycles);
            list[1 + atomicAdd(list, 1)] = it;
        }
        dead = true;
        __syncthreads();
    };

    int following = total;
#pragma unroll 1
    for (int item = first; item < total; item = following, ++iter) {
        const int ch = item % nch, h = (item / nch) % H, b = item / (nch * H);
        following = next_item(item + gridDim.x);
        int n;
        size_t row0;
        seq_chunk(sq, b, ch, row0, n, nullptr);
        uint8_t *pack = scratch + pack_slot(sq, b, h, ch, row0, H) * PK::bytes;
        if (dead) {  // block-uniform
            if (tid == 0) list[1 + atomicAdd(list, 1)] = item;
            continue;
        }
        bool ok = mbar_wait(gbar, iter & 1, kWaitCycles);
        if (tid < C) sB[tid] = bnext;
        if (tid == 0) bulk_wait_read();  // the previous item's staged results have left R1
        if (!__syncthreads_and(ok)) {
            give_up(gbar, iter & 1, item);
            continue;
        }
        // ---- Gamma: inclusive cumulative sum over tokens, thread (channel, range of TPQ tokens).
        //      The range lives in registers: one pass of loads, the prefix sum, the other ranges'
        //      totals added, the reference-bound check, one pass of stores.
        bool safe = true;
        {
            constexpr int QT = NT / D;  // 2 (D=128) or 4 (D=64) token ranges
            constexpr int TPQ = C / QT;
            const int c = tid % D, qr = tid / D, i0 = qr * TPQ;
            float gv[TPQ];
            if constexpr (GRAW) {
                // g = -exp(a_log) softplus(g_raw + dt_bias) (0 past the chunk's end), FP32 over g_raw's box
                const uint16_t *gr = reinterpret_cast<const uint16_t *>(gdst);
#pragma unroll
                for (int r = 0; r < TPQ; ++r) gv[r] = bf16_to_f32(gr[(i0 + r) * D + c]);
                const float nea = -expf(in.a_log[h]), dtb = in.dt_bias[static_cast<size_t>(h) * D + c];
#pragma unroll
                for (int r = 0; r < TPQ; ++r) gv[r] = i0 + r < n ? kda_gate_f32(gv[r], dtb, nea) : 0.f;
            } else {
#pragma unroll
                for (int r = 0; r < TPQ; ++r) gv[r] = i0 + r < n ? sG[(i0 + r) * D + c] : 0.f;  // rows past the end decay nothing
            }
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < TPQ; ++r) {
                acc += gv[r];
                gv[r] = acc;
            }
            sTmp[qr * D + c] = acc;
            __syncthreads();  // every range's total is in sTmp; g_raw's box has been read
            float pre = 0.f;
            for (int r = 0; r < qr; ++r) pre += sTmp[r * D + c];
#pragma unroll
            for (int r = 0; r < TPQ; ++r) {
                gv[r] += pre;
                sG[(i0 + r) * D + c] = gv[r];
            }
            if (in.tables) {  // verify mode: keep Gamma for the fold
                float *gt = in.tables + ((static_cast<size_t>(b) * H + h) * 2 + 1) * C * D;
#pragma unroll
                for (int r = 0; r < TPQ; ++r) gt[(i0 + r) * D + c] = gv[r];
            }
            // the reference bound of the 16-token blocks in this thread's range: every factor
            // e^{+-(Gamma_i - Gamma_m)} of the L/M operands stays within e^{kRefBound}
#pragma unroll
            for (int a = 0; a < TPQ / 16; ++a) {
                const float gm = gv[16 * a + 7];
#pragma unroll
                for (int r = 16 * a; r < 16 * a + 16; ++r) safe = safe && fabsf(gv[r] - gm) <= kRefBound;
            }
            safe = __syncthreads_and(safe) != 0;
        }
        if (tid < D) {
            const int c = tid;
            const float gm[4] = {sG[7 * D + c], sG[23 * D + c], sG[39 * D + c], sG[55 * D + c]};
            const float gc = sG[63 * D + c];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                sTab[a * D + c] = __expf(gm[a]);
                sTab[(4 + a) * D + c] = __expf(gc - gm[a]);
            }
            sTab[8 * D + c] = __expf(gm[1] - gm[0]);
            sTab[9 * D + c] = __expf(gm[2] - gm[0]);
            sTab[10 * D + c] = __expf(gm[2] - gm[1]);
            sTab[11 * D + c] = __expf(gm[3] - gm[0]);
            sTab[12 * D + c] = __expf(gm[3] - gm[1]);
            sTab[13 * D + c] = __expf(gm[3] - gm[2]);
            reinterpret_cast<float *>(pack + PK::OFF_AC)[c] = __expf(gc);
        }
        __syncthreads();
        // ---- the L/M operands, 64 channels at a time: thread units (token i, 8-channel group),
        //      A (mid-block reference) and B (all references) in shared memory, and the pack's
        //      state-independent operands Q o e^Gamma (A1 rows 64..127) and K o e^{Gamma_C - Gamma}
        //      (A3) written out. (The pack is written for unsafe chunks too; the CUDA-core body
        //      then rewrites it.)
#pragma unroll 1
        for (int hf = 0; hf < NH; ++hf) {
            if (hf > 0) {  // the previous part's MMA has finished reading the operand buffer
                ok = mbar_wait(bar, mph & 1, kWaitCycles);
                tc_fence_after();
                ok = __syncthreads_and(ok) != 0;
                if (!ok) break;
                ++mph;
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int u = tid + NT * j, i = u >> 3, cl = 8 * (u & 7), cb = 64 * hf + cl, a = i >> 4;
                float k8[8], q8[8], gi[8], gm[8], ef[8], ei[8], x[8];
                if (i < n) {
                    load8_in<D, QKV16>(in, 1, row0 + i, H, h, cb, k8);
                    load8_in<D, QKV16>(in, 0, row0 + i, H, h, cb, q8, true, pol_first);
                } else {
#pragma unroll
                    for (int w = 0; w < 8; ++w) { k8[w] = 0.f; q8[w] = 0.f; }
                }
                ld8f(sG + i * D + cb, gi);
                ld8f(sG + (16 * a + 7) * D + cb, gm);
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    const float r = gi[w] - gm[w];
                    ef[w] = __expf(r);
                    ei[w] = __expf(-r);
                }
#pragma unroll
                for (int w = 0; w < 8; ++w) x[w] = k8[w] * ef[w];
                st_pair(sA, I::A_H / 2, kmaj_off(i, cl, 128), x);
#pragma unroll
                for (int w = 0; w < 8; ++w) x[w] = q8[w] * ef[w];
                st_pair(sA, I::A_H / 2, kmaj_off(64 + i, cl, 128), x);
                // B rows for every reference block a2 >= a (column offsets 0, 16, 48, 96)
#pragma unroll
                for (int a2 = 0; a2 < 4; ++a2) {
                    if (a2 < a) continue;
                    const int off2 = 8 * a2 * (a2 + 1);
                    if (a2 == a) {
#pragma unroll
                        for (int w = 0; w < 8; ++w) x[w] = k8[w] * ei[w];
                    } else {
                        const int tix = a2 == 1 ? 8 : (a2 == 2 ? (a == 0 ? 9 : 10) : (a == 0 ? 11 : (a == 1 ? 12 : 13)));
                        float tb[8];
                        ld8f(sTab + tix * D + cb, tb);
#pragma unroll
                        for (int w = 0; w < 8; ++w) x[w] = k8[w] * ei[w] * tb[w];
                    }
                    st_pair(sBt, I::B_H / 2, kmaj_off(off2 + i, cl, I::NB), x);
                }
                // pack operands: e^{Gamma_i} = ef e^{Gamma_m}, e^{Gamma_C - Gamma_i} = ei e^{Gamma_C - Gamma_m}
                float em[8];
                ld8f(sTab + a * D + cb, em);
#pragma unroll
                for (int w = 0; w < 8; ++w) x[w] = q8[w] * (ef[w] * em[w]);
                st_pair_g(pack + PK::OFF_A1, PK::A1 / 2, kmaj_off(64 + i, cb, 128), x, pol_pack);
                ld8f(sTab + (4 + a) * D + cb, em);
#pragma unroll
                for (int w = 0; w < 8; ++w) x[w] = k8[w] * (ei[w] * em[w]);
                st_pair_g(pack + PK::OFF_A3, PK::A3 / 2, mnmaj_off(cb, i, C), x, pol_pack);
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            // D[128 x 160] (+)= A . B^T over this part's 64 channels (L' in rows 0..63, M in 64..127)
            if (tid == 0) {
                constexpr uint32_t id = idesc_bf16(128, I::NB, false, false);
                const uint64_t dah = kmaj_desc(smem_u32(sA), 128, 0, 0), dal = kmaj_desc(smem_u32(sA) + I::A_H / 2, 128, 0, 0);
                const uint64_t dbh = kmaj_desc(smem_u32(sBt), I::NB, 0, 0);
                const uint64_t dbl = kmaj_desc(smem_u32(sBt) + I::B_H / 2, I::NB, 0, 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ah = dah + kmaj_step(128, ks), al = dal + kmaj_step(128, ks);
                    const uint64_t bh = dbh + kmaj_step(I::NB, ks), bl = dbl + kmaj_step(I::NB, ks);
                    mma_bf16(tmem, ah, bh, id, (hf > 0 || ks > 0) ? 1u : 0u);
                    mma_bf16(tmem, ah, bl, id, 1);
                    mma_bf16(tmem, al, bh, id, 1);
                }
                mma_commit(bar);
            }
        }
        if (!ok) {  // a part's wait gave up (block-uniform)
            give_up(bar, mph & 1, item);
            continue;
        }
        ok = mbar_wait(bar, mph & 1, kWaitCycles);  // the last part's MMA
        tc_fence_after();
        if (!__syncthreads_and(ok)) {
            give_up(bar, mph & 1, item);
            continue;
        }
        ++mph;
        if (!safe) {  // the CUDA-core body redoes this chunk (it rewrites the whole pack)
            if (tid == 0) list[1 + atomicAdd(list, 1)] = item;
            if (following < total) fetch_g(following);  // R2 (Gamma) is free
            continue;
        }
        // ---- read back: warp (quad, part); row r = 32 quad + lane (i = r % 64, block a = i / 16)
        //      needs columns [off_a, off_a + 16(a+1)); the quad's window is [0, 48) for rows in
        //      blocks 0-1 and [48, 160) for blocks 2-3, its 8-column chunks split over two warps.
        //      L = diag(beta) L' (strictly lower) to shared memory; M (lower with diagonal, zero
        //      above) straight into the pack.
        {
            const int quad = warp & 3, part = warp >> 2;
            const int r = 32 * quad + lane, i = r & 63, a = i >> 4;
            const int off_a = 8 * a * (a + 1), seg = 16 * (a + 1);
            const int w0 = (quad & 1) ? 48 : 0, wlen = (quad & 1) ? 112 : 48;
            const bool is_l = r < 64;
            const float bi = sB[i];
#pragma unroll 1
            for (int c8 = part * 8; c8 < wlen; c8 += 16) {
                float x[8];
                tmem_ld8(tmem_lane_base(tmem, warp) + w0 + c8, x);
                tmem_ld_wait();
                const int j0 = w0 + c8 - off_a;
                if (j0 >= 0 && j0 < seg) {
                    if (is_l) {
#pragma unroll
                        for (int w = 0; w < 8; ++w)
                            if (j0 + w < i) sL[i * PC + j0 + w] = x[w] * bi;
                    } else {
#pragma unroll
                        for (int w = 0; w < 8; ++w) x[w] = j0 + w <= i ? x[w] : 0.f;
                        st_pair_g(pack + PK::OFF_AM, PK::AM / 2, kmaj_off(i, j0, 64), x, pol_pack);
                    }
                }
            }
            if (!is_l) {
                const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int jc = seg / 8 + part; jc < 8; jc += 2) st_pair_g(pack + PK::OFF_AM, PK::AM / 2, kmaj_off(i, 8 * jc, 64), z, pol_pack);
            }
        }
        tc_fence_before();
        __syncthreads();
        invert_unit_lower64<NT>(sL, sT, sTmp);
        // ---- Tb = T diag(beta) as the A operand (64 x 64 K-major, zero above the diagonal)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int u = tid + NT * j, r = u >> 3, c0 = 8 * (u & 7);
            float tr[8], bc[8], x[8];
            ld8f(sT + r * PT + c0, tr);
            ld8f(sB + c0, bc);
#pragma unroll
            for (int w = 0; w < 8; ++w) x[w] = c0 + w <= r ? tr[w] * bc[w] : 0.f;
            st_pair(sTb, 8192, kmaj_off(r, c0, 64), x);
        }
        __syncthreads();  // T is dead: the K o A operand part may overwrite it
        // ---- the W|U~ B operand, MN-major (n = channel, k = token): K o A = K o e^Gamma over the
        //      dead L and T, then V over Gamma (v held in registers across the barrier)
        float vv[UB][8];
#pragma unroll
        for (int j = 0; j < UB; ++j) {
            const int u = tid + NT * j, i = u / (D / 8), cb = 8 * (u % (D / 8));
            float k8[8], gi[8], x[8];
            if (i < n) {
                load8_in<D, QKV16>(in, 1, row0 + i, H, h, cb, k8, true, pol_first);
                load8_in<D, QKV16>(in, 2, row0 + i, H, h, cb, vv[j], true, pol_first);
            } else {
#pragma unroll
                for (int w = 0; w < 8; ++w) { k8[w] = 0.f; vv[j][w] = 0.f; }
            }
            ld8f(sG + i * D + cb, gi);
#pragma unroll
            for (int w = 0; w < 8; ++w) x[w] = k8[w] * __expf(gi[w]);
            st_pair(sKA, I::KA / 2, mnmaj_off(cb, i, C), x);
        }
        __syncthreads();  // Gamma is dead
#pragma unroll
        for (int j = 0; j < UB; ++j) {
            const int u = tid + NT * j, i = u / (D / 8), cb = 8 * (u % (D / 8));
            st_pair(sR2, I::KA / 2, mnmaj_off(cb, i, C), vv[j]);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- [W | U~] = Tb . [K o A | V]  (M = 64, N = D each, K = 64) into TMEM columns 0..2D-1
        if (tid == 0) {
            constexpr uint32_t id = idesc_bf16(64, D, false, true);
            const uint64_t dah = kmaj_desc(smem_u32(sTb), 64, 0, 0), dal = kmaj_desc(smem_u32(sTb) + 8192, 64, 0, 0);
            const uint64_t dkh = mnmaj_desc(smem_u32(sKA), C, 0, 0), dkl = mnmaj_desc(smem_u32(sKA) + I::KA / 2, C, 0, 0);
            const uint64_t dvh = mnmaj_desc(smem_u32(sR2), C, 0, 0), dvl = mnmaj_desc(smem_u32(sR2) + I::KA / 2, C, 0, 0);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t ah = dah + kmaj_step(64, ks), al = dal + kmaj_step(64, ks);
                const uint64_t kh = dkh + mnmaj_step(ks), kl = dkl + mnmaj_step(ks);
                const uint64_t vh = dvh + mnmaj_step(ks), vl = dvl + mnmaj_step(ks);
                const uint32_t acc = ks > 0 ? 1u : 0u;
                mma_bf16(tmem, ah, kh, id, acc);
                mma_bf16(tmem, ah, kl, id, 1);
                mma_bf16(tmem, al, kh, id, 1);
                mma_bf16(tmem + D, ah, vh, id, acc);
                mma_bf16(tmem + D, ah, vl, id, 1);
                mma_bf16(tmem + D, al, vh, id, 1);
            }
            mma_commit(bar);
        }
        ok = mbar_wait(bar, mph & 1, kWaitCycles);
        tc_fence_after();
        if (!__syncthreads_and(ok)) {
            give_up(bar, mph & 1, item);
            continue;
        }
        ++mph;
        if (following < total) fetch_g(following);  // R2 is free: the next item's g box comes in
        // ---- read back (M = 64 layout: row 16 quad + lane in lanes < 16 of the quad); warp part 0
        //      takes W (columns 0..D-1: rows 0..63 of A1, BF16 hi + lo), part 1 U~ (FP32), staged in
        //      R1 in the pack's own layout (the operands there are dead) and written out by bulk copies
        {
            uint8_t *sWs = sm;                                          // W: [hi|lo][D/64 panels][64 rows x 128 B]
            float *sUs = reinterpret_cast<float *>(sm + I::W_STAGE);  // U~: the pack's UT layout
            const int quad = warp & 3, part = warp >> 2, row = 16 * quad + lane;
#pragma unroll 1
            for (int c32 = 0; c32 < D; c32 += 32) {
                float x[2][16];
                tmem_ld16(tmem_lane_base(tmem, warp) + part * D + c32, x[0]);
                tmem_ld16(tmem_lane_base(tmem, warp) + part * D + c32 + 16, x[1]);
                tmem_ld_wait();
                if (lane < 16) {
#pragma unroll
                    for (int hl = 0; hl < 4; ++hl) {
                        const int cc = c32 + 8 * hl;
                        const float(&x8)[8] = *reinterpret_cast<const float(*)[8]>(&x[hl >> 1][8 * (hl & 1)]);
                        if (part == 0) {
                            st_pair(sWs, I::W_STAGE / 2, (cc >> 6) * 8192 + kmaj_off(row, cc & 63, 64), x8);
                        } else {
                            float *dst = sUs + (cc >> 5) * (PK::UG_BYTES / 4) + row * PK::UP + (cc & 31);
                            *reinterpret_cast<float4 *>(dst) = make_float4(x8[0], x8[1], x8[2], x8[3]);
                            *reinterpret_cast<float4 *>(dst + 4) = make_float4(x8[4], x8[5], x8[6], x8[7]);
                        }
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();  // TMEM is read: the next item's MMAs may overwrite it
            if (tid == 0) {
#pragma unroll
                for (int p = 0; p < D / 64; ++p) {
                    bulk_store(pack + PK::OFF_A1 + p * 16384, sWs + p * 8192, 8192, pol_pack);
                    bulk_store(pack + PK::OFF_A1 + PK::A1 / 2 + p * 16384, sWs + I::W_STAGE / 2 + p * 8192, 8192, pol_pack);
                }
                bulk_store(pack + PK::OFF_UT, sUs, PK::UT, pol_pack);
                bulk_commit();
            }
        }
    }
    if (tid == 0) bulk_wait_all();  // every staged result is in global memory
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ================================================================ phase 2: state pass

template <int D, int DVS>
struct State {
    using PK = Pack<D>;
    static constexpr int NB = DVS < 64 ? 64 : DVS;  // MN-major B tiles span whole 64-wide atoms
    static constexpr int A2 = 2 * kTileBytes;       // [0; M]: 128 x 64 K-major hi + lo, rows 0..63 zero
    static constexpr int B1 = 2 * NB * D * 2;       // S0 hi + lo, MN-major (N = value columns, K = D keys)
    static constexpr int B2 = 2 * NB * C * 2;       // U hi + lo, MN-major (N = value columns, K = 64)
    // two U operands where they fit: a chunk's output group (D1 += [0; M] U) then runs after the
    // next chunk's D1, beside its epilogue, instead of ahead of it in the tensor pipe
    static constexpr int NU = PK::A1 + 2 * kTileBytes + PK::A3 + B1 + 2 * B2 + 2048 <= 232448 ? 2 : 1;
    static constexpr int OFF_A1 = 0, OFF_A2 = PK::A1, OFF_A3 = OFF_A2 + A2, OFF_B1 = OFF_A3 + PK::A3,
                         OFF_B2 = OFF_B1 + B1, OFF_MISC = OFF_B2 + NU * B2;
    static constexpr int MISC = 1024;
    static constexpr int bytes = OFF_MISC + MISC + 1024;  // + alignment slack
    static_assert(bytes <= 232448, "one CTA per SM");
    // D1 twice (chunk parity: a chunk's outputs are read while the next chunk's D1 is computed), D3,
    // and the FP32 master copy of the state slice (key row = lane, value column = column)
    static constexpr uint32_t TMEM_COLS = 4 * DVS;
    static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512, "TMEM columns");
};

// A bulk global -> shared copy completing on `bar`, whose expected bytes were already
// announced by the caller (several copies on one barrier).
__device__ __forceinline__ void bulk_copy_nx(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Issue a bulk global -> shared copy of `bytes` (multiple of 16) completing on `bar`.
__device__ __forceinline__ void bulk_copy(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// The chain of one (stream, head, value slice of DVS columns) over its chunks. Per chunk:
//   MMA group 1   D1 = [W; Q o A] . S0                       (M = 128, N = DVS, K = D)
//   epilogue 1    U = U~ - D1[0:64] into shared memory
//   MMA group 2   D3 = (K o e^{Gamma_C - Gamma})^T . U        (M = D, N = DVS, K = 64)
//   MMA group 3   D1 += [0; M] . U                            (so D1[64:128] = (Q o A) S0 + M U)
//   epilogue 2    S = A_C o S0 + D3 (the FP32 master copy lives in TMEM) into the S operand
// Groups 1 and 2 and the two epilogues are the critical path. Two control threads issue every
// copy and every MMA, so that the epilogue warps never wait behind MMA issue: the chain thread
// (warp kEpiWarps) issues groups 1 and 2 and the copies of their operands; with two U operands in
// shared memory the output thread (warp kEpiWarps + 1) issues group 3 of a chunk once its group 2
// has completed (it then runs while epilogue 2 does) and copies the next M; with one U operand the
// chain thread issues group 3 right after group 2. The output rows O = scale D1[64:128] of chunk c
// are read while group 2 of chunk c + 1 runs. Epilogue and control warps hand over through
// mbarriers. Epilogue warps: 8 (4 TMEM lane quarters x 2 column groups), 16 for 128-column
// slices (x 4), so that a thread's share of an epilogue stays at 32 columns or fewer.
template <int DVS>
constexpr int kEpiWarpsFor = DVS >= 128 ? 16 : 8;
template <int DVS>
constexpr int kStateThreadsFor = 32 * (kEpiWarpsFor<DVS> + 2);  // + the two control warps

template <int D, int DVS>
__global__ void __launch_bounds__(kStateThreadsFor<DVS>, 1)
state_kernel(const uint8_t *__restrict__ scratch, float *const *__restrict__ h_state, float *__restrict__ core,
             const Seqs sq, int H, float scale, float *__restrict__ tables, int *__restrict__ status) {
    using S = State<D, DVS>;
    using PK = Pack<D>;
    constexpr int kEpiWarps = kEpiWarpsFor<DVS>, kStateThreads = kStateThreadsFor<DVS>;
    constexpr int HALF = DVS / (kEpiWarps / 4);  // value columns per epilogue thread
    // U~ read into registers while group 1 runs (slices up to 64 columns; wider slices read it one
    // 8-column group ahead: with 9 warps one scheduler holds three, so a thread has about 168 registers)
    constexpr bool kPreU = HALF <= 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA1 = sm + S::OFF_A1, *sA2 = sm + S::OFF_A2, *sA3 = sm + S::OFF_A3, *sB1 = sm + S::OFF_B1,
            *sB2 = sm + S::OFF_B2;
    // barriers: copies 0 A1, 1 M, 2 A3; MMA groups 4 (D1), 5 (D3), 6 (D1 += [0; M] U); 7 and 10 the
    // final drains after a timeout (chain and output threads); 8 "U is in B2" and 9 "S is in B1, D3
    // read" (one arrival per epilogue warp, after the warp's own writes and TMEM reads)
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::OFF_MISC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::OFF_MISC + 128);
    int *fail = reinterpret_cast<int *>(sm + S::OFF_MISC + 136);  // a role gave up waiting

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int c0 = slice * DVS;
    const size_t rs = static_cast<size_t>(H) * D;
    const int nch = sq.nch;  // chunk slots per stream in the scratch
    int nb = nch;            // this stream's chunks
    size_t first_row = 0;    // its first row (varlen mode)
    if (sq.cu) {
        const int s0 = sq.cu[b], s1 = sq.cu[b + 1];
        if (s0 < 0 || s1 < s0 || s1 > sq.total || s1 - s0 > nch * C) {  // a bad cu_seqlens entry
            if (tid == 0 && slice == 0 && h == 0) atomicExch(status, KDA_ERR_INVALID_ARG);
            return;
        }
        nb = (s1 - s0 + C - 1) / C;
        first_row = static_cast<size_t>(s0);
    }
    if (nb == 0) return;  // an empty stream keeps its state
    float *Sg = h_state[b] + static_cast<size_t>(h) * D * D;
    const uint8_t *packs = scratch + pack_slot(sq, b, h, 0, first_row, H) * PK::bytes;  // chunks follow
    const bool ctl = warp == kEpiWarps && lane == 0;      // the chain thread
    const bool ctl2 = warp == kEpiWarps + 1 && lane == 0;  // the output thread

    auto copy_m = [&](const uint8_t *pk) {  // M's hi and lo halves into rows 64..127 of A2
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&bars[1])),
                     "r"(static_cast<uint32_t>(PK::AM))
                     : "memory");
        bulk_copy_nx(sA2 + 8192, pk + PK::OFF_AM, PK::AM / 2, &bars[1]);
        bulk_copy_nx(sA2 + kTileBytes + 8192, pk + PK::OFF_AM + PK::AM / 2, PK::AM / 2, &bars[1]);
    };
    // A1 ([W; Q o A], hi then lo) in k-parts of 64 channels: a part is one 64-channel atom column
    // of the hi half and of the lo half, so group 1 can start on part 0 while part 1 lands, and
    // part 0 of the next chunk can come in once the MMAs of part 0 have completed
    constexpr int kA1Parts = D / 64, kA1Part = PK::A1 / 2 / kA1Parts;
    auto copy_a1 = [&](const uint8_t *pk, int part) {  // part 0 completes on bars[0], part 1 on bars[11]
        uint64_t *bar = part ? &bars[11] : &bars[0];
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                     "r"(static_cast<uint32_t>(2 * kA1Part))
                     : "memory");
        bulk_copy_nx(sA1 + part * kA1Part, pk + PK::OFF_A1 + part * kA1Part, kA1Part, bar);
        bulk_copy_nx(sA1 + PK::A1 / 2 + part * kA1Part, pk + PK::OFF_A1 + PK::A1 / 2 + part * kA1Part, kA1Part, bar);
    };
    if (ctl) {
        for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
        mbar_init(&bars[8], kEpiWarps);  // one arrival per epilogue warp
        mbar_init(&bars[9], kEpiWarps);
        mbar_init(&bars[10], 1);
        mbar_init(&bars[11], 1);
        mbar_init(&bars[12], 1);
        *fail = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
    }
    // rows 0..63 of both halves of A2 stay zero: D1 += [0; M] U adds nothing to rows 0..63
    for (int e = tid; e < 2 * 8192 / 16; e += kStateThreads) {
        const int half = e / (8192 / 16), off = (e % (8192 / 16)) * 16;
        *reinterpret_cast<uint4 *>(sA2 + half * kTileBytes + off) = make_uint4(0u, 0u, 0u, 0u);
    }
    // Epilogue roles: for an M = 128 accumulator warp w reads TMEM lanes 32(w%4)..+31 (rows),
    // value columns [(w/4) HALF, + HALF). D3 with D = 64 (M = 64) has rows 16 (w%4) + lane, lane < 16.
    static_assert(DVS % (kEpiWarps / 4) == 0 && HALF % 8 == 0, "epilogue column groups");
    const int quad = warp & 3, colh = warp >> 2;
    const int erow = 32 * quad + lane;
    const int ccol = colh * HALF;
    const int srow = warp >= kEpiWarps ? -1 : ((D == 128) ? erow : ((lane < 16) ? 16 * quad + lane : -1));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tD3 = tmem + 2 * DVS;
    // the FP32 master state slice lives in TMEM: key row srow in this thread's own lane, value
    // columns [ccol, ccol + HALF) of the slice at tS (lanes of rows that do not exist hold zeros)
    const uint32_t tS = tmem_lane_base(tmem + 3 * DVS, warp) + ccol;
    if (warp < kEpiWarps) {
#pragma unroll
        for (int j = 0; j < HALF; j += 8) {
            float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (srow >= 0) {
                const float *src = Sg + static_cast<size_t>(srow) * D + c0 + ccol + j;
                const float4 a = *reinterpret_cast<const float4 *>(src), c = *reinterpret_cast<const float4 *>(src + 4);
                x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = c.x; x[5] = c.y; x[6] = c.z; x[7] = c.w;
                // S0 into B1 (MN-major: element (n = value column, k = key row)), 16-byte chunks
                st_pair(sB1, S::B1 / 2, mnmaj_off(ccol + j, srow, D), x);
            }
            tmem_st8(tS + j, x);
        }
        tmem_st_wait();
    }
    // the packs: written by the passes before this one (everything above reads none of them)
    pdl_acquire();
    if (ctl) {
        for (int part = 0; part < kA1Parts; ++part) copy_a1(packs, part);
        copy_m(packs);
        bulk_copy(sA3, packs + PK::OFF_A3, PK::A3, &bars[2]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    bool ok = true;

    if (warp >= kEpiWarps) {
        // ================================================= control warps (lane 0 of each works)
        // K-step-0 descriptors of every operand (the buffers never move)
        const uint64_t dA2h = kmaj_desc(smem_u32(sA2), 128, 0, 0), dA2l = kmaj_desc(smem_u32(sA2) + kTileBytes, 128, 0, 0);
        const uint64_t dB2h = mnmaj_desc(smem_u32(sB2), C, 0, 0), dB2l = mnmaj_desc(smem_u32(sB2) + S::B2 / 2, C, 0, 0);
        constexpr uint64_t kB2Buf = static_cast<uint64_t>(S::B2 >> 4);  // one U buffer, in descriptor units
        // the output group (D1 += [0; M] U) of chunk c: U from B2 buffer c % NU, M from A2
        auto issue_out_group = [&](int c) {
            constexpr uint32_t idm = idesc_bf16(128, DVS, false, true);
            const uint64_t ub = (c % S::NU) * kB2Buf;
            const uint32_t tD1c = tmem + (c & 1) * DVS;
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t bh = dB2h + ub + mnmaj_step(ks), bl = dB2l + ub + mnmaj_step(ks);
                const uint64_t mh = dA2h + kmaj_step(128, ks), ml = dA2l + kmaj_step(128, ks);
                mma_bf16(tD1c, mh, bh, idm, 1);
                mma_bf16(tD1c, mh, bl, idm, 1);
                mma_bf16(tD1c, ml, bh, idm, 1);
            }
            mma_commit(&bars[6]);
        };
        // copy barriers this thread issues on (A1 part 0, M, A3, A1 part 1): copies issued and
        // phases waited for (so that a timed-out thread can drain what is still in flight)
        constexpr int kCopyBar[4] = {0, 1, 2, 11};
        uint32_t issued[4] = {1, 1, 1, kA1Parts > 1 ? 1u : 0u}, waited[4] = {0, 0, 0, 0};
        auto wait_copy = [&](int k) {
            const bool r = mbar_wait(&bars[kCopyBar[k]], waited[k] & 1, kWaitCycles);
            if (r) ++waited[k];
            return r;
        };
        auto give_up = [&]() {
            ok = false;
            atomicExch(fail, 1);
        };
        if (ctl) {
            const uint64_t dA1h = kmaj_desc(smem_u32(sA1), 128, 0, 0), dA1l = kmaj_desc(smem_u32(sA1) + PK::A1 / 2, 128, 0, 0);
            const uint64_t dB1h = mnmaj_desc(smem_u32(sB1), D, 0, 0), dB1l = mnmaj_desc(smem_u32(sB1) + S::B1 / 2, D, 0, 0);
            const uint64_t dA3h = mnmaj_desc(smem_u32(sA3), C, 0, 0), dA3l = mnmaj_desc(smem_u32(sA3) + PK::A3 / 2, C, 0, 0);
            if (S::NU == 2) issued[1] = 0;  // the output thread owns the M copies
#pragma unroll 1
            for (int ch = 0; ch < nb && ok; ++ch) {
                const uint32_t par = ch & 1;
                const uint32_t tD1 = tmem + par * DVS;
                const uint8_t *cur = packs + static_cast<size_t>(ch) * PK::bytes;
                const uint8_t *next = cur + PK::bytes;
                const bool more = ch + 1 < nb;
                // S of this chunk is in B1 (the epilogue's previous round), A1 has landed
                if (ch > 0 && !mbar_wait(&bars[9], (ch - 1) & 1, kWaitCycles)) { give_up(); break; }
                {
                    constexpr uint32_t id = idesc_bf16(128, DVS, false, true);
                    bool got = true;
#pragma unroll
                    for (int part = 0; part < kA1Parts; ++part) {
                        if (!wait_copy(part ? 3 : 0)) { got = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const int ks = 4 * part + kk;
                            const uint64_t ah = dA1h + kmaj_step(128, ks), al = dA1l + kmaj_step(128, ks);
                            const uint64_t bh = dB1h + mnmaj_step(ks), bl = dB1l + mnmaj_step(ks);
                            mma_bf16(tD1, ah, bh, id, ks > 0 ? 1u : 0u);
                            mma_bf16(tD1, ah, bl, id, 1);
                            mma_bf16(tD1, al, bh, id, 1);
                        }
                        if (part + 1 < kA1Parts) mma_commit(&bars[12]);  // part 0 has been read
                    }
                    if (!got) { give_up(); break; }
                    mma_commit(&bars[4]);
                }
                if (S::NU == 1 && ch > 0) {  // the previous output group has read M: this chunk's M
                    if (!mbar_wait(&bars[6], (ch - 1) & 1, kWaitCycles)) { give_up(); break; }
                    copy_m(cur);
                    ++issued[1];
                }
                if (kA1Parts > 1 && more) {  // A1 part 0 is free again
                    if (!mbar_wait(&bars[12], par, kWaitCycles)) { give_up(); break; }
                    copy_a1(next, 0);
                    ++issued[0];
                }
                if (!mbar_wait(&bars[4], par, kWaitCycles)) { give_up(); break; }
                if (more) {  // the rest of A1 is free again
                    copy_a1(next, kA1Parts - 1);
                    ++issued[kA1Parts > 1 ? 3 : 0];
                }
                // U is in B2
                if (!mbar_wait(&bars[8], par, kWaitCycles)) { give_up(); break; }
                if (!wait_copy(2)) { give_up(); break; }
                tc_fence_after();
                {
                    constexpr uint32_t id3 = idesc_bf16(D, DVS, true, true);
                    const uint64_t ub = (ch % S::NU) * kB2Buf;
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks) {
                        const uint64_t bh = dB2h + ub + mnmaj_step(ks), bl = dB2l + ub + mnmaj_step(ks);
                        const uint64_t ah = dA3h + mnmaj_step(ks), al = dA3l + mnmaj_step(ks);
                        mma_bf16(tD3, ah, bh, id3, ks > 0 ? 1u : 0u);
                        mma_bf16(tD3, ah, bl, id3, 1);
                        mma_bf16(tD3, al, bh, id3, 1);
                    }
                    mma_commit(&bars[5]);
                }
                if (S::NU == 1) {  // one U buffer: the output group now, behind group 2
                    if (!wait_copy(1)) { give_up(); break; }
                    issue_out_group(ch);
                }
                if (more) {  // A3 is free once group 2 has completed
                    if (!mbar_wait(&bars[5], par, kWaitCycles)) { give_up(); break; }
                    bulk_copy(sA3, next + PK::OFF_A3, PK::A3, &bars[2]);
                    ++issued[2];
                }
            }
            if (!ok) {
                // drain (bounded): every MMA issued, then every copy still in flight
                mma_commit(&bars[7]);
                mbar_wait(&bars[7], 0, kWaitCycles);
                for (int k = 0; k < 4; ++k)
                    while (waited[k] < issued[k] && wait_copy(k)) {
                    }
            }
        } else if (ctl2 && S::NU == 2) {
            issued[0] = issued[2] = issued[3] = 0;  // the chain thread owns the A1 and A3 copies
#pragma unroll 1
            for (int ch = 0; ch < nb && ok; ++ch) {
                // group 2 of this chunk has completed: its output group runs while epilogue 2 does
                if (!mbar_wait(&bars[5], ch & 1, kWaitCycles)) { give_up(); break; }
                if (!wait_copy(1)) { give_up(); break; }
                tc_fence_after();
                issue_out_group(ch);
                if (ch + 1 < nb) {  // the output group has read M: the next chunk's M may come in
                    if (!mbar_wait(&bars[6], ch & 1, kWaitCycles)) { give_up(); break; }
                    copy_m(packs + static_cast<size_t>(ch + 1) * PK::bytes);
                    ++issued[1];
                }
            }
            if (!ok) {
                mma_commit(&bars[10]);
                mbar_wait(&bars[10], 0, kWaitCycles);
                while (waited[1] < issued[1] && wait_copy(1)) {
                }
            }
        }
    } else {
        // ================================================= epilogue warps
        // O = scale D1[64:128] of chunk c (quads 2 and 3: TMEM lanes 64..127 = the chunk's tokens),
        // once group 3 of chunk c has completed
        auto out_epilogue = [&](int c) {  // the caller has waited for the output group of chunk c
            tc_fence_after();
            const int i = erow - 64;
            int nn;
            size_t r0;
            seq_chunk(sq, b, c, r0, nn, nullptr);
            const uint32_t tD1c = tmem + (c & 1) * DVS;
#pragma unroll
            for (int j = 0; j < HALF; j += 8) {
                float x[8];
                tmem_ld8(tmem_lane_base(tD1c, warp) + ccol + j, x);
                tmem_ld_wait();
                if (i < nn && ok) {
                    float *dst = core + (r0 + i) * rs + static_cast<size_t>(h) * D + c0 + ccol + j;
                    *reinterpret_cast<float4 *>(dst) =
                        make_float4(scale * x[0], scale * x[1], scale * x[2], scale * x[3]);
                    *reinterpret_cast<float4 *>(dst + 4) =
                        make_float4(scale * x[4], scale * x[5], scale * x[6], scale * x[7]);
                }
            }
        };
#pragma unroll 1
        for (int ch = 0; ch < nb; ++ch) {
            const uint32_t par = ch & 1;
            const uint32_t tD1 = tmem + par * DVS;
            const uint8_t *cur = packs + static_cast<size_t>(ch) * PK::bytes;
            const float ac = srow >= 0 ? reinterpret_cast<const float *>(cur + PK::OFF_AC)[srow] : 0.f;
            auto ut_ptr = [&](int j) {  // U~ of this thread's row, value columns c0 + ccol + j ..
                const int c = c0 + ccol + j;
                return reinterpret_cast<const float *>(cur + PK::OFF_UT + (c >> 5) * PK::UG_BYTES) + erow * PK::UP +
                       (c & 31);
            };
            float ut[kPreU ? HALF : 1];
            if (kPreU && quad < 2) {
#pragma unroll
                for (int j = 0; j < (kPreU ? HALF : 0); j += 4) {
                    const float4 u4 = *reinterpret_cast<const float4 *>(ut_ptr(j));
                    ut[j] = u4.x; ut[j + 1] = u4.y; ut[j + 2] = u4.z; ut[j + 3] = u4.w;
                }
            }
            ok = ok && mbar_wait(&bars[4], par, kWaitCycles);
            tc_fence_after();
            // ---- epilogue 1: U = U~ - D1[0:64] -> B2 (MN-major: element (n = value column, k = token))
            if (quad < 2) {
                float4 un0 = make_float4(0.f, 0.f, 0.f, 0.f), un1 = un0;  // the next group of U~ (wide slices)
                if (!kPreU) {
                    un0 = *reinterpret_cast<const float4 *>(ut_ptr(0));
                    un1 = *reinterpret_cast<const float4 *>(ut_ptr(0) + 4);
                }
#pragma unroll
                for (int j = 0; j < HALF; j += 8) {
                    float x[8];
                    tmem_ld8(tmem_lane_base(tD1, warp) + ccol + j, x);
                    float u8[8];
                    if constexpr (kPreU) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) u8[u] = ut[j + u];
                    } else {
                        u8[0] = un0.x; u8[1] = un0.y; u8[2] = un0.z; u8[3] = un0.w;
                        u8[4] = un1.x; u8[5] = un1.y; u8[6] = un1.z; u8[7] = un1.w;
                        if (j + 8 < HALF) {
                            un0 = *reinterpret_cast<const float4 *>(ut_ptr(j + 8));
                            un1 = *reinterpret_cast<const float4 *>(ut_ptr(j + 8) + 4);
                        }
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 8; ++u) x[u] = u8[u] - x[u];
                    if (tables && ok) {  // verify mode: U of every row, for the fold
                        float *utab = tables + (static_cast<size_t>(b) * H + h) * 2 * C * D + erow * D + c0 + ccol + j;
                        *reinterpret_cast<float4 *>(utab) = make_float4(x[0], x[1], x[2], x[3]);
                        *reinterpret_cast<float4 *>(utab + 4) = make_float4(x[4], x[5], x[6], x[7]);
                    }
                    st_pair(sB2 + (ch % S::NU) * S::B2, S::B2 / 2, mnmaj_off(ccol + j, erow, C), x);
                }
            }
            // the previous chunk's output group has completed (waited for before this warp's arrival:
            // the next output group cannot complete before that arrival, so the phase is unambiguous)
            if (ch > 0 && quad >= 2) ok = ok && mbar_wait(&bars[6], (ch - 1) & 1, kWaitCycles);
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[8]);
            // the previous chunk's output rows, while group 2 runs
            if (ch > 0 && quad >= 2) out_epilogue(ch - 1);
            // ---- epilogue 2: S = A_C o S0 + D3 (the FP32 master copy in TMEM), S into B1
            ok = ok && mbar_wait(&bars[5], par, kWaitCycles);
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < HALF; j += 8) {
                float x[8], sv[8];
                tmem_ld8(tmem_lane_base(tD3, warp) + ccol + j, x);
                tmem_ld8(tS + j, sv);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 8; ++u) sv[u] = fmaf(ac, sv[u], x[u]);
                tmem_st8(tS + j, sv);
                if (srow >= 0) st_pair(sB1, S::B1 / 2, mnmaj_off(ccol + j, srow, D), sv);
            }
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[9]);
            if (!ok || *reinterpret_cast<volatile int *>(fail)) {
                ok = false;
                break;
            }
        }
        if (quad >= 2) ok = ok && mbar_wait(&bars[6], (nb - 1) & 1, kWaitCycles);
        if (ok && quad >= 2) out_epilogue(nb - 1);
    }
    ok = __syncthreads_and(ok && *reinterpret_cast<volatile int *>(fail) == 0) != 0;
    if (!ok) {
        if (tid == 0) atomicExch(status, KDA_ERR_TIMEOUT);
    } else if (warp < kEpiWarps && !tables) {  // verify mode leaves the state as it was
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < HALF; j += 8) {
            float sv[8];
            tmem_ld8(tS + j, sv);
            tmem_ld_wait();
            if (srow >= 0) {
                float *dst = Sg + static_cast<size_t>(srow) * D + c0 + ccol + j;
                *reinterpret_cast<float4 *>(dst) = make_float4(sv[0], sv[1], sv[2], sv[3]);
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(sv[4], sv[5], sv[6], sv[7]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, S::TMEM_COLS);
}

// Scratch layout: the operand packs, then a 256-byte slot with the count of chunks the
// tensor-core intra kernel handed to the CUDA-core body, then their (b, h, chunk) ids.
template <int D>
size_t packs_bytes(long long npacks) { return static_cast<size_t>(npacks) * Pack<D>::bytes; }

// Packs the call's layout holds: one per (stream, head, chunk slot), or H x slots (compact).
long long pack_count(int B, int H, const Seqs &sq) {
    return static_cast<long long>(H) * (sq.slots ? sq.slots : static_cast<long long>(B) * sq.nch);
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int D, int DVS, int MODE>
int launch_tc(const PrefillIn &in, float *const *h_state, float *core, int B, const Seqs &sq, int H, float scale,
              void *scratch, cudaStream_t s) {
    const int nch = sq.nch;
    int *status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    static std::atomic<unsigned long long> attr_intra{0}, attr_fix{0}, attr_state{0};
    KDA_TRY(smem_opt_in(intra_tc_kernel<D, MODE>, IntraTC<D>::bytes, attr_intra, true));
    KDA_TRY(smem_opt_in(intra_fix_kernel<D, MODE>, static_cast<int>(Intra<D>::bytes), attr_fix));
    KDA_TRY(smem_opt_in(state_kernel<D, DVS>, State<D, DVS>::bytes, attr_state));
    uint8_t *sc = static_cast<uint8_t *>(scratch);
    int *list = reinterpret_cast<int *>(sc + packs_bytes<D>(pack_count(B, H, sq)));
    if (cudaMemsetAsync(list, 0, sizeof(int), s) != cudaSuccess) return KDA_ERR_CUDA;
    const int sms = sm_count();
    const long long items = static_cast<long long>(B) * H * nch;
    if (items > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;  // item ids are int
    // two tensor-core intra CTAs per SM; the CUDA-core fix-up runs one per SM
    const int grid = static_cast<int>(std::min<long long>(items, 2LL * sms));
    const int grid_fix = static_cast<int>(std::min<long long>(items, sms));
    // row maps: (stream, row in stream) for equal-length streams; the packed rows in varlen mode
    const int mT = sq.cu ? sq.total : sq.T, mTp = sq.cu ? sq.total : sq.T_pad, mB = sq.cu ? 1 : B;
    InMaps maps;
    if (kGraw<MODE>)
        KDA_TRY(make_rows_map(&maps.g, in.g_raw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H * D, mT, mTp, mB, D, C));
    else
        KDA_TRY(make_rows_map(&maps.g, in.gate, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H * D, mT, mTp, mB, D, C));
    // packs that overflow half of L2 go out evict-first: they are read back only by the state
    // pass, and the inputs prefetched for the coming items need the room
    PrefillIn inp = in;
    inp.stream_pack = packs_bytes<D>(pack_count(B, H, sq)) > (size_t{64} << 20) ? 1 : 0;
    intra_tc_kernel<D, MODE><<<grid, kTcThreads, IntraTC<D>::bytes, s>>>(maps, inp, sc, list, B, sq, H, status);
    KDA_TRY(launch_status());
    // the fix-up and state passes launch programmatically: each waits in-kernel for its predecessor
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(kIntraThreads);
    cfg.gridDim = dim3(grid_fix);
    cfg.dynamicSmemBytes = Intra<D>::bytes;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, intra_fix_kernel<D, MODE>, in, sc, static_cast<const int *>(list), sq, H) != cudaSuccess)
        return KDA_ERR_CUDA;
    cfg.blockDim = dim3(kStateThreadsFor<DVS>);
    cfg.gridDim = dim3(D / DVS, H, B);
    cfg.dynamicSmemBytes = State<D, DVS>::bytes;
    if (cudaLaunchKernelEx(&cfg, state_kernel<D, DVS>, static_cast<const uint8_t *>(sc), h_state, core, sq, H, scale,
                           in.tables, status) != cudaSuccess)
        return KDA_ERR_CUDA;
    return launch_status();
}

// Value slice width. One state CTA fills an SM and walks its (stream, head)'s chunks in order,
// so the pass takes (waves of CTAs) x (chunks) x (one chunk's chain). Measured chains per chunk:
// about 4.9 K cycles with 32 value columns, 6 K with 64, 10 K with 128 (16 epilogue warps; the
// MMAs cost the same up to N = 64 and the epilogues grow with the columns). The width with the
// smallest waves x chain is taken: 32 columns while four slices per unit fit in one wave, 64
// while two do, 128 for one wave of whole heads beyond that.
template <int MODE>
int launch_any(const PrefillIn &in, float *const *h_state, float *core, int B, const Seqs &sq, const kda_dims *dims,
               void *scratch, cudaStream_t s) {
    const int H = dims->heads;
    const float sc = dims->scale;
    if (dims->head_dim == 64) return launch_tc<64, 32, MODE>(in, h_state, core, B, sq, H, sc, scratch, s);
    const long long units = static_cast<long long>(B) * H, sms = sm_count();
    auto cost = [&](long long slices, long long chain) { return (units * slices + sms - 1) / sms * chain; };
    const long long c32 = cost(4, 49), c64 = cost(2, 60), c128 = cost(1, 100);
    if (c32 <= c64 && c32 <= c128) return launch_tc<128, 32, MODE>(in, h_state, core, B, sq, H, sc, scratch, s);
    if (c64 <= c128) return launch_tc<128, 64, MODE>(in, h_state, core, B, sq, H, sc, scratch, s);
    return launch_tc<128, 128, MODE>(in, h_state, core, B, sq, H, sc, scratch, s);
}

Seqs equal_seqs(int T) {
    const int T_pad = static_cast<int>(kda_t_pad(static_cast<size_t>(T), C));
    return Seqs{nullptr, T, T_pad, T_pad / C, 0, 0};
}

size_t scratch_for_packs(long long npacks, int D) {
    const size_t packs = D == 64 ? packs_bytes<64>(npacks) : packs_bytes<128>(npacks);
    const size_t list = (4 + 4 * static_cast<size_t>(npacks) + 255) / 256 * 256;
    return packs + list;
}

// Packed streams: the compact layout when it takes fewer slots than one per (stream, chunk).
Seqs varlen_seqs(const int *cu, int B, int max_chunks, int total) {
    const long long rect = static_cast<long long>(B) * max_chunks;
    const long long compact = (static_cast<long long>(total) + C - 1) / C + B - 1;
    const int slots = compact < rect ? static_cast<int>(compact) : 0;
    return Seqs{cu, 0, 0, max_chunks, total, slots};
}

}  // namespace

size_t chunk_prefill_scratch_bytes(int B, int T, int H, int D) {
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    return chunk_prefill_slots_scratch_bytes(B, static_cast<int>(kda_t_pad(static_cast<size_t>(T), C) / C), H, D);
}

size_t chunk_prefill_slots_scratch_bytes(int B, int nch, int H, int D) {
    if (B <= 0 || nch <= 0 || H <= 0) return 0;
    return scratch_for_packs(static_cast<long long>(B) * H * nch, D);
}

size_t chunk_prefill_varlen_need_bytes(int B, int max_chunks, int total, int H, int D) {
    if (B <= 0 || max_chunks <= 0 || H <= 0) return 0;
    return scratch_for_packs(pack_count(B, H, varlen_seqs(nullptr, B, max_chunks, total)), D);
}

size_t chunk_prefill_packed_bytes(int max_seqs, int max_total, int H, int D) {
    if (max_seqs <= 0 || max_total <= 0 || H <= 0) return 0;
    return scratch_for_packs(static_cast<long long>(H) * ((static_cast<long long>(max_total) + C - 1) / C + max_seqs - 1),
                             D);
}

int chunk_prefill_tc(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                     float *const *h_state, float *core, int B, int T, const kda_dims *dims, void *scratch,
                     cudaStream_t s) {
    const PrefillIn in{q, k, v, gate, nullptr, nullptr, nullptr, nullptr, beta, nullptr};
    return launch_any<kInF32>(in, h_state, core, B, equal_seqs(T), dims, scratch, s);
}

int chunk_prefill_tc_varlen(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                            const int *cu_seqlens, int B, int max_chunks, int total, float *const *h_state,
                            float *core, const kda_dims *dims, void *scratch, cudaStream_t s) {
    const PrefillIn in{q, k, v, gate, nullptr, nullptr, nullptr, nullptr, beta, nullptr};
    return launch_any<kInF32>(in, h_state, core, B, varlen_seqs(cu_seqlens, B, max_chunks, total), dims, scratch, s);
}

int chunk_verify_tc(const float *q, const float *k, const float *v, const float *gate, const float *beta,
                    const int *cu_seqlens, int B, int total, float *const *h_state, float *core, float *tables,
                    const kda_dims *dims, void *scratch, cudaStream_t s) {
    const PrefillIn in{q, k, v, gate, nullptr, nullptr, nullptr, nullptr, beta, tables};
    return launch_any<kInF32>(in, h_state, core, B, varlen_seqs(cu_seqlens, B, 1, total), dims, scratch, s);
}

int chunk_prefill_tc_fused(const uint16_t *qkv, const uint16_t *g_raw, const float *dt_bias, const float *a_log,
                           const float *beta, float *const *h_state, float *core, int B, int T, const kda_dims *dims,
                           void *scratch, cudaStream_t s) {
    const PrefillIn in{nullptr, nullptr, nullptr, nullptr, qkv, g_raw, dt_bias, a_log, beta, nullptr};
    return launch_any<kInFused>(in, h_state, core, B, equal_seqs(T), dims, scratch, s);
}

int chunk_prefill_tc_fused_varlen(const uint16_t *qkv, const uint16_t *g_raw, const float *dt_bias, const float *a_log,
                                  const float *beta, const int *cu_seqlens, int B, int max_chunks, int total,
                                  float *const *h_state, float *core, const kda_dims *dims, void *scratch,
                                  cudaStream_t s) {
    const PrefillIn in{nullptr, nullptr, nullptr, nullptr, qkv, g_raw, dt_bias, a_log, beta, nullptr};
    return launch_any<kInFused>(in, h_state, core, B, varlen_seqs(cu_seqlens, B, max_chunks, total), dims, scratch,
                                s);
}

int chunk_verify_tc_fused(const uint16_t *qkv, const uint16_t *g_raw, const float *dt_bias, const float *a_log,
                          const float *beta, const int *cu_seqlens, int B, int total, float *const *h_state,
                          float *core, float *tables, const kda_dims *dims, void *scratch, cudaStream_t s) {
    const PrefillIn in{nullptr, nullptr, nullptr, nullptr, qkv, g_raw, dt_bias, a_log, beta, tables};
    return launch_any<kInFused>(in, h_state, core, B, varlen_seqs(cu_seqlens, B, 1, total), dims, scratch, s);
}

int chunk_prefill_tc_graw(const float *q, const float *k, const float *v, const uint16_t *g_raw,
                          const float *dt_bias, const float *a_log, const float *beta, float *const *h_state,
                          float *core, int B, int T, const kda_dims *dims, void *scratch, cudaStream_t s) {
    const PrefillIn in{q, k, v, nullptr, nullptr, g_raw, dt_bias, a_log, beta, nullptr};
    return launch_any<kInGraw>(in, h_state, core, B, equal_seqs(T), dims, scratch, s);
}

}  // namespace kda
