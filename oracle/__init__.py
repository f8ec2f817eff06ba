"""KDA oracle: a plain, slow, FP64 CPU statement of what the KDA core and block compute.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs may import this package. The product (kda_gated_delta_gate_b200)
never imports it, and this package imports nothing from the product: the two share
no code. Both read their inputs from the seeded generators in `synth`.

Sources, cited by page title and section:
  * Glm5NextKdaWorkspace page: the stage buffers and their storage precision
    (qkv_parts / qkv_proj / conv_out / g_raw / out_gate / o_norm_out / final_out BF16;
    q_f32.. / gate / beta / core FP32), and where each stage rounds.
  * Glm5NextKdaLayer page: `decode` (conv fuses SiLU and L2; q/k reach the recurrence
    pre-normalised), `decode_k` (K rows of one sequence, snapshots after each row),
    `prefill` (chunked, from the carried state), `prefill_with_pad_fill` (pad tail).
  * Glm5NextKdaWeights page: [out, in] Linear weights, conv [conv_dim, conv_kernel],
    dt_bias per channel, a_log per head, o_norm [head_dim].
The gate is g = -exp(a_log[h]) * softplus(g_raw + dt_bias[c]) (bounded above by 0),
beta = sigmoid(b_proj(h)), and the core is the gated delta rule implemented in
kda_recurrence.c. All accumulation is FP64; BF16 rounding (round-to-nearest-even) is
applied exactly at the storage points the workspace page lists.

Where the pages leave a point open, the function that depends on it states the reading taken.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle_kda.so")
_SRC = os.path.join(_HERE, "kda_recurrence.c")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C part of the oracle (gcc, -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-o",
                               _LIB_PATH, _SRC, "-lm", "-lpthread"])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_recurrence.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] + [dp] * 7 + [ctypes.c_int]
        lib.oracle_recurrence.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # noqa: WPS433 (torch tensors only reach here from the harness)
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


# ----------------------------------------------------------------------------- numerics

def bf16_round(x) -> np.ndarray:
    """Round FP64 values to the nearest BF16 value (ties to even), returned as FP64.

    BF16 keeps 8 significant bits with FP32's exponent range: the quantum of a value
    in [2^(e-1), 2^e) is 2^(e-8), never finer than the subnormal quantum 2^-133.
    Values at or beyond the rounding boundary above the largest finite BF16 become inf.
    """
    x = _f64(x)
    m, e = np.frexp(x)
    qexp = np.maximum(e - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(x, -qexp)), qexp)
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = np.where(np.abs(r) > bf16_max, np.copysign(np.inf, x), r)
    return np.where(np.isfinite(x), r, x)


def softplus(x) -> np.ndarray:
    """log(1 + e^x) in the overflow-free form max(x, 0) + log1p(exp(-|x|))."""
    x = _f64(x)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x) -> np.ndarray:
    """1 / (1 + e^-x), evaluated without overflow on either side."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def silu(x) -> np.ndarray:
    x = _f64(x)
    return x * sigmoid(x)


def gate(g_raw, dt_bias, a_log, H: int, D: int) -> np.ndarray:
    """kda_gate: g[t, h, d] = -exp(a_log[h]) * softplus(g_raw[t, h*D+d] + dt_bias[h*D+d]).

    Glm5NextKdaWorkspace, field `gate` ([T_pad, heads, head_dim] FP32, the bounded
    log-decay) from field `g_raw` ([T, qkv] BF16); Glm5NextKdaWeights, fields `dt_bias`
    ([heads*head_dim] F32, per channel) and `a_log` ([heads] F32, per head).
    Returns shape [..., H, D] for g_raw of shape [..., H*D].
    """
    g_raw = _f64(g_raw)
    dt_bias = _f64(dt_bias).reshape(H * D)
    a_log = _f64(a_log).reshape(H)
    z = (g_raw + dt_bias).reshape(g_raw.shape[:-1] + (H, D))
    return -np.exp(a_log)[:, None] * softplus(z)


def recurrence(q, k, v, g, beta, s0, scale: float = 1.0, nthreads: int | None = None):
    """The KDA core over T valid tokens of B sequences (kda_recurrence.c).

    q, k, v, g: [B, T, H, D]; beta: [B, T, H]; s0: [B, H, D, D] (row = key channel).
    Returns (o [B, T, H, D], S_T [B, H, D, D]) in FP64. s0 is not modified.
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    S = _f64(s0).copy()
    B, T, H, D = q.shape
    assert k.shape == v.shape == g.shape == q.shape and beta.shape == (B, T, H)
    assert S.shape == (B, H, D, D)
    o = np.zeros((B, T, H, D), dtype=np.float64)
    rc = _load().oracle_recurrence(B, T, H, D, float(scale), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                   _ptr(beta), _ptr(S), _ptr(o), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_recurrence: bad arguments")
    return o, S


def linear(x, w) -> np.ndarray:
    """Torch Linear without bias: x @ w^T in FP64 (Glm5NextKdaWeights: [out, in])."""
    return _f64(x) @ _f64(w).T


def causal_conv_silu(x, conv_state, conv_w):
    """Depthwise causal conv (kernel 4) from the carried conv state, then SiLU.

    x: [T, C] (qkv_proj rows); conv_state: [C, 3], columns oldest -> newest;
    conv_w: [C, 4], tap 3 multiplies the current token. Returns (y [T, C] FP64 after SiLU,
    new_state [C, 3] = the last three inputs of (state || x)).
    """
    x = _f64(x)
    st = _f64(conv_state)
    w = _f64(conv_w)
    T, C = x.shape
    xx = np.concatenate([st.T, x], axis=0)  # [3 + T, C]
    y = np.zeros((T, C), dtype=np.float64)
    for j in range(4):
        y += w[:, j][None, :] * xx[j:j + T, :]
    new_state = xx[T:T + 3, :].T.copy()
    return silu(y), new_state


def _l2_heads(x, H: int, D: int, eps: float):
    xs = x.reshape(x.shape[:-1] + (H, D))
    n = np.sqrt(np.sum(xs * xs, axis=-1, keepdims=True) + eps)
    return (xs / n).reshape(x.shape)


def front_prefill(x, conv_state, conv_w, H: int, D: int, l2_eps: float = 1e-6):
    """Prefill front end: conv + SiLU -> BF16 conv_out, then l2_norm_bf16 in place on q|k.

    Glm5NextKdaWorkspace, field `conv_out`: [T, conv_dim] BF16 after conv + SiLU, with
    q|k L2-normalised by l2_norm_bf16 in place on prefill (so q/k are rounded twice).
    Returns (conv_out [T, 3*H*D] on the BF16 grid, new conv state [3*H*D, 3]).
    """
    qkv = H * D
    y, new_state = causal_conv_silu(x, conv_state, conv_w)
    c = bf16_round(y)
    c[:, :qkv] = bf16_round(_l2_heads(c[:, :qkv], H, D, l2_eps))
    c[:, qkv:2 * qkv] = bf16_round(_l2_heads(c[:, qkv:2 * qkv], H, D, l2_eps))
    return c, new_state


def front_decode_row(x_row, conv_state, conv_w, H: int, D: int, l2_eps: float = 1e-6):
    """Decode front end: the conv kernel fuses SiLU and L2 before its single BF16 write.

    Glm5NextKdaLayer, `decode`; Glm5NextKdaWorkspace, field `conv_out`.
    Returns (conv_out row [3*H*D] on the BF16 grid, new conv state [3*H*D, 3]).
    """
    qkv = H * D
    y, new_state = causal_conv_silu(_f64(x_row).reshape(1, -1), conv_state, conv_w)
    y = y[0]
    out = np.empty_like(y)
    out[:qkv] = bf16_round(_l2_heads(y[:qkv], H, D, l2_eps))
    out[qkv:2 * qkv] = bf16_round(_l2_heads(y[qkv:2 * qkv], H, D, l2_eps))
    out[2 * qkv:] = bf16_round(y[2 * qkv:])
    return out, new_state


def gated_rmsnorm(core, out_gate, w, eps: float = 1e-6) -> np.ndarray:
    """o_norm: per head, core / sqrt(mean_d core^2 + eps) * w[d] * sigmoid(out_gate) -> BF16.

    Glm5NextKdaWorkspace, field `o_norm_out` (after the sigmoid-gated RMSNorm);
    Glm5NextKdaWeights, field `o_norm` ([head_dim] BF16).
    core: [T, H, D]; out_gate: [T, H*D]. Returns [T, H*D] on the BF16 grid.
    """
    core = _f64(core)
    T, H, D = core.shape
    r = core / np.sqrt(np.mean(core * core, axis=-1, keepdims=True) + eps)
    y = r * _f64(w).reshape(1, 1, D) * sigmoid(_f64(out_gate).reshape(T, H, D))
    return bf16_round(y.reshape(T, H * D))


def block_prefill(W, hidden, h_state, conv_state, *, scale: float = 1.0, l2_eps: float = 1e-6,
                  rms_eps: float = 1e-6, nthreads: int | None = None) -> dict:
    """One KDA block prefill over T tokens of one sequence, stage by stage, in page order.

    Glm5NextKdaLayer `prefill`; stage buffers from Glm5NextKdaWorkspace. W is a
    synth.BlockWeights; hidden [T, hidden]; h_state [H, D, D]; conv_state [3*H*D, 3].
    Every stage's result is returned so each can be compared on its own.
    """
    H, D = W.H, W.D
    h = _f64(hidden)
    T = h.shape[0]
    q = bf16_round(linear(h, W.w_q))
    k = bf16_round(linear(h, W.w_k))
    v = bf16_round(linear(h, W.w_v))
    qkv_proj = np.concatenate([q, k, v], axis=1)
    conv_out, new_conv = front_prefill(qkv_proj, conv_state, W.conv_w, H, D, l2_eps)
    qkv = H * D
    qf = conv_out[:, :qkv].reshape(1, T, H, D)
    kf = conv_out[:, qkv:2 * qkv].reshape(1, T, H, D)
    vf = conv_out[:, 2 * qkv:].reshape(1, T, H, D)
    f_a = bf16_round(linear(h, W.f_a))
    g_raw = bf16_round(linear(f_a, W.f_b))
    g = gate(g_raw, W.dt_bias, W.a_log, H, D).reshape(1, T, H, D)
    b_logit = linear(h, W.b_proj)
    beta = sigmoid(b_logit).reshape(1, T, H)
    core, S = recurrence(qf, kf, vf, g, beta, _f64(h_state)[None], scale, nthreads)
    g_a = bf16_round(linear(h, W.g_a))
    out_gate = bf16_round(linear(g_a, W.g_b))
    o_norm_out = gated_rmsnorm(core[0], out_gate, W.o_norm, rms_eps)
    final_out = bf16_round(linear(o_norm_out, W.o_proj))
    return dict(qkv_proj=qkv_proj, conv_out=conv_out, g_raw=g_raw, gate=g[0], b_logit=b_logit,
                beta=beta[0], core=core[0], out_gate=out_gate, o_norm_out=o_norm_out,
                final_out=final_out, h_state=S[0], conv_state=new_conv)


def decode_rows(x_rows, conv_state, conv_w, g_raw, dt_bias, a_log, b_logit, out_gate, o_norm_w,
                h_state, H: int, D: int, *, scale: float = 1.0, l2_eps: float = 1e-6,
                rms_eps: float = 1e-6) -> dict:
    """K rows of ONE sequence, one token at a time, exactly as K serial decodes would do.

    Glm5NextKdaLayer `decode` / `decode_k`: conv (+SiLU+L2) -> gate -> beta -> one
    recurrence step -> o_norm, state carried row to row; snapshot[t] is the state
    (recurrent, conv) AFTER row t.
    x_rows [K, 3*H*D]; g_raw, out_gate [K, H*D]; b_logit [K, H]; h_state [H, D, D].
    """
    x_rows, g_raw, b_logit, out_gate = (_f64(a) for a in (x_rows, g_raw, b_logit, out_gate))
    K = x_rows.shape[0]
    qkv = H * D
    cs = _f64(conv_state)
    S = _f64(h_state)[None].copy()
    conv_out = np.zeros((K, 3 * qkv))
    core = np.zeros((K, H, D))
    onorm = np.zeros((K, qkv))
    snaps = []
    for t in range(K):
        row, cs = front_decode_row(x_rows[t], cs, conv_w, H, D, l2_eps)
        conv_out[t] = row
        q = row[:qkv].reshape(1, 1, H, D)
        k = row[qkv:2 * qkv].reshape(1, 1, H, D)
        v = row[2 * qkv:].reshape(1, 1, H, D)
        g = gate(g_raw[t], dt_bias, a_log, H, D).reshape(1, 1, H, D)
        beta = sigmoid(b_logit[t]).reshape(1, 1, H)
        o, S = recurrence(q, k, v, g, beta, S, scale, 1)
        core[t] = o[0, 0]
        onorm[t] = gated_rmsnorm(o[0], out_gate[t:t + 1], o_norm_w, rms_eps)[0]
        snaps.append((S[0].copy(), cs.copy()))
    return dict(conv_out=conv_out, core=core, o_norm_out=onorm, h_state=S[0], conv_state=cs,
                snapshots=snaps)


def block_decode(W, hidden_rows, h_state, conv_state, *, scale: float = 1.0, l2_eps: float = 1e-6,
                 rms_eps: float = 1e-6) -> dict:
    """K rows of ONE sequence through the whole block, one token at a time.

    Glm5NextKdaLayer `decode` / `decode_k` with the block's projections: every row's
    q/k/v, f_b(f_a(h)), b_proj(h) and g_b(g_a(h)) (BF16 outputs, FP32 beta logits, as on
    prefill), then decode_rows' stateful row (conv + SiLU + L2, gate, beta, recurrence,
    o_norm), then o_proj -> BF16. hidden_rows [K, hidden]; h_state [H, D, D];
    conv_state [3*H*D, 3]. Returns decode_rows' dict plus the projection stages and final_out.
    """
    H, D = W.H, W.D
    h = _f64(hidden_rows)
    x_rows = np.concatenate([bf16_round(linear(h, W.w_q)), bf16_round(linear(h, W.w_k)),
                             bf16_round(linear(h, W.w_v))], axis=1)
    g_raw = bf16_round(linear(bf16_round(linear(h, W.f_a)), W.f_b))
    b_logit = linear(h, W.b_proj)
    out_gate = bf16_round(linear(bf16_round(linear(h, W.g_a)), W.g_b))
    r = decode_rows(x_rows, conv_state, W.conv_w, g_raw, W.dt_bias, W.a_log, b_logit, out_gate, W.o_norm,
                    h_state, H, D, scale=scale, l2_eps=l2_eps, rms_eps=rms_eps)
    r.update(qkv_proj=x_rows, g_raw=g_raw, b_logit=b_logit, out_gate=out_gate,
             final_out=bf16_round(linear(r["o_norm_out"], W.o_proj)))
    return r
