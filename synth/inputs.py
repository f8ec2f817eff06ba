"""Seeded synthetic workloads for the KDA core and block.

Shapes and layouts follow the Glm5NextKdaWorkspace page (token-major activations,
[T, heads, head_dim]; prefill buffers padded to whole 64-token chunks) and the
Glm5NextKdaWeights page (torch Linear [out, in] BF16 weights, per-channel F32
dt_bias, per-head F32 a_log, conv weight [conv_dim, conv_kernel]).

Distributions (one torch.Generator per call, seeded; draws in a fixed order):
  q, k   N(0,1) FP32, then scaled to unit length per (token, head): this is the
         "L2-normalised" input distribution of the core-only workloads (points on
         the unit sphere), not the front end's l2 step.
  v      N(0,1);  g_raw N(0,1) rounded to BF16;  b_logit N(0,1) FP32.
  dt_bias U(-1,1) per channel;  a_log U(-1,1) per head;  initial state N(0, s0_std).
  Block weights N(0, 0.02) BF16; hidden states N(0,1) BF16.
Optionally q/k/v are rounded to BF16 and widened back to FP32 ("BF16 widened to FP32").

Nothing here computes the method: no gate, sigmoid, recurrence, convolution or norm.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


def t_pad(T: int, chunk: int = 64) -> int:
    """Rows a prefill buffer holds for T tokens: T rounded up to whole chunks."""
    return ((T + chunk - 1) // chunk) * chunk


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, device, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x * std if std != 1.0 else x


def _uniform(shape, gen, device, lo=-1.0, hi=1.0):
    x = torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    return x * (hi - lo) + lo


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return (x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)).contiguous()


def _bf16_exact(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16).to(torch.float32)


@dataclass
class CoreInputs:
    """Inputs of the KDA core for B sequences of T tokens (unpadded)."""
    B: int
    T: int
    H: int
    D: int
    q: torch.Tensor        # [B, T, H, D] f32
    k: torch.Tensor        # [B, T, H, D] f32
    v: torch.Tensor        # [B, T, H, D] f32
    g_raw: torch.Tensor    # [B, T, H*D] bf16
    dt_bias: torch.Tensor  # [H*D] f32
    a_log: torch.Tensor    # [H] f32
    b_logit: torch.Tensor  # [B, T, H] f32
    s0: torch.Tensor       # [B, H, D, D] f32 (row = key channel, column = value channel)


def core_inputs(B: int, T: int, H: int, D: int, seed: int, *, bf16_inputs: bool = False,
                s0_std: float = 0.0, device="cpu") -> CoreInputs:
    gen = _gen(seed, device)
    q = _unit_rows(_randn((B, T, H, D), gen, device))
    k = _unit_rows(_randn((B, T, H, D), gen, device))
    v = _randn((B, T, H, D), gen, device)
    g_raw = _randn((B, T, H * D), gen, device).to(torch.bfloat16)
    dt_bias = _uniform((H * D,), gen, device)
    a_log = _uniform((H,), gen, device)
    b_logit = _randn((B, T, H), gen, device)
    if s0_std > 0:
        s0 = _randn((B, H, D, D), gen, device, std=s0_std)
    else:
        s0 = torch.zeros((B, H, D, D), dtype=torch.float32, device=device)
    if bf16_inputs:
        q, k, v = _bf16_exact(q), _bf16_exact(k), _bf16_exact(v)
    return CoreInputs(B, T, H, D, q, k, v, g_raw, dt_bias, a_log, b_logit, s0)


def pad_rows(x: torch.Tensor, T_pad: int, fill: float) -> torch.Tensor:
    """[B, T, ...] -> [B*T_pad, ...]: each sequence's rows back to back, tail rows = fill."""
    B, T = x.shape[0], x.shape[1]
    out = torch.full((B, T_pad) + tuple(x.shape[2:]), float(fill), dtype=x.dtype, device=x.device)
    out[:, :T] = x
    return out.reshape((B * T_pad,) + tuple(x.shape[2:])).contiguous()


@dataclass
class BlockWeights:
    """One KDA block's weights, torch Linear layout [out, in]."""
    hidden: int
    H: int
    D: int
    rank: int
    w_q: torch.Tensor      # [H*D, hidden] bf16
    w_k: torch.Tensor
    w_v: torch.Tensor
    conv_w: torch.Tensor   # [3*H*D, 4] bf16
    f_a: torch.Tensor      # [rank, hidden] bf16
    f_b: torch.Tensor      # [H*D, rank] bf16
    dt_bias: torch.Tensor  # [H*D] f32
    a_log: torch.Tensor    # [H] f32
    b_proj: torch.Tensor   # [H, hidden] bf16
    g_a: torch.Tensor      # [rank, hidden] bf16
    g_b: torch.Tensor      # [H*D, rank] bf16
    o_norm: torch.Tensor   # [D] bf16
    o_proj: torch.Tensor   # [hidden, H*D] bf16


def block_weights(hidden: int, H: int, D: int, rank: int, seed: int, *, std: float = 0.02,
                  device="cpu") -> BlockWeights:
    gen = _gen(seed, device)
    qkv = H * D

    def w(shape):
        return _randn(shape, gen, device, std=std).to(torch.bfloat16)

    w_q, w_k, w_v = w((qkv, hidden)), w((qkv, hidden)), w((qkv, hidden))
    conv_w = w((3 * qkv, 4))
    f_a, f_b = w((rank, hidden)), w((qkv, rank))
    dt_bias = _uniform((qkv,), gen, device)
    a_log = _uniform((H,), gen, device)
    b_proj = w((H, hidden))
    g_a, g_b = w((rank, hidden)), w((qkv, rank))
    o_norm = w((D,))
    o_proj = w((hidden, qkv))
    return BlockWeights(hidden, H, D, rank, w_q, w_k, w_v, conv_w, f_a, f_b, dt_bias, a_log,
                        b_proj, g_a, g_b, o_norm, o_proj)


def block_hidden(T: int, hidden: int, seed: int, device="cpu") -> torch.Tensor:
    gen = _gen(seed + 1000, device)
    return _randn((T, hidden), gen, device).to(torch.bfloat16)


@dataclass
class DecodeInputs:
    """Rows of the stateful decode: N sequences x K rows each (row-major, sequence-major)."""
    N: int
    K: int
    H: int
    D: int
    x: torch.Tensor           # [N*K, 3*H*D] bf16: q|k|v projection rows before the conv
    conv_state: torch.Tensor  # [N, 3*H*D, 3] bf16, columns oldest -> newest
    conv_w: torch.Tensor      # [3*H*D, 4] bf16
    g_raw: torch.Tensor       # [N*K, H*D] bf16
    dt_bias: torch.Tensor     # [H*D] f32
    a_log: torch.Tensor       # [H] f32
    b_logit: torch.Tensor     # [N*K, H] f32
    out_gate: torch.Tensor    # [N*K, H*D] bf16
    o_norm: torch.Tensor      # [D] bf16
    s0: torch.Tensor          # [N, H, D, D] f32


def decode_inputs(N: int, H: int, D: int, seed: int, *, K: int = 1, s0_std: float = 0.1,
                  conv_std: float = 0.5, device="cpu") -> DecodeInputs:
    gen = _gen(seed, device)
    cd = 3 * H * D
    x = _randn((N * K, cd), gen, device).to(torch.bfloat16)
    conv_state = _randn((N, cd, 3), gen, device).to(torch.bfloat16)
    conv_w = _randn((cd, 4), gen, device, std=conv_std).to(torch.bfloat16)
    g_raw = _randn((N * K, H * D), gen, device).to(torch.bfloat16)
    dt_bias = _uniform((H * D,), gen, device)
    a_log = _uniform((H,), gen, device)
    b_logit = _randn((N * K, H), gen, device)
    out_gate = _randn((N * K, H * D), gen, device).to(torch.bfloat16)
    o_norm = (1.0 + _randn((D,), gen, device, std=0.1)).to(torch.bfloat16)
    s0 = _randn((N, H, D, D), gen, device, std=s0_std)
    return DecodeInputs(N, K, H, D, x, conv_state, conv_w, g_raw, dt_bias, a_log, b_logit,
                        out_gate, o_norm, s0)
