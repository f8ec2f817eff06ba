"""Tensor-parallel head sharding of the KDA block (Glm5NextLayer `mixer_all_reduce`).

Every stage of the block up to the gated RMSNorm is independent per head, so `world` ranks
each take H / world heads: the output channels of those heads in q/k/v, f_b, g_b, the conv
rows of their q, k and v channels, their dt_bias and a_log entries, their b_proj rows, and
the matching input columns of o_proj; f_a, g_a and o_norm are replicated. Each rank runs the
block on its heads (kda_block_prefill / kda_block_decode with o_proj = NULL, so the calls stop
at o_norm_out), multiplies by its o_proj slice into a [rows, hidden] partial, and the partials
are summed across ranks by one all-reduce (torch.distributed: NCCL over NVLink on GPUs, gloo on
CPU). By default the partial is the BF16 block output of this rank's heads and the all-reduce
runs on BF16, as the mixer all-reduce of the pages moves the block output (2 bytes per value);
reduce_dtype="fp32" keeps the partials in FP32 and rounds the sum once, as the unsharded o_proj
rounds its FP32 accumulation once, at twice the bytes on the links.

This module is plumbing around the C ABI: every step of the block runs in libkda's kernels.
"""
from __future__ import annotations

import dataclasses
import types

import kda_gated_delta_gate_b200 as kda

# weights whose output rows are the block's q|k|v / gate channels (sliced by head)
_ROWS = ("w_q", "w_k", "w_v", "f_b", "g_b", "dt_bias")


def head_range(H: int, rank: int, world: int) -> tuple[int, int]:
    """Heads [h0, h1) of `rank` when H heads are split evenly over `world` ranks."""
    if world < 1 or not 0 <= rank < world or H % world:
        raise ValueError(f"cannot split {H} heads over {world} ranks (rank {rank})")
    n = H // world
    return rank * n, (rank + 1) * n


def shard_block_weights(W, rank: int, world: int):
    """This rank's share of block weights W (fields w_q, w_k, w_v, conv_w, f_a, f_b, dt_bias,
    a_log, b_proj, g_a, g_b, o_norm, o_proj, H, D, hidden, rank; torch tensors on any device).
    Returns an object of the same kind with H = H / world and the sliced tensors."""
    h0, h1 = head_range(W.H, rank, world)
    D, qkv = W.D, W.H * W.D
    c0, c1 = h0 * D, h1 * D
    import torch
    fields = {n: getattr(W, n)[c0:c1].contiguous() for n in _ROWS}
    fields["conv_w"] = torch.cat([W.conv_w[c0:c1], W.conv_w[qkv + c0:qkv + c1], W.conv_w[2 * qkv + c0:2 * qkv + c1]])
    fields["a_log"] = W.a_log[h0:h1].contiguous()
    fields["b_proj"] = W.b_proj[h0:h1].contiguous()
    fields["o_proj"] = W.o_proj[:, c0:c1].contiguous()
    fields["H"] = h1 - h0
    if dataclasses.is_dataclass(W):
        return dataclasses.replace(W, **fields)
    out = types.SimpleNamespace(**vars(W))
    for k, v in fields.items():
        setattr(out, k, v)
    return out


class TPBlock:
    """One rank's share of the KDA block on the current CUDA device.

    shard: the output of shard_block_weights with device tensors. max_tokens sizes the
    workspace. group: a torch.distributed process group (None: the default group if
    torch.distributed is initialised, else no reduction: the caller sums the partials).
    reduce_dtype: "bf16" (the partials and the all-reduce in BF16) or "fp32"."""

    def __init__(self, shard, max_tokens: int, group=None, l2_eps: float = 1e-6, rms_eps: float = 1e-6,
                 scale: float = 1.0, reduce_dtype: str = "bf16"):
        import torch
        if reduce_dtype not in ("bf16", "fp32"):
            raise ValueError(f"reduce_dtype must be bf16 or fp32, not {reduce_dtype}")
        self.w = shard
        self.H, self.D, self.hidden = shard.H, shard.D, shard.hidden
        self.dw = types.SimpleNamespace(
            q_proj=shard.w_q, k_proj=shard.w_k, v_proj=shard.w_v, conv=shard.conv_w, f_a=shard.f_a, f_b=shard.f_b,
            dt_bias=shard.dt_bias, a_log=shard.a_log, b_proj=shard.b_proj, g_a=shard.g_a, g_b=shard.g_b,
            o_norm=shard.o_norm, o_proj=None, hidden=shard.hidden, rank=shard.rank)
        self.st = kda.block_weights_struct(self.dw)
        self.ws = kda.Workspace(kda.dims(self.H, self.D, scale=scale, l2_eps=l2_eps, rms_eps=rms_eps), shard.hidden,
                                shard.rank, max_tokens)
        dt = torch.bfloat16 if reduce_dtype == "bf16" else torch.float32
        self.partial = torch.empty((max_tokens, shard.hidden), dtype=dt, device=shard.w_q.device)
        self.group = group

    def _reduce(self, rows: int):
        import torch
        import torch.distributed as dist
        part = self.partial[:rows]
        kda.kda_gemm_bf16(self.ws.view("o_norm_out", (rows, self.H * self.D), torch.bfloat16), self.w.o_proj, part,
                          rows, self.hidden, self.H * self.D)
        if dist.is_available() and dist.is_initialized():
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)
        return part

    def prefill(self, hidden, T: int, h_state, conv_state, pad_fill: float = 0.0):
        """The block prefill of T rows on this rank's heads; returns the [T, hidden] output summed
        over the group (BF16; with reduce_dtype "fp32" the FP32 sum, to be rounded to BF16)."""
        kda.kda_block_prefill(self.st, hidden, T, h_state, conv_state, pad_fill, self.ws)
        return self._reduce(T)

    def decode(self, hidden, N: int, h_state_ptrs, conv_state_ptrs):
        """N sequences x 1 token on this rank's heads (kda_block_decode); [N, hidden] summed."""
        kda.kda_block_decode(self.st, hidden, N, h_state_ptrs, conv_state_ptrs, self.ws)
        return self._reduce(N)

    def close(self):
        self.ws.close()
