"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI on seeded
inputs from `synth`, and run the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import pad_rows, t_pad


def rel_l2(got, ref) -> float:
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / (den if den > 0 else 1.0))


def worst_head_rel_l2(got, ref) -> float:
    """got/ref [..., H, D]: the worst relative L2 error over heads."""
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    H = r.shape[-2]
    g = np.moveaxis(g, -2, 0).reshape(H, -1)
    r = np.moveaxis(r, -2, 0).reshape(H, -1)
    return float(max(np.linalg.norm(g[h] - r[h]) / max(np.linalg.norm(r[h]), 1e-300) for h in range(H)))


def np64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def gpu_prefill(ci, *, impl="tc", pad_fill=0.0, scale=1.0, states=None, stream=None):
    """Gate + beta + chunked prefill on the GPU for synth.CoreInputs `ci` (padded buffers
    with every tail - q, k, v, gate, beta - set to pad_fill). Returns (core [B,T,H,D] f32
    of the valid rows, final states [B,H,D,D], device tensors dict)."""
    B, T, H, D = ci.B, ci.T, ci.H, ci.D
    Tp = t_pad(T)
    dev = "cuda"
    d = kda.dims(H, D, scale=scale)
    q = pad_rows(ci.q, Tp, pad_fill).to(dev)
    k = pad_rows(ci.k, Tp, pad_fill).to(dev)
    v = pad_rows(ci.v, Tp, pad_fill).to(dev)
    g_raw = pad_rows(ci.g_raw, Tp, 0.0).to(dev)
    gate = torch.empty((B * Tp, H, D), dtype=torch.float32, device=dev)
    kda.kda_gate(g_raw, ci.dt_bias.to(dev), ci.a_log.to(dev), gate, B * Tp, d, stream)
    beta = pad_rows(ci.b_logit, Tp, 0.0).to(dev)
    kda.kda_beta(beta, beta, beta.numel(), stream)
    gate.view(B, Tp, H, D)[:, T:] = pad_fill
    beta.view(B, Tp, H)[:, T:] = pad_fill
    if states is None:
        states = [ci.s0[b].to(dev).clone() for b in range(B)]
    ptrs = kda.ptr_array(states)
    core = torch.full((B * Tp, H, D), float("nan"), dtype=torch.float32, device=dev)
    kda.kda_chunk_prefill(q, k, v, gate, beta, ptrs, core, B, T, d, stream, impl=impl)
    torch.cuda.synchronize()
    return core.view(B, Tp, H, D)[:, :T], torch.stack(states), dict(gate=gate, beta=beta)


def oracle_prefill(ci, *, scale=1.0, s0=None, heads=None, seqs=None):
    """The oracle on the same inputs; optionally only some heads / sequences."""
    H, D = ci.H, ci.D
    sel_b = list(range(ci.B)) if seqs is None else list(seqs)
    sel_h = list(range(H)) if heads is None else list(heads)
    nb, nh, T = len(sel_b), len(sel_h), ci.T
    q = ci.q[sel_b][:, :, sel_h]
    k = ci.k[sel_b][:, :, sel_h]
    v = ci.v[sel_b][:, :, sel_h]
    g_raw = ci.g_raw[sel_b].reshape(nb, T, H, D)[:, :, sel_h].reshape(nb, T, nh * D).float()
    dt = ci.dt_bias.reshape(H, D)[sel_h].reshape(-1)
    g = oracle.gate(g_raw.cpu(), dt.cpu(), ci.a_log[sel_h].cpu(), nh, D)
    beta = oracle.sigmoid(ci.b_logit[sel_b][:, :, sel_h].cpu())
    S0 = (ci.s0 if s0 is None else s0)[sel_b][:, sel_h]
    return oracle.recurrence(q.cpu(), k.cpu(), v.cpu(), g, beta, S0.cpu(), scale)
