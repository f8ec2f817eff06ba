"""kda_chunk_prefill_noalloc: the prefill entry point for callers that cannot allocate device
memory (for example an engine whose memory pools already hold all free HBM). Through the C
ABI, two calls in a row must each reproduce kda_chunk_prefill's results on the same inputs,
within the prefill tolerance (relative L2 <= 1e-4); a request beyond the library's fixed
32 MiB scratch array is refused with KDA_ERR_CAPACITY before anything runs. This file is
collected last so that a failure here leaves every other test already run."""
import ctypes

import pytest
import torch

import kda_gated_delta_gate_b200 as kda
from synth import core_inputs, pad_rows, t_pad
from tests.gpu_harness import np64, rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _inputs(B, T, H, D, seed):
    ci = core_inputs(B, T, H, D, seed=seed, bf16_inputs=True, s0_std=0.1)
    Tp = t_pad(T)
    d = kda.dims(H, D)
    dev = "cuda"
    q, k, v = (pad_rows(x, Tp, 0.0).to(dev) for x in (ci.q, ci.k, ci.v))
    g_raw = pad_rows(ci.g_raw, Tp, 0.0).to(dev)
    gate = torch.empty((B * Tp, H, D), device=dev)
    kda.kda_gate(g_raw, ci.dt_bias.to(dev), ci.a_log.to(dev), gate, B * Tp, d)
    beta = pad_rows(ci.b_logit, Tp, 0.0).to(dev)
    kda.kda_beta(beta, beta, beta.numel())
    return ci, d, q, k, v, gate, beta


def _run(fn, ci, d, q, k, v, gate, beta):
    B, T, H, D = ci.B, ci.T, ci.H, ci.D
    states = [ci.s0[b].cuda().clone() for b in range(B)]
    core = torch.zeros((B * t_pad(T), H, D), device="cuda")
    fn(q, k, v, gate, beta, kda.ptr_array(states), core, B, T, d)
    torch.cuda.synchronize()
    return core.view(B, t_pad(T), H, D)[:, :T].clone(), torch.stack(states)


def test_noalloc_matches_scratch_entry_point_twice(cuda_ok):
    args = _inputs(2, 384, 16, 128, seed=21)  # 2 x 16 x 6 chunk packs of 149 KB: 27.9 MiB of scratch
    ref_core, ref_S = _run(kda.kda_chunk_prefill, *args)
    for _ in range(2):
        core, S = _run(kda.kda_chunk_prefill_noalloc, *args)
        assert rel_l2(np64(core), np64(ref_core)) <= TOL
        assert rel_l2(np64(S), np64(ref_S)) <= TOL
    assert kda.device_status() == 0


def test_noalloc_refuses_requests_beyond_its_array(cuda_ok):
    L = kda.lib()
    limit = L.kda_chunk_prefill_noalloc_max_scratch_bytes()
    assert limit == 32 << 20
    d = kda.dims(32, 128)
    assert kda.kda_chunk_prefill_scratch_bytes(1, 4096, d) > limit
    bogus = 0x10000  # never dereferenced: the size check comes first
    rc = L.kda_chunk_prefill_noalloc(*([bogus] * 7), 1, 4096, ctypes.byref(d), None)
    assert rc == 3  # KDA_ERR_CAPACITY
