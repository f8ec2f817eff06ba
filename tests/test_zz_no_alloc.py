"""kda_chunk_prefill_noalloc: the prefill entry point for callers that cannot allocate device
memory (for example an engine whose memory pools already hold all free HBM, or a plug-in whose
host framework owns the device memory budget). Through the C ABI, two calls in a row must each
reproduce kda_chunk_prefill's results on the same inputs bit for bit (the same kernels on the
same inputs: any difference would be a scratch-reuse race between the calls); the second call
must leave the device's free memory exactly as it was (nothing allocated); a call with B = 0
reserves the array and runs nothing; a request beyond the library's fixed 32 MiB scratch array
is refused with KDA_ERR_CAPACITY before anything runs. This file is collected last so that a
failure here leaves every other test already run."""
import ctypes

import pytest
import torch

import kda_gated_delta_gate_b200 as kda
from synth import core_inputs, pad_rows, t_pad

pytestmark = pytest.mark.gpu


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


def _run(fn, ci, d, q, k, v, gate, beta, core, states):
    B, T = ci.B, ci.T
    for b in range(B):
        states[b].copy_(ci.s0[b])
    core.zero_()
    torch.cuda.synchronize()
    fn(q, k, v, gate, beta, kda.ptr_array(states), core, B, T, d)
    torch.cuda.synchronize()


def test_noalloc_matches_scratch_entry_point_twice(cuda_ok):
    args = _inputs(2, 384, 16, 128, seed=21)  # 2 x 16 x 6 chunk packs of 149 KB: 27.9 MiB of scratch
    ci = args[0]
    B, T, H, D = ci.B, ci.T, ci.H, ci.D
    states = [torch.empty((H, D, D), device="cuda") for _ in range(B)]
    core = torch.empty((B * t_pad(T), H, D), device="cuda")
    _run(kda.kda_chunk_prefill, *args, core, states)
    ref_core, ref_S = core.clone(), torch.stack(states).clone()
    free = []
    for _ in range(2):
        _run(kda.kda_chunk_prefill_noalloc, *args, core, states)
        free.append(torch.cuda.mem_get_info()[0])
        assert torch.equal(core, ref_core)
        assert torch.equal(torch.stack(states), ref_S)
    assert free[1] == free[0]  # the second call took no device memory
    assert kda.device_status() == 0


def test_noalloc_empty_call_reserves_and_runs_nothing(cuda_ok):
    L = kda.lib()
    d = kda.dims(16, 128)
    bogus = 0x10000  # never dereferenced: nothing runs for B = 0
    assert L.kda_chunk_prefill_noalloc(*([bogus] * 7), 0, 384, ctypes.byref(d), None) == 0
    torch.cuda.synchronize()
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
