"""GPU parity of the chunked prefill (kda_gate + kda_beta + kda_chunk_prefill) with the FP64
oracle, through the C ABI. Tolerance: relative L2 <= 1e-4 on the valid core rows and on the
final state (FP32 paths), over the whole tensor and per head."""
import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import core_inputs, t_pad
from tests.gpu_harness import gpu_prefill, np64, oracle_prefill, rel_l2, worst_head_rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-4
IMPLS = ["tc", "simt"]


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


def _check(ci, core, S, scale=1.0):
    o_ref, S_ref = oracle_prefill(ci, scale=scale)
    c = np64(core)
    s = np64(S)
    assert np.all(np.isfinite(c)) and np.all(np.isfinite(s))
    e_o, e_s = rel_l2(c, o_ref), rel_l2(s, S_ref)
    e_oh = worst_head_rel_l2(c, o_ref)
    e_sh = worst_head_rel_l2(np.swapaxes(s, 1, 2), np.swapaxes(S_ref, 1, 2))
    assert e_o <= TOL and e_s <= TOL and e_oh <= TOL and e_sh <= TOL, (e_o, e_s, e_oh, e_sh)
    return e_o, e_s


def test_gate_and_beta_match_oracle():
    ci = core_inputs(1, 300, 32, 128, seed=1)
    d = kda.dims(32, 128)
    g_raw = ci.g_raw[0].cuda()
    gate = torch.empty((300, 32, 128), device="cuda")
    kda.kda_gate(g_raw, ci.dt_bias.cuda(), ci.a_log.cuda(), gate, 300, d)
    ref = oracle.gate(ci.g_raw[0].float(), ci.dt_bias, ci.a_log, 32, 128)
    got = np64(gate)
    assert np.all(got <= 0)
    np.testing.assert_allclose(got, ref, rtol=2e-6, atol=1e-30)
    b = ci.b_logit[0].cuda().reshape(-1)
    beta = torch.empty_like(b)
    kda.kda_beta(b, beta, b.numel())
    np.testing.assert_allclose(np64(beta), oracle.sigmoid(ci.b_logit[0].reshape(-1)), rtol=1e-6)


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_small_config(impl):
    """B=1, T=64, H=2, D=64, zero initial state, FP32 inputs (the CPU-checkable workload)."""
    ci = core_inputs(1, 64, 2, 64, seed=0)
    core, S, _ = gpu_prefill(ci, impl=impl)
    _check(ci, core, S)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("B,T,H,D", [(2, 150, 3, 128), (3, 1, 2, 64), (1, 64, 4, 128), (2, 257, 2, 64),
                                     (1, 129, 1, 128)])
def test_prefill_ragged_and_edges(impl, B, T, H, D):
    ci = core_inputs(B, T, H, D, seed=7 + T, s0_std=0.1)
    core, S, _ = gpu_prefill(ci, impl=impl, scale=0.5)
    _check(ci, core, S, scale=0.5)


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_4096_tokens_32_heads(impl):
    """B=1, T=4096, H=32, D=128, BF16-exact inputs, initial state N(0, 0.1): the full prefill workload."""
    ci = core_inputs(1, 4096, 32, 128, seed=1, bf16_inputs=True, s0_std=0.1)
    core, S, _ = gpu_prefill(ci, impl=impl)
    _check(ci, core, S)


@pytest.mark.parametrize("impl", IMPLS)
def test_split_prefill_equals_whole(impl):
    """prefill(1536) then prefill(2560) from the carried state == the oracle over 4096 tokens."""
    ci = core_inputs(1, 4096, 32, 128, seed=1, bf16_inputs=True, s0_std=0.1)
    from synth.inputs import CoreInputs

    def part(a, b_):
        return CoreInputs(1, b_ - a, 32, 128, ci.q[:, a:b_], ci.k[:, a:b_], ci.v[:, a:b_], ci.g_raw[:, a:b_],
                          ci.dt_bias, ci.a_log, ci.b_logit[:, a:b_], ci.s0)

    states = [ci.s0[0].cuda().clone()]
    c1, _, _ = gpu_prefill(part(0, 1536), impl=impl, states=states)
    c2, S, _ = gpu_prefill(part(1536, 4096), impl=impl, states=states)
    _check(ci, torch.cat([c1, c2], dim=1), S)


@pytest.mark.parametrize("impl", IMPLS)
def test_poison_pad_tail(impl):
    """Rows >= T hold NaN, 1e30 or 0 in q, k, v, gate and beta: the final state and the valid
    outputs are bit-identical across the three, and match the oracle."""
    ci = core_inputs(2, 100, 4, 128, seed=4, s0_std=0.1)
    outs = [gpu_prefill(ci, impl=impl, pad_fill=f) for f in (0.0, float("nan"), 1e30)]
    for core, S, _ in outs[1:]:
        assert torch.equal(S, outs[0][1])
        assert torch.equal(core, outs[0][0])
    _check(ci, outs[1][0], outs[1][1])


@pytest.mark.parametrize("D", [128, 64])
def test_prefill_extreme_decay_takes_exact_path(D):
    """One head with a decay of hundreds of nats per token in some channels (beyond what the
    tensor-core intra path accepts inside a 16-token block): those chunks are recomputed by the
    exact CUDA-core path; all heads still match the oracle."""
    ci = core_inputs(1, 200, 3, D, seed=31, s0_std=0.1)
    ci.a_log[1] = 3.0                      # exp(3) = 20 on head 1
    ci.dt_bias[1 * D + 5] = 20.0           # softplus ~ 20: g ~ -400 per token on one channel
    ci.dt_bias[1 * D + 9] = 6.0
    for impl in IMPLS:
        core, S, _ = gpu_prefill(ci, impl=impl)
        _check(ci, core, S)


def test_tc_and_simt_agree():
    ci = core_inputs(2, 333, 4, 128, seed=12, s0_std=0.1)
    a, Sa, _ = gpu_prefill(ci, impl="tc")
    b, Sb, _ = gpu_prefill(ci, impl="simt")
    assert rel_l2(np64(a), np64(b)) <= TOL and rel_l2(np64(Sa), np64(Sb)) <= TOL


@pytest.mark.parametrize("impl", ["tc"])
def test_long_prefill_poison_full_size(impl):
    """B=4 streams of T=65500 (T_pad 65536), H=32, D=128, pad_fill NaN vs 0: full final states
    bit-identical; sampled (stream, head) pairs within tolerance of the oracle."""
    B, T, H, D = 4, 65500, 32, 128
    ci = core_inputs(B, T, H, D, seed=4, bf16_inputs=True, s0_std=0.1, device="cuda")
    core_n, S_n, _ = gpu_prefill(ci, impl=impl, pad_fill=float("nan"))
    core_n = core_n.clone()
    core_0, S_0, _ = gpu_prefill(ci, impl=impl, pad_fill=0.0)
    assert torch.equal(S_n, S_0)
    assert torch.equal(core_n, core_0)
    for b, h in [(0, 0), (1, 17), (2, 31), (3, 5)]:
        o_ref, S_ref = oracle_prefill(ci, seqs=[b], heads=[h])
        got_o = np64(core_n[b, :, h])
        got_s = np64(S_n[b, h])
        assert rel_l2(got_o, o_ref[0, :, 0]) <= TOL
        assert rel_l2(got_s, S_ref[0, 0]) <= TOL
    del core_n, core_0
    torch.cuda.empty_cache()
