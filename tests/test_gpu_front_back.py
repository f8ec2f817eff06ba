"""GPU parity of the prefill front end (conv + SiLU + q|k L2 + widen/pad) and the back end
(sigmoid-gated RMSNorm) with the oracle. BF16 outputs: relative L2 <= 2e-2 and every element
within one BF16 step of the oracle's value per rounding site on its path (the two sides
round FP32 vs FP64 values, and a value near a rounding boundary may go either way; q|k
pass two sites on prefill); the carried conv state is exact."""
import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import decode_inputs, t_pad
from tests.gpu_harness import np64, rel_l2

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


def _within_bf16_steps(got, ref, steps=1, frac=0.01):
    """Every element within `steps` BF16 steps of the oracle (one step is at most 2^-7 of the
    value), and at most `frac` of the elements differ at all."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = np.abs(got - ref)
    assert np.all(diff <= steps * 2.0 ** -7 * np.abs(ref) + 1e-30), float(np.max(diff / (np.abs(ref) + 1e-30)))
    assert np.mean(diff > 0) <= frac


def _front(x, cs, w, T, H, D, pad_fill):
    qkv = H * D
    Tp = t_pad(T)
    conv_out = torch.empty((T, 3 * qkv), dtype=torch.bfloat16, device="cuda")
    f = [torch.empty((Tp, qkv), device="cuda") for _ in range(3)]
    kda.kda_front_conv_silu_l2(x, cs, w, conv_out, f[0], f[1], f[2], pad_fill, T, kda.dims(H, D))
    return conv_out, f


@pytest.mark.parametrize("T,H,D", [(200, 2, 64), (300, 32, 128), (2, 3, 128), (64, 1, 64)])
def test_front_prefill_matches_oracle(T, H, D):
    di = decode_inputs(1, H, D, seed=T, K=T)
    cs = di.conv_state[0].cuda().clone()
    conv_out, f = _front(di.x.cuda(), cs, di.conv_w.cuda(), T, H, D, float("nan"))
    torch.cuda.synchronize()
    ref, ref_state = oracle.front_prefill(di.x, di.conv_state[0], di.conv_w, H, D)
    got = np64(conv_out)
    assert rel_l2(got, ref) <= TOL_BF16
    qkv = H * D
    # q|k are rounded twice on prefill (conv+SiLU write, then l2_norm_bf16 in place): two steps
    _within_bf16_steps(got[:, :2 * qkv], ref[:, :2 * qkv], steps=2)
    _within_bf16_steps(got[:, 2 * qkv:], ref[:, 2 * qkv:], steps=1)
    assert np.array_equal(np64(cs), ref_state)
    for m in range(3):
        assert torch.equal(f[m][:T], conv_out[:, m * qkv:(m + 1) * qkv].float())
        assert torch.all(torch.isnan(f[m][T:]))


def test_front_prefill_split_equals_whole():
    H, D, T, T1 = 4, 128, 300, 131
    di = decode_inputs(1, H, D, seed=9, K=T)
    x, w = di.x.cuda(), di.conv_w.cuda()
    cs = di.conv_state[0].cuda().clone()
    whole, _ = _front(x, cs, w, T, H, D, 0.0)
    cs2 = di.conv_state[0].cuda().clone()
    a, _ = _front(x[:T1].contiguous(), cs2, w, T1, H, D, 0.0)
    b, _ = _front(x[T1:].contiguous(), cs2, w, T - T1, H, D, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([a, b]), whole) and torch.equal(cs2, cs)


@pytest.mark.parametrize("T,H,D", [(300, 32, 128), (17, 2, 64)])
def test_back_gated_rmsnorm_matches_oracle(T, H, D):
    g = torch.Generator().manual_seed(T)
    core = torch.randn((T, H, D), generator=g)
    out_gate = torch.randn((T, H * D), generator=g).to(torch.bfloat16)
    w = (1 + 0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16)
    out = torch.empty((T, H * D), dtype=torch.bfloat16, device="cuda")
    kda.kda_back_gated_rmsnorm(core.cuda(), out_gate.cuda(), w.cuda(), out, T, kda.dims(H, D))
    torch.cuda.synchronize()
    ref = oracle.gated_rmsnorm(core, out_gate, w)
    got = np64(out)
    assert rel_l2(got, ref) <= TOL_BF16
    _within_bf16_steps(got, ref, steps=1, frac=0.05)
