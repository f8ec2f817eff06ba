"""GPU parity of the decode paths with the oracle, and the decode_k identity
(Glm5NextKdaLayer `decode_k`: bit-identical to K serial decodes; snapshot t = state after row t)."""
import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import core_inputs, decode_inputs
from tests.gpu_harness import np64, oracle_prefill, rel_l2, worst_head_rel_l2

pytestmark = pytest.mark.gpu
TOL = 1e-4
TOL_BF16 = 2e-2


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


@pytest.mark.parametrize("N,H,D", [(256, 32, 128), (5, 3, 64)])
def test_recurrent_decode(N, H, D):
    ci = core_inputs(N, 1, H, D, seed=3, s0_std=0.1)
    d = kda.dims(H, D, scale=0.8)
    gate = torch.empty((N, H, D), device="cuda")
    kda.kda_gate(ci.g_raw.reshape(N, H * D).cuda(), ci.dt_bias.cuda(), ci.a_log.cuda(), gate, N, d)
    beta = ci.b_logit.reshape(N, H).cuda().contiguous()
    kda.kda_beta(beta, beta, beta.numel())
    states = [ci.s0[n].cuda().clone() for n in range(N)]
    o = torch.empty((N, H, D), device="cuda")
    kda.kda_recurrent_decode(ci.q.reshape(N, H, D).cuda(), ci.k.reshape(N, H, D).cuda(),
                             ci.v.reshape(N, H, D).cuda(), gate, beta, kda.ptr_array(states), o, N, d)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(ci, scale=0.8)
    assert rel_l2(np64(o), o_ref[:, 0]) <= TOL
    assert worst_head_rel_l2(np64(o), o_ref[:, 0]) <= TOL
    assert rel_l2(np64(torch.stack(states)), S_ref) <= TOL


def _dev(di):
    return {k: getattr(di, k).cuda() for k in ("x", "conv_w", "g_raw", "dt_bias", "a_log", "b_logit", "out_gate",
                                               "o_norm")}


def _fused(di, dv, conv_states, h_states, rows, N, d):
    qkv = di.H * di.D
    onorm = torch.empty((N, qkv), dtype=torch.bfloat16, device="cuda")
    conv_out = torch.empty((N, 3 * qkv), dtype=torch.bfloat16, device="cuda")
    core = torch.empty((N, di.H, di.D), device="cuda")
    kda.kda_decode_fused(dv["x"][rows], kda.ptr_array(conv_states), dv["conv_w"], dv["g_raw"][rows], dv["dt_bias"],
                         dv["a_log"], dv["b_logit"][rows], kda.ptr_array(h_states), dv["out_gate"][rows], dv["o_norm"],
                         onorm, conv_out, core, N, d)
    return onorm, conv_out, core


@pytest.mark.parametrize("N,H,D", [(256, 32, 128), (7, 2, 64)])
def test_decode_fused_matches_oracle(N, H, D):
    di = decode_inputs(N, H, D, seed=3)
    d = kda.dims(H, D)
    dv = _dev(di)
    cs = [di.conv_state[n].cuda().clone() for n in range(N)]
    hs = [di.s0[n].cuda().clone() for n in range(N)]
    onorm, conv_out, core = _fused(di, dv, cs, hs, slice(0, N), N, d)
    torch.cuda.synchronize()
    ref = [oracle.decode_rows(di.x[n:n + 1], di.conv_state[n], di.conv_w, di.g_raw[n:n + 1], di.dt_bias, di.a_log,
                              di.b_logit[n:n + 1], di.out_gate[n:n + 1], di.o_norm, di.s0[n], H, D)
           for n in range(N)]
    r_on = np.stack([r["o_norm_out"][0] for r in ref])
    r_core = np.stack([r["core"][0] for r in ref])
    r_S = np.stack([r["h_state"] for r in ref])
    r_cs = np.stack([r["conv_state"] for r in ref])
    r_co = np.stack([r["conv_out"][0] for r in ref])
    assert rel_l2(np64(onorm), r_on) <= TOL_BF16
    assert rel_l2(np64(conv_out), r_co) <= TOL_BF16
    assert rel_l2(np64(core), r_core) <= TOL
    assert rel_l2(np64(torch.stack(hs)), r_S) <= TOL
    assert np.array_equal(np64(torch.stack(cs)), r_cs)


@pytest.mark.parametrize("K", [4, 32, 33, 70])
def test_decode_k_bit_identical_to_serial_decodes(K):
    """K rows in one decode_k call give the bits of K serial one-row decodes, snapshots included:
    32 rows fill one launch (31 snapshots); 33 and 70 rows run as chained launches of 31 rows
    plus the rest, each group's last snapshot copied from the state it leaves."""
    H, D = 32, 128
    di = decode_inputs(1, H, D, seed=3, K=K)
    d = kda.dims(H, D)
    dv = _dev(di)
    qkv = H * D
    # K serial one-row decodes
    cs = [di.conv_state[0].cuda().clone()]
    hs = [di.s0[0].cuda().clone()]
    serial, snaps = [], []
    for t in range(K):
        serial.append(_fused(di, dv, cs, hs, slice(t, t + 1), 1, d))
        snaps.append((hs[0].clone(), cs[0].clone()))
    # one decode_k call with K-1 snapshots
    h_k = di.s0[0].cuda().clone()
    c_k = di.conv_state[0].cuda().clone()
    h_snap = [torch.empty_like(h_k) for _ in range(K - 1)]
    c_snap = [torch.empty_like(c_k) for _ in range(K - 1)]
    onorm = torch.empty((K, qkv), dtype=torch.bfloat16, device="cuda")
    conv_out = torch.empty((K, 3 * qkv), dtype=torch.bfloat16, device="cuda")
    core = torch.empty((K, H, D), device="cuda")
    kda.kda_decode_k(dv["x"], c_k, dv["conv_w"], dv["g_raw"], dv["dt_bias"], dv["a_log"], dv["b_logit"], h_k,
                     dv["out_gate"], dv["o_norm"], onorm, conv_out, core, K, h_snap, c_snap, d)
    torch.cuda.synchronize()
    for t in range(K):
        assert torch.equal(onorm[t], serial[t][0][0])
        assert torch.equal(conv_out[t], serial[t][1][0])
        assert torch.equal(core[t], serial[t][2][0])
    for t in range(K - 1):
        assert torch.equal(h_snap[t], snaps[t][0]) and torch.equal(c_snap[t], snaps[t][1])
    assert torch.equal(h_k, hs[0]) and torch.equal(c_k, cs[0])
    ref = oracle.decode_rows(di.x, di.conv_state[0], di.conv_w, di.g_raw, di.dt_bias, di.a_log, di.b_logit,
                             di.out_gate, di.o_norm, di.s0[0], H, D)
    assert rel_l2(np64(core), ref["core"]) <= TOL
    assert rel_l2(np64(h_k), ref["h_state"]) <= TOL
    for t in range(K - 1):
        assert rel_l2(np64(h_snap[t]), ref["snapshots"][t][0]) <= TOL
        assert np.array_equal(np64(c_snap[t]), ref["snapshots"][t][1])


def test_decode_k_without_snapshots_and_k1():
    H, D = 4, 64
    di = decode_inputs(1, H, D, seed=5, K=3)
    d = kda.dims(H, D)
    dv = _dev(di)
    h_a, c_a = di.s0[0].cuda().clone(), di.conv_state[0].cuda().clone()
    out = torch.empty((3, H * D), dtype=torch.bfloat16, device="cuda")
    kda.kda_decode_k(dv["x"], c_a, dv["conv_w"], dv["g_raw"], dv["dt_bias"], dv["a_log"], dv["b_logit"], h_a,
                     dv["out_gate"], dv["o_norm"], out, None, None, 3, [], [], d)
    h_b, c_b = di.s0[0].cuda().clone(), di.conv_state[0].cuda().clone()
    out_b = torch.empty((3, H * D), dtype=torch.bfloat16, device="cuda")
    for t in range(3):
        kda.kda_decode_k(dv["x"][t:t + 1], c_b, dv["conv_w"], dv["g_raw"][t:t + 1], dv["dt_bias"], dv["a_log"],
                         dv["b_logit"][t:t + 1], h_b, dv["out_gate"][t:t + 1], dv["o_norm"], out_b[t:t + 1], None,
                         None, 1, [], [], d)
    torch.cuda.synchronize()
    assert torch.equal(out, out_b) and torch.equal(h_a, h_b) and torch.equal(c_a, c_b)


def test_misaligned_state_pointer_is_skipped():
    """A state pointer 4 bytes off a 16-byte boundary (the state copies need 16): that
    sequence's heads are left untouched and KDA_ERR_MISALIGNED is latched; the aligned
    sequence in the same call is still updated correctly."""
    N, H, D = 2, 2, 64
    ci = core_inputs(N, 1, H, D, seed=5, s0_std=0.1)
    d = kda.dims(H, D)
    gate = torch.empty((N, H, D), device="cuda")
    kda.kda_gate(ci.g_raw.reshape(N, H * D).cuda(), ci.dt_bias.cuda(), ci.a_log.cuda(), gate, N, d)
    beta = ci.b_logit.reshape(N, H).cuda().contiguous()
    kda.kda_beta(beta, beta, beta.numel())
    good = ci.s0[0].cuda().clone()
    buf = torch.zeros(H * D * D + 4, device="cuda")
    bad = buf[1:1 + H * D * D].view(H, D, D)
    bad.copy_(ci.s0[1].cuda())
    before = bad.clone()
    o = torch.empty((N, H, D), device="cuda")
    kda.kda_recurrent_decode(ci.q.reshape(N, H, D).cuda(), ci.k.reshape(N, H, D).cuda(),
                             ci.v.reshape(N, H, D).cuda(), gate, beta, kda.ptr_array([good, bad]), o, N, d)
    torch.cuda.synchronize()
    assert kda.device_status(clear=True) == 7  # KDA_ERR_MISALIGNED
    assert torch.equal(bad, before)
    o_ref, S_ref = oracle_prefill(ci)
    assert rel_l2(np64(o[0]), o_ref[0, 0]) <= TOL
    assert rel_l2(np64(good), S_ref[0]) <= TOL


def test_decode_k_groups_without_snapshots():
    """70 rows without snapshots (launches of 32, 32, 6 rows) equal 70 rows with snapshots
    (launches of 31, 31, 8): the grouping never changes a bit."""
    H, D, K = 4, 64, 70
    di = decode_inputs(1, H, D, seed=9, K=K)
    d = kda.dims(H, D)
    dv = _dev(di)
    res = []
    for snaps in (False, True):
        h_, c_ = di.s0[0].cuda().clone(), di.conv_state[0].cuda().clone()
        out = torch.empty((K, H * D), dtype=torch.bfloat16, device="cuda")
        core = torch.empty((K, H, D), device="cuda")
        hsn = [torch.empty_like(h_) for _ in range(K - 1)] if snaps else []
        csn = [torch.empty_like(c_) for _ in range(K - 1)] if snaps else []
        kda.kda_decode_k(dv["x"], c_, dv["conv_w"], dv["g_raw"], dv["dt_bias"], dv["a_log"], dv["b_logit"], h_,
                         dv["out_gate"], dv["o_norm"], out, None, core, K, hsn, csn, d)
        torch.cuda.synchronize()
        res.append((out, core, h_, c_))
    for a_, b_ in zip(*res):
        assert torch.equal(a_, b_)
