"""GPU parity of the chunked prefill (kda_gate + kda_beta + kda_chunk_prefill) with the FP64
oracle, through the C ABI. Tolerance: relative L2 <= 1e-4 on the valid core rows and on the
final state (FP32 paths), over the whole tensor and per head."""
import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import core_inputs, pad_rows, t_pad
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


def test_gate_softplus_sweep_against_fp64():
    """The kernels' softplus (SFU exponential, atanh series below y = 1/8, SFU logarithm above)
    over x in [-40, 40] on a fine grid, x = g_raw + dt_bias with g_raw in {0, +-1/8} and a_log = 0,
    so that g = -softplus(x): relative error within 2e-6 + 1.2e-7 |x| of the FP64 oracle
    everywhere, both branches and the switch between them included. The |x| term is the FP32
    rounding of x itself (and of the exponential's scaled argument): for x << 0 softplus is
    about e^x, whose relative error is the absolute error of x. It changes e^g by less than
    one FP32 step."""
    H, D, T = 32, 128, 3
    d = kda.dims(H, D)
    dt = torch.linspace(-40.0, 40.0, H * D, dtype=torch.float64).float()
    g_raw = torch.tensor([0.0, 0.125, -0.125]).repeat_interleave(H * D).reshape(T, H * D).to(torch.bfloat16)
    a_log = torch.zeros(H)
    gate = torch.empty((T, H, D), device="cuda")
    kda.kda_gate(g_raw.cuda(), dt.cuda(), a_log.cuda(), gate, T, d)
    torch.cuda.synchronize()
    ref = oracle.gate(g_raw.float(), dt, a_log, H, D).reshape(T, H * D)
    x = np64(g_raw) + np64(dt)[None, :]
    rel = np.abs(np64(gate).reshape(T, H * D) - ref) / np.abs(ref)
    assert np.all(rel <= 2e-6 + 1.2e-7 * np.abs(x)), float(np.max(rel / (2e-6 + 1.2e-7 * np.abs(x))))


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
    bit-identical; 16 (stream, head) pairs, four heads of every stream, within tolerance of the
    oracle (outputs of every token and final state)."""
    B, T, H, D = 4, 65500, 32, 128
    ci = core_inputs(B, T, H, D, seed=4, bf16_inputs=True, s0_std=0.1, device="cuda")
    core_n, S_n, _ = gpu_prefill(ci, impl=impl, pad_fill=float("nan"))
    core_n = core_n.clone()
    core_0, S_0, _ = gpu_prefill(ci, impl=impl, pad_fill=0.0)
    assert torch.equal(S_n, S_0)
    assert torch.equal(core_n, core_0)
    heads = {0: [0, 9, 17, 31], 1: [3, 12, 20, 28], 2: [5, 14, 22, 30], 3: [1, 7, 19, 26]}
    for b, hs in heads.items():
        o_ref, S_ref = oracle_prefill(ci, seqs=[b], heads=hs)  # the four heads in parallel
        for j, h in enumerate(hs):
            assert rel_l2(np64(core_n[b, :, h]), o_ref[0, :, j]) <= TOL, (b, h)
            assert rel_l2(np64(S_n[b, h]), S_ref[0, j]) <= TOL, (b, h)
    del core_n, core_0
    torch.cuda.empty_cache()


def _gpu_prefill_fused(ci, *, pad_fill=float("nan"), scale=1.0):
    """kda_chunk_prefill_fused on BF16 q|k|v rows and BF16 g_raw; every tail row of qkv,
    g_raw and beta holds pad_fill."""
    B, T, H, D = ci.B, ci.T, ci.H, ci.D
    Tp = t_pad(T)
    d = kda.dims(H, D, scale=scale)
    qkv = torch.cat([ci.q.reshape(B, T, H * D), ci.k.reshape(B, T, H * D), ci.v.reshape(B, T, H * D)], dim=-1)
    qkv = pad_rows(qkv.to(torch.bfloat16), Tp, pad_fill).cuda()
    g_raw = pad_rows(ci.g_raw, Tp, pad_fill).cuda()
    beta = pad_rows(ci.b_logit, Tp, 0.0).cuda()
    kda.kda_beta(beta, beta, beta.numel())
    beta.view(B, Tp, H)[:, T:] = pad_fill
    states = [ci.s0[b].cuda().clone() for b in range(B)]
    core = torch.full((B * Tp, H, D), float("nan"), dtype=torch.float32, device="cuda")
    kda.kda_chunk_prefill_fused(qkv, g_raw, ci.dt_bias.cuda(), ci.a_log.cuda(), beta, kda.ptr_array(states), core, B,
                                T, d)
    torch.cuda.synchronize()
    return core.view(B, Tp, H, D)[:, :T], torch.stack(states)


@pytest.mark.parametrize("B,T,H,D", [(1, 4096, 32, 128), (2, 150, 3, 128), (3, 1, 2, 64), (2, 257, 2, 64),
                                     (1, 129, 1, 128)])
def test_fused_prefill_matches_f32_path_and_oracle(B, T, H, D):
    """The fused-input prefill (BF16 conv_out rows and g_raw, gate formed in-kernel) against
    the FP32 path on the widened inputs (same operands: equal to within FP32 rounding) and
    against the oracle; tails poisoned with NaN."""
    ci = core_inputs(B, T, H, D, seed=40 + T, bf16_inputs=True, s0_std=0.1)
    core_f, S_f = _gpu_prefill_fused(ci, scale=0.7)
    core, S, _ = gpu_prefill(ci, scale=0.7)
    assert rel_l2(np64(core_f), np64(core)) <= 1e-6 and rel_l2(np64(S_f), np64(S)) <= 1e-6
    _check(ci, core_f, S_f, scale=0.7)


def test_fused_prefill_extreme_decay_takes_exact_path():
    """Strong decay on some channels sends chunks to the exact CUDA-core body, which forms the
    gate from g_raw itself in this mode."""
    ci = core_inputs(1, 200, 3, 128, seed=31, bf16_inputs=True, s0_std=0.1)
    ci.a_log[1] = 3.0
    ci.dt_bias[1 * 128 + 5] = 20.0
    ci.dt_bias[1 * 128 + 9] = 6.0
    core_f, S_f = _gpu_prefill_fused(ci)
    _check(ci, core_f, S_f)


@pytest.mark.parametrize("B,T,H,D,strong", [(1, 4096, 32, 128, False), (2, 150, 3, 128, False),
                                            (3, 1, 2, 64, False), (2, 257, 2, 64, False), (1, 200, 3, 128, True)])
def test_graw_prefill_bit_identical_to_gate_then_prefill(B, T, H, D, strong):
    """kda_chunk_prefill_graw (the gate formed in the kernel from BF16 g_raw) gives the same
    bits as kda_gate + kda_chunk_prefill on the same inputs, and matches the oracle; the tails
    of q, k, v, g_raw and beta hold NaN. `strong`: decay strong enough on some channels to send
    chunks to the exact CUDA-core body, which forms the gate itself in this mode."""
    ci = core_inputs(B, T, H, D, seed=70 + T, s0_std=0.1)
    if strong:
        ci.a_log[1] = 3.0
        ci.dt_bias[1 * D + 5] = 20.0
        ci.dt_bias[1 * D + 9] = 6.0
    Tp, nan = t_pad(T), float("nan")
    d = kda.dims(H, D, scale=0.7)
    q, k, v = (pad_rows(x, Tp, nan).cuda() for x in (ci.q, ci.k, ci.v))
    g_raw = pad_rows(ci.g_raw, Tp, nan).cuda()
    dt, al = ci.dt_bias.cuda(), ci.a_log.cuda()
    beta = pad_rows(ci.b_logit, Tp, 0.0).cuda()
    kda.kda_beta(beta, beta, beta.numel())
    beta.view(B, Tp, H)[:, T:] = nan
    gate = torch.full((B * Tp, H, D), nan, device="cuda")
    for b in range(B):  # valid rows only: the gate of the tail stays NaN
        kda.kda_gate(g_raw[b * Tp:b * Tp + T], dt, al, gate[b * Tp:b * Tp + T], T, d)
    outs = []
    for use_graw in (False, True):
        states = [ci.s0[b].cuda().clone() for b in range(B)]
        core = torch.full((B * Tp, H, D), nan, device="cuda")
        if use_graw:
            kda.kda_chunk_prefill_graw(q, k, v, g_raw, dt, al, beta, kda.ptr_array(states), core, B, T, d)
        else:
            kda.kda_chunk_prefill(q, k, v, gate, beta, kda.ptr_array(states), core, B, T, d)
        torch.cuda.synchronize()
        outs.append((core.view(B, Tp, H, D)[:, :T].clone(), torch.stack(states)))
    (c0, s0), (c1, s1) = outs
    assert torch.equal(c0, c1) and torch.equal(s0, s1)
    _check(ci, c1, s1, scale=0.7)


@pytest.mark.parametrize("T,H,D,seg", [(4096, 32, 128, 512), (1000, 4, 128, 256), (130, 3, 64, 64),
                                      (70, 2, 128, 512)])
def test_host_prefill_bit_identical_to_device_calls(T, H, D, seg):
    """kda_chunk_prefill_host (pinned host inputs and outputs, segments of whole chunks with
    copies and compute overlapped) gives the same bits as kda_beta + kda_chunk_prefill_fused over
    all T rows on the device, and matches the oracle."""
    ci = core_inputs(1, T, H, D, seed=90 + T, bf16_inputs=True, s0_std=0.1)
    Tp = t_pad(T)
    d = kda.dims(H, D, scale=0.7)
    qkv = torch.cat([ci.q.reshape(T, H * D), ci.k.reshape(T, H * D), ci.v.reshape(T, H * D)], dim=-1)
    qkv = qkv.to(torch.bfloat16).contiguous()
    g_raw = ci.g_raw[0].contiguous()
    b_logit = ci.b_logit[0].contiguous()
    dt, al = ci.dt_bias.cuda(), ci.a_log.cuda()
    # on the device, whole
    qkv_d = pad_rows(qkv[None], Tp, 0.0).cuda()
    g_d = pad_rows(g_raw[None], Tp, 0.0).cuda()
    beta_d = pad_rows(b_logit[None], Tp, 0.0).cuda()
    kda.kda_beta(beta_d, beta_d, beta_d.numel())
    st_dev = ci.s0[0].cuda().clone()
    core_dev = torch.zeros((Tp, H, D), device="cuda")
    kda.kda_chunk_prefill_fused(qkv_d, g_d, dt, al, beta_d, kda.ptr_array([st_dev]), core_dev, 1, T, d)
    # from host buffers, segmented
    hq, hg, hb = qkv.pin_memory(), g_raw.pin_memory(), b_logit.pin_memory()
    hs = ci.s0[0].clone().pin_memory()
    hc = torch.full((T, H, D), float("nan")).pin_memory()
    buf = torch.empty(kda.kda_chunk_prefill_host_bytes(T, seg, d), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()
    kda.kda_chunk_prefill_host(hq, hg, hb, dt, al, hs, hc, T, seg, buf, d, s.cuda_stream)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(hc, core_dev[:T].cpu()) and torch.equal(hs, st_dev.cpu())
    if T <= 1000:
        _check(ci, hc.reshape(1, T, H, D), hs.reshape(1, H, D, D), scale=0.7)


@pytest.mark.parametrize("T,H,D,seg", [(4096, 32, 128, 1024), (1000, 4, 128, 256), (70, 2, 64, 512)])
def test_host_f32_prefill_bit_identical_to_device_calls(T, H, D, seg):
    """kda_chunk_prefill_host_f32 (pinned FP32 q, k, v, BF16 g_raw and FP32 beta logits in; core
    and state out; segments overlapped) gives the bits of kda_gate + kda_beta +
    kda_chunk_prefill over all T rows on the device, and matches the oracle."""
    ci = core_inputs(1, T, H, D, seed=95 + T, bf16_inputs=False, s0_std=0.1)
    Tp = t_pad(T)
    d = kda.dims(H, D)
    q, k, v = (x[0].reshape(T, H * D).contiguous() for x in (ci.q, ci.k, ci.v))
    g_raw, b_logit = ci.g_raw[0].contiguous(), ci.b_logit[0].contiguous()
    dt, al = ci.dt_bias.cuda(), ci.a_log.cuda()
    # on the device, whole
    dq, dk, dv = (pad_rows(x[None], Tp, 0.0).cuda() for x in (q, k, v))
    gate = torch.zeros((Tp, H * D), device="cuda")
    kda.kda_gate(pad_rows(g_raw[None], Tp, 0.0).cuda(), dt, al, gate, T, d)
    beta = pad_rows(b_logit[None], Tp, 0.0).cuda()
    kda.kda_beta(beta, beta, beta.numel())
    st_dev = ci.s0[0].cuda().clone()
    core_dev = torch.zeros((Tp, H, D), device="cuda")
    kda.kda_chunk_prefill(dq, dk, dv, gate, beta, kda.ptr_array([st_dev]), core_dev, 1, T, d)
    # from host buffers, segmented
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    hg, hb = g_raw.pin_memory(), b_logit.pin_memory()
    hs = ci.s0[0].clone().pin_memory()
    hc = torch.full((T, H, D), float("nan")).pin_memory()
    buf = torch.empty(kda.kda_chunk_prefill_host_f32_bytes(T, seg, d), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()
    kda.kda_chunk_prefill_host_f32(hq, hk, hv, hg, hb, dt, al, hs, hc, T, seg, buf, d, s.cuda_stream)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(hc, core_dev[:T].cpu()) and torch.equal(hs, st_dev.cpu())
    if T <= 1000:
        _check(ci, hc.reshape(1, T, H, D), hs.reshape(1, H, D, D))


def _varlen_case(lens, H, D, seed):
    """Packed sequences of the given lengths: q, k, v [total, H, D], gate and beta formed on the
    GPU from the packed g_raw / b_logit, per-sequence initial states, cu_seqlens on the device."""
    total = sum(lens)
    ci = core_inputs(1, max(total, 1), H, D, seed=seed, bf16_inputs=True, s0_std=0.0)
    g = torch.Generator().manual_seed(seed + 1)
    s0 = torch.randn((len(lens), H, D, D), generator=g) * 0.1
    d = kda.dims(H, D)
    dev = dict(q=ci.q[0, :total].cuda().contiguous(), k=ci.k[0, :total].cuda().contiguous(),
               v=ci.v[0, :total].cuda().contiguous())
    gate = torch.empty((total, H, D), device="cuda")
    kda.kda_gate(ci.g_raw[0, :total].cuda().contiguous(), ci.dt_bias.cuda(), ci.a_log.cuda(), gate, total, d)
    beta = ci.b_logit[0, :total].cuda().contiguous()
    kda.kda_beta(beta, beta, beta.numel())
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    return ci, s0, dev, gate, beta, cu, d


@pytest.mark.parametrize("lens,H,D", [([100, 0, 257, 64, 1], 2, 64), ([300, 129, 7], 4, 128)])
def test_varlen_prefill_matches_per_sequence_path_and_oracle(lens, H, D):
    """kda_chunk_prefill_varlen on back-to-back sequences: each sequence's outputs and final state
    are the bits kda_chunk_prefill gives on that sequence alone, and match the oracle; an empty
    sequence keeps its state."""
    from synth.inputs import CoreInputs
    ci, s0, dev, gate, beta, cu, d = _varlen_case(lens, H, D, seed=60 + len(lens))
    total, B = sum(lens), len(lens)
    states = [s0[b].cuda().clone() for b in range(B)]
    core = torch.full((total, H, D), float("nan"), device="cuda")
    max_chunks = max((L + 63) // 64 for L in lens) + 1  # one spare slot per sequence
    kda.kda_chunk_prefill_varlen(dev["q"], dev["k"], dev["v"], gate, beta, cu, B, max_chunks, total,
                                 kda.ptr_array(states), core, d)
    torch.cuda.synchronize()
    start = 0
    for b, L in enumerate(lens):
        if L == 0:
            assert torch.equal(states[b], s0[b].cuda())
            continue
        sl = slice(start, start + L)
        one = CoreInputs(1, L, H, D, ci.q[:, sl], ci.k[:, sl], ci.v[:, sl], ci.g_raw[:, sl], ci.dt_bias, ci.a_log,
                         ci.b_logit[:, sl], s0[b:b + 1])
        c1, S1, _ = gpu_prefill(one)
        assert torch.equal(core[sl], c1[0]), b
        assert torch.equal(states[b], S1[0]), b
        _check(one, core[sl].unsqueeze(0), states[b].unsqueeze(0))
        start += L


def test_varlen_many_sequences_and_batched_verify_at_serving_shapes():
    """64 packed sequences of mixed lengths (0..300 tokens) through the varlen prefill, then
    256 sequences x 4 draft rows through the batched verify and fold (H 32, D 128): sampled
    sequences bit-identical to the per-sequence path; every verify row equal to the varlen
    prefill's; the folded states equal to the prefill of the accepted rows (sampled) and the
    oracle's."""
    from synth.inputs import CoreInputs
    rng = np.random.default_rng(7)
    lens = [int(x) for x in rng.integers(0, 301, size=64)]
    lens[3] = 0
    lens[10] = 300
    H, D = 4, 128
    ci, s0, dev, gate, beta, cu, d = _varlen_case(lens, H, D, seed=120)
    total, B = sum(lens), len(lens)
    states = [s0[b].cuda().clone() for b in range(B)]
    core = torch.full((total, H, D), float("nan"), device="cuda")
    kda.kda_chunk_prefill_varlen(dev["q"], dev["k"], dev["v"], gate, beta, cu, B, 5, total, kda.ptr_array(states),
                                 core, d)
    torch.cuda.synchronize()
    starts = np.concatenate([[0], np.cumsum(lens)])
    for b in [0, 3, 10, 33, 63]:
        L, st = lens[b], int(starts[b])
        if L == 0:
            assert torch.equal(states[b], s0[b].cuda())
            continue
        sl = slice(st, st + L)
        one = CoreInputs(1, L, H, D, ci.q[:, sl], ci.k[:, sl], ci.v[:, sl], ci.g_raw[:, sl], ci.dt_bias, ci.a_log,
                         ci.b_logit[:, sl], s0[b:b + 1])
        c1, S1, _ = gpu_prefill(one)
        assert torch.equal(core[sl], c1[0]) and torch.equal(states[b], S1[0]), b
    # batched verify: 256 sequences x 4 rows, H 32
    H, D, Bv, K = 32, 128, 256, 4
    vlens = [K] * Bv
    ci, s0, dev, gate, beta, cu, d = _varlen_case(vlens, H, D, seed=121)
    total = Bv * K
    states = [s0[b].cuda().clone() for b in range(Bv)]
    ptrs = kda.ptr_array(states)
    core = torch.full((total, H, D), float("nan"), device="cuda")
    tables = torch.empty(kda.kda_chunk_verify_tables_bytes(Bv, d) // 4, device="cuda")
    kda.kda_chunk_verify(dev["q"], dev["k"], dev["v"], gate, beta, cu, Bv, total, ptrs, core, tables, d)
    fresh = [s0[b].cuda().clone() for b in range(Bv)]
    core_p = torch.full((total, H, D), float("nan"), device="cuda")
    kda.kda_chunk_prefill_varlen(dev["q"], dev["k"], dev["v"], gate, beta, cu, Bv, 1, total, kda.ptr_array(fresh),
                                 core_p, d)
    torch.cuda.synchronize()
    assert torch.equal(core, core_p)
    assert all(torch.equal(states[b], s0[b].cuda()) for b in range(0, Bv, 17))
    for b in [0, 77, 128, 255]:  # sampled sequences' draft rows against the oracle
        sl = slice(b * K, b * K + K)
        one = CoreInputs(1, K, H, D, ci.q[:, sl], ci.k[:, sl], ci.v[:, sl], ci.g_raw[:, sl], ci.dt_bias, ci.a_log,
                         ci.b_logit[:, sl], s0[b:b + 1])
        o_ref, _ = oracle_prefill(one)
        assert rel_l2(np64(core[sl]), o_ref[0]) <= TOL, b
    accepted = [int(x) for x in rng.integers(0, K + 1, size=Bv)]
    kda.kda_chunk_verify_fold(dev["k"], cu, torch.tensor(accepted, dtype=torch.int32, device="cuda"), Bv, total,
                              tables, ptrs, d)
    torch.cuda.synchronize()
    for b in [0, 1, 100, 255]:
        r, st = accepted[b], b * K
        if r == 0:
            assert torch.equal(states[b], s0[b].cuda())
            continue
        sl = slice(st, st + r)
        one = CoreInputs(1, r, H, D, ci.q[:, sl], ci.k[:, sl], ci.v[:, sl], ci.g_raw[:, sl], ci.dt_bias, ci.a_log,
                         ci.b_logit[:, sl], s0[b:b + 1])
        _, S1, _ = gpu_prefill(one)
        assert rel_l2(np64(states[b]), np64(S1[0])) <= 1e-5, b
        _, S_ref = oracle_prefill(one)
        assert rel_l2(np64(states[b]), S_ref[0]) <= TOL, b


def test_varlen_prefill_rejects_a_sequence_longer_than_its_slots():
    """With max_num_chunks = 1 a 100-token sequence does not fit: it is skipped, its state left
    as it was, and KDA_ERR_INVALID_ARG is latched; the 50-token sequence beside it is exact."""
    from synth.inputs import CoreInputs
    lens, H, D = [100, 50], 2, 64
    ci, s0, dev, gate, beta, cu, d = _varlen_case(lens, H, D, seed=77)
    states = [s0[b].cuda().clone() for b in range(2)]
    core = torch.zeros((150, H, D), device="cuda")
    kda.kda_chunk_prefill_varlen(dev["q"], dev["k"], dev["v"], gate, beta, cu, 2, 1, 150, kda.ptr_array(states), core,
                                 d)
    torch.cuda.synchronize()
    assert kda.device_status(clear=True) == 1  # KDA_ERR_INVALID_ARG
    assert torch.equal(states[0], s0[0].cuda())
    one = CoreInputs(1, 50, H, D, ci.q[:, 100:], ci.k[:, 100:], ci.v[:, 100:], ci.g_raw[:, 100:], ci.dt_bias,
                     ci.a_log, ci.b_logit[:, 100:], s0[1:2])
    _check(one, core[100:].unsqueeze(0), states[1].unsqueeze(0))


@pytest.mark.parametrize("D", [128, 64])
def test_verify_then_fold_accepted_rows(D):
    """Batched verify under the WY tables: every draft row's output equals the varlen prefill's
    (bit for bit) while the states stay; folding accepted[b] rows gives the state the prefill of
    exactly those rows gives (and the oracle's); accepted = 0 leaves the state."""
    from synth.inputs import CoreInputs
    lens, H = [5, 64, 1, 17], 4
    accepted = [3, 64, 0, 17]
    ci, s0, dev, gate, beta, cu, d = _varlen_case(lens, H, D, seed=90 + D)
    total, B = sum(lens), len(lens)
    states = [s0[b].cuda().clone() for b in range(B)]
    core = torch.full((total, H, D), float("nan"), device="cuda")
    tables = torch.empty(kda.kda_chunk_verify_tables_bytes(B, d) // 4, device="cuda")
    ptrs = kda.ptr_array(states)
    kda.kda_chunk_verify(dev["q"], dev["k"], dev["v"], gate, beta, cu, B, total, ptrs, core, tables, d)
    torch.cuda.synchronize()
    for b in range(B):
        assert torch.equal(states[b], s0[b].cuda())
    fresh = [s0[b].cuda().clone() for b in range(B)]
    core_p = torch.full((total, H, D), float("nan"), device="cuda")
    kda.kda_chunk_prefill_varlen(dev["q"], dev["k"], dev["v"], gate, beta, cu, B, 1, total, kda.ptr_array(fresh),
                                 core_p, d)
    torch.cuda.synchronize()
    assert torch.equal(core, core_p)
    start = 0
    for b, L in enumerate(lens):  # every draft row against the oracle from the unchanged state
        sl = slice(start, start + L)
        one = CoreInputs(1, L, H, D, ci.q[:, sl], ci.k[:, sl], ci.v[:, sl], ci.g_raw[:, sl], ci.dt_bias, ci.a_log,
                         ci.b_logit[:, sl], s0[b:b + 1])
        o_ref, _ = oracle_prefill(one)
        assert rel_l2(np64(core[sl]), o_ref[0]) <= TOL, b
        start += L
    acc = torch.tensor(accepted, dtype=torch.int32, device="cuda")
    kda.kda_chunk_verify_fold(dev["k"], cu, acc, B, total, tables, ptrs, d)
    torch.cuda.synchronize()
    start = 0
    for b, (L, r) in enumerate(zip(lens, accepted)):
        if r == 0:
            assert torch.equal(states[b], s0[b].cuda())
        else:
            sl = slice(start, start + r)
            one = CoreInputs(1, r, H, D, ci.q[:, sl], ci.k[:, sl], ci.v[:, sl], ci.g_raw[:, sl], ci.dt_bias,
                             ci.a_log, ci.b_logit[:, sl], s0[b:b + 1])
            _, S1, _ = gpu_prefill(one)
            assert rel_l2(np64(states[b]), np64(S1[0])) <= 1e-5, b
            o_ref, S_ref = oracle_prefill(one)
            assert rel_l2(np64(states[b]), S_ref[0]) <= TOL, b
        start += L
