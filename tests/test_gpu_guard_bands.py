"""Guard bands: every output and scratch buffer of the C ABI sits inside a larger allocation
whose margins hold a canary byte pattern; after the call the margins (and the rows a call
documents as untouched, such as the pad rows of the prefill core) must still hold it. This is
the race / out-of-bounds check the build uses in place of compute-sanitizer: it catches any
write past a buffer's end, before its start, or into rows the contract leaves alone."""
import ctypes
import math

import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
from synth import core_inputs, decode_inputs, pad_rows, t_pad

pytestmark = pytest.mark.gpu
CANARY = 0xA5
MARGIN = 4096  # bytes on each side (keeps every view 16-byte aligned)


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


class Guarded:
    """A tensor of `shape` and `dtype` in the middle of a canary-filled allocation."""

    def __init__(self, shape, dtype, device="cuda", pin=False):
        es = torch.empty((), dtype=dtype).element_size()
        self.nbytes = math.prod(shape) * es
        raw = torch.full((2 * MARGIN + self.nbytes,), CANARY, dtype=torch.uint8)
        self.raw = raw.pin_memory() if pin else raw.to(device)
        self.t = self.raw[MARGIN:MARGIN + self.nbytes].view(dtype).view(shape)

    def margins_intact(self):
        return bool(torch.all(self.raw[:MARGIN] == CANARY)) and bool(torch.all(self.raw[MARGIN + self.nbytes:] == CANARY))

    def canary_bytes(self, t):
        """True if every byte of the view `t` (part of self.t) still holds the canary."""
        return bool(torch.all(t.contiguous().view(torch.uint8) == CANARY))


def _varlen_scratch_bytes(B, max_chunks, d):
    return int(kda.lib().kda_chunk_prefill_varlen_scratch_bytes(B, max_chunks, ctypes.byref(d)))


def _prefill_inputs(B, T, H, D, seed):
    ci = core_inputs(B, T, H, D, seed=seed, s0_std=0.1)
    Tp = t_pad(T)
    d = kda.dims(H, D)
    q, k, v = (pad_rows(x, Tp, 0.0).cuda() for x in (ci.q, ci.k, ci.v))
    g_raw = pad_rows(ci.g_raw, Tp, 0.0).cuda()
    gate = torch.empty((B * Tp, H, D), device="cuda")
    kda.kda_gate(g_raw, ci.dt_bias.cuda(), ci.a_log.cuda(), gate, B * Tp, d)
    beta = pad_rows(ci.b_logit, Tp, 0.0).cuda()
    kda.kda_beta(beta, beta, beta.numel())
    return ci, d, q, k, v, g_raw, gate, beta


@pytest.mark.parametrize("mode", ["f32", "graw"])
def test_prefill_writes_only_its_outputs(mode):
    B, T, H, D = 2, 150, 3, 128
    ci, d, q, k, v, g_raw, gate, beta = _prefill_inputs(B, T, H, D, seed=5)
    Tp = t_pad(T)
    core = Guarded((B * Tp, H, D), torch.float32)
    states = [Guarded((H, D, D), torch.float32) for _ in range(B)]
    for b in range(B):
        states[b].t.copy_(ci.s0[b])
    sb = kda.kda_chunk_prefill_scratch_bytes(B, T, d)
    scratch = Guarded((sb,), torch.uint8)
    ptrs = kda.ptr_array([s.t for s in states])
    if mode == "f32":
        kda.kda_chunk_prefill(q, k, v, gate, beta, ptrs, core.t, B, T, d, scratch=scratch.t)
    else:
        kda.kda_chunk_prefill_graw(q, k, v, g_raw, ci.dt_bias.cuda(), ci.a_log.cuda(), beta, ptrs, core.t, B, T, d,
                                   scratch=scratch.t)
    torch.cuda.synchronize()
    assert core.margins_intact() and scratch.margins_intact() and all(s.margins_intact() for s in states)
    pad = core.t.view(B, Tp, H, D)[:, T:]
    assert core.canary_bytes(pad), "pad rows of core were written"
    assert torch.all(torch.isfinite(core.t.view(B, Tp, H, D)[:, :T]))


def test_varlen_verify_fold_write_only_their_outputs():
    lens, H, D = [100, 0, 70, 1], 2, 64
    total = sum(lens)
    ci, d, q, k, v, _, gate, beta = _prefill_inputs(1, total, H, D, seed=6)
    q, k, v, gate, beta = (x[:total].contiguous() for x in (q, k, v, gate, beta))
    cu = torch.tensor([0, 100, 100, 170, 171], dtype=torch.int32, device="cuda")
    nb = len(lens)
    core = Guarded((total, H, D), torch.float32)
    states = [Guarded((H, D, D), torch.float32) for _ in range(nb)]
    for s in states:
        s.t.normal_(0.0, 0.1)
    sb = _varlen_scratch_bytes(nb, 2, d)
    scratch = Guarded((sb,), torch.uint8)
    ptrs = kda.ptr_array([s.t for s in states])
    kda.kda_chunk_prefill_varlen(q, k, v, gate, beta, cu, nb, 2, total, ptrs, core.t, d, scratch=scratch.t)
    torch.cuda.synchronize()
    assert core.margins_intact() and scratch.margins_intact() and all(s.margins_intact() for s in states)
    # verify (at most 64 rows per sequence) and fold
    vl = [5, 0, 64, 1]
    vt = sum(vl)
    cu_v = torch.tensor([0, 5, 5, 69, 70], dtype=torch.int32, device="cuda")
    tables = Guarded((kda.kda_chunk_verify_tables_bytes(nb, d),), torch.uint8)
    vcore = Guarded((vt, H, D), torch.float32)
    vscratch = Guarded((_varlen_scratch_bytes(nb, 1, d),), torch.uint8)
    before = [s.t.clone() for s in states]
    kda.kda_chunk_verify(q[:vt], k[:vt], v[:vt], gate[:vt], beta[:vt], cu_v, nb, vt, ptrs, vcore.t, tables.t, d,
                         scratch=vscratch.t)
    torch.cuda.synchronize()
    assert all(torch.equal(s.t, b) for s, b in zip(states, before)), "verify changed a state"
    acc = torch.tensor([3, 0, 64, 1], dtype=torch.int32, device="cuda")
    kda.kda_chunk_verify_fold(k[:vt], cu_v, acc, nb, vt, tables.t, ptrs, d)
    torch.cuda.synchronize()
    assert tables.margins_intact() and vcore.margins_intact() and vscratch.margins_intact()
    assert all(s.margins_intact() for s in states)


def test_decode_paths_write_only_their_outputs():
    N, H, D, K = 5, 3, 64, 4
    di = decode_inputs(N, H, D, seed=7, K=K)
    d = kda.dims(H, D)
    qkv = H * D
    dv = {n: getattr(di, n).cuda() for n in ("x", "conv_w", "g_raw", "dt_bias", "a_log", "b_logit", "out_gate",
                                             "o_norm")}
    cs = [Guarded((3 * qkv, 3), torch.bfloat16) for _ in range(N)]
    hs = [Guarded((H, D, D), torch.float32) for _ in range(N)]
    for n in range(N):
        cs[n].t.copy_(di.conv_state[n])
        hs[n].t.copy_(di.s0[n])
    onorm, conv_out = Guarded((N, qkv), torch.bfloat16), Guarded((N, 3 * qkv), torch.bfloat16)
    core = Guarded((N, H, D), torch.float32)
    kda.kda_decode_fused(dv["x"][:N], kda.ptr_array([c.t for c in cs]), dv["conv_w"], dv["g_raw"][:N], dv["dt_bias"],
                         dv["a_log"], dv["b_logit"][:N], kda.ptr_array([h.t for h in hs]), dv["out_gate"][:N],
                         dv["o_norm"], onorm.t, conv_out.t, core.t, N, d)
    torch.cuda.synchronize()
    for g in [onorm, conv_out, core] + cs + hs:
        assert g.margins_intact()
    # decode_k: K rows of one sequence with a snapshot after each of rows 0..K-2
    h1, c1 = Guarded((H, D, D), torch.float32), Guarded((3 * qkv, 3), torch.bfloat16)
    h1.t.copy_(di.s0[0])
    c1.t.copy_(di.conv_state[0])
    hsn = [Guarded((H, D, D), torch.float32) for _ in range(K - 1)]
    csn = [Guarded((3 * qkv, 3), torch.bfloat16) for _ in range(K - 1)]
    onk, cok = Guarded((K, qkv), torch.bfloat16), Guarded((K, 3 * qkv), torch.bfloat16)
    corek = Guarded((K, H, D), torch.float32)
    kda.kda_decode_k(dv["x"][:K], c1.t, dv["conv_w"], dv["g_raw"][:K], dv["dt_bias"], dv["a_log"], dv["b_logit"][:K],
                     h1.t, dv["out_gate"][:K], dv["o_norm"], onk.t, cok.t, corek.t, K, [h.t for h in hsn],
                     [c.t for c in csn], d)
    torch.cuda.synchronize()
    for g in [h1, c1, onk, cok, corek] + hsn + csn:
        assert g.margins_intact()


def test_front_back_gemm_gemv_write_only_their_outputs():
    T, H, D = 70, 2, 128
    qkv, cd = H * D, 3 * H * D
    d = kda.dims(H, D)
    g = torch.Generator(device="cuda").manual_seed(8)
    x = torch.randn((T, cd), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((cd, 4), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    cs = Guarded((cd, 3), torch.bfloat16)
    cs.t.zero_()
    Tp = t_pad(T)
    conv_out = Guarded((T, cd), torch.bfloat16)
    wide = [Guarded((Tp, qkv), torch.float32) for _ in range(3)]
    kda.kda_front_conv_silu_l2(x, cs.t, w, conv_out.t, wide[0].t, wide[1].t, wide[2].t, 0.0, T, d)
    core = torch.randn((T, H, D), generator=g, device="cuda")
    gate = torch.randn((T, qkv), generator=g, device="cuda").to(torch.bfloat16)
    onw = torch.ones((D,), device="cuda").to(torch.bfloat16)
    out = Guarded((T, qkv), torch.bfloat16)
    kda.kda_back_gated_rmsnorm(core, gate, onw, out.t, T, d)
    # GEMM / GEMV into a column range of wider rows: the other columns stay untouched
    M, N, Kd, ldc = 96, 128, 256, 384
    A = torch.randn((M, Kd), generator=g, device="cuda").to(torch.bfloat16)
    W = torch.randn((N, Kd), generator=g, device="cuda").to(torch.bfloat16)
    Cg = Guarded((M, ldc), torch.bfloat16)
    kda.kda_gemm_bf16(A, W, Cg.t[:, 128:128 + N], M, N, Kd, ldc=ldc)
    Cv = Guarded((3, ldc), torch.float32)
    kda.kda_gemv_bf16(A[:3], W, Cv.t[:, 128:128 + N], 3, N, Kd, ldy=ldc)
    torch.cuda.synchronize()
    for gb in [cs, conv_out, out, Cg, Cv] + wide:
        assert gb.margins_intact()
    for gb in (Cg, Cv):
        assert gb.canary_bytes(gb.t[:, :128]) and gb.canary_bytes(gb.t[:, 128 + N:])


def test_host_prefill_writes_only_its_outputs():
    T, H, D, seg = 200, 2, 128, 64
    ci = core_inputs(1, T, H, D, seed=9, bf16_inputs=True, s0_std=0.1)
    d = kda.dims(H, D)
    qkv = torch.cat([ci.q.reshape(T, H * D), ci.k.reshape(T, H * D), ci.v.reshape(T, H * D)], dim=-1)
    hq = qkv.to(torch.bfloat16).contiguous().pin_memory()
    hg, hb = ci.g_raw[0].contiguous().pin_memory(), ci.b_logit[0].contiguous().pin_memory()
    hs = Guarded((H, D, D), torch.float32, pin=True)
    hs.t.copy_(ci.s0[0])
    hc = Guarded((T, H, D), torch.float32, pin=True)
    buf = Guarded((kda.kda_chunk_prefill_host_bytes(T, seg, d),), torch.uint8)
    s = torch.cuda.current_stream()
    kda.kda_chunk_prefill_host(hq, hg, hb, ci.dt_bias.cuda(), ci.a_log.cuda(), hs.t, hc.t, T, seg, buf.t, d,
                               s.cuda_stream)
    s.synchronize()
    torch.cuda.synchronize()
    assert hs.margins_intact() and hc.margins_intact() and buf.margins_intact()
    assert torch.all(torch.isfinite(hc.t))


def test_packed_scratch_is_enough_for_the_compact_layout():
    """Packed sequences whose chunks start mid-chunk everywhere, with scratch sized exactly by
    kda_chunk_prefill_packed_scratch_bytes (ceil(total/64) + B - 1 pack slots per head): the
    compact layout stays inside it, and the results are the bits of the one-slot-per-chunk
    layout (a larger scratch)."""
    lens, H, D = [63, 1, 65, 130, 2], 2, 128
    total, nb = sum(lens), len(lens)
    ci, d, q, k, v, _, gate, beta = _prefill_inputs(1, total, H, D, seed=12)
    q, k, v, gate, beta = (x[:total].contiguous() for x in (q, k, v, gate, beta))
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32, device="cuda")
    s0 = torch.randn((nb, H, D, D), generator=torch.Generator().manual_seed(12)) * 0.1
    out = []
    for sb in (kda.kda_chunk_prefill_packed_scratch_bytes(nb, total, d), _varlen_scratch_bytes(nb, 3, d)):
        core = Guarded((total, H, D), torch.float32)
        states = [Guarded((H, D, D), torch.float32) for _ in range(nb)]
        for b in range(nb):
            states[b].t.copy_(s0[b])
        scratch = Guarded((sb,), torch.uint8)
        kda.kda_chunk_prefill_varlen(q, k, v, gate, beta, cu, nb, 3, total, kda.ptr_array([s.t for s in states]),
                                     core.t, d, scratch=scratch.t)
        torch.cuda.synchronize()
        assert core.margins_intact() and scratch.margins_intact() and all(s.margins_intact() for s in states)
        out.append((core.t.clone(), [s.t.clone() for s in states]))
    (c0, s0_), (c1, s1_) = out
    assert torch.equal(c0, c1) and all(torch.equal(a, b) for a, b in zip(s0_, s1_))
    assert (kda.kda_chunk_prefill_packed_scratch_bytes(nb, total, d) < _varlen_scratch_bytes(nb, 3, d))


def test_packed_front_end_and_conv_fold_write_only_their_outputs():
    """kda_front_conv_silu_l2_varlen (reading and advancing B conv states) and kda_conv_state_fold
    keep to conv_out and the states; sequences start inside 16-token tiles, one is empty."""
    H, D = 2, 64
    lens = [5, 0, 30, 1, 19]
    total, nb, cd = sum(lens), len(lens), 3 * H * D
    g = torch.Generator().manual_seed(13)
    x = (torch.randn((total, cd), generator=g)).to(torch.bfloat16).cuda()
    cw = (torch.randn((cd, 4), generator=g) * 0.5).to(torch.bfloat16).cuda()
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32, device="cuda")
    states = [Guarded((cd, 3), torch.bfloat16) for _ in range(nb)]
    for s in states:
        s.t.copy_(torch.randn((cd, 3), generator=g).to(torch.bfloat16))
    out = Guarded((total, cd), torch.bfloat16)
    d = kda.dims(H, D)
    kda.kda_front_conv_silu_l2_varlen(x, kda.ptr_array([s.t for s in states]), cw, out.t, cu, nb, total, True, d)
    acc = torch.tensor([3, 0, 30, 1, 0], dtype=torch.int32, device="cuda")
    kda.kda_conv_state_fold(x, kda.ptr_array([s.t for s in states]), cu, acc, nb, total, d)
    torch.cuda.synchronize()
    assert out.margins_intact() and all(s.margins_intact() for s in states)


def test_host_f32_prefill_writes_only_its_outputs():
    T, H, D, seg = 200, 2, 128, 128
    ci = core_inputs(1, T, H, D, seed=14, s0_std=0.1)
    d = kda.dims(H, D)
    hq, hk, hv = (x[0].reshape(T, H * D).contiguous().pin_memory() for x in (ci.q, ci.k, ci.v))
    hg, hb = ci.g_raw[0].contiguous().pin_memory(), ci.b_logit[0].contiguous().pin_memory()
    hs = Guarded((H, D, D), torch.float32, pin=True)
    hs.t.copy_(ci.s0[0])
    hc = Guarded((T, H, D), torch.float32, pin=True)
    buf = Guarded((kda.kda_chunk_prefill_host_f32_bytes(T, seg, d),), torch.uint8)
    s = torch.cuda.current_stream()
    kda.kda_chunk_prefill_host_f32(hq, hk, hv, hg, hb, ci.dt_bias.cuda(), ci.a_log.cuda(), hs.t, hc.t, T, seg, buf.t,
                                   d, s.cuda_stream)
    s.synchronize()
    torch.cuda.synchronize()
    assert hs.margins_intact() and hc.margins_intact() and buf.margins_intact()
    assert torch.all(torch.isfinite(hc.t))


@pytest.mark.parametrize("lens,acc", [([7, 64, 1], [7, 10, 0]),   # 72 rows: the chunked verify
                                      ([7, 16, 1], [7, 10, 0])])  # 24 rows: row by row
def test_block_verify_and_fold_write_only_their_outputs(lens, acc):
    """kda_block_verify reads the guarded recurrent and conv states and leaves them as they were;
    kda_block_verify_fold writes only inside them; the tables stay inside their allocation. Both
    routes: the chunked verify and the row-by-row one of short drafts."""
    from synth import block_hidden, block_weights
    from tests.test_gpu_block import _device_weights
    hidden, H, D, rank = 256, 2, 64, 64
    total, nb = sum(lens), len(lens)
    Wt = block_weights(hidden, H, D, rank, seed=15, std=0.05)
    h = block_hidden(total, hidden, seed=15).cuda()
    d = kda.dims(H, D)
    ws = kda.Workspace(d, hidden, rank, max_tokens=total, max_seqs=nb)
    g = torch.Generator().manual_seed(15)
    hs = [Guarded((H, D, D), torch.float32) for _ in range(nb)]
    cs = [Guarded((3 * H * D, 3), torch.bfloat16) for _ in range(nb)]
    for a, c in zip(hs, cs):
        a.t.copy_(torch.randn((H, D, D), generator=g) * 0.1)
        c.t.copy_(torch.randn((3 * H * D, 3), generator=g).to(torch.bfloat16))
    before = [(a.t.clone(), c.t.clone()) for a, c in zip(hs, cs)]
    tables = Guarded((kda.kda_chunk_verify_tables_bytes(nb, d) // 4,), torch.float32)
    cu = torch.tensor([0] + [int(x) for x in np.cumsum(lens)], dtype=torch.int32, device="cuda")
    dw = _device_weights(Wt)
    st = kda.block_weights_struct(dw)
    hp, cp = kda.ptr_array([a.t for a in hs]), kda.ptr_array([c.t for c in cs])
    kda.kda_block_verify(st, h, cu, nb, total, hp, cp, tables.t, ws)
    torch.cuda.synchronize()
    assert all(torch.equal(a.t, b0) and torch.equal(c.t, b1) for (a, c), (b0, b1) in zip(zip(hs, cs), before))
    kda.kda_block_verify_fold(cu, torch.tensor(acc, dtype=torch.int32, device="cuda"), nb, total, tables.t, hp, cp, ws)
    torch.cuda.synchronize()
    assert tables.margins_intact() and all(a.margins_intact() and c.margins_intact() for a, c in zip(hs, cs))
    assert torch.equal(hs[2].t, before[2][0]) and torch.equal(cs[2].t, before[2][1])  # accepted 0
    ws.close()
