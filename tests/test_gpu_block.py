"""GPU parity of the projection GEMM and of the whole block prefill (Glm5NextKdaLayer `prefill`)
with the FP64 oracle. BF16 block outputs: relative L2 <= 2e-2 (the block path rounds to BF16 at
every stage the workspace page lists, on both sides, from FP32 vs FP64 arithmetic). The block's
FP32 core and state are held to 1e-4: the block's core stage is the fused-input chunked prefill
bit for bit, and that call on the oracle's own stage values matches the oracle's core."""
import types

import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import block_hidden, block_weights, t_pad
from tests.gpu_harness import np64, rel_l2

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


def _bf16(shape, g, std=1.0):
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K,f32", [(200, 4096, 256, False), (300, 128, 512, False), (64, 32, 128, True),
                                       (1000, 384, 64, False), (129, 256, 4096, True), (7, 48, 192, False)])
def test_gemm_matches_fp64(M, N, K, f32):
    g = torch.Generator().manual_seed(M + N + K)
    A, W = _bf16((M, K), g), _bf16((N, K), g, 0.05)
    C = torch.empty((M, N), dtype=torch.float32 if f32 else torch.bfloat16, device="cuda")
    kda.kda_gemm_bf16(A.cuda(), W.cuda(), C, M, N, K)
    torch.cuda.synchronize()
    ref = A.double().numpy() @ W.double().numpy().T
    got = np64(C)
    if f32:
        assert np.max(np.abs(got - ref)) <= 1e-5 * np.max(np.abs(ref)) + 1e-6
    else:
        assert rel_l2(got, ref) <= 4e-3
        assert np.all(np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-3 * np.max(np.abs(ref)))


def test_gemm_writes_a_column_range_of_wider_rows():
    """ldc > N: three projections into the packed q|k|v row, untouched columns stay as they were."""
    g = torch.Generator().manual_seed(5)
    M, N, K = 200, 256, 256
    A = _bf16((M, K), g).cuda()
    C = torch.full((M, 3 * N), 7.0, dtype=torch.bfloat16, device="cuda")
    Ws = [_bf16((N, K), g, 0.05).cuda() for _ in range(2)]
    kda.kda_gemm_bf16(A, Ws[0], C, M, N, K, ldc=3 * N)
    kda.kda_gemm_bf16(A, Ws[1], C[:, 2 * N:], M, N, K, ldc=3 * N)
    torch.cuda.synchronize()
    for idx, W in zip((0, 2), Ws):
        ref = A.double().cpu().numpy() @ W.double().cpu().numpy().T
        assert rel_l2(np64(C[:, idx * N:(idx + 1) * N]), ref) <= 4e-3
    assert torch.all(C[:, N:2 * N] == 7.0)


def test_gemm_full_size_sampled():
    """M = 8192, N = 4096, K = 4096 (an o_proj / q_proj of the full block): sampled entries
    against FP64 dot products."""
    g = torch.Generator(device="cuda").manual_seed(3)
    M, N, K = 8192, 4096, 4096
    A = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    kda.kda_gemm_bf16(A, W, C, M, N, K)
    torch.cuda.synchronize()
    r = np.random.default_rng(0)
    rows, cols = r.integers(0, M, 3000), r.integers(0, N, 3000)
    Ad = A[torch.as_tensor(rows, device="cuda")].double().cpu().numpy()
    Wd = W[torch.as_tensor(cols, device="cuda")].double().cpu().numpy()
    ref = np.sum(Ad * Wd, axis=1)
    got = C[torch.as_tensor(rows, device="cuda"), torch.as_tensor(cols, device="cuda")].double().cpu().numpy()
    assert np.max(np.abs(got - ref)) <= 1e-5 * np.max(np.abs(ref)) + 1e-5


def _device_weights(Wt):
    return types.SimpleNamespace(
        q_proj=Wt.w_q.cuda(), k_proj=Wt.w_k.cuda(), v_proj=Wt.w_v.cuda(), conv=Wt.conv_w.cuda(), f_a=Wt.f_a.cuda(),
        f_b=Wt.f_b.cuda(), dt_bias=Wt.dt_bias.cuda(), a_log=Wt.a_log.cuda(), b_proj=Wt.b_proj.cuda(),
        g_a=Wt.g_a.cuda(), g_b=Wt.g_b.cuda(), o_norm=Wt.o_norm.cuda(), o_proj=Wt.o_proj.cuda(), hidden=Wt.hidden,
        rank=Wt.rank)


def _run_block(Wt, h, T, ws, hs, cs, pad_fill=0.0):
    dw = _device_weights(Wt)
    st = kda.block_weights_struct(dw)
    kda.kda_block_prefill(st, h, T, hs, cs, pad_fill, ws)
    torch.cuda.synchronize()
    return dw


def _stages(ws, T, Wt):
    H, D, qkv = Wt.H, Wt.D, Wt.H * Wt.D
    v = lambda n, shp, dt: ws.view(n, shp, dt).clone()  # noqa: E731
    return dict(qkv_proj=v("qkv_proj", (T, 3 * qkv), torch.bfloat16), conv_out=v("conv_out", (T, 3 * qkv), torch.bfloat16),
                g_raw=v("g_raw", (T, qkv), torch.bfloat16),
                beta=v("beta", (T, H), torch.float32), core=v("core", (T, H, D), torch.float32),
                out_gate=v("out_gate", (T, qkv), torch.bfloat16), o_norm_out=v("o_norm_out", (T, qkv), torch.bfloat16),
                final_out=v("final_out", (T, Wt.hidden), torch.bfloat16))


def _fused_core(conv_out, g_raw, beta, Wt, T, s0):
    """kda_chunk_prefill_fused on given BF16 conv_out rows [T, 3HD], BF16 g_raw [T, HD] and FP32
    beta [T, H] (rows past T zero), from state s0: (core [T, H, D], final state)."""
    H, D = Wt.H, Wt.D
    Tp = t_pad(T)
    qkv = torch.zeros((Tp, 3 * H * D), dtype=torch.bfloat16, device="cuda")
    qkv[:T] = torch.as_tensor(conv_out).to("cuda", torch.bfloat16)
    gr = torch.zeros((Tp, H * D), dtype=torch.bfloat16, device="cuda")
    gr[:T] = torch.as_tensor(g_raw).to("cuda", torch.bfloat16)
    be = torch.zeros((Tp, H), dtype=torch.float32, device="cuda")
    be[:T] = torch.as_tensor(beta).reshape(T, H).to("cuda", torch.float32)
    hs = torch.as_tensor(s0).to("cuda", torch.float32).clone()
    core = torch.full((Tp, H, D), float("nan"), device="cuda")
    kda.kda_chunk_prefill_fused(qkv, gr, Wt.dt_bias.cuda(), Wt.a_log.cuda(), be, kda.ptr_array([hs]), core, 1, T,
                                kda.dims(H, D))
    torch.cuda.synchronize()
    return core[:T], hs


def _check_block_core(ws, hs, Wt, T, ref):
    """The block's FP32 core and state at the FP32 tolerance, in two steps that never feed a GPU
    value to the oracle: (a) the block's core stage is kda_chunk_prefill_fused on the block's own
    stage buffers, bit for bit; (b) kda_chunk_prefill_fused on the oracle's stage values (its
    BF16 conv_out and g_raw, its beta) matches the oracle's core and state to 1e-4."""
    H, D, qkv = Wt.H, Wt.D, Wt.H * Wt.D
    core_b = ws.view("core", (T, H, D), torch.float32)
    c_a, s_a = _fused_core(ws.view("conv_out", (T, 3 * qkv), torch.bfloat16), ws.view("g_raw", (T, qkv), torch.bfloat16),
                           ws.view("beta", (T, H), torch.float32), Wt, T, torch.zeros((H, D, D)))
    assert torch.equal(c_a, core_b) and torch.equal(s_a, hs)
    c_b, s_b = _fused_core(ref["conv_out"], ref["g_raw"], ref["beta"], Wt, T, np.zeros((H, D, D)))
    assert rel_l2(np64(c_b), ref["core"]) <= 1e-4
    assert rel_l2(np64(s_b), ref["h_state"]) <= 1e-4


@pytest.mark.parametrize("hidden,H,D,rank,T", [(256, 2, 64, 64, 200), (512, 4, 128, 128, 130)])
def test_block_prefill_stages_match_oracle(hidden, H, D, rank, T):
    Wt = block_weights(hidden, H, D, rank, seed=2, std=0.05)
    h = block_hidden(T, hidden, seed=2)
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=256)
    hs = torch.zeros((H, D, D), device="cuda")
    cs = torch.zeros((3 * H * D, 3), dtype=torch.bfloat16, device="cuda")
    _run_block(Wt, h.cuda(), T, ws, hs, cs)
    got = _stages(ws, T, Wt)
    ref = oracle.block_prefill(Wt, h, np.zeros((H, D, D)), np.zeros((3 * H * D, 3)))
    errs = {k_: rel_l2(np64(got[k_]), ref[k_]) for k_ in got}
    errs["h_state"] = rel_l2(np64(hs), ref["h_state"])
    errs["conv_state"] = rel_l2(np64(cs), ref["conv_state"])
    assert errs["qkv_proj"] <= 4e-3 and errs["conv_state"] <= 4e-3, errs
    assert all(e <= TOL_BF16 for e in errs.values()), errs
    _check_block_core(ws, hs, Wt, T, ref)
    ws.close()


def test_block_prefill_split_and_poison():
    """prefill(200) == prefill(120) then prefill(80) from the carried recurrent and conv states;
    a NaN pad tail (prefill_with_pad_fill) changes nothing."""
    hidden, H, D, rank = 256, 2, 64, 64
    Wt = block_weights(hidden, H, D, rank, seed=4, std=0.05)
    h = block_hidden(200, hidden, seed=4).cuda()
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=256)
    hs, cs = torch.zeros((H, D, D), device="cuda"), torch.zeros((3 * H * D, 3), dtype=torch.bfloat16, device="cuda")
    _run_block(Wt, h, 200, ws, hs, cs)
    whole = ws.view("final_out", (200, hidden), torch.bfloat16).clone()
    hs2, cs2 = torch.zeros_like(hs), torch.zeros_like(cs)
    _run_block(Wt, h[:120].contiguous(), 120, ws, hs2, cs2, pad_fill=float("nan"))
    first = ws.view("final_out", (120, hidden), torch.bfloat16).clone()
    _run_block(Wt, h[120:].contiguous(), 80, ws, hs2, cs2, pad_fill=float("nan"))
    second = ws.view("final_out", (80, hidden), torch.bfloat16).clone()
    assert rel_l2(np64(torch.cat([first, second])), np64(whole)) <= 1e-2
    assert rel_l2(np64(hs2), np64(hs)) <= 1e-3
    assert torch.equal(cs2, cs)
    with pytest.raises(kda.KdaError):
        _run_block(Wt, torch.zeros((300, hidden), dtype=torch.bfloat16, device="cuda"), 300, ws, hs2, cs2)
    ws.close()


def test_block_prefill_full_size():
    """The full block: hidden 4096, H 32, D 128, rank 128, T 8192, weights N(0, 0.02), zero
    states; final_out and the carried state against the FP64 oracle."""
    hidden, H, D, rank, T = 4096, 32, 128, 128, 8192
    Wt = block_weights(hidden, H, D, rank, seed=2)
    h = block_hidden(T, hidden, seed=2)
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=T)
    hs = torch.zeros((H, D, D), device="cuda")
    cs = torch.zeros((3 * H * D, 3), dtype=torch.bfloat16, device="cuda")
    _run_block(Wt, h.cuda(), T, ws, hs, cs)
    final = np64(ws.view("final_out", (T, hidden), torch.bfloat16))
    ref = oracle.block_prefill(Wt, h, np.zeros((H, D, D)), np.zeros((3 * H * D, 3)))
    assert rel_l2(final, ref["final_out"]) <= TOL_BF16
    assert rel_l2(np64(hs), ref["h_state"]) <= TOL_BF16
    _check_block_core(ws, hs, Wt, T, ref)
    ws.close()
