"""GPU block decode (Glm5NextKdaLayer `decode`: N sequences x 1 token through the whole block)
and block decode_k (`decode_k`: K rows of one sequence, projections read once for all rows)
against the oracle, and the decode_k identity through the whole block: K rows in one call
are bit-identical to K one-row calls, snapshots included. BF16 block outputs at 2e-2; the FP32
core and states at 1e-4 through the stateful row's own entry point (never feeding a GPU value
to the oracle)."""
import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import block_hidden, block_weights
from tests.gpu_harness import np64, rel_l2
from tests.test_gpu_block import _device_weights

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


def _states(n, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    hs = torch.randn((n, H, D, D), generator=g) * 0.1
    cs = torch.randn((n, 3 * H * D, 3), generator=g).to(torch.bfloat16)
    return hs, cs


def _decode_fused(x_rows, g_raw, b_logit, out_gate, hs, cs, Wt):
    """kda_decode_fused on given stage rows (one token for each of N sequences) from copies of
    the states hs [N, H, D, D] and conv states cs [N, 3HD, 3]: (core, states, conv states, o_norm_out)."""
    H, D = Wt.H, Wt.D
    N = len(hs)
    dev = "cuda"
    x = torch.as_tensor(x_rows).to(dev, torch.bfloat16).contiguous()
    gr = torch.as_tensor(g_raw).to(dev, torch.bfloat16).contiguous()
    bl = torch.as_tensor(b_logit).to(dev, torch.float32).contiguous()
    og = torch.as_tensor(out_gate).to(dev, torch.bfloat16).contiguous()
    hd = [torch.as_tensor(hs[n]).to(dev, torch.float32).clone() for n in range(N)]
    cd = [torch.as_tensor(cs[n]).to(dev, torch.bfloat16).clone() for n in range(N)]
    out = torch.empty((N, H * D), dtype=torch.bfloat16, device=dev)
    core = torch.empty((N, H, D), device=dev)
    kda.kda_decode_fused(x, kda.ptr_array(cd), Wt.conv_w.cuda(), gr, Wt.dt_bias.cuda(), Wt.a_log.cuda(), bl,
                         kda.ptr_array(hd), og, Wt.o_norm.cuda(), out, None, core, N, kda.dims(H, D))
    torch.cuda.synchronize()
    return core, hd, cd, out


@pytest.mark.parametrize("hidden,H,D,rank,N,std", [(256, 2, 64, 64, 3, 0.05), (4096, 32, 128, 128, 4, 0.02)])
def test_block_decode_matches_oracle(hidden, H, D, rank, N, std):
    Wt = block_weights(hidden, H, D, rank, seed=7, std=std)
    h = block_hidden(N, hidden, seed=7)
    hs, cs = _states(N, H, D, seed=7)
    dw = _device_weights(Wt)
    st = kda.block_weights_struct(dw)
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=8)
    hd = [hs[n].cuda().clone() for n in range(N)]
    cd = [cs[n].cuda().clone() for n in range(N)]
    kda.kda_block_decode(st, h.cuda(), N, kda.ptr_array(hd), kda.ptr_array(cd), ws)
    torch.cuda.synchronize()
    final = np64(ws.view("final_out", (N, hidden), torch.bfloat16))
    refs = [oracle.block_decode(Wt, h[n:n + 1], hs[n], cs[n]) for n in range(N)]
    for n, ref in enumerate(refs):
        assert rel_l2(final[n:n + 1], ref["final_out"]) <= TOL_BF16
        assert rel_l2(np64(hd[n]), ref["h_state"]) <= TOL_BF16
        assert rel_l2(np64(cd[n]), ref["conv_state"]) <= 4e-3
    # the FP32 core and state at 1e-4, with no GPU value fed to the oracle: (a) the block's
    # stateful row is kda_decode_fused on the block's own stage buffers, bit for bit; (b) that
    # call on the oracle's stage values matches the oracle's core and state
    qkv = H * D
    c_a, h_a, c_sa, o_a = _decode_fused(ws.view("qkv_proj", (N, 3 * qkv), torch.bfloat16),
                                        ws.view("g_raw", (N, qkv), torch.bfloat16),
                                        ws.view("beta", (N, H), torch.float32),
                                        ws.view("out_gate", (N, qkv), torch.bfloat16), hs, cs, Wt)
    assert torch.equal(c_a, ws.view("core", (N, H, D), torch.float32))
    assert torch.equal(o_a, ws.view("o_norm_out", (N, qkv), torch.bfloat16))
    assert all(torch.equal(h_a[n], hd[n]) and torch.equal(c_sa[n], cd[n]) for n in range(N))
    stack = lambda key: np.concatenate([r[key] for r in refs])  # noqa: E731
    c_b, h_b, _, _ = _decode_fused(stack("qkv_proj"), stack("g_raw"), stack("b_logit"), stack("out_gate"), hs, cs, Wt)
    for n, ref in enumerate(refs):
        assert rel_l2(np64(c_b[n]), ref["core"][0]) <= 1e-4
        assert rel_l2(np64(h_b[n]), ref["h_state"]) <= 1e-4
    ws.close()


@pytest.mark.parametrize("hidden,H,D,rank,N", [(256, 2, 64, 64, 3), (4096, 32, 128, 128, 1)])
def test_block_decode_graph_replays_the_call(hidden, H, D, rank, N):
    """kda_block_decode_graph records one kda_block_decode (recording runs nothing); three
    replays with new hidden rows each time give the same bits as three direct calls on a copy
    of the same states (outputs, states and conv states)."""
    Wt = block_weights(hidden, H, D, rank, seed=13, std=0.02)
    hs, cs = _states(N, H, D, seed=13)
    dw = _device_weights(Wt)
    st = kda.block_weights_struct(dw)
    steps = [block_hidden(N, hidden, seed=20 + i).cuda() for i in range(3)]
    # direct calls
    ws_a = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=8)
    ha = [hs[n].cuda().clone() for n in range(N)]
    ca = [cs[n].cuda().clone() for n in range(N)]
    pa, pca = kda.ptr_array(ha), kda.ptr_array(ca)
    outs_a = []
    for x in steps:
        kda.kda_block_decode(st, x, N, pa, pca, ws_a)
        outs_a.append(ws_a.view("final_out", (N, hidden), torch.bfloat16).clone())
    # recorded once, replayed with the hidden buffer refilled between replays
    ws_b = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=8)
    hb = [hs[n].cuda().clone() for n in range(N)]
    cb = [cs[n].cuda().clone() for n in range(N)]
    pb, pcb = kda.ptr_array(hb), kda.ptr_array(cb)
    xin = torch.empty_like(steps[0])
    graph = kda.kda_block_decode_graph(st, xin, N, pb, pcb, ws_b)
    torch.cuda.synchronize()
    assert all(torch.equal(hb[n], hs[n].cuda()) for n in range(N)), "recording changed a state"
    outs_b = []
    for x in steps:
        xin.copy_(x)
        graph.launch()
        outs_b.append(ws_b.view("final_out", (N, hidden), torch.bfloat16).clone())
    torch.cuda.synchronize()
    for a_, b_ in zip(outs_a, outs_b):
        assert torch.equal(a_, b_)
    assert all(torch.equal(ha[n], hb[n]) and torch.equal(ca[n], cb[n]) for n in range(N))
    graph.close()
    ws_a.close()
    ws_b.close()


@pytest.mark.parametrize("hidden,H,D,rank,K,std", [(256, 2, 64, 64, 5, 0.05), (4096, 32, 128, 128, 4, 0.02),
                                                   (256, 2, 64, 64, 40, 0.05)])
def test_block_decode_k_bit_identical_to_serial_block_decodes(hidden, H, D, rank, K, std):
    """K rows in one call are the bits of K one-row calls; at K = 40 the projections and o_proj
    run on groups of 32 and 8 rows and the stateful rows on launches of 31 and 9."""
    Wt = block_weights(hidden, H, D, rank, seed=11, std=std)
    h = block_hidden(K, hidden, seed=11).cuda()
    hs, cs = _states(1, H, D, seed=11)
    dw = _device_weights(Wt)
    st = kda.block_weights_struct(dw)
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=K)
    # one call of K rows, snapshots after rows 0..K-2
    ha, ca = hs[0].cuda().clone(), cs[0].cuda().clone()
    h_snaps = [torch.full_like(ha, float("nan")) for _ in range(K - 1)]
    c_snaps = [torch.zeros_like(ca) for _ in range(K - 1)]
    kda.kda_block_decode_k(st, h, K, ha, ca, h_snaps, c_snaps, ws)
    torch.cuda.synchronize()
    final_k = ws.view("final_out", (K, hidden), torch.bfloat16).clone()
    onorm_k = ws.view("o_norm_out", (K, H * D), torch.bfloat16).clone()
    # K serial one-row calls
    hb, cb = hs[0].cuda().clone(), cs[0].cuda().clone()
    rows, onorms = [], []
    for t in range(K):
        kda.kda_block_decode(st, h[t:t + 1].contiguous(), 1, kda.ptr_array([hb]), kda.ptr_array([cb]), ws)
        torch.cuda.synchronize()
        rows.append(ws.view("final_out", (1, hidden), torch.bfloat16).clone())
        onorms.append(ws.view("o_norm_out", (1, H * D), torch.bfloat16).clone())
        if t < K - 1:
            assert torch.equal(hb, h_snaps[t]) and torch.equal(cb, c_snaps[t]), t
    assert torch.equal(torch.cat(onorms), onorm_k)
    assert torch.equal(torch.cat(rows), final_k)
    assert torch.equal(ha, hb) and torch.equal(ca, cb)
    ref = oracle.block_decode(Wt, h.cpu(), hs[0], cs[0])
    assert rel_l2(np64(final_k), ref["final_out"]) <= TOL_BF16
    assert rel_l2(np64(ha), ref["h_state"]) <= TOL_BF16
    for t in range(K - 1):
        assert rel_l2(np64(h_snaps[t]), ref["snapshots"][t][0]) <= TOL_BF16
    ws.close()


def test_block_decode_argument_checks():
    Wt = block_weights(256, 2, 64, 64, seed=1, std=0.05)
    dw = _device_weights(Wt)  # held: the struct keeps only raw pointers
    st = kda.block_weights_struct(dw)
    ws = kda.Workspace(kda.dims(2, 64), 256, 64, max_tokens=4)
    hs = torch.zeros((2, 64, 64), device="cuda")
    cs = torch.zeros((384, 3), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((40, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kda.KdaError):  # more rows than the workspace holds
        kda.kda_block_decode(st, h, 5, kda.ptr_array([hs] * 5), kda.ptr_array([cs] * 5), ws)
    with pytest.raises(kda.KdaError):  # K > max_tokens
        kda.kda_block_decode_k(st, h, 5, hs, cs, [], [], ws)
    ws.close()


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (5, 4096, 128), (13, 96, 4096), (32, 32, 4096)])
def test_gemv_matches_fp64_and_is_row_invariant(M, N, K):
    """kda_gemv_bf16 against an FP64 product (FP32 output: accumulation error only; BF16 output:
    one rounding), and every row's bits equal to a call with that row alone."""
    g = torch.Generator().manual_seed(M * 7 + N)
    x = torch.randn((M, K), generator=g).to(torch.bfloat16).cuda()
    W = (torch.randn((N, K), generator=g) * 0.05).to(torch.bfloat16).cuda()
    y32 = torch.empty((M, N), device="cuda")
    y16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    kda.kda_gemv_bf16(x, W, y32, M, N, K)
    kda.kda_gemv_bf16(x, W, y16, M, N, K)
    torch.cuda.synchronize()
    ref = np64(x) @ np64(W).T
    scale = np.abs(np64(x)) @ np.abs(np64(W)).T
    assert np.all(np.abs(np64(y32) - ref) <= 1e-5 * scale + 1e-30)
    assert np.all(np.abs(np64(y16) - np64(y32)) <= 2.0 ** -8 * np.abs(np64(y32)) + 1e-30)
    for m in {0, M // 2, M - 1}:
        one = torch.empty((1, N), device="cuda")
        kda.kda_gemv_bf16(x[m:m + 1].contiguous(), W, one, 1, N, K)
        torch.cuda.synchronize()
        assert torch.equal(one[0], y32[m])
