"""GPU parity of the packed-sequence block calls (Glm5NextLayer batched prefill and its varlen
form) and of the block-level batched verify and accepted-row fold (Glm5NextLayer speculative
verify and `gdn_fold_accepted`; Glm5NextKdaLayer `decode_k` at layer level).

A verify of at most 16 draft rows per sequence on average runs row by row in the stateful decode
row. Its exact check is decode_k's: every draft row's outputs, and the states its fold leaves,
equal kda_decode_k run on that sequence's own stage rows, bit for bit. Longer drafts take the
chunked verify, checked as the prefill is below.

Each sequence is checked on its own against the FP64 oracle run on that sequence alone:
- the BF16 stage buffers at 2e-2 (BF16 rounding at every stage, on both sides);
- the conv state bit for bit against the last three inputs of (old state || the sequence's
  qkv_proj rows), which the conv state is by definition;
- the FP32 core and state at 1e-4 in two steps that never feed a GPU value to the oracle:
  (a) the packed call's core rows and state equal kda_chunk_prefill_fused on that sequence's
  own stage rows, bit for bit; (b) kda_chunk_prefill_fused on the oracle's stage values matches
  the oracle's core and state to 1e-4.
"""
import numpy as np
import pytest
import torch

import kda_gated_delta_gate_b200 as kda
import oracle
from synth import block_hidden, block_weights
from tests.gpu_harness import np64, rel_l2
from tests.test_gpu_block import _device_weights, _fused_core, _stages

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2
KDA_ERR_INVALID_ARG = 1


@pytest.fixture(autouse=True)
def _status(cuda_ok):
    kda.device_status(clear=True)
    yield
    assert kda.device_status(clear=True) == 0


def _cu(lens):
    return [0] + [int(x) for x in np.cumsum(lens)]


def _states(n, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    hs = torch.randn((n, H, D, D), generator=g) * 0.1
    cs = torch.randn((n, 3 * H * D, 3), generator=g).to(torch.bfloat16)
    return hs, cs


def _decode_k_rows(dw, got, sl, hs0_b, cs0_b, d):
    """kda_decode_k over the stage rows sl (pre-conv qkv_proj rows, g_raw, beta logits, out_gate)
    from copies of one sequence's states: (o_norm_out, core, conv_out, state, conv state)."""
    K, qkv = sl.stop - sl.start, d.heads * d.head_dim
    hs, cs = hs0_b.cuda().clone(), cs0_b.cuda().clone()
    on = torch.empty((K, qkv), dtype=torch.bfloat16, device="cuda")
    co = torch.empty((K, 3 * qkv), dtype=torch.bfloat16, device="cuda")
    core = torch.empty((K, d.heads, d.head_dim), dtype=torch.float32, device="cuda")
    kda.kda_decode_k(got["qkv_proj"][sl].contiguous(), cs, dw.conv, got["g_raw"][sl].contiguous(), dw.dt_bias,
                     dw.a_log, got["beta"][sl].contiguous(), hs, got["out_gate"][sl].contiguous(), dw.o_norm, on, co,
                     core, K, [], [], d)
    torch.cuda.synchronize()
    return on, core, co, hs, cs


def _conv_after(cs0, qkv_rows):
    """The conv state after the rows qkv_rows [L, 3HD] from cs0 [3HD, 3]: the last three inputs
    of (state || rows), oldest first."""
    return torch.cat([cs0, qkv_rows.T], dim=1)[:, -3:].contiguous()


def _check_core(got, r0, L, Wt, s0, core_rows, state, ref):
    """Steps (a) and (b) of the module docstring for one sequence of L rows from row r0."""
    sl = slice(r0, r0 + L)
    c_a, s_a = _fused_core(got["conv_out"][sl], got["g_raw"][sl], got["beta"][sl], Wt, L, s0)
    assert torch.equal(c_a, core_rows)
    if state is not None:
        assert torch.equal(s_a, state)
    c_b, s_b = _fused_core(ref["conv_out"], ref["g_raw"], ref["beta"], Wt, L, np64(s0))
    assert rel_l2(np64(c_b), ref["core"]) <= 1e-4
    assert rel_l2(np64(s_b), ref["h_state"]) <= 1e-4


def _run_varlen(Wt, h, lens, hs0, cs0, max_seqs=None):
    """kda_block_prefill_varlen over the packed rows h from copies of the states: (workspace,
    stage buffers, states, conv states)."""
    H, D, B, total = Wt.H, Wt.D, len(lens), sum(lens)
    ws = kda.Workspace(kda.dims(H, D), Wt.hidden, Wt.rank, max_tokens=total, max_seqs=max_seqs or B)
    hs = [hs0[b].cuda().clone() for b in range(B)]
    cs = [cs0[b].cuda().clone() for b in range(B)]
    cu = torch.tensor(_cu(lens), dtype=torch.int32, device="cuda")
    dw = _device_weights(Wt)  # held: the struct keeps only raw pointers
    nch = max(1, max((L + 63) // 64 for L in lens))
    kda.kda_block_prefill_varlen(kda.block_weights_struct(dw), h.cuda(), cu, B, nch, total, kda.ptr_array(hs),
                                 kda.ptr_array(cs), ws)
    torch.cuda.synchronize()
    return ws, _stages(ws, total, Wt), hs, cs


@pytest.mark.parametrize("hidden,H,D,rank,lens", [(256, 2, 64, 64, [70, 0, 1, 130, 64]),
                                                  (512, 4, 128, 128, [3, 200, 65])])
def test_block_prefill_varlen_matches_each_sequence_alone(hidden, H, D, rank, lens):
    """Packed sequences (one of them empty, one of one row, one exactly a chunk) from nonzero
    recurrent and conv states: every sequence's stages, states and outputs against the oracle
    on that sequence alone."""
    Wt = block_weights(hidden, H, D, rank, seed=31, std=0.05)
    B, total, cu = len(lens), sum(lens), _cu(lens)
    h = block_hidden(total, hidden, seed=31)
    hs0, cs0 = _states(B, H, D, seed=31)
    ws, got, hs, cs = _run_varlen(Wt, h, lens, hs0, cs0)
    for b in range(B):
        r0, L = cu[b], lens[b]
        if L == 0:
            assert torch.equal(hs[b], hs0[b].cuda()) and torch.equal(cs[b], cs0[b].cuda())
            continue
        sl = slice(r0, r0 + L)
        ref = oracle.block_prefill(Wt, h[sl], np64(hs0[b]), np64(cs0[b]))
        errs = {k_: rel_l2(np64(got[k_][sl]), ref[k_]) for k_ in ("qkv_proj", "conv_out", "g_raw", "out_gate",
                                                                   "o_norm_out", "final_out")}
        assert all(e <= TOL_BF16 for e in errs.values()), (b, errs)
        assert torch.equal(cs[b], _conv_after(cs0[b].cuda(), got["qkv_proj"][sl])), b
        assert rel_l2(np64(cs[b]), ref["conv_state"]) <= 4e-3, b
        _check_core(got, r0, L, Wt, hs0[b], got["core"][sl], hs[b], ref)
    ws.close()


def test_block_prefill_batched_equals_varlen_and_single_calls():
    """B equal-length sequences through kda_block_prefill_batched: the bits of the packed call with
    cu_seqlens = (0, T, 2T, ...), and each sequence within BF16 rounding of kda_block_prefill on it
    alone (the same stages; only the projection GEMM sees more rows)."""
    hidden, H, D, rank, B, T = 256, 2, 64, 64, 3, 50
    Wt = block_weights(hidden, H, D, rank, seed=33, std=0.05)
    h = block_hidden(B * T, hidden, seed=33)
    hs0, cs0 = _states(B, H, D, seed=33)
    ws_v, got_v, hs_v, cs_v = _run_varlen(Wt, h, [T] * B, hs0, cs0)
    ws = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=B * T, max_seqs=B)
    hs = [hs0[b].cuda().clone() for b in range(B)]
    cs = [cs0[b].cuda().clone() for b in range(B)]
    dw = _device_weights(Wt)
    st = kda.block_weights_struct(dw)
    kda.kda_block_prefill_batched(st, h.cuda(), B, T, kda.ptr_array(hs), kda.ptr_array(cs), ws)
    torch.cuda.synchronize()
    got = _stages(ws, B * T, Wt)
    assert torch.equal(got["final_out"], got_v["final_out"]) and torch.equal(got["core"], got_v["core"])
    assert all(torch.equal(hs[b], hs_v[b]) and torch.equal(cs[b], cs_v[b]) for b in range(B))
    one = kda.Workspace(kda.dims(H, D), hidden, rank, max_tokens=T)
    for b in range(B):
        h1, c1 = hs0[b].cuda().clone(), cs0[b].cuda().clone()
        kda.kda_block_prefill(st, h[b * T:(b + 1) * T].cuda().contiguous(), T, h1, c1, 0.0, one)
        torch.cuda.synchronize()
        f1 = one.view("final_out", (T, hidden), torch.bfloat16)
        assert rel_l2(np64(f1), np64(got["final_out"][b * T:(b + 1) * T])) <= 1e-2, b
        assert rel_l2(np64(h1), np64(hs[b])) <= 1e-3, b
    with pytest.raises(kda.KdaError):  # more sequences than the workspace was made for
        kda.kda_block_prefill_batched(st, h.cuda(), B + 1, 10, kda.ptr_array(hs + hs[:1]),
                                      kda.ptr_array(cs + cs[:1]), ws)
    one.close()
    ws.close()
    ws_v.close()


@pytest.mark.parametrize("hidden,H,D,rank,lens,acc", [
    (256, 2, 64, 64, [5, 1, 17], [3, 0, 17]),        # 23 rows: the matrix-vector projections
    (256, 2, 64, 64, [40, 3, 64, 0], [40, 1, 10, 0]),  # 107 rows: the GEMM projections; an empty draft
    (512, 4, 128, 128, [8, 8], [8, 2]),
])
def test_block_verify_then_fold(hidden, H, D, rank, lens, acc):
    """kda_block_verify leaves every state as it was and gives each draft row the output of the
    block prefill of that sequence's rows (oracle); kda_block_verify_fold then moves each
    recurrent state to the state after its accepted rows (oracle; and bit for bit decode_k's on
    the same stage rows for a row-by-row verify, within 1e-5 of the chunked prefill of those
    rows for a chunked one) and each conv state to the last three accepted inputs, bit for bit;
    accepted = 0 leaves both states."""
    Wt = block_weights(hidden, H, D, rank, seed=41, std=0.05)
    B, total, cu = len(lens), sum(lens), _cu(lens)
    d = kda.dims(H, D)
    h = block_hidden(total, hidden, seed=41)
    hs0, cs0 = _states(B, H, D, seed=41)
    ws = kda.Workspace(d, hidden, rank, max_tokens=total, max_seqs=B)
    hs = [hs0[b].cuda().clone() for b in range(B)]
    cs = [cs0[b].cuda().clone() for b in range(B)]
    hp, cp = kda.ptr_array(hs), kda.ptr_array(cs)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    tables = torch.empty(kda.kda_chunk_verify_tables_bytes(B, d) // 4, device="cuda")
    dw = _device_weights(Wt)
    st = kda.block_weights_struct(dw)
    kda.kda_block_verify(st, h.cuda(), cu_d, B, total, hp, cp, tables, ws)
    torch.cuda.synchronize()
    assert all(torch.equal(hs[b], hs0[b].cuda()) and torch.equal(cs[b], cs0[b].cuda()) for b in range(B))
    got = _stages(ws, total, Wt)
    by_rows = total <= 16 * B  # kda_block_verify's rule: short drafts run row by row
    for b in range(B):
        r0, L = cu[b], lens[b]
        if L == 0:
            continue
        sl = slice(r0, r0 + L)
        ref = oracle.block_prefill(Wt, h[sl], np64(hs0[b]), np64(cs0[b]))
        errs = {k_: rel_l2(np64(got[k_][sl]), ref[k_]) for k_ in ("conv_out", "g_raw", "o_norm_out", "final_out")}
        assert all(e <= TOL_BF16 for e in errs.values()), (b, errs)
        if by_rows:
            on, core, co, _, _ = _decode_k_rows(dw, got, sl, hs0[b], cs0[b], d)
            assert torch.equal(on, got["o_norm_out"][sl]) and torch.equal(co, got["conv_out"][sl]), b
            assert torch.equal(core, got["core"][sl]), b
        else:
            _check_core(got, r0, L, Wt, hs0[b], got["core"][sl], None, ref)
    kda.kda_block_verify_fold(cu_d, torch.tensor(acc, dtype=torch.int32, device="cuda"), B, total, tables, hp, cp,
                              ws)
    torch.cuda.synchronize()
    for b in range(B):
        r0, r = cu[b], acc[b]
        if r == 0:
            assert torch.equal(hs[b], hs0[b].cuda()) and torch.equal(cs[b], cs0[b].cuda()), b
            continue
        sl = slice(r0, r0 + r)
        assert torch.equal(cs[b], _conv_after(cs0[b].cuda(), got["qkv_proj"][sl])), b
        if by_rows:
            _, _, _, s_r, c_r = _decode_k_rows(dw, got, sl, hs0[b], cs0[b], d)
            assert torch.equal(hs[b], s_r) and torch.equal(cs[b], c_r), b
        else:
            _, s_r = _fused_core(got["conv_out"][sl], got["g_raw"][sl], got["beta"][sl], Wt, r, hs0[b])
            assert rel_l2(np64(hs[b]), np64(s_r)) <= 1e-5, b
        ref = oracle.block_prefill(Wt, h[sl], np64(hs0[b]), np64(cs0[b]))
        assert rel_l2(np64(hs[b]), ref["h_state"]) <= TOL_BF16, b
        assert rel_l2(np64(cs[b]), ref["conv_state"]) <= 4e-3, b
    ws.close()


def test_block_verify_refuses_a_draft_longer_than_a_chunk():
    """A sequence of 65 draft rows is skipped with KDA_ERR_INVALID_ARG latched; its states stay,
    and the other sequence of the call is verified as usual."""
    hidden, H, D, rank, lens = 256, 2, 64, 64, [65, 4]
    Wt = block_weights(hidden, H, D, rank, seed=43, std=0.05)
    B, total, cu = len(lens), sum(lens), _cu(lens)
    d = kda.dims(H, D)
    h = block_hidden(total, hidden, seed=43)
    hs0, cs0 = _states(B, H, D, seed=43)
    ws = kda.Workspace(d, hidden, rank, max_tokens=total, max_seqs=B)
    hs = [hs0[b].cuda().clone() for b in range(B)]
    cs = [cs0[b].cuda().clone() for b in range(B)]
    tables = torch.empty(kda.kda_chunk_verify_tables_bytes(B, d) // 4, device="cuda")
    dw = _device_weights(Wt)
    kda.kda_block_verify(kda.block_weights_struct(dw), h.cuda(), torch.tensor(cu, dtype=torch.int32, device="cuda"),
                         B, total, kda.ptr_array(hs), kda.ptr_array(cs), tables, ws)
    torch.cuda.synchronize()
    assert kda.device_status(clear=True) == KDA_ERR_INVALID_ARG
    assert all(torch.equal(hs[b], hs0[b].cuda()) and torch.equal(cs[b], cs0[b].cuda()) for b in range(B))
    got = _stages(ws, total, Wt)
    ref = oracle.block_prefill(Wt, h[65:69], np64(hs0[1]), np64(cs0[1]))
    assert rel_l2(np64(got["final_out"][65:69]), ref["final_out"]) <= TOL_BF16
    ws.close()


def test_block_verify_full_size_short_drafts():
    """hidden 4096, H 32, D 128, rank 128: 16 sequences x 4 draft rows run row by row, with
    o_proj's 32 weight tiles each splitting K = 4096 over four CTAs. Sampled sequences' stage
    buffers and block outputs against the oracle (2e-2), every sampled row's o_norm_out and core
    bit for bit kda_decode_k's on its stage rows, and both states untouched."""
    hidden, H, D, rank, B, K = 4096, 32, 128, 128, 16, 4
    Wt = block_weights(hidden, H, D, rank, seed=47, std=0.02)
    lens = [K] * B
    total, cu = B * K, _cu(lens)
    d = kda.dims(H, D)
    h = block_hidden(total, hidden, seed=47)
    hs0, cs0 = _states(B, H, D, seed=47)
    ws = kda.Workspace(d, hidden, rank, max_tokens=total, max_seqs=B)
    hs = [hs0[b].cuda().clone() for b in range(B)]
    cs = [cs0[b].cuda().clone() for b in range(B)]
    tables = torch.empty(kda.kda_chunk_verify_tables_bytes(B, d) // 4, device="cuda")
    dw = _device_weights(Wt)
    kda.kda_block_verify(kda.block_weights_struct(dw), h.cuda(), torch.tensor(cu, dtype=torch.int32, device="cuda"), B,
                         total, kda.ptr_array(hs), kda.ptr_array(cs), tables, ws)
    torch.cuda.synchronize()
    assert all(torch.equal(hs[b], hs0[b].cuda()) and torch.equal(cs[b], cs0[b].cuda()) for b in range(B))
    got = _stages(ws, total, Wt)
    for b in (0, 7, 15):
        sl = slice(cu[b], cu[b] + K)
        ref = oracle.block_prefill(Wt, h[sl], np64(hs0[b]), np64(cs0[b]))
        errs = {k_: rel_l2(np64(got[k_][sl]), ref[k_]) for k_ in ("conv_out", "g_raw", "o_norm_out", "final_out")}
        assert all(e <= TOL_BF16 for e in errs.values()), (b, errs)
        on, core, _, _, _ = _decode_k_rows(dw, got, sl, hs0[b], cs0[b], d)
        assert torch.equal(on, got["o_norm_out"][sl]) and torch.equal(core, got["core"][sl]), b
    ws.close()


def test_block_fold_without_a_row_route_verify_refuses():
    """A fold whose (B, total) picks the row-by-row route, on a workspace where no such verify ran,
    is refused (KDA_ERR_INVALID_ARG) before any launch: both states stay."""
    hidden, H, D, rank, lens = 256, 2, 64, 64, [3, 2]
    B, total, cu = len(lens), sum(lens), _cu(lens)
    d = kda.dims(H, D)
    hs0, cs0 = _states(B, H, D, seed=49)
    ws = kda.Workspace(d, hidden, rank, max_tokens=total, max_seqs=B)
    hs = [hs0[b].cuda().clone() for b in range(B)]
    cs = [cs0[b].cuda().clone() for b in range(B)]
    tables = torch.empty(kda.kda_chunk_verify_tables_bytes(B, d) // 4, device="cuda")
    with pytest.raises(kda.KdaError) as err:
        kda.kda_block_verify_fold(torch.tensor(cu, dtype=torch.int32, device="cuda"),
                                  torch.tensor([1, 1], dtype=torch.int32, device="cuda"), B, total, tables,
                                  kda.ptr_array(hs), kda.ptr_array(cs), ws)
    assert err.value.status == KDA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert all(torch.equal(hs[b], hs0[b].cuda()) and torch.equal(cs[b], cs0[b].cuda()) for b in range(B))
    ws.close()
