"""The C-ABI library without a GPU: it loads, exports every symbol include/kda.h declares,
and rejects bad arguments on the host before anything reaches the device."""
import ctypes

import pytest

import kda_gated_delta_gate_b200 as kda

BOGUS = 0x10000  # never dereferenced: every case below fails validation first


@pytest.fixture(scope="module")
def L():
    from kda_gated_delta_gate_b200 import build
    build.build()
    return kda.lib()


def test_exports_every_declared_symbol(L):
    names = kda.header_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(kda._SIGS), "binding and header disagree"


def test_version_status_tpad(L):
    assert L.kda_version() >= 100
    for s in range(8):
        assert L.kda_status_string(s)
    assert L.kda_status_string(99) == b"unknown status"
    assert [kda.t_pad(t) for t in (0, 1, 63, 64, 65, 65500, 4096)] == [0, 64, 64, 64, 128, 65536, 4096]


def _d(**kw):
    base = dict(heads=2, head_dim=64)
    base.update(kw)
    return kda.dims(**base)


def test_gate_argument_checks(L):
    rc = L.kda_gate(None, BOGUS, BOGUS, BOGUS, 4, ctypes.byref(_d()), None)
    assert rc == 1
    assert L.kda_gate(BOGUS, BOGUS, BOGUS, BOGUS, 4, ctypes.byref(_d(head_dim=96)), None) == 4
    assert L.kda_gate(BOGUS, BOGUS, BOGUS, BOGUS, 4, ctypes.byref(_d(chunk=32)), None) == 4
    assert L.kda_gate(BOGUS + 2, BOGUS, BOGUS, BOGUS, 4, ctypes.byref(_d()), None) == 7
    assert L.kda_gate(BOGUS, BOGUS, BOGUS, BOGUS, -1, ctypes.byref(_d()), None) == 1
    assert L.kda_gate(BOGUS, BOGUS, BOGUS, BOGUS, 0, ctypes.byref(_d()), None) == 0  # empty: nothing runs
    assert L.kda_gate(BOGUS, BOGUS, BOGUS, BOGUS, 4, None, None) == 1


def test_prefill_argument_checks(L):
    d = ctypes.byref(_d())
    args = [BOGUS] * 7
    need = L.kda_chunk_prefill_scratch_bytes(2, 100, d)
    # B * H * chunks operand packs (D = 64: [W; Q o A], M, K o e^{Gamma_C - Gamma} as BF16 hi/lo
    # tiles, U~ in FP32 with a 4-float row skew, e^{Gamma_C}) + the list of chunks handed to the
    # CUDA-core path
    assert need == 2 * 2 * 2 * (32768 + 16384 + 16384 + 2 * 64 * 36 * 4 + 1024) + 256
    assert L.kda_chunk_prefill_scratch_bytes(0, 100, d) == 0
    assert L.kda_chunk_prefill(*args, 1, 0, BOGUS, 0, d, None) == 0  # T = 0: nothing to do
    assert L.kda_chunk_prefill(*args, 0, 10, BOGUS, 0, d, None) == 0  # B = 0
    assert L.kda_chunk_prefill(*args, -1, 10, BOGUS, need, d, None) == 1
    assert L.kda_chunk_prefill(*args, 2, 100, BOGUS, need - 16, d, None) == 3  # scratch too small
    assert L.kda_chunk_prefill(*args, 2, 100, None, need, d, None) == 1
    assert L.kda_chunk_prefill(*args, 2, 100, BOGUS + 8, need, d, None) == 7
    bad = list(args)
    bad[5] = None
    assert L.kda_chunk_prefill(*bad, 1, 10, BOGUS, need, d, None) == 1
    bad = list(args)
    bad[6] = BOGUS + 4
    assert L.kda_chunk_prefill(*bad, 1, 10, BOGUS, need, d, None) == 7
    assert L.kda_chunk_prefill_simt(*args, 1, 10, ctypes.byref(_d(head_dim=32)), None) == 4


def test_decode_alias_and_snapshot_checks(L):
    d = ctypes.byref(_d())
    g_raw = BOGUS
    out_gate = BOGUS + 64  # overlaps g_raw's [N, H*D] BF16 range
    rc = L.kda_decode_fused(BOGUS, BOGUS, BOGUS, g_raw, BOGUS, BOGUS, BOGUS, BOGUS, out_gate, BOGUS, BOGUS,
                            None, None, 2, d, None)
    assert rc == 2
    far = BOGUS + (1 << 20)
    common = [BOGUS, BOGUS, BOGUS, g_raw, BOGUS, BOGUS, BOGUS, BOGUS, far, BOGUS, BOGUS, None, None]
    assert L.kda_decode_k(*common, 0, None, None, 0, d, None) == 1          # K < 1
    assert L.kda_decode_k(*common, 40, None, None, 39, d, None) == 1       # K > 32 is taken; snapshots missing
    assert L.kda_decode_k(*common, 4, None, None, 2, d, None) == 1          # n_snap not 0 or K-1
    assert L.kda_decode_k(*common, 4, None, None, 3, d, None) == 1          # snapshots missing
    assert L.kda_recurrent_decode(*([BOGUS] * 7), -3, d, None) == 1


def test_host_prefill_argument_checks(L):
    d = ctypes.byref(_d())
    # staging rows (T_pad = 128) for qkv, g_raw, beta, core, the state, the slot, one segment's scratch
    hd, tp = 2 * 64, 128
    r256 = lambda x: (x + 255) // 256 * 256
    seg_scratch = L.kda_chunk_prefill_scratch_bytes(1, 64, d)
    need = (r256(tp * 3 * hd * 2) + r256(tp * hd * 2) + r256(tp * 2 * 4) + r256(tp * hd * 4) + r256(hd * 64 * 4)
            + 256 + r256(seg_scratch))
    assert L.kda_chunk_prefill_host_bytes(100, 64, d) == need
    assert L.kda_chunk_prefill_host_bytes(100, 96, d) == 0  # not whole chunks
    assert L.kda_chunk_prefill_host_bytes(0, 64, d) == 0
    args = [BOGUS] * 7
    assert L.kda_chunk_prefill_host(*args, 0, 64, BOGUS, 0, d, None) == 0  # T = 0: nothing to do
    assert L.kda_chunk_prefill_host(*args, 100, 0, BOGUS, need, d, None) == 1
    assert L.kda_chunk_prefill_host(*args, 100, 100, BOGUS, need, d, None) == 1
    assert L.kda_chunk_prefill_host(*args, -1, 64, BOGUS, need, d, None) == 1
    assert L.kda_chunk_prefill_host(*args, 100, 64, None, need, d, None) == 1
    assert L.kda_chunk_prefill_host(*args, 100, 64, BOGUS + 8, need, d, None) == 7
    assert L.kda_chunk_prefill_host(*args, 100, 64, BOGUS, need - 16, d, None) == 3
    bad = list(args)
    bad[5] = None
    assert L.kda_chunk_prefill_host(*bad, 100, 64, BOGUS, need, d, None) == 1
    assert L.kda_chunk_prefill_host(*args, 100, 64, BOGUS, need, ctypes.byref(_d(head_dim=96)), None) == 4


def test_graph_argument_checks(L):
    out = ctypes.c_void_p(BOGUS)
    assert L.kda_block_decode_graph(BOGUS, BOGUS, 1, BOGUS, BOGUS, BOGUS, None) == 1
    assert L.kda_block_decode_graph(BOGUS, BOGUS, 0, BOGUS, BOGUS, BOGUS, ctypes.byref(out)) == 1
    assert out.value is None  # cleared on error
    assert L.kda_block_decode_graph(None, BOGUS, 1, BOGUS, BOGUS, BOGUS, ctypes.byref(out)) == 1
    assert L.kda_graph_launch(None, None) == 1
    assert L.kda_graph_destroy(None) == 0


def test_front_back_argument_checks(L):
    d = ctypes.byref(_d())
    assert L.kda_front_conv_silu_l2(BOGUS, BOGUS, BOGUS, BOGUS, BOGUS, None, None, 0.0, 8, d, None) == 1
    assert L.kda_front_conv_silu_l2(BOGUS, BOGUS, BOGUS, BOGUS, None, None, None, 0.0, 0, d, None) == 0
    assert L.kda_back_gated_rmsnorm(BOGUS, BOGUS, BOGUS, BOGUS + 8, 8, d, None) == 7
    assert L.kda_back_gated_rmsnorm(None, BOGUS, BOGUS, BOGUS, 8, d, None) == 1


def test_binding_raises_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(kda, "_lib", None)
    monkeypatch.setattr(kda, "LIB_PATH", str(tmp_path / "libkda.so"))
    with pytest.raises(ImportError):
        kda.lib()


def test_packed_block_argument_checks(L):
    """The packed-sequence block calls, the batched verify and the fold refuse bad arguments
    before any launch (no device memory is touched)."""
    d = _d()
    dp = ctypes.byref(d)
    ws = ctypes.c_void_p()
    assert L.kda_workspace_create_batched(dp, 256, 64, 128, 0, ctypes.byref(ws)) == 1       # max_seqs 0
    assert L.kda_workspace_create_batched(dp, 256, 64, 0, 2, ctypes.byref(ws)) == 1         # max_tokens 0
    assert L.kda_workspace_create_batched(dp, 200, 64, 128, 2, ctypes.byref(ws)) == 4       # hidden % 64
    assert L.kda_workspace_max_seqs(None) == 0
    assert L.kda_block_prefill_varlen(None, BOGUS, BOGUS, 2, 1, 100, BOGUS, BOGUS, None, None) == 1
    assert L.kda_block_prefill_batched(None, BOGUS, 2, 50, BOGUS, BOGUS, None, None) == 1
    assert L.kda_block_verify(None, BOGUS, BOGUS, 2, 10, BOGUS, BOGUS, BOGUS, 1 << 20, None, None) == 1
    assert L.kda_block_verify_fold(BOGUS, BOGUS, 2, 10, BOGUS, BOGUS, BOGUS, None, None) == 1   # no workspace
    assert L.kda_front_conv_silu_l2_varlen(BOGUS, BOGUS, BOGUS, BOGUS, None, 2, 10, 1, dp, None) == 1
    assert L.kda_front_conv_silu_l2_varlen(BOGUS + 8, BOGUS, BOGUS, BOGUS, BOGUS, 2, 10, 1, dp, None) == 7
    assert L.kda_front_conv_silu_l2_varlen(BOGUS, BOGUS, BOGUS, BOGUS, BOGUS, 0, 0, 1, dp, None) == 0
    assert L.kda_conv_state_fold(BOGUS, BOGUS, BOGUS, BOGUS, -1, 10, dp, None) == 1
    assert L.kda_conv_state_fold(BOGUS, BOGUS, BOGUS, BOGUS, 0, 10, dp, None) == 0


def test_packed_scratch_bounds(L):
    """The compact chunk-slot layout: a head needs ceil(total / 64) + B - 1 pack slots, never more
    than the one-slot-per-(sequence, chunk) layout asks for a long enough max_num_chunks."""
    d = ctypes.byref(_d())
    one = L.kda_chunk_prefill_scratch_bytes(1, 64, d)          # one chunk per head, plus the list
    for seqs, total in [(1, 64), (1, 4096), (8, 4096), (64, 100), (3, 1)]:
        slots = -(-total // 64) + seqs - 1
        got = L.kda_chunk_prefill_packed_scratch_bytes(seqs, total, d)
        assert got == L.kda_chunk_prefill_varlen_scratch_bytes(1, slots, d), (seqs, total)
        assert got >= one
    # a single sequence: the same bytes as the equal-length call of that length
    assert L.kda_chunk_prefill_packed_scratch_bytes(1, 1000, d) == L.kda_chunk_prefill_scratch_bytes(1, 1000, d)
    assert L.kda_chunk_prefill_packed_scratch_bytes(0, 10, d) == 0
