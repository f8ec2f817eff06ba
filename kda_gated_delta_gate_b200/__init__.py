"""Python binding of libkda.so, the B200 KDA core library (C ABI: include/kda.h).

Argument marshalling only: every function here passes device pointers, sizes and the
current CUDA stream to the C entry point of the same name; all computation happens in
the library's sm_100a kernels. PyTorch supplies device memory and streams.

There is no fallback: if libkda.so is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Iterable, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "kda.h")

KDA_OK = 0
STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_ALIAS", 3: "KDA_ERR_CAPACITY",
          4: "KDA_ERR_UNSUPPORTED", 5: "KDA_ERR_CUDA", 6: "KDA_ERR_TIMEOUT", 7: "KDA_ERR_MISALIGNED"}


class KdaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


class KdaDims(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("chunk", ctypes.c_int),
                ("scale", ctypes.c_float), ("l2_eps", ctypes.c_float), ("rms_eps", ctypes.c_float)]


def dims(heads: int, head_dim: int, chunk: int = 64, scale: float = 1.0, l2_eps: float = 1e-6,
         rms_eps: float = 1e-6) -> KdaDims:
    return KdaDims(heads, head_dim, chunk, scale, l2_eps, rms_eps)


class KdaBlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q_proj", "k_proj", "v_proj", "conv", "f_a", "f_b", "dt_bias",
                                                  "a_log", "b_proj", "g_a", "g_b", "o_norm", "o_proj")] + \
               [("hidden", ctypes.c_int), ("rank", ctypes.c_int)]


# workspace stage buffers (include/kda.h, KDA_BUF_*)
BUFFERS = ("qkv_proj", "conv_out", "q_f32", "k_f32", "v_f32", "gate", "beta", "core", "g_raw", "out_gate",
           "o_norm_out", "final_out", "f_a_out", "g_a_out", "prefill_scratch")

_lib = None
_VP = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_DIMS = ctypes.POINTER(KdaDims)

_SIGS = {
    "kda_version": ([], _I),
    "kda_status_string": ([_I], ctypes.c_char_p),
    "kda_t_pad": ([ctypes.c_size_t, _I], ctypes.c_size_t),
    "kda_device_status": ([ctypes.POINTER(_I), _I], _I),
    "kda_gate": ([_VP, _VP, _VP, _VP, _I, _DIMS, _VP], _I),
    "kda_beta": ([_VP, _VP, _I, _VP], _I),
    "kda_chunk_prefill": ([_VP] * 7 + [_I, _I, _VP, ctypes.c_size_t, _DIMS, _VP], _I),
    "kda_chunk_prefill_scratch_bytes": ([_I, _I, _DIMS], ctypes.c_size_t),
    "kda_chunk_prefill_fused": ([_VP] * 7 + [_I, _I, _VP, ctypes.c_size_t, _DIMS, _VP], _I),
    "kda_chunk_prefill_graw": ([_VP] * 9 + [_I, _I, _VP, ctypes.c_size_t, _DIMS, _VP], _I),
    "kda_chunk_prefill_host": ([_VP] * 7 + [_I, _I, _VP, ctypes.c_size_t, _DIMS, _VP], _I),
    "kda_chunk_prefill_host_bytes": ([_I, _I, _DIMS], ctypes.c_size_t),
    "kda_chunk_prefill_host_f32": ([_VP] * 9 + [_I, _I, _VP, ctypes.c_size_t, _DIMS, _VP], _I),
    "kda_chunk_prefill_host_f32_bytes": ([_I, _I, _DIMS], ctypes.c_size_t),
    "kda_chunk_prefill_varlen": ([_VP] * 6 + [_I, _I, _I, _VP, _VP, _VP, ctypes.c_size_t, _DIMS, _VP], _I),
    "kda_chunk_prefill_varlen_scratch_bytes": ([_I, _I, _DIMS], ctypes.c_size_t),
    "kda_chunk_verify": ([_VP] * 6 + [_I, _I, _VP, _VP, _VP, ctypes.c_size_t, _VP, ctypes.c_size_t, _DIMS, _VP], _I),
    "kda_chunk_verify_tables_bytes": ([_I, _DIMS], ctypes.c_size_t),
    "kda_chunk_verify_fold": ([_VP, _VP, _VP, _I, _I, _VP, _VP, _DIMS, _VP], _I),
    "kda_chunk_prefill_simt": ([_VP] * 7 + [_I, _I, _DIMS, _VP], _I),
    "kda_chunk_prefill_noalloc": ([_VP] * 7 + [_I, _I, _DIMS, _VP], _I),
    "kda_chunk_prefill_noalloc_max_scratch_bytes": ([], ctypes.c_size_t),
    "kda_recurrent_decode": ([_VP] * 7 + [_I, _DIMS, _VP], _I),
    "kda_decode_fused": ([_VP] * 13 + [_I, _DIMS, _VP], _I),
    "kda_decode_k": ([_VP] * 13 + [_I, _VP, _VP, _I, _DIMS, _VP], _I),
    "kda_front_conv_silu_l2": ([_VP] * 7 + [_F, _I, _DIMS, _VP], _I),
    "kda_back_gated_rmsnorm": ([_VP] * 4 + [_I, _DIMS, _VP], _I),
    "kda_gemm_bf16": ([_VP, _I, _VP, _I, _VP, _I, _I, _I, _I, _I, _VP], _I),
    "kda_workspace_create": ([_DIMS, _I, _I, ctypes.c_size_t, ctypes.POINTER(_VP)], _I),
    "kda_workspace_destroy": ([_VP], _I),
    "kda_workspace_max_tokens": ([_VP], ctypes.c_size_t),
    "kda_workspace_buffer": ([_VP, _I, ctypes.POINTER(_VP), ctypes.POINTER(ctypes.c_size_t)], _I),
    "kda_block_prefill": ([_VP, _VP, _I, _VP, _VP, _F, _VP, _VP], _I),
    "kda_block_decode": ([_VP, _VP, _I, _VP, _VP, _VP, _VP], _I),
    "kda_gemv_bf16": ([_VP, _I, _VP, _I, _VP, _I, _I, _I, _I, _I, _VP], _I),
    "kda_block_decode_k": ([_VP, _VP, _I, _VP, _VP, _VP, _VP, _I, _VP, _VP], _I),
    "kda_block_decode_graph": ([_VP, _VP, _I, _VP, _VP, _VP, ctypes.POINTER(_VP)], _I),
    "kda_graph_launch": ([_VP, _VP], _I),
    "kda_graph_destroy": ([_VP], _I),
    "kda_chunk_prefill_packed_scratch_bytes": ([_I, _I, _DIMS], ctypes.c_size_t),
    "kda_front_conv_silu_l2_varlen": ([_VP] * 5 + [_I, _I, _I, _DIMS, _VP], _I),
    "kda_conv_state_fold": ([_VP] * 4 + [_I, _I, _DIMS, _VP], _I),
    "kda_workspace_create_batched": ([_DIMS, _I, _I, ctypes.c_size_t, _I, ctypes.POINTER(_VP)], _I),
    "kda_workspace_max_seqs": ([_VP], _I),
    "kda_block_prefill_varlen": ([_VP, _VP, _VP, _I, _I, _I, _VP, _VP, _VP, _VP], _I),
    "kda_block_prefill_batched": ([_VP, _VP, _I, _I, _VP, _VP, _VP, _VP], _I),
    "kda_block_verify": ([_VP, _VP, _VP, _I, _I, _VP, _VP, _VP, ctypes.c_size_t, _VP, _VP], _I),
    "kda_block_verify_fold": ([_VP, _VP, _I, _I, _VP, _VP, _VP, _VP, _VP], _I),
}


def lib():
    """Load libkda.so (built in-tree by kda_gated_delta_gate_b200.build). Raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kda_gated_delta_gate_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def header_symbols() -> list:
    """Every function name include/kda.h declares."""
    with open(HEADER_PATH) as f:
        return re.findall(r"^KDA_API\s+[\w\s\*]*?\b(kda_\w+)\s*\(", f.read(), flags=re.M)


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _call(name: str, *args) -> int:
    rc = getattr(lib(), name)(*args)
    if rc != KDA_OK:
        raise KdaError(name, rc)
    return rc


def ptr_array(tensors: Sequence, device="cuda"):
    """Device int64 tensor holding the data pointers of `tensors` (a `T* const*` argument)."""
    import torch
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def host_ptr_array(tensors: Iterable):
    ts = list(tensors)
    return (ctypes.c_void_p * max(1, len(ts)))(*[t.data_ptr() for t in ts])


def t_pad(T: int, chunk: int = 64) -> int:
    return int(lib().kda_t_pad(T, chunk))


# One scratch buffer per (device, stream), grown on demand and kept: the chunked prefill, varlen
# and verify wrappers take it when the caller passes no `scratch`, so a hot call allocates only
# the first time it needs more bytes on that stream. Calls on one stream are ordered, so they may
# share its buffer; calls on different streams never do.
_SCRATCH = {}


def scratch_buffer(nbytes: int, device, stream_handle: int):
    """The cached scratch of (device, stream): a uint8 device tensor of at least nbytes."""
    import torch
    dev = torch.device(device)
    key = (dev.index if dev.index is not None else torch.cuda.current_device(), int(stream_handle))
    buf = _SCRATCH.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=dev)
        _SCRATCH[key] = buf
    return buf


def device_status(clear: bool = True) -> int:
    out = ctypes.c_int(0)
    _call("kda_device_status", ctypes.byref(out), 1 if clear else 0)
    return out.value


# ----------------------------------------------------------------------------- entry points

def kda_gate(g_raw, dt_bias, a_log, gate, n_rows: int, d: KdaDims, stream=None):
    return _call("kda_gate", _p(g_raw), _p(dt_bias), _p(a_log), _p(gate), n_rows, ctypes.byref(d), _stream(stream))


def kda_beta(b_logit, beta, n: int, stream=None):
    return _call("kda_beta", _p(b_logit), _p(beta), n, _stream(stream))


def kda_chunk_prefill_scratch_bytes(B: int, T: int, d: KdaDims) -> int:
    return int(lib().kda_chunk_prefill_scratch_bytes(B, T, ctypes.byref(d)))


def kda_chunk_prefill(q, k, v, gate, beta, h_state_ptrs, core, B: int, T: int, d: KdaDims, stream=None,
                      impl: str = "tc", scratch=None):
    """impl "tc": the tensor-core path (needs `scratch`, a device buffer of at least
    kda_chunk_prefill_scratch_bytes bytes; the stream's cached buffer when None). impl "simt":
    the CUDA-core path (no scratch)."""
    if impl == "simt":
        return _call("kda_chunk_prefill_simt", _p(q), _p(k), _p(v), _p(gate), _p(beta), _p(h_state_ptrs), _p(core),
                     B, T, ctypes.byref(d), _stream(stream))
    st = _stream(stream)
    if scratch is None:
        scratch = scratch_buffer(kda_chunk_prefill_scratch_bytes(B, T, d), core.device, st)
    return _call("kda_chunk_prefill", _p(q), _p(k), _p(v), _p(gate), _p(beta), _p(h_state_ptrs), _p(core), B, T,
                 _p(scratch), scratch.numel() * scratch.element_size(), ctypes.byref(d), st)


def kda_chunk_prefill_fused(qkv, g_raw, dt_bias, a_log, beta, h_state_ptrs, core, B: int, T: int, d: KdaDims,
                            stream=None, scratch=None):
    """The chunked prefill on the front end's BF16 q|k|v rows and the raw BF16 gate input
    (the gate is formed in the kernel). `scratch` as for kda_chunk_prefill."""
    st = _stream(stream)
    if scratch is None:
        scratch = scratch_buffer(kda_chunk_prefill_scratch_bytes(B, T, d), core.device, st)
    return _call("kda_chunk_prefill_fused", _p(qkv), _p(g_raw), _p(dt_bias), _p(a_log), _p(beta), _p(h_state_ptrs),
                 _p(core), B, T, _p(scratch), scratch.numel() * scratch.element_size(), ctypes.byref(d), st)


def kda_chunk_prefill_graw(q, k, v, g_raw, dt_bias, a_log, beta, h_state_ptrs, core, B: int, T: int, d: KdaDims,
                           stream=None, scratch=None):
    """kda_chunk_prefill on FP32 q, k, v with the gate formed in the kernel from the raw BF16
    g_raw, dt_bias and a_log (bit-identical to kda_gate + kda_chunk_prefill)."""
    st = _stream(stream)
    if scratch is None:
        scratch = scratch_buffer(kda_chunk_prefill_scratch_bytes(B, T, d), core.device, st)
    return _call("kda_chunk_prefill_graw", _p(q), _p(k), _p(v), _p(g_raw), _p(dt_bias), _p(a_log), _p(beta),
                 _p(h_state_ptrs), _p(core), B, T, _p(scratch), scratch.numel() * scratch.element_size(),
                 ctypes.byref(d), st)


def kda_chunk_prefill_host_bytes(T: int, segment_tokens: int, d: KdaDims) -> int:
    return int(lib().kda_chunk_prefill_host_bytes(T, segment_tokens, ctypes.byref(d)))


def kda_chunk_prefill_host(qkv, g_raw, b_logit, dt_bias, a_log, h_state, core, T: int, segment_tokens: int,
                           device_buffer, d: KdaDims, stream=None):
    """kda_beta + kda_chunk_prefill_fused on HOST (pinned) qkv, g_raw, b_logit, h_state and core,
    copies and compute of consecutive segments overlapped. Outputs are complete once `stream`
    has completed. `device_buffer`: a device tensor of kda_chunk_prefill_host_bytes bytes."""
    return _call("kda_chunk_prefill_host", _p(qkv), _p(g_raw), _p(b_logit), _p(dt_bias), _p(a_log), _p(h_state),
                 _p(core), T, segment_tokens, _p(device_buffer), device_buffer.numel() * device_buffer.element_size(),
                 ctypes.byref(d), _stream(stream))


def kda_chunk_prefill_host_f32_bytes(T: int, segment_tokens: int, d: KdaDims) -> int:
    return int(lib().kda_chunk_prefill_host_f32_bytes(T, segment_tokens, ctypes.byref(d)))


def kda_chunk_prefill_host_f32(q, k, v, g_raw, b_logit, dt_bias, a_log, h_state, core, T: int, segment_tokens: int,
                               device_buffer, d: KdaDims, stream=None):
    """kda_gate + kda_beta + kda_chunk_prefill on HOST (pinned) FP32 q, k, v, BF16 g_raw, FP32
    b_logit, h_state and core, copies and compute of consecutive segments overlapped.
    `device_buffer`: a device tensor of kda_chunk_prefill_host_f32_bytes bytes."""
    return _call("kda_chunk_prefill_host_f32", _p(q), _p(k), _p(v), _p(g_raw), _p(b_logit), _p(dt_bias), _p(a_log),
                 _p(h_state), _p(core), T, segment_tokens, _p(device_buffer),
                 device_buffer.numel() * device_buffer.element_size(), ctypes.byref(d), _stream(stream))


def kda_chunk_prefill_noalloc(q, k, v, gate, beta, h_state_ptrs, core, B: int, T: int, d: KdaDims, stream=None):
    """kda_chunk_prefill without a scratch argument, for callers that cannot allocate: the
    library's own 32 MiB device array is used (calls must not overlap on the GPU)."""
    return _call("kda_chunk_prefill_noalloc", _p(q), _p(k), _p(v), _p(gate), _p(beta), _p(h_state_ptrs), _p(core),
                 B, T, ctypes.byref(d), _stream(stream))


def kda_recurrent_decode(q, k, v, gate, beta, h_state_ptrs, o, N: int, d: KdaDims, stream=None):
    return _call("kda_recurrent_decode", _p(q), _p(k), _p(v), _p(gate), _p(beta), _p(h_state_ptrs), _p(o), N,
                 ctypes.byref(d), _stream(stream))


def kda_decode_fused(x, conv_state_ptrs, conv_w, g_raw, dt_bias, a_log, b_logit, h_state_ptrs, out_gate,
                     o_norm_w, o_norm_out, conv_out, core, N: int, d: KdaDims, stream=None):
    return _call("kda_decode_fused", _p(x), _p(conv_state_ptrs), _p(conv_w), _p(g_raw), _p(dt_bias), _p(a_log),
                 _p(b_logit), _p(h_state_ptrs), _p(out_gate), _p(o_norm_w), _p(o_norm_out), _p(conv_out), _p(core),
                 N, ctypes.byref(d), _stream(stream))


def kda_decode_k(x, conv_state, conv_w, g_raw, dt_bias, a_log, b_logit, h_state, out_gate, o_norm_w, o_norm_out,
                 conv_out, core, K: int, h_snaps: Sequence, conv_snaps: Sequence, d: KdaDims, stream=None):
    n = len(h_snaps)
    hs = host_ptr_array(h_snaps) if n else None
    cs = host_ptr_array(conv_snaps) if n else None
    return _call("kda_decode_k", _p(x), _p(conv_state), _p(conv_w), _p(g_raw), _p(dt_bias), _p(a_log), _p(b_logit),
                 _p(h_state), _p(out_gate), _p(o_norm_w), _p(o_norm_out), _p(conv_out), _p(core), K,
                 ctypes.cast(hs, _VP) if hs is not None else None, ctypes.cast(cs, _VP) if cs is not None else None,
                 n, ctypes.byref(d), _stream(stream))


def kda_front_conv_silu_l2(x, conv_state, conv_w, conv_out, q_f32, k_f32, v_f32, pad_fill: float, T: int,
                           d: KdaDims, stream=None):
    return _call("kda_front_conv_silu_l2", _p(x), _p(conv_state), _p(conv_w), _p(conv_out), _p(q_f32), _p(k_f32),
                 _p(v_f32), float(pad_fill), T, ctypes.byref(d), _stream(stream))


def kda_back_gated_rmsnorm(core, out_gate, w, out, T: int, d: KdaDims, stream=None):
    return _call("kda_back_gated_rmsnorm", _p(core), _p(out_gate), _p(w), _p(out), T, ctypes.byref(d),
                 _stream(stream))


def kda_gemm_bf16(A, W, C, M: int, N: int, K: int, *, lda=None, ldw=None, ldc=None, stream=None):
    """C[M x N] = A[M x K] . W[N x K]^T (BF16 in, FP32 accumulate); C's dtype picks the output."""
    import torch
    out_f32 = 1 if C.dtype == torch.float32 else 0
    return _call("kda_gemm_bf16", _p(A), lda if lda is not None else A.stride(0), _p(W),
                 ldw if ldw is not None else W.stride(0), _p(C), ldc if ldc is not None else C.stride(0), M, N, K,
                 out_f32, _stream(stream))


def block_weights_struct(w) -> KdaBlockWeights:
    """KdaBlockWeights from an object with device tensors q_proj, ..., o_proj and ints hidden, rank.
    The struct holds raw pointers only: keep `w` (and its tensors) alive while calls use it."""
    return KdaBlockWeights(*[_p(getattr(w, n)) for n in ("q_proj", "k_proj", "v_proj", "conv", "f_a", "f_b",
                                                          "dt_bias", "a_log", "b_proj", "g_a", "g_b", "o_norm",
                                                          "o_proj")], w.hidden, w.rank)


class Workspace:
    """The block's stage buffers, allocated once for max_tokens rows and, for packed calls
    (kda_block_prefill_varlen / _batched, kda_block_verify), max_seqs sequences
    (kda_workspace_create_batched; max_seqs = 1 is kda_workspace_create)."""

    def __init__(self, d: KdaDims, hidden: int, rank: int, max_tokens: int, max_seqs: int = 1):
        self.dims = d
        self._h = ctypes.c_void_p()
        _call("kda_workspace_create_batched", ctypes.byref(d), hidden, rank, max_tokens, max_seqs,
              ctypes.byref(self._h))

    @property
    def handle(self):
        return self._h

    def buffer(self, name: str):
        """(device pointer, bytes) of a stage buffer."""
        ptr, nb = ctypes.c_void_p(), ctypes.c_size_t()
        _call("kda_workspace_buffer", self._h, BUFFERS.index(name), ctypes.byref(ptr), ctypes.byref(nb))
        return ptr.value, nb.value

    def view(self, name: str, shape, dtype):
        """A torch view of (the front of) a stage buffer; the workspace must outlive it."""
        import torch
        ptr, nb = self.buffer(name)
        n = 1
        for x in shape:
            n *= x
        es = torch.empty((), dtype=dtype).element_size()
        assert n * es <= nb
        return _device_view(ptr, shape, dtype)

    def close(self):
        if self._h:
            lib().kda_workspace_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _device_view(ptr: int, shape, dtype):
    """Wrap device memory owned by the library as a torch tensor (no copy, no ownership)."""
    import torch

    class _Holder:
        def __init__(self, p, nbytes):
            self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (p, False),
                                             "version": 3, "strides": None}

    n = 1
    for x in shape:
        n *= x
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    raw = torch.as_tensor(_Holder(ptr, nbytes), device="cuda")
    return raw.view(dtype).view(tuple(shape))


def kda_block_prefill(weights: KdaBlockWeights, hidden, T: int, h_state, conv_state, pad_fill: float,
                      ws: Workspace, stream=None):
    return _call("kda_block_prefill", ctypes.byref(weights), _p(hidden), T, _p(h_state), _p(conv_state),
                 float(pad_fill), ws.handle, _stream(stream))


def kda_block_decode(weights: KdaBlockWeights, hidden, N: int, h_state_ptrs, conv_state_ptrs, ws: Workspace,
                     stream=None):
    """N sequences x 1 token through the whole block; h_state_ptrs / conv_state_ptrs are device
    int64 arrays of N pointers (ptr_array). The output is in ws buffer "final_out"."""
    return _call("kda_block_decode", ctypes.byref(weights), _p(hidden), N, _p(h_state_ptrs), _p(conv_state_ptrs),
                 ws.handle, _stream(stream))


def kda_block_decode_k(weights: KdaBlockWeights, hidden, K: int, h_state, conv_state, h_snaps: Sequence,
                       conv_snaps: Sequence, ws: Workspace, stream=None):
    """K rows of one sequence through the whole block (snapshots after every row but the last)."""
    n = len(h_snaps)
    hs = host_ptr_array(h_snaps) if n else None
    cs = host_ptr_array(conv_snaps) if n else None
    return _call("kda_block_decode_k", ctypes.byref(weights), _p(hidden), K, _p(h_state), _p(conv_state),
                 ctypes.cast(hs, _VP) if hs is not None else None, ctypes.cast(cs, _VP) if cs is not None else None,
                 n, ws.handle, _stream(stream))


def kda_block_prefill_varlen(weights: KdaBlockWeights, hidden, cu_seqlens, B: int, max_num_chunks: int,
                             total_tokens: int, h_state_ptrs, conv_state_ptrs, ws: Workspace, stream=None):
    """B packed sequences (cu_seqlens: device int32 [B+1]) through the whole block; the states are
    device pointer arrays (ptr_array), carried and updated. Output in ws buffer "final_out"."""
    return _call("kda_block_prefill_varlen", ctypes.byref(weights), _p(hidden), _p(cu_seqlens), B, max_num_chunks,
                 total_tokens, _p(h_state_ptrs), _p(conv_state_ptrs), ws.handle, _stream(stream))


def kda_block_prefill_batched(weights: KdaBlockWeights, hidden, B: int, T: int, h_state_ptrs, conv_state_ptrs,
                              ws: Workspace, stream=None):
    """B sequences of T rows each (hidden [B*T, hidden]) through the whole block."""
    return _call("kda_block_prefill_batched", ctypes.byref(weights), _p(hidden), B, T, _p(h_state_ptrs),
                 _p(conv_state_ptrs), ws.handle, _stream(stream))


def kda_block_verify(weights: KdaBlockWeights, hidden, cu_seqlens, B: int, total_tokens: int, h_state_ptrs,
                     conv_state_ptrs, tables, ws: Workspace, stream=None):
    """Draft rows of B sequences (at most 64 each) through the whole block; no state changes;
    tables (kda_chunk_verify_tables_bytes(B) bytes) kept for kda_block_verify_fold."""
    return _call("kda_block_verify", ctypes.byref(weights), _p(hidden), _p(cu_seqlens), B, total_tokens,
                 _p(h_state_ptrs), _p(conv_state_ptrs), _p(tables), tables.numel() * tables.element_size(),
                 ws.handle, _stream(stream))


def kda_block_verify_fold(cu_seqlens, accepted, B: int, total_tokens: int, tables, h_state_ptrs, conv_state_ptrs,
                          ws: Workspace, stream=None):
    """Advance each sequence's recurrent and conv state past its accepted rows (device int32 [B])."""
    return _call("kda_block_verify_fold", _p(cu_seqlens), _p(accepted), B, total_tokens, _p(tables),
                 _p(h_state_ptrs), _p(conv_state_ptrs), ws.handle, _stream(stream))


def kda_front_conv_silu_l2_varlen(x, conv_state_ptrs, conv_w, conv_out, cu_seqlens, B: int, total_tokens: int,
                                  advance_state: bool, d: KdaDims, stream=None):
    return _call("kda_front_conv_silu_l2_varlen", _p(x), _p(conv_state_ptrs), _p(conv_w), _p(conv_out),
                 _p(cu_seqlens), B, total_tokens, 1 if advance_state else 0, ctypes.byref(d), _stream(stream))


def kda_conv_state_fold(x, conv_state_ptrs, cu_seqlens, accepted, B: int, total_tokens: int, d: KdaDims,
                        stream=None):
    return _call("kda_conv_state_fold", _p(x), _p(conv_state_ptrs), _p(cu_seqlens), _p(accepted), B, total_tokens,
                 ctypes.byref(d), _stream(stream))


def kda_chunk_prefill_packed_scratch_bytes(max_seqs: int, max_total_tokens: int, d: KdaDims) -> int:
    return int(lib().kda_chunk_prefill_packed_scratch_bytes(max_seqs, max_total_tokens, ctypes.byref(d)))


def kda_gemv_bf16(x, W, y, M: int, N: int, K: int, ldx=None, ldw=None, ldy=None, stream=None):
    """y[M, N] = x[M, K] . W[N, K]^T for a few rows (BF16 in; y's dtype picks BF16 or FP32)."""
    import torch
    return _call("kda_gemv_bf16", _p(x), ldx or K, _p(W), ldw or K, _p(y), ldy or N, M, N, K,
                 1 if y.dtype == torch.float32 else 0, _stream(stream))


def kda_chunk_prefill_varlen(q, k, v, gate, beta, cu_seqlens, B: int, max_num_chunks: int, total_tokens: int,
                             h_state_ptrs, core, d: KdaDims, stream=None, scratch=None):
    """Chunked prefill over B packed sequences of unequal lengths (cu_seqlens: device int32 [B+1])."""
    st = _stream(stream)
    if scratch is None:
        need = int(lib().kda_chunk_prefill_varlen_scratch_bytes(B, max_num_chunks, ctypes.byref(d)))
        scratch = scratch_buffer(need, core.device, st)
    return _call("kda_chunk_prefill_varlen", _p(q), _p(k), _p(v), _p(gate), _p(beta), _p(cu_seqlens), B,
                 max_num_chunks, total_tokens, _p(h_state_ptrs), _p(core), _p(scratch),
                 scratch.numel() * scratch.element_size(), ctypes.byref(d), st)


def kda_chunk_verify(q, k, v, gate, beta, cu_seqlens, B: int, total_tokens: int, h_state_ptrs, core, tables,
                     d: KdaDims, stream=None, scratch=None):
    """Batched verify: outputs for every draft row, states unchanged, tables kept for the fold."""
    st = _stream(stream)
    if scratch is None:
        need = int(lib().kda_chunk_prefill_varlen_scratch_bytes(B, 1, ctypes.byref(d)))
        scratch = scratch_buffer(need, core.device, st)
    return _call("kda_chunk_verify", _p(q), _p(k), _p(v), _p(gate), _p(beta), _p(cu_seqlens), B, total_tokens,
                 _p(h_state_ptrs), _p(core), _p(tables), tables.numel() * tables.element_size(), _p(scratch),
                 scratch.numel() * scratch.element_size(), ctypes.byref(d), st)


def kda_chunk_verify_tables_bytes(B: int, d: KdaDims) -> int:
    return int(lib().kda_chunk_verify_tables_bytes(B, ctypes.byref(d)))


def kda_chunk_verify_fold(k, cu_seqlens, accepted, B: int, total_tokens: int, tables, h_state_ptrs, d: KdaDims,
                          stream=None):
    """Advance every state by its accepted rows (device int32 [B]) from the verify tables."""
    return _call("kda_chunk_verify_fold", _p(k), _p(cu_seqlens), _p(accepted), B, total_tokens, _p(tables),
                 _p(h_state_ptrs), ctypes.byref(d), _stream(stream))


class Graph:
    """A recorded kda_block_decode (kda_block_decode_graph); launch() replays it."""

    def __init__(self, handle):
        self._h = handle

    def launch(self, stream=None):
        _call("kda_graph_launch", self._h, _stream(stream))

    def close(self):
        if self._h:
            lib().kda_graph_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def kda_block_decode_graph(weights: KdaBlockWeights, hidden, N: int, h_state_ptrs, conv_state_ptrs,
                           ws: Workspace) -> Graph:
    """Record kda_block_decode of N rows into a CUDA graph (nothing runs). The graph keeps the
    buffers' addresses: keep `weights`' tensors, hidden, the states, the pointer arrays and `ws`
    alive and in place while it is used."""
    h = ctypes.c_void_p()
    _call("kda_block_decode_graph", ctypes.byref(weights), _p(hidden), N, _p(h_state_ptrs), _p(conv_state_ptrs),
          ws.handle, ctypes.byref(h))
    return Graph(h)
