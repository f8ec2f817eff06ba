"""The tcgen05 building blocks (umma.cuh) on the GPU: for every probed shape and operand
layout (K-major / MN-major, 128-byte swizzle, M = 64 or 128, N = 16..256) the MMA result
read back from TMEM equals the exact product of the BF16-exact operands (FP32 accumulate)."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def probe(cuda_ok):
    from kda_gated_delta_gate_b200 import build
    L = ctypes.CDLL(build.build_probe())
    L.probe_run.argtypes = [ctypes.c_int] + [ctypes.c_void_p] * 4
    L.probe_shape.argtypes = [ctypes.c_int, ctypes.c_void_p]
    return L


def _shapes(L):
    out = []
    for i in range(L.probe_count()):
        s = (ctypes.c_int * 5)()
        L.probe_shape(i, s)
        out.append((i, *list(s)))
    return out


def test_umma_shapes_and_layouts(probe):
    failures = []
    for i, M, N, K, amn, bmn in _shapes(probe):
        g = torch.Generator().manual_seed(i)
        A = torch.randn((M, K), generator=g).to(torch.bfloat16).float()
        B = torch.randn((N, K), generator=g).to(torch.bfloat16).float()
        Ad, Bd = A.cuda(), B.cuda()
        Dd = torch.full((M, N), float("nan"), device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = probe.probe_run(i, Ad.data_ptr(), Bd.data_ptr(), Dd.data_ptr(), st.data_ptr())
        torch.cuda.synchronize()
        assert rc == 0, (i, rc)
        ref = A.double().numpy() @ B.double().numpy().T
        got = Dd.cpu().double().numpy()
        err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
        if st.item() != 0 or not np.isfinite(err) or err > 1e-5:
            failures.append((i, M, N, K, amn, bmn, st.item(), float(err)))
    assert not failures, failures


def test_bounded_wait_gives_up_and_context_survives(probe):
    """Failure detection without a GPU fault: a wait on a barrier nothing arrives on returns
    after its limit (about 1 ms here), the kernel reports it in a status word the host reads,
    and the context stays usable for the next launch."""
    probe.probe_timeout.argtypes = [ctypes.c_void_p, ctypes.c_longlong]
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    assert probe.probe_timeout(st.data_ptr(), 2_000_000) == 0
    torch.cuda.synchronize()
    assert st.item() == 1
    A = torch.ones((128, 128), device="cuda")
    D = torch.empty((128, 16), device="cuda")
    s2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert probe.probe_run(0, A.data_ptr(), A.data_ptr(), D.data_ptr(), s2.data_ptr()) == 0
    torch.cuda.synchronize()
    assert s2.item() == 0 and torch.all(D == 128.0)
