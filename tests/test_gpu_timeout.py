"""The bounded on-chip wait, made to run out on purpose without any fault: a
one-CTA probe kernel (tests/cuda/timeout_probe.cu, built from the library's
own wait, status and tensor-memory helpers) waits on an mbarrier that nothing
arrives on.  The wait must give up after the library's limit, report
QLIN_ERR_TIMEOUT through dev_status, free its tensor memory and return; the
context must stay usable: the library's kernels that follow (tensor-memory
allocating ones included) still match the oracle."""
import ctypes as C
import os

import numpy as np
import pytest
import torch

import oracle
import quantized_weight_linear_qlin_b200 as q
import synth

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEV = "cuda"


@pytest.fixture(scope="module")
def probe():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    L = C.CDLL(__graft_entry__.build_probe())
    L.probe_never_arrived.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
    L.probe_never_arrived.restype = C.c_int
    L.probe_wait_limit_ns.restype = C.c_ulonglong
    return L


def bits16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_wait_runs_out_reports_timeout_and_context_survives(probe):
    limit_ns = probe.probe_wait_limit_ns()
    assert 1e7 <= limit_ns <= 2e9          # a bounded wait of at most a couple of seconds
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.zeros(2, dtype=torch.int64, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    assert probe.probe_never_arrived(C.c_void_p(status.data_ptr()), C.c_void_p(out.data_ptr()),
                                     C.c_void_p(stream)) == 0
    torch.cuda.synchronize()               # returns: the kernel ended by itself
    assert status.item() == q.ERR_TIMEOUT
    took, waited = out.cpu().tolist()
    assert took == 2
    assert limit_ns <= waited < limit_ns + 1_000_000_000

    # the context is intact and the probe's tensor memory was released: the
    # library's tensor-core kernels allocate it on every SM and still agree
    # with the oracle
    for fmt, n, k, t in ((q.Q4_G64, 4096, 5120, 4), (q.FP8_ROW, 2048, 1024, 1)):
        w = synth.weights_f32(n, k, seed=70 + t)
        x = synth.activations_bf16(t, k, seed=71 + t)
        ref = oracle.pack(fmt, w.numpy())
        pw = q.PackedWeights(fmt, n, k, device=DEV)
        q.qlin_pack_weights(q.SRC_F32, w.to(DEV), pw)
        y = torch.empty(t, n, dtype=torch.float32, device=DEV)
        ws = q.Workspace(DEV).ensure(q.qlin_gemv_workspace_bytes(pw, t))
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        q.qlin_gemv(pw, x.to(DEV), y, q.OUT_F32, workspace=ws, dev_status=st)
        yr, br = oracle.gemv(ref, bits16(x), nthreads=8)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - yr) <= 1e-3 * br)
