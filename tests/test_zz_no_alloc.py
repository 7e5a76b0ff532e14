"""qlin_gemv_noalloc: the decode GEMV with its scratch in the library's fixed
device array must give what qlin_gemv gives with a caller workspace, call after
call, and must refuse requests that need more scratch than the array holds.

Collected last on purpose (file name), so it also runs after every other test
has used the device."""
import numpy as np
import pytest
import torch

import quantized_weight_linear_qlin_b200 as q
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _packed(fmt, n, k, seed):
    w = synth.weights_f32(n, k, seed=seed, device=DEV)
    pw = q.PackedWeights(fmt, n, k, device=DEV)
    q.qlin_pack_weights(q.SRC_F32, w, pw)
    return pw


@pytest.mark.parametrize("fmt,n,k,t", [
    (q.Q4_G64, 34816, 5120, 1),    # gate+up, decode
    (q.Q5_G64, 5120, 17408, 33),   # down, verify step: split tiles
    (q.Q8_G32, 1000, 2048, 5),     # ragged rows
    (q.FP8_ROW, 4096, 5120, 17),
    (q.Q5_G64, 200, 1216, 3),      # K not whole tensor-core units: CUDA-core kernel
])
def test_noalloc_matches_workspace_path_twice(fmt, n, k, t):
    pw = _packed(fmt, n, k, seed=11)
    x = synth.activations_bf16(t, k, seed=12, device=DEV)
    ws = q.Workspace(DEV).ensure(q.qlin_gemv_workspace_bytes(pw, t))
    y_ref = torch.empty(t, n, dtype=torch.float32, device=DEV)
    q.qlin_gemv(pw, x, y_ref, q.OUT_F32, workspace=ws)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for _ in range(2):  # two calls in a row on the same fixed scratch
        y = torch.full((t, n), float("nan"), dtype=torch.float32, device=DEV)
        q.qlin_gemv_noalloc(pw, x, y, q.OUT_F32, dev_status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        a, b = y.cpu().numpy(), y_ref.cpu().numpy()
        # same kernels, same reduction order: equal up to FP32 rounding noise
        assert np.allclose(a, b, rtol=1e-6, atol=1e-6 * np.abs(b).max())


def test_noalloc_rejects_requests_beyond_the_array():
    # BF16 weights whose K is not a whole number of tensor-core units run on
    # the general CUDA-core kernel; with K beyond its 2048-column stage it
    # splits K and needs a T * N FP32 accumulator: 32 MiB here, above the
    # 16 MiB array
    n, k, t = 4096, 4160, 2048
    pw = q.PackedWeights(q.BF16, n, k, device=DEV)
    x = torch.zeros(t, k, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(t, n, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(q.QlinError) as e:
        q.qlin_gemv_noalloc(pw, x, y, q.OUT_BF16)
    assert e.value.status == q.ERR_WORKSPACE


def test_noalloc_reports_argument_errors_like_qlin_gemv():
    """Quantized weights at T = 65: QLIN_ERR_UNSUPPORTED (as qlin_gemv), not a
    workspace error, and nothing is enqueued."""
    n, k, t = 34816, 5120, 65
    pw = q.PackedWeights(q.Q4_G64, n, k, device=DEV)
    x = torch.zeros(t, k, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(t, n, dtype=torch.bfloat16, device=DEV)
    for call in (lambda: q.qlin_gemv_noalloc(pw, x, y, q.OUT_BF16),
                 lambda: q.qlin_gemv(pw, x, y, q.OUT_BF16, workspace=q.Workspace(DEV))):
        with pytest.raises(q.QlinError) as e:
            call()
        assert e.value.status == q.ERR_UNSUPPORTED


def test_noalloc_rejects_quantized_cuda_core_shape_beyond_the_array():
    """Q4 with K = 5184 (not a whole number of tensor-core column units) runs on
    the CUDA-core kernel, whose split-K accumulator needs T * N * 4 = 39 MB at
    N = 152064, T = 64: above the 16 MiB array."""
    n, k, t = 152064, 5184, 64
    pw = q.PackedWeights(q.Q4_G64, n, k, device=DEV)
    assert q.qlin_gemv_workspace_bytes(pw, t) == t * n * 4
    x = torch.zeros(t, k, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(t, n, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(q.QlinError) as e:
        q.qlin_gemv_noalloc(pw, x, y, q.OUT_BF16)
    assert e.value.status == q.ERR_WORKSPACE
