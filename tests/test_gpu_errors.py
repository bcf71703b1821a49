"""Device-side failure detection without faulting the GPU.

The bounded-wait self-test waits on a barrier nothing completes, gives up after
a few milliseconds and reports OB_ERR_DEVICE_TIMEOUT; the context stays usable.
Host-side checks on real device pointers return their status without launching.
"""
import numpy as np
import pytest
import torch

from binary_weight_gemm_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


def test_bounded_wait_reports_timeout_and_context_survives(ops):
    assert ops.ob_last_device_error() == 0
    assert ops.ob_selftest_timeout(2_000_000) == 8  # OB_ERR_DEVICE_TIMEOUT
    assert ops.ob_last_device_error() == 0           # read clears it
    # The context still works: run a real kernel afterwards.
    W = torch.from_numpy(synth.weights(0, 8, 64)).cuda()
    P = ops.ob_pack_signs(W)
    torch.cuda.synchronize()
    assert P.shape == (8, 2)


def test_misaligned_device_pointer_rejected(ops):
    from binary_weight_gemm_b200 import _lib
    buf = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    base = buf.data_ptr()
    st = _lib.lib().ob_pack_signs(base + 4, 2, 32, base + 512, torch.cuda.current_stream().cuda_stream)
    assert st == 3  # OB_ERR_ALIGN


def test_binding_raises_on_status(ops):
    from binary_weight_gemm_b200._lib import ObError
    X = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    P = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    a = torch.ones(4, device="cuda")
    b = torch.ones(64, device="cuda")
    with pytest.raises(ObError):
        ops.ob_linear(X, P, a, b, path=42)


def test_no_device_error_after_normal_work(ops):
    W = torch.from_numpy(synth.weights(1, 256, 256)).cuda()
    a, b, _, _, _ = ops.ob_svid_rank1(W)
    P = ops.ob_pack_signs(W)
    xb, _ = synth.activations(1, 40, 256)
    X = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    for path in (0, 1, 3, 4, 5, 0x100, 0x104):
        ops.ob_linear(X, P, a, b, path=path)
    from binary_weight_gemm_b200._lib import ObError
    with pytest.raises(ObError):  # value 2 named a kernel that was removed
        ops.ob_linear(X, P, a, b, path=2)
    assert ops.ob_last_device_error() == 0
