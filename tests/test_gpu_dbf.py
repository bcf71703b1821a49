"""GPU parity of the DBF linear layer against the fp64 oracle (direct form W_hat = diag(a) S_A diag(m) S_B diag(b))."""
import numpy as np
import pytest
import torch

import oracle
from binary_weight_gemm_b200 import synth
from helpers import Guarded, assert_gemm_close

pytestmark = pytest.mark.gpu

PATHS = {"simt": 1, "tc": 3, "mma_decode": 4, "i8": 5, "auto": 0, "stack": 6, "simt_static": 0x101,
         "mma_static": 0x104, "auto_static": 0x100}


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


def _cuda(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _run(ops, xb, f, path, out_dtype=torch.bfloat16):
    SB = ops.ob_pack_signs(_cuda(f["S_B"].astype(np.float32)))
    SA = ops.ob_pack_signs(_cuda(f["S_A"].astype(np.float32)))
    X = _cuda(xb.view(np.int16)).view(torch.bfloat16)
    M, r, N = xb.shape[0], SB.shape[0], SA.shape[0]
    g = Guarded((M, N), out_dtype)
    ws = Guarded((max(1, ops.dbf_workspace_size(M, r)),), torch.uint8)
    Y = ops.dbf_linear(X, SB, _cuda(f["m"]), SA, _cuda(f["a"]), _cuda(f["b"]), out_dtype=out_dtype, path=path,
                       out=g.t, workspace=ws.t)
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    g.check("dbf_linear output")
    ws.check("dbf_linear workspace")
    return Y


def _ref(x, f):
    return oracle.dbf_linear(x, f["S_A"], f["S_B"], f["a"], f["m"], f["b"])


@pytest.mark.parametrize("path", ["simt", "tc", "mma_decode", "i8", "auto", "stack", "simt_static", "mma_static"])
@pytest.mark.parametrize("M,N,r,K", [(1, 128, 32, 64), (4, 256, 96, 256), (7, 200, 160, 96), (33, 130, 64, 128),
                                     (260, 256, 128, 320)])
def test_dbf_small_shapes(ops, path, M, N, r, K):
    f = synth.dbf_factors(M + N + r + K, N, r, K)
    xb, x = synth.activations(M + N, M, K)
    if path == "stack" and M > 16:  # the one-launch form is for decode sizes only
        from binary_weight_gemm_b200._lib import ObError
        with pytest.raises(ObError):
            _run(ops, xb, f, PATHS[path])
        return
    assert_gemm_close(_run(ops, xb, f, PATHS[path]), _ref(x, f), what=f"dbf {path} {M},{N},{r},{K}")


@pytest.mark.parametrize("M,path", [(1, "auto"), (2, "auto"), (16, "auto"), (512, "auto"), (1, "auto_static"),
                                    (16, "auto_static"), (1, "stack"), (2, "stack"), (16, "stack")])
def test_dbf_workload_full(ops, M, path):
    # DBF: K = N = 4096, r = 2048; S_A, S_B random +/-1; a, m, b ~ |N(0,1)|*0.02+1e-3.
    f = synth.dbf_factors(3, 4096, 2048, 4096)
    xb, x = synth.activations(3, M, 4096)
    Y = _run(ops, xb, f, PATHS[path])
    assert_gemm_close(Y, _ref(x, f), what=f"dbf workload M={M} {path}")


# Middle dimensions for about 0.5, 1.5, 1.8 and 2.3 bits per weight at K = N = 4096
# (bits ~ r (K + N) / (N K)): non-uniform r per layer, with tile tails in both sign GEMMs.
# At M = 512 both products of r <= 3680 run on the CTA-pair kernel's 128-token tiles; at
# r = 4704 both are split over K on the one-CTA kernel.
@pytest.mark.parametrize("r", [1056, 3072, 3680, 4704])
@pytest.mark.parametrize("M", [1, 16, 300, 512])
def test_dbf_general_r(ops, r, M):
    f = synth.dbf_factors(r + M, 4096, r, 4096)
    xb, x = synth.activations(r, M, 4096)
    Y = _run(ops, xb, f, PATHS["auto"])
    ref = oracle.dbf_linear_chain(x, f["S_A"], f["S_B"], f["a"], f["m"], f["b"])
    assert_gemm_close(Y, ref, what=f"dbf r={r} M={M}")


@pytest.mark.parametrize("M", [1, 4])
def test_dbf_decode_with_the_smallest_workspace(ops, M):
    # A workspace that holds only T is enough for AUTO (two launches); the one-launch form
    # needs the barrier word after T and rejects it.
    f = synth.dbf_factors(14 + M, 512, 256, 384)
    xb, x = synth.activations(14, M, 384)
    SB = ops.ob_pack_signs(_cuda(f["S_B"].astype(np.float32)))
    SA = ops.ob_pack_signs(_cuda(f["S_A"].astype(np.float32)))
    X = _cuda(xb.view(np.int16)).view(torch.bfloat16)
    t_bytes = (M * 256 * 2 + 255) // 256 * 256
    for ws_bytes in (t_bytes, ops.dbf_workspace_size(M, 256)):
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
        Y = ops.dbf_linear(X, SB, _cuda(f["m"]), SA, _cuda(f["a"]), _cuda(f["b"]), workspace=ws)
        torch.cuda.synchronize()
        assert ops.ob_last_device_error() == 0
        assert_gemm_close(Y, _ref(x, f), what=f"dbf M={M} workspace {ws_bytes}")
    from binary_weight_gemm_b200._lib import ObError
    with pytest.raises(ObError):
        ops.dbf_linear(X, SB, _cuda(f["m"]), SA, _cuda(f["a"]), _cuda(f["b"]),
                       workspace=torch.zeros(t_bytes, dtype=torch.uint8, device="cuda"), path=ops.OB_PATH_STACK)


def test_dbf_fp32_output(ops):
    # Smallest middle dimension (one packed word per S_A row), fp32 output.
    f = synth.dbf_factors(11, 256, 32, 256)
    xb, x = synth.activations(11, 3, 256)
    Y = _run(ops, xb, f, PATHS["auto"], out_dtype=torch.float32)
    assert Y.dtype == torch.float32
    assert_gemm_close(Y, _ref(x, f), what="dbf fp32")


def test_dbf_one_hot_input(ops):
    f = synth.dbf_factors(12, 128, 64, 128)
    ks = [0, 5, 31, 32, 127]
    x = np.zeros((len(ks), 128), dtype=np.float32)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    xb, x = synth.bf16_round(x)
    Y = _run(ops, xb, f, PATHS["auto"], out_dtype=torch.float32)
    assert_gemm_close(Y, _ref(x, f), what="dbf one-hot")


def test_dbf_degenerate(ops):
    f = synth.dbf_factors(13, 64, 32, 64)
    X = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    SB = ops.ob_pack_signs(_cuda(f["S_B"].astype(np.float32)))
    SA = ops.ob_pack_signs(_cuda(f["S_A"].astype(np.float32)))
    Y = ops.dbf_linear(X, SB, _cuda(f["m"]), SA, _cuda(f["a"]), _cuda(f["b"]))
    assert Y.shape == (0, 64)
