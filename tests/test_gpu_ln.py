"""GPU parity of the OneBit layer followed by LayerNorm (Z = LayerNorm(Y)) against the fp64 oracle.

Z has unit scale per row; the same tolerances as the GEMMs apply (relative
Frobenius <= 5e-3, max |dZ| <= 1e-2 max |Z_ref|).  a, b are the oracle's SVID
vectors cast to fp32 and given to both sides.
"""
import numpy as np
import pytest
import torch

import oracle
from binary_weight_gemm_b200 import synth
from helpers import Guarded, assert_gemm_close, oracle_svid

pytestmark = pytest.mark.gpu

PATHS = {"auto": 0, "simt": 1, "tc": 3, "mma_decode": 4, "i8": 5}


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


def _cuda(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _run(ops, xb, W, a, b, path=0, eps=1e-5, out_dtype=torch.bfloat16):
    P = ops.ob_pack_signs(_cuda(W))
    X = _cuda(xb.view(np.int16)).view(torch.bfloat16)
    g = Guarded((xb.shape[0], W.shape[0]), out_dtype)
    Z = ops.ob_linear_ln(X, P, _cuda(a), _cuda(b), eps=eps, out_dtype=out_dtype, path=path, out=g.t)
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    g.check("ob_linear_ln output")
    return Z


def _svid32(W):
    a, b, _ = oracle.svid_rank1(W)
    return a.astype(np.float32), b.astype(np.float32)


@pytest.mark.parametrize("path", ["simt", "tc", "mma_decode", "i8"])
@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (4, 256, 256), (3, 200, 96), (17, 130, 160), (300, 264, 192)])
def test_ln_small_shapes(ops, path, M, N, K):
    W = synth.weights(M + N + K, N, K)
    a, b = _svid32(W)
    xb, x = synth.activations(M + N, M, K)
    Z = _run(ops, xb, W, a, b, PATHS[path])
    assert_gemm_close(Z, oracle.onebit_linear_ln(x, oracle.sign_pm1(W), a, b), what=f"ln {path} {M}x{N}x{K}")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_ln_decode_full(ops, M):
    W, a, b, _ = oracle_svid(1, 4096, 4096)
    xb, x = synth.activations(1, M, 4096, outliers=True)
    Z = _run(ops, xb, W, a, b)
    assert_gemm_close(Z, oracle.onebit_linear_ln(x, oracle.sign_pm1(W), a, b), what=f"ln decode M={M}")


def test_ln_prefill_sampled_rows(ops):
    W, a, b, _ = oracle_svid(2, 11008, 4096)
    xb, x = synth.activations(2, 2048, 4096)
    Z = _run(ops, xb, W, a, b)
    rows = np.random.default_rng(0).choice(2048, 48, replace=False)
    rows[:2] = [0, 2047]
    ref = oracle.onebit_linear_ln(x[rows], oracle.sign_pm1(W), a, b)
    assert_gemm_close(Z[torch.from_numpy(rows).cuda()], ref, what="ln prefill rows")


def test_ln_fp32_output_and_eps(ops):
    W = synth.weights(41, 384, 512)
    a, b = _svid32(W)
    xb, x = synth.activations(41, 8, 512)
    for eps in (0.0, 1e-5, 0.25):
        Z = _run(ops, xb, W, a, b, eps=eps, out_dtype=torch.float32)
        assert Z.dtype == torch.float32
        ref = oracle.layernorm(oracle.onebit_linear(x, oracle.sign_pm1(W), a, b), eps=eps)
        assert_gemm_close(Z, ref, what=f"ln fp32 eps={eps}")
        # Invariants of the normalised rows (fp32 output, statistics from fp32 Y).
        Zn = Z.double().cpu().numpy()
        np.testing.assert_allclose(Zn.mean(axis=1), 0.0, atol=1e-4)


def test_ln_degenerate(ops):
    # One output feature: every row normalises to 0.  K = 0: Y = 0, so Z = 0.
    W = synth.weights(43, 1, 64)
    a, b = _svid32(W)
    xb, _ = synth.activations(43, 5, 64)
    assert not _run(ops, xb, W, a, b).any()
    Z = ops.ob_linear_ln(torch.zeros((3, 0), dtype=torch.bfloat16, device="cuda"),
                         torch.zeros((8, 0), dtype=torch.int32, device="cuda"), torch.ones(8, device="cuda"),
                         torch.ones(0, device="cuda"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert Z.shape == (3, 8) and not Z.any()


def test_ln_rejects_bad_eps(ops):
    from binary_weight_gemm_b200._lib import ObError
    X = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    P = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    for eps in (-1.0, float("nan"), float("inf")):
        with pytest.raises(ObError):
            ops.ob_linear_ln(X, P, torch.ones(4, device="cuda"), torch.ones(64, device="cuda"), eps=eps)
