"""GPU parity of the CTA-pair tcgen05 GEMM (linear_tc2.cu) against the fp64 oracle.

OB_PATH_TC (and AUTO above 16 tokens) with bf16 output, M >= 512 and N >= 256 runs
the pair kernel (OB_PATH_TC1 forces the one-CTA kernel); these shapes exercise its
ragged tiles: N not a multiple of 256
(a pair whose second CTA has no valid rows), M not a multiple of the token tile, K with a
partial 128-k stage.  On 148 SMs the pair kernel takes 128-token tiles when twice the
256-token tiles fit the 74 SM pairs: every shape below up to (2048, 384, 1056) takes the
narrow tiles (777 tokens: the last tile's second CTA loads no valid token), the last two
the 256-token tiles.
"""
import numpy as np
import pytest
import torch

import oracle
from binary_weight_gemm_b200 import synth
from helpers import assert_gemm_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


def _cuda(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("M,N,K", [(512, 256, 128), (600, 300, 160), (777, 520, 96), (1030, 1000, 4096),
                                   (2048, 384, 1056), (2304, 4000, 544), (4100, 2600, 1056)])
def test_tc2_shapes(ops, M, N, K):
    seed = M + N + K
    W = synth.weights(seed, N, K)
    a, b, _ = oracle.svid_rank1(W)
    a, b = a.astype(np.float32), b.astype(np.float32)
    xb, x = synth.activations(seed, M, K)
    P = ops.ob_pack_signs(_cuda(W))
    X = _cuda(xb.view(np.int16)).view(torch.bfloat16)
    Y = ops.ob_linear(X, P, _cuda(a), _cuda(b), path=ops.OB_PATH_TC)
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    rows = np.arange(M) if M * N * K <= 2**30 else np.random.default_rng(seed).choice(M, 64, replace=False)
    ref = oracle.onebit_linear(x[rows], oracle.sign_pm1(W), a, b)
    assert_gemm_close(Y[torch.from_numpy(rows).cuda()], ref, what=f"tc2 {M}x{N}x{K}")


def test_tc2_matches_one_cta_kernel(ops):
    # The same problem on the pair kernel (OB_PATH_TC) and on the one-CTA kernel (OB_PATH_TC1).
    M, N, K = 1024, 768, 2048
    W = synth.weights(77, N, K)
    a, b, _ = oracle.svid_rank1(W)
    xb, _ = synth.activations(77, M, K)
    P = ops.ob_pack_signs(_cuda(W))
    X = _cuda(xb.view(np.int16)).view(torch.bfloat16)
    A, B = _cuda(a.astype(np.float32)), _cuda(b.astype(np.float32))
    Y2 = ops.ob_linear(X, P, A, B, path=ops.OB_PATH_TC)
    Y1 = ops.ob_linear(X, P, A, B, path=ops.OB_PATH_TC1)
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    assert_gemm_close(Y2, Y1.double().cpu().numpy(), what="pair vs one-CTA")
