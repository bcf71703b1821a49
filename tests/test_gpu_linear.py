"""GPU parity of the OneBit linear layer against the fp64 oracle (direct form).

Tolerances (bf16 inputs, fp32 accumulation): relative Frobenius error <= 5e-3 and
max |dY| <= 1e-2 * max |Y_ref|.  a, b are the oracle's SVID vectors cast to
fp32 and given to both sides, so the GEMM is tested in isolation; one test runs
the whole GPU pipeline (pack, SVID, linear) against the whole oracle pipeline.
"""
import numpy as np
import pytest
import torch

import oracle
from binary_weight_gemm_b200 import synth
from helpers import Guarded, assert_gemm_close, oracle_svid

pytestmark = pytest.mark.gpu

PATHS = {"simt": 1, "tc": 3, "mma_decode": 4, "i8": 5, "tc1": 7, "auto_static": 0x100, "simt_static": 0x101}


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


def _cuda(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _x_bf16(x_bits):
    return _cuda(x_bits.view(np.int16)).view(torch.bfloat16)


def _run(ops, x_bits, W, a, b, path, out_dtype=torch.bfloat16):
    P = ops.ob_pack_signs(_cuda(W))
    g = Guarded((x_bits.shape[0], W.shape[0]), out_dtype)
    Y = ops.ob_linear(_x_bf16(x_bits), P, _cuda(a), _cuda(b), out_dtype=out_dtype, path=path, out=g.t)
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    g.check("ob_linear output")
    return Y


def _ref(x, W, a, b):
    return oracle.onebit_linear(x, oracle.sign_pm1(W), a, b)


# ---------------------------------------------------------------- small and ragged shapes, every path

SHAPES = [  # (M, N, K)
    (4, 256, 256),     # the tiny workload
    (1, 128, 64),
    (3, 200, 96),      # ragged N (not a multiple of 128), K with a half 64-stage
    (5, 129, 32),      # one packed word per row
    (16, 384, 1024),
    (17, 130, 160),    # M over one decode pass
    (300, 260, 192),   # ragged M and N tiles for the large-M kernel
    (513, 128, 4096),
    (300, 264, 192),   # ragged M and N, Y rows 16-byte aligned (TMA-stored output tile)
]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_linear_small_shapes(ops, path, M, N, K):
    seed = M * 7 + N + K
    W = synth.weights(seed, N, K)
    a, b, _ = oracle.svid_rank1(W)
    a, b = a.astype(np.float32), b.astype(np.float32)
    xb, x = synth.activations(seed, M, K)
    Y = _run(ops, xb, W, a, b, PATHS[path])
    assert_gemm_close(Y, _ref(x, W, a, b), what=f"{path} {M}x{N}x{K}")


@pytest.mark.parametrize("path", list(PATHS))
def test_linear_one_hot_rows_pin_layout(ops, path):
    # X = e_k picks column k of W_hat: Y[:, n] = a_n s_nk b_k.  Pins bit order and orientation.
    N, K = 256, 256
    W = synth.weights(21, N, K)
    a, b, _ = oracle.svid_rank1(W)
    a, b = a.astype(np.float32), b.astype(np.float32)
    ks = [0, 1, 15, 16, 17, 31, 32, 63, 64, 100, 255]
    x = np.zeros((len(ks), K), dtype=np.float32)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    xb, x = synth.bf16_round(x)
    Y = _run(ops, xb, W, a, b, PATHS[path], out_dtype=torch.float32).cpu().numpy()
    ref = _ref(x, W, a, b)
    np.testing.assert_allclose(Y, ref, rtol=1e-2, atol=1e-7)
    assert np.array_equal(np.sign(Y), np.sign(ref))


@pytest.mark.parametrize("path", list(PATHS))
def test_linear_fp32_output_and_outliers(ops, path):
    M, N, K = 8, 384, 512
    W = synth.weights(31, N, K)
    a, b, _ = oracle.svid_rank1(W)
    a, b = a.astype(np.float32), b.astype(np.float32)
    xb, x = synth.activations(31, M, K, outliers=True)
    Y = _run(ops, xb, W, a, b, PATHS[path], out_dtype=torch.float32)
    assert Y.dtype == torch.float32
    assert_gemm_close(Y, _ref(x, W, a, b), what=path)


def test_linear_exact_rank1_pipeline(ops):
    # |W| rank 1: GPU SVID is exact and the OneBit layer reproduces the dense X W^T.
    rng = np.random.default_rng(5)
    N, K, M = 256, 512, 4
    p = rng.uniform(0.5, 2.0, N).astype(np.float32) * 0.02
    q = rng.uniform(0.5, 2.0, K).astype(np.float32)
    W = (np.where(rng.random((N, K)) < 0.5, -1, 1) * np.outer(p, q)).astype(np.float32)
    xb, x = synth.activations(5, M, K)
    a, b, _, _, st = ops.ob_svid_rank1(_cuda(W))
    P = ops.ob_pack_signs(_cuda(W))
    for path in PATHS.values():
        Y = ops.ob_linear(_x_bf16(xb), P, a, b, out_dtype=torch.float32, path=path)
        assert_gemm_close(Y, x.astype(np.float64) @ W.astype(np.float64).T, what=f"path {path}")


def test_linear_end_to_end_pipeline_vs_oracle_pipeline(ops):
    # GPU: pack + SVID + linear.  Oracle: Sign + full-SVD SVID + direct form.
    W = synth.weights(0, 256, 256)
    xb, x = synth.activations(0, 4, 256)
    a_g, b_g, _, _, _ = ops.ob_svid_rank1(_cuda(W))
    P = ops.ob_pack_signs(_cuda(W))
    a_r, b_r, _ = oracle.svid_rank1(W)
    ref = oracle.onebit_linear(x, oracle.sign_pm1(W), a_r, b_r)
    for path in PATHS.values():
        Y = ops.ob_linear(_x_bf16(xb), P, a_g, b_g, path=path)
        assert_gemm_close(Y, ref, what=f"pipeline path {path}")


@pytest.mark.parametrize("M,K,path", [(260, 20480, "tc"), (40, 20480, "auto"), (20, 36864, "auto")])
def test_linear_long_k(ops, M, K, path):
    # K past 16384 runs the three-stage tcgen05 kernel; past 32768 AUTO takes the
    # warp-level MMA kernel in 16-token launches.
    N = 136
    seed = K + M
    W = synth.weights(seed, N, K)
    a, b, _ = oracle.svid_rank1(W)
    a, b = a.astype(np.float32), b.astype(np.float32)
    xb, x = synth.activations(seed, M, K)
    Y = _run(ops, xb, W, a, b, PATHS.get(path, 0))
    assert_gemm_close(Y, _ref(x, W, a, b), what=f"long K {M}x{N}x{K} {path}")


def test_tc_path_rejects_k_beyond_limit(ops):
    from binary_weight_gemm_b200._lib import ObError
    K = 32768 + 32
    X = torch.zeros((32, K), dtype=torch.bfloat16, device="cuda")
    P = torch.zeros((128, K // 32), dtype=torch.int32, device="cuda")
    for path in ("tc", "tc1"):
        with pytest.raises(ObError):
            ops.ob_linear(X, P, torch.ones(128, device="cuda"), torch.ones(K, device="cuda"), path=PATHS[path])


def test_linear_degenerate_sizes(ops):
    P = torch.zeros((8, 2), dtype=torch.int32, device="cuda")
    a = torch.ones(8, device="cuda")
    b = torch.ones(64, device="cuda")
    Y = ops.ob_linear(torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda"), P, a, b)
    assert Y.shape == (0, 8)
    # K = 0: empty sum, Y = 0.
    Y = ops.ob_linear(torch.zeros((3, 0), dtype=torch.bfloat16, device="cuda"),
                      torch.zeros((8, 0), dtype=torch.int32, device="cuda"), a,
                      torch.ones(0, device="cuda"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert Y.shape == (3, 8) and not Y.any()


# ---------------------------------------------------------------- full-size workloads

@pytest.mark.parametrize("path", ["mma_decode", "simt", "i8", "auto_static"])
@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_decode_workload_full(ops, path, M):
    # OneBit decode GEMV: X M x 4096, W 4096 x 4096 -> 2 MiB packed, a, b from SVID.
    W, a, b, _ = oracle_svid(1, 4096, 4096)
    xb, x = synth.activations(1, M, 4096)
    Y = _run(ops, xb, W, a, b, PATHS[path])
    assert_gemm_close(Y, _ref(x, W, a, b), what=f"decode M={M} {path}")


def test_prefill_workload_full_every_element(ops):
    # OneBit prefill: X 2048 x 4096, W 11008 x 4096; all 22.5 M outputs against the fp64
    # oracle (about 92 GFLOP on the host), on the path AUTO takes (the CTA-pair kernel).
    W, a, b, _ = oracle_svid(2, 11008, 4096)
    xb, x = synth.activations(2, 2048, 4096)
    Y = _run(ops, xb, W, a, b, 0)
    assert torch.isfinite(Y.float()).all()
    assert_gemm_close(Y, _ref(x, W, a, b), what="prefill, every element")


def test_prefill_one_cta_kernel_sampled_rows(ops):
    # The one-CTA tcgen05 kernel (forced: AUTO takes the CTA pair here) on the prefill
    # workload; oracle on 64 sampled token rows.
    W, a, b, _ = oracle_svid(2, 11008, 4096)
    xb, x = synth.activations(2, 2048, 4096)
    Y = _run(ops, xb, W, a, b, PATHS["tc1"])
    rows = np.random.default_rng(0).choice(2048, 64, replace=False)
    rows[:2] = [0, 2047]
    assert_gemm_close(Y[torch.from_numpy(rows).cuda()], _ref(x[rows], W, a, b), what="prefill rows")


SWEEP = [(4096, 4096), (4096, 11008), (11008, 4096)]  # (K, N): K -> N


@pytest.mark.parametrize("shape_idx", range(3))
@pytest.mark.parametrize("M", [1, 16, 256, 4096])
def test_sweep_with_outliers(ops, shape_idx, M):
    K, N = SWEEP[shape_idx]
    W, a, b, _ = oracle_svid(4 + shape_idx, N, K)
    xb, x = synth.activations(4 + shape_idx, M, K, outliers=True)
    Y = _run(ops, xb, W, a, b, 0)
    # every element, M = 4096 included (up to 370 GFLOP of fp64 on the host)
    assert_gemm_close(Y, _ref(x, W, a, b), what=f"sweep {K}->{N} M={M}")


@pytest.mark.parametrize("M,N,K,path", [(256, 4096, 4096, 0), (64, 1024, 2048, 0), (300, 512, 11008, 0),
                                        (128, 2048, 8192, 0), (17, 1000, 160, 0), (256, 4096, 4096, 7),
                                        (600, 512, 2048, 0), (256, 132, 512, 0)])
def test_linear_ws_split_over_k(ops, M, N, K, path):
    # ob_linear_ws: few output tiles on the one-CTA tcgen05 GEMM split over K through the
    # workspace (fp32 partial sums); every element against the oracle; a workspace one byte
    # short, and none, run unsplit with the same result.
    from helpers import Guarded
    W = synth.weights(M + N + K, N, K)
    a, b, _ = oracle.svid_rank1(W)
    a, b = a.astype(np.float32), b.astype(np.float32)
    xb, x = synth.activations(M + K, M, K)
    P = ops.ob_pack_signs(_cuda(W))
    X, A, B = _x_bf16(xb), _cuda(a), _cuda(b)
    ref = _ref(x, W, a, b)
    need = ops.ob_linear_workspace_size(M, N, K)
    for ws_bytes in sorted({need, max(need - 1, 0), 0}):
        ws = Guarded((max(ws_bytes, 1),), torch.uint8) if ws_bytes else None
        out = Guarded((M, N), torch.bfloat16)
        ops.ob_linear(X, P, A, B, out=out.t, path=path,
                      workspace=None if ws is None else ws.t[:ws_bytes] if ws_bytes else None)
        torch.cuda.synchronize()
        assert ops.ob_last_device_error() == 0
        out.check("ob_linear_ws output")
        if ws is not None:
            ws.check("ob_linear_ws workspace")
        assert_gemm_close(out.t, ref, what=f"ob_linear_ws {M}x{N}x{K} path {path} ws {ws_bytes}")


def test_cuda_graph_replay_matches(ops):
    W, a, b, _ = oracle_svid(1, 4096, 4096)
    xb, x = synth.activations(1, 4, 4096)
    P = ops.ob_pack_signs(_cuda(W))
    X, A, B = _x_bf16(xb), _cuda(a), _cuda(b)
    Y = torch.empty((4, 4096), dtype=torch.bfloat16, device="cuda")
    ops.ob_linear(X, P, A, B, out=Y)  # warm up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            ops.ob_linear(X, P, A, B, out=Y, stream=s)
    Y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert_gemm_close(Y, _ref(x, W, a, b), what="graph replay")


@pytest.mark.parametrize("M,path", [(1, "auto"), (4, "auto"), (16, "auto"), (40, "auto"), (1, "i8"), (2, "i8"), (3, "i8"),
                                    (16, "i8"), (1, "auto_static"), (3, "simt_static"), (16, "auto_static")])
def test_chained_layers_in_graph(ops, M, path):
    # Eight 512 x 512 layers chained through their outputs (layer i+1 reads layer i's Y),
    # captured in one CUDA graph; calls may launch before their predecessor has finished
    # (programmatic dependent launch), so each must read its input only after it is complete.
    # Every layer is checked against the oracle on the bf16 input it actually received.
    K = 512
    layers = []
    for i in range(8):
        W = synth.weights(100 + i, K, K)
        a, b, _ = oracle.svid_rank1(W)
        layers.append((W, a.astype(np.float32), b.astype(np.float32)))
    dev = [(ops.ob_pack_signs(_cuda(W)), _cuda(a), _cuda(b)) for W, a, b in layers]
    xb, _ = synth.activations(100, M, K)
    X = _x_bf16(xb)
    Ys = [torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for _ in layers]
    torch.cuda.synchronize()
    s = torch.cuda.Stream()

    def chain():
        x = X
        for (P, a, b), Y in zip(dev, Ys):
            ops.ob_linear(x, P, a, b, out=Y, stream=s, path=PATHS.get(path, 0))
            x = Y

    with torch.cuda.stream(s):
        chain()  # warm up outside capture
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            chain()
    for Y in Ys:
        Y.zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    x_in = X.float().cpu().numpy().astype(np.float64)
    for i, ((W, a, b), Y) in enumerate(zip(layers, Ys)):
        assert_gemm_close(Y, _ref(x_in, W, a, b), what=f"chained layer {i} M={M}")
        x_in = Y.float().cpu().numpy().astype(np.float64)
