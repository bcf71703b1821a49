"""GPU parity of ob_linear_stack (a list of OneBit layers in one persistent launch).

Every layer is checked against the fp64 oracle on the bf16 input it actually
received (its X, possibly an earlier layer's Y), with the GEMM tolerances.  AUTO takes
the int8 form for one and two tokens and the bf16 warp-MMA form above; tests that name a
path force one form.
"""
import numpy as np
import pytest
import torch

import oracle
from binary_weight_gemm_b200 import synth
from helpers import Guarded, assert_gemm_close, oracle_svid

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import ops as _ops
    torch.cuda.init()
    return _ops


MMA, I8 = 4, 5


def _cuda(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _x(xb):
    return _cuda(xb.view(np.int16)).view(torch.bfloat16)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _layer(seed, N, K, scale_in=True):
    W = synth.weights(seed, N, K)
    a, b, _ = oracle.svid_rank1(W)
    a, b = a.astype(np.float32), b.astype(np.float32)
    if not scale_in:
        b = np.ones(K, dtype=np.float32)
    return W, a, b


def _check(layers_host, layer_io, what):
    """layers_host: (W, a, b) per layer; layer_io: (X tensor, Y tensor) per layer after the run."""
    for i, ((W, a, b), (X, Y)) in enumerate(zip(layers_host, layer_io)):
        ref = oracle.onebit_linear(_np(X), oracle.sign_pm1(W), a, b)
        assert_gemm_close(Y, ref, what=f"{what} layer {i}")


def _run(ops, spec, M, path=0, dataflow=False):
    """ob_linear_stack; dataflow: with the workspace of ob_linear_stack_workspace_size (tagged
    outputs instead of grid barriers), which must exceed the barrier-only size, between canary
    guard words and pre-filled with their pattern (so a tag area the library failed to clear
    would read as ready)."""
    ws = None
    if dataflow:
        n = ops.ob_linear_stack_workspace_size(spec, M)
        assert n > ops.ob_stack_workspace_size()
        ws = Guarded((n,), torch.uint8)
    elif M == 2:  # two tokens keep the grid barriers whatever the workspace
        assert ops.ob_linear_stack_workspace_size(spec, M) == ops.ob_stack_workspace_size()
    ops.ob_linear_stack(spec, M, path=path, workspace=None if ws is None else ws.t)
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    if ws is not None:
        ws.check("stack workspace")


@pytest.mark.parametrize("M,path,df", [(1, 0, False), (2, 0, False), (4, 0, False), (9, 0, False), (16, 0, False),
                                       (1, MMA, False), (2, MMA, False), (1, 0, True)])
def test_stack_chain(ops, M, path, df):
    K = 512
    host = [_layer(200 + i, K, K) for i in range(8)]
    X0 = _x(synth.activations(200, M, K)[0])
    gs = [Guarded((M, K), torch.bfloat16) for _ in host]
    spec, x = [], X0
    for i, ((W, a, b), g) in enumerate(zip(host, gs)):
        spec.append((x, ops.ob_pack_signs(_cuda(W)), _cuda(a), _cuda(b), g.t, i > 0))
        x = g.t
    _run(ops, spec, M, path, df)
    for i, g in enumerate(gs):
        g.check(f"chain layer {i} output")
    _check(host, [(s[0], s[4]) for s in spec], f"chain M={M} path={path} dataflow={df}")


@pytest.mark.parametrize("M,df", [(1, False), (2, False), (1, True)])
def test_stack_i8_tiles_chunks_and_tails(ops, M, df):
    # int8 form.  Group 1 (all read X0, K = 128): 60 layers of 32 rows (a CTA's tile range
    # crosses layers; the first writes fp32), one of 30000 rows (about 12.7 tiles per CTA:
    # more than one 12-tile pass), one of 1152 rows.  Group 2 reads the 1152-wide output:
    # K = 1152 is two full super-blocks and a 128-k tail; 300 rows (a ragged last tile), no
    # input scale.  Group 3: a layer with K = 12832 (25 super-blocks and a tail: more than
    # one staging chunk) on a separate input with outliers.
    X0 = _x(synth.activations(270, M, 128)[0])
    shapes = [(32, 128)] * 60 + [(30000, 128), (1152, 128), (300, 1152)]
    host, spec = [], []
    for i, (N, K) in enumerate(shapes):
        last = i == len(shapes) - 1
        W, a, b = _layer(300 + i, N, K, scale_in=not last)
        host.append((W, a, b))
        Y = torch.empty((M, N), dtype=torch.float32 if i == 0 else torch.bfloat16, device="cuda")
        X = spec[-1][4] if last else X0
        spec.append((X, ops.ob_pack_signs(_cuda(W)), _cuda(a), None if last else _cuda(b), Y, last))
    # A long-K layer (25 super-blocks and a 32-k tail: two staging chunks), after a barrier.
    Kl = 12832
    W, a, b = _layer(399, 96, Kl)
    host.append((W, a, b))
    Xl = _x(synth.activations(271, M, Kl, outliers=True)[0])
    spec.append((Xl, ops.ob_pack_signs(_cuda(W)), _cuda(a), _cuda(b),
                 torch.empty((M, 96), dtype=torch.bfloat16, device="cuda"), True))
    _run(ops, spec, M, I8, df)
    _check(host, [(sp[0], sp[4]) for sp in spec], f"i8 stack M={M} dataflow={df}")


@pytest.mark.parametrize("M,df", [(1, False), (2, False), (5, False), (16, False), (1, True)])
def test_stack_groups_ragged(ops, M, df):
    # Group 1 (independent, all read X0): A 96->224, B 96->130 (fp32 out), C 96->64 without input
    # scale.  Group 2 (after a barrier): D reads A (224->200), E reads A too (224->128, vector path).
    X0 = _x(synth.activations(210, M, 96)[0])
    shapes = [("A", 224, 96), ("B", 130, 96), ("C", 64, 96), ("D", 200, 224), ("E", 128, 224)]
    host = {n: _layer(210 + i, N, K, scale_in=(n != "C")) for i, (n, N, K) in enumerate(shapes)}
    out = {"A": torch.empty((M, 224), dtype=torch.bfloat16, device="cuda"),
           "B": torch.empty((M, 130), dtype=torch.float32, device="cuda"),
           "C": torch.empty((M, 64), dtype=torch.bfloat16, device="cuda"),
           "D": torch.empty((M, 200), dtype=torch.bfloat16, device="cuda"),
           "E": torch.empty((M, 128), dtype=torch.bfloat16, device="cuda")}
    src = {"A": X0, "B": X0, "C": X0, "D": out["A"], "E": out["A"]}
    spec = []
    for n, N, K in shapes:
        W, a, b = host[n]
        spec.append((src[n], ops.ob_pack_signs(_cuda(W)), _cuda(a), None if n == "C" else _cuda(b), out[n],
                     n == "D"))
    _run(ops, spec, M, 0, df)
    _check([host[n] for n, _, _ in shapes], [(src[n], out[n]) for n, _, _ in shapes], f"groups M={M} dataflow={df}")


@pytest.mark.parametrize("M,path,df", [(1, 0, False), (2, 0, False), (16, 0, False), (1, MMA, False), (1, 0, True)])
def test_stack_dbf(ops, M, path, df):
    # DBF as two layers: T = ((X ⊙ b) S_B^T) ⊙ m, then Y = (T S_A^T) ⊙ a (no input scale).
    f = synth.dbf_factors(220, 1024, 512, 768)
    xb, x = synth.activations(220, M, 768)
    X = _x(xb)
    T = torch.empty((M, 512), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((M, 1024), dtype=torch.bfloat16, device="cuda")
    SB = ops.ob_pack_signs(_cuda(f["S_B"].astype(np.float32)))
    SA = ops.ob_pack_signs(_cuda(f["S_A"].astype(np.float32)))
    _run(ops, [(X, SB, _cuda(f["m"]), _cuda(f["b"]), T, False), (T, SA, _cuda(f["a"]), None, Y, True)], M, path, df)
    assert_gemm_close(Y, oracle.dbf_linear(x, f["S_A"], f["S_B"], f["a"], f["m"], f["b"]), what=f"dbf stack M={M}")


@pytest.mark.parametrize("M,df", [(3, False), (1, True)])
def test_stack_longer_than_one_launch(ops, M, df):
    # 400 chained 64 x 64 layers: more than one launch's worth of descriptors (320 per launch;
    # with the dataflow form the second launch reads the first one's last output as an input).
    K, L = 64, 400
    host = [_layer(1000 + i, K, K) for i in range(L)]
    xb0, x = synth.activations(230, M, K)
    X0 = _x(xb0)
    # Each layer's output scale is divided by the rms of its output in the oracle's chain, so
    # the activations stay O(1): unscaled, these layers shrink them about 7x per layer, into
    # bf16's sub-normal range (spacing 9e-41) after about 45 layers, where a relative
    # tolerance says nothing.
    for i, (W, a, b) in enumerate(host):
        y = oracle.onebit_linear(x, oracle.sign_pm1(W), a, b)
        s = float(np.sqrt(np.mean(y * y)))
        host[i] = (W, (a / s).astype(np.float32), b)
        x = y / s
    Ys = [torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    spec, x = [], X0
    for i, ((W, a, b), Y) in enumerate(zip(host, Ys)):
        spec.append((x, ops.ob_pack_signs(_cuda(W)), _cuda(a), _cuda(b), Y, i > 0))
        x = Y
    _run(ops, spec, M, 0, df)
    for i in (0, 1, 318, 319, 320, 321, 382, 383, 384, 385, L - 1):
        W, a, b = host[i]
        assert_gemm_close(Ys[i], oracle.onebit_linear(_np(spec[i][0]), oracle.sign_pm1(W), a, b),
                          what=f"long stack layer {i}")


@pytest.mark.parametrize("M,df", [(1, False), (4, False), (1, True)])
def test_stack_in_cuda_graph(ops, M, df):
    # Replayed twice: the dataflow form's tag area is cleared inside the graph before each launch.
    K = 512
    host = [_layer(240 + i, K, K) for i in range(4)]
    X0 = _x(synth.activations(240, M, K)[0])
    Ys = [torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for _ in host]
    spec, x = [], X0
    for i, ((W, a, b), Y) in enumerate(zip(host, Ys)):
        spec.append((x, ops.ob_pack_signs(_cuda(W)), _cuda(a), _cuda(b), Y, i > 0))
        x = Y
    nws = ops.ob_linear_stack_workspace_size(spec, M) if df else ops.ob_stack_workspace_size()
    assert (nws > ops.ob_stack_workspace_size()) == df
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ops.ob_linear_stack(spec, M, workspace=ws, stream=s)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            ops.ob_linear_stack(spec, M, workspace=ws, stream=s)
    for Y in Ys:
        Y.zero_()
    torch.cuda.synchronize()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    _check(host, [(sp[0], sp[4]) for sp in spec], "graph stack")


@pytest.mark.parametrize("M,path,df", [(1, 0, False), (1, MMA, False), (2, 0, False), (16, 0, False), (1, 0, True)],
                         ids=["M1", "M1-mma", "M2", "M16", "M1-dataflow"])
def test_stack_7b_block(ops, M, path, df):
    # One 7B-shaped block: q, k, v, o (4096 -> 4096), gate, up (4096 -> 11008), down (11008 -> 4096).
    Wq, aq, bq, _ = oracle_svid(1, 4096, 4096)
    Wg, ag, bg, _ = oracle_svid(5, 11008, 4096)
    Wd, ad, bd, _ = oracle_svid(6, 4096, 11008)
    X0 = _x(synth.activations(250, M, 4096, outliers=True)[0])
    Pq, Pg, Pd = (ops.ob_pack_signs(_cuda(W)) for W in (Wq, Wg, Wd))
    buf = {n: torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
           for n, N in (("q", 4096), ("k", 4096), ("v", 4096), ("o", 4096), ("gate", 11008), ("up", 11008),
                        ("down", 4096))}
    P = {"q": (Pq, aq, bq, Wq), "k": (Pq, aq, bq, Wq), "v": (Pq, aq, bq, Wq), "o": (Pq, aq, bq, Wq),
         "gate": (Pg, ag, bg, Wg), "up": (Pg, ag, bg, Wg), "down": (Pd, ad, bd, Wd)}
    src = {"q": X0, "k": X0, "v": X0, "o": buf["q"], "gate": buf["o"], "up": buf["o"], "down": buf["gate"]}
    after = {"o": True, "gate": True, "down": True}
    order = ["q", "k", "v", "o", "gate", "up", "down"]
    spec = [(src[n], P[n][0], _cuda(P[n][1]), _cuda(P[n][2]), buf[n], after.get(n, False)) for n in order]
    _run(ops, spec, M, path, df)
    for n in order:
        W, a, b = P[n][3], P[n][1], P[n][2]
        assert_gemm_close(buf[n], oracle.onebit_linear(_np(src[n]), oracle.sign_pm1(W), a, b),
                          what=f"7b block {n} M={M}")


def test_stack_list_that_needs_barriers_with_a_large_workspace(ops):
    # A list whose third layer writes the buffer the first layer wrote (A -> B, B -> C, C -> B)
    # does not qualify for the dataflow form: its size is the barrier-only size, and with a
    # workspace as large as a qualifying list's it still runs with grid barriers.
    M, K = 1, 256
    host = [_layer(280 + i, K, K) for i in range(3)]
    X0 = _x(synth.activations(280, M, K)[0])
    B = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    C = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    P = [ops.ob_pack_signs(_cuda(W)) for W, _, _ in host]
    spec = [(X0, P[0], _cuda(host[0][1]), _cuda(host[0][2]), B, False),
            (B, P[1], _cuda(host[1][1]), _cuda(host[1][2]), C, True),
            (C, P[2], _cuda(host[2][1]), _cuda(host[2][2]), B, True)]
    assert ops.ob_linear_stack_workspace_size(spec, M) == ops.ob_stack_workspace_size()
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    ops.ob_linear_stack(spec, M, workspace=ws)
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    b1 = oracle.onebit_linear(_np(X0), oracle.sign_pm1(host[0][0]), host[0][1], host[0][2])
    # layer 1 read layer 0's output, since overwritten: the oracle's, rounded to bf16 as the GPU's was
    c = oracle.onebit_linear(_np(torch.from_numpy(b1).to(torch.bfloat16)), oracle.sign_pm1(host[1][0]), host[1][1],
                             host[1][2])
    assert_gemm_close(C, c, what="barrier list layer 1")
    assert_gemm_close(B, oracle.onebit_linear(_np(C), oracle.sign_pm1(host[2][0]), host[2][1], host[2][2]),
                      what="barrier list layer 2")


def test_stack_argument_errors(ops):
    from binary_weight_gemm_b200._lib import ObError
    K = 64
    W, a, b = _layer(260, 32, K)
    P = ops.ob_pack_signs(_cuda(W))
    X = torch.zeros((17, K), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((17, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ObError):  # M > 16
        ops.ob_linear_stack([(X, P, _cuda(a), _cuda(b), Y, False)], 17)
    X4, Y4 = X[:4].contiguous(), Y[:4].contiguous()
    with pytest.raises(ObError):  # workspace too small
        ops.ob_linear_stack([(X4, P, _cuda(a), _cuda(b), Y4, False)], 4,
                            workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(ObError):  # the int8 form takes at most two tokens
        ops.ob_linear_stack([(X4, P, _cuda(a), _cuda(b), Y4, False)], 4, path=I8)
    with pytest.raises(ObError):  # not a stack form
        ops.ob_linear_stack([(X4, P, _cuda(a), _cuda(b), Y4, False)], 4, path=3)
    ops.ob_linear_stack([], 4)  # empty list: nothing to do
    assert ops.ob_last_device_error() == 0
