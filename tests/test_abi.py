"""The C-ABI library builds, loads, and exports every declared symbol (CPU only).

Host-side argument checks are exercised too: they run before any CUDA call, so
they return their status without a GPU.
"""
import ctypes
import os

import pytest

from conftest import ROOT
from helpers import header_functions

HEADER = os.path.join(ROOT, "include", "obgemm.h")


@pytest.fixture(scope="module")
def lib():
    from binary_weight_gemm_b200 import build, _lib
    build.build()
    return _lib.lib()


def test_header_declares_the_boundary():
    names = header_functions(HEADER)
    for required in ["ob_pack_signs", "ob_svid_rank1", "ob_linear", "dbf_linear", "ob_last_device_error",
                     "ob_status_string", "ob_svid_workspace_size", "dbf_workspace_size"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from binary_weight_gemm_b200 import _lib
    names = header_functions(HEADER)
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} declared in obgemm.h but not exported"
    assert sorted(names) == sorted(_lib.SIGNATURES), "ctypes signatures and header disagree"


def test_library_exports_nothing_else():
    from binary_weight_gemm_b200 import _lib
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(line.split()[-1] for line in out.splitlines() if " T " in line)
    assert exported == sorted(_lib.SIGNATURES)


def test_status_strings_and_version(lib):
    for code in range(11):
        assert lib.ob_status_string(code)
    assert b"unknown" in lib.ob_status_string(99)
    assert lib.ob_version() >= 10000


def test_linear_workspace_size_and_checks(lib):
    # fp32 partial sums of the K slices for few-tile tcgen05 problems; 0 where no split applies
    assert lib.ob_linear_workspace_size(256, 4096, 4096) == 4 * 256 * 4096 * 4   # 32 tiles: 4 slices
    assert lib.ob_linear_workspace_size(16, 4096, 4096) == 0     # decode sizes
    assert lib.ob_linear_workspace_size(256, 4098, 4096) == 0    # N % 4 != 0
    assert lib.ob_linear_workspace_size(2048, 11008, 4096) == 0  # enough tiles
    assert lib.ob_linear_workspace_size(256, 4096, 40960) == 0   # K past the tcgen05 limit
    assert lib.ob_linear_workspace_size(-1, 4096, 4096) == 0
    assert lib.ob_linear_workspace_size(1 << 40, 1 << 40, 32) == 0
    OK, NULL, SHAPE, ALIGN, UNSUP = 0, 1, 2, 3, 9
    p, bad = ctypes.c_void_p(4096), ctypes.c_void_p(4100)
    assert lib.ob_linear_ws(p, 256, 64, p, 4, p, p, p, 0, bad, 1 << 20, 0, None) == ALIGN
    assert lib.ob_linear_ws(p, 256, 48, p, 4, p, p, p, 0, p, 1 << 20, 0, None) == SHAPE
    assert lib.ob_linear_ws(p, 256, 64, p, 4, p, p, p, 0, p, 1 << 20, 6, None) == UNSUP
    assert lib.ob_linear_ws(None, 0, 64, None, 4, None, None, None, 0, None, 0, 0, None) == OK


def test_workspace_sizes(lib):
    assert lib.dbf_workspace_size(512, 2048) >= 512 * 2048 * 2
    assert lib.dbf_workspace_size(0, 32) == 0
    assert lib.ob_svid_workspace_size(4096, 4096) >= 4 * (2 * 4096 + 4096)
    assert lib.ob_svid_workspace_size(-1, 3) == 0


def test_host_argument_checks_without_gpu(lib):
    OK, NULL, SHAPE, ALIGN, UNSUP = 0, 1, 2, 3, 9
    p = ctypes.c_void_p(4096)      # never dereferenced: each check returns first
    bad = ctypes.c_void_p(4100)    # not 16-byte aligned
    # shapes
    assert lib.ob_pack_signs(p, 4, 33, p, None) == SHAPE
    assert lib.ob_pack_signs(p, -1, 32, p, None) == SHAPE
    assert lib.ob_linear(p, 1, 48, p, 4, p, p, p, 0, None) == SHAPE
    assert lib.dbf_linear(p, 1, 64, p, 40, p, p, 4, p, p, p, 0, p, 1 << 20, None) == SHAPE
    # empty problems are no-ops
    assert lib.ob_pack_signs(None, 0, 64, None, None) == OK
    assert lib.ob_linear(None, 0, 64, None, 8, None, None, None, 0, None) == OK
    assert lib.ob_linear(None, 3, 64, None, 0, None, None, None, 0, None) == OK
    # options
    assert lib.ob_linear(p, 1, 64, p, 4, p, p, p, 7, None) == UNSUP
    assert lib.ob_linear_ex(p, 1, 64, p, 4, p, p, p, 0, 42, None) == UNSUP
    assert lib.ob_linear_ex(p, 1, 64, p, 4, p, p, p, 0, 0x200, None) == UNSUP   # unknown flag
    assert lib.ob_linear_ex(p, 1, 64, p, 4, p, p, p, 0, 0x102, None) == UNSUP   # removed path, with a flag
    assert lib.ob_linear_ex(p, 1, 64, p, 4, p, p, p, 0, -1, None) == UNSUP
    assert lib.ob_linear_ex(None, 0, 64, None, 8, None, None, None, 0, 0x100, None) == OK  # static weights
    assert lib.ob_linear_ex(p, 1, 64, p, 4, p, p, p, 0, 6, None) == UNSUP   # the one-launch DBF form
    assert lib.ob_linear_ex(p, 1, 64, p, 4, p, p, p, 0, 8, None) == UNSUP
    assert lib.ob_linear_ex(None, 0, 64, None, 8, None, None, None, 0, 7, None) == OK  # the one-CTA tcgen05 GEMM
    assert lib.dbf_linear_ex(p, 1, 64, p, 32, p, p, 4, p, p, p, 0, p, 1 << 20, 7, None) == UNSUP
    # dbf_linear_ex: the one-launch form only at decode sizes; unknown flags rejected
    assert lib.dbf_linear_ex(p, 17, 64, p, 32, p, p, 4, p, p, p, 0, p, 1 << 20, 6, None) == UNSUP
    assert lib.dbf_linear_ex(p, 1, 64, p, 32, p, p, 4, p, p, p, 0, p, 1 << 20, 0x400, None) == UNSUP
    assert lib.dbf_linear_ex(p, 1, 64, p, 32, p, p, 4, p, p, p, 0, p, 1 << 20, 7, None) == UNSUP
    # null and alignment
    assert lib.ob_linear(None, 1, 64, p, 4, p, p, p, 0, None) == NULL
    assert lib.ob_linear(p, 1, 64, p, 4, p, p, None, 0, None) == NULL
    assert lib.ob_linear(bad, 1, 64, p, 4, p, p, p, 0, None) == ALIGN
    assert lib.ob_pack_signs(bad, 2, 64, p, None) == ALIGN
    assert lib.dbf_linear(p, 1, 64, p, 32, p, p, 4, p, p, p, 0, None, 0, None) == 6  # workspace
    assert lib.dbf_linear(p, 1, 64, p, 32, None, p, 4, p, p, p, 0, p, 1 << 20, None) == NULL
    iters = ctypes.c_int(-1)
    assert lib.ob_svid_rank1(p, 4, 64, p, p, None, 0, 0.0, ctypes.byref(iters), None, 0, None) == 6
    assert iters.value == 0
    assert lib.ob_svid_rank1(p, 4, 62, p, p, None, 0, 0.0, None, p, 1 << 20, None) == SHAPE


def test_python_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from binary_weight_gemm_b200 import _lib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_LIB", None)
    with pytest.raises(ImportError):
        _lib.lib()


def test_layernorm_and_stack_argument_checks_without_gpu(lib):
    from binary_weight_gemm_b200._lib import ObLayer
    OK, NULL, SHAPE, ALIGN, WS, UNSUP = 0, 1, 2, 3, 6, 9
    p = ctypes.c_void_p(4096)
    bad = ctypes.c_void_p(4100)
    # ob_linear_ln: eps is checked before anything else; then the ob_linear checks.
    for eps in (-1.0, float("nan"), float("inf")):
        assert lib.ob_linear_ln(p, 1, 64, p, 4, p, p, p, 0, eps, 0, None) == UNSUP
    assert lib.ob_linear_ln(p, 1, 48, p, 4, p, p, p, 0, 1e-5, 0, None) == SHAPE
    assert lib.ob_linear_ln(None, 0, 64, None, 8, None, None, None, 0, 1e-5, 0, None) == OK
    assert lib.ob_linear_ln(p, 1, 64, p, 4, p, p, None, 0, 1e-5, 0, None) == NULL
    # ob_linear_stack: every descriptor is validated before a launch.
    assert lib.ob_stack_workspace_size() >= 8

    def layers(*descs):
        arr = (ObLayer * len(descs))()
        for i, d in enumerate(descs):
            arr[i] = d
        return arr

    good = ObLayer(p, p, p, p, p, 64, 32, 0, 0)
    ws, wsn = p, lib.ob_stack_workspace_size()
    assert lib.ob_linear_stack(layers(good), 1, 17, ws, wsn, None) == SHAPE       # M > 16
    assert lib.ob_linear_stack(layers(good), 0, 4, ws, wsn, None) == OK           # no layers
    assert lib.ob_linear_stack(layers(good), 1, 0, ws, wsn, None) == OK           # no tokens
    assert lib.ob_linear_stack(None, 1, 4, ws, wsn, None) == NULL
    assert lib.ob_linear_stack(layers(good), 1, 4, None, wsn, None) == NULL
    assert lib.ob_linear_stack(layers(good), 1, 4, bad, wsn, None) == ALIGN
    assert lib.ob_linear_stack(layers(good), 1, 4, ws, 4, None) == WS
    assert lib.ob_linear_stack(layers(good, ObLayer(p, p, p, p, p, 48, 32, 0, 1)), 2, 4, ws, wsn, None) == SHAPE
    assert lib.ob_linear_stack(layers(ObLayer(p, p, p, p, p, 64, 0, 0, 0)), 1, 4, ws, wsn, None) == SHAPE
    assert lib.ob_linear_stack(layers(ObLayer(p, p, p, p, p, 64, 32, 5, 0)), 1, 4, ws, wsn, None) == UNSUP
    assert lib.ob_linear_stack(layers(ObLayer(p, None, p, p, p, 64, 32, 0, 0)), 1, 4, ws, wsn, None) == NULL
    assert lib.ob_linear_stack(layers(ObLayer(p, p, p, bad, p, 64, 32, 0, 0)), 1, 4, ws, wsn, None) == ALIGN
    # a null input scale is allowed (no scale); the next check that fails is the device context
    st = lib.ob_linear_stack(layers(ObLayer(p, p, p, None, p, 64, 32, 0, 0)), 1, 4, ws, wsn, None)
    assert st not in (NULL, SHAPE, ALIGN, WS, UNSUP)


def test_stack_dataflow_workspace_analysis_without_gpu(lib):
    # The dataflow form of ob_linear_stack (tagged outputs instead of grid barriers) needs every
    # layer to write its own buffer and every input to be outside all outputs or exactly an
    # earlier layer's bf16 output; otherwise the size is the barrier-only size.
    from binary_weight_gemm_b200._lib import ObLayer
    base = lib.ob_stack_workspace_size()

    def size(descs, M):
        arr = (ObLayer * len(descs))()
        for i, d in enumerate(descs):
            arr[i] = ObLayer(*d)
        return lib.ob_linear_stack_workspace_size(arr, len(descs), M)

    def align256(x):
        return (x + 255) // 256 * 256

    X0, W, A = 1 << 20, 2 << 20, 3 << 20
    Y = [(8 + i) << 20 for i in range(4)]  # distinct 1 MB buffers
    # chain X0 -> Y0 -> Y1 -> Y2 (K = N = 64): Y0 and Y1 are read by later layers
    chain = [(X0, W, A, None, Y[0], 64, 64, 0, 0), (Y[0], W, A, None, Y[1], 64, 64, 0, 1),
             (Y[1], W, A, None, Y[2], 64, 64, 0, 1)]
    assert size(chain, 1) == base + align256(2 * 64 * 4)
    assert size(chain, 2) == base                       # one token only (two measured slower)
    assert size(chain, 3) == base
    # q, k, v read one input; o reads q: only q's output is tagged
    block = [(X0, W, A, None, Y[0], 64, 128, 0, 0), (X0, W, A, None, Y[1], 64, 128, 0, 0),
             (X0, W, A, None, Y[2], 64, 128, 0, 0), (Y[0], W, A, None, Y[3], 128, 64, 0, 1)]
    assert size(block, 1) == base + align256(128 * 4)
    # every tagged output starts on 256 bytes: 128 words each for two 96-wide outputs at M = 1
    odd = [(X0, W, A, None, Y[0], 64, 96, 0, 0), (X0, W, A, None, Y[1], 64, 96, 0, 0),
           (Y[0], W, A, None, Y[2], 96, 32, 0, 1), (Y[1], W, A, None, Y[3], 96, 32, 0, 1)]
    assert size(odd, 1) == base + 2 * 512
    # two layers writing one buffer, a later layer writing an earlier layer's input, an input
    # that only overlaps an output, a producer with fp32 output: barriers only
    assert size([chain[0], (Y[0], W, A, None, Y[0], 64, 64, 0, 1)], 1) == base
    assert size([(X0, W, A, None, Y[0], 64, 64, 0, 0), (Y[0], W, A, None, X0, 64, 64, 0, 1)], 1) == base
    assert size([chain[0], (Y[0] + 64, W, A, None, Y[1], 32, 64, 0, 1)], 1) == base
    assert size([(X0, W, A, None, Y[0], 64, 64, 1, 0), (Y[0], W, A, None, Y[1], 64, 64, 0, 1)], 1) == base
    # no consumer inside the list: nothing to tag
    assert size([chain[0]], 1) == base
    assert lib.ob_linear_stack_workspace_size(None, 3, 1) == base


def test_factorize_argument_checks_without_gpu(lib):
    NULL, SHAPE, ALIGN, WS, UNSUP = 1, 2, 3, 6, 9
    p = ctypes.c_void_p(4096)
    bad = ctypes.c_void_p(4100)
    ws = lib.dbf_factorize_workspace_size(64, 128, 32)
    assert ws >= 4 * (5 * 64 * 32 + 5 * 128 * 32 + 3 * 128 * 32 + 2 * 32 * 32 + 64 * 128)
    assert lib.dbf_factorize_workspace_size(64, 100, 32) == 0   # K not a multiple of 32
    assert lib.dbf_factorize_workspace_size(64, 128, 48) == 0   # r not a multiple of 32
    assert lib.dbf_factorize_workspace_size(0, 128, 32) == 0

    def call(W=p, N=64, K=128, r=32, omega=p, sweeps=2, admm=3, cg=25, rho=1.0, refit=2, SA=p, SB=p, a=p, m=p,
             b=p, work=p, wsb=ws):
        return lib.dbf_factorize(W, N, K, r, omega, sweeps, admm, cg, rho, refit, SA, SB, a, m, b, None, None, None,
                                 work, wsb, None)

    assert call(K=100) == SHAPE
    assert call(r=48) == SHAPE
    assert call(r=0) == SHAPE
    assert call(N=0) == SHAPE
    assert call(sweeps=-1) == UNSUP
    assert call(admm=0) == UNSUP
    assert call(cg=0) == UNSUP
    assert call(rho=0.0) == UNSUP
    assert call(rho=float("nan")) == UNSUP
    assert call(refit=-1) == UNSUP
    assert call(W=None) == NULL
    assert call(omega=None) == NULL
    assert call(m=None) == NULL
    assert call(work=None) == NULL
    assert call(SB=bad) == ALIGN
    assert call(wsb=ws - 1) == WS
    # valid arguments: the next check is the device context (no GPU here)
    assert call() not in (NULL, SHAPE, ALIGN, WS, UNSUP)


def test_sizes_whose_products_wrap_are_rejected_without_gpu(lib):
    # Shapes whose element counts overflow 64 bits when multiplied must be refused by the
    # host checks (OB_ERR_SHAPE / OB_ERR_WORKSPACE), never reach a launch.
    SHAPE, WS = 2, 6
    p = ctypes.c_void_p(4096)
    M, r = 1 << 37, 1 << 26          # M * r * 2 == 2**64: wraps to 0 in size_t
    assert lib.dbf_linear_noalloc(p, M, 64, p, r, p, p, 4, p, p, p, 0, None) == WS
    assert lib.dbf_linear(p, M, 64, p, r, p, p, 4, p, p, p, 0, p, 1 << 20, None) == SHAPE
    assert lib.dbf_workspace_size(M, r) == 0
    big = 1 << 40
    assert lib.ob_linear(p, big, big, p, 4, p, p, p, 0, None) == SHAPE
    assert lib.ob_linear(p, 4, big, p, big, p, p, p, 0, None) == SHAPE
    assert lib.ob_pack_signs(p, big, big, p, None) == SHAPE
    assert lib.ob_svid_workspace_size(big, big) == 0
    assert lib.ob_svid_rank1(p, big, big, p, p, None, 0, 0.0, None, p, 1 << 20, None) == SHAPE
