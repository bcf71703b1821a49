"""dbf_linear_noalloc: the DBF layer for callers that cannot allocate device memory.

Such callers (code running under CUDA graph capture, engines with a fixed
memory plan, plugins whose memory belongs to another allocator) cannot hand
dbf_linear a workspace, so this entry point keeps the M x r intermediate in a
static device array.  Its results must match dbf_linear's on the same inputs,
call after call, because every call reuses the same array.  This file sorts
last so that a run stopping at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from binary_weight_gemm_b200 import synth
from helpers import assert_gemm_close

pytestmark = pytest.mark.gpu


def _cuda(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _problem(ops, seed, M, N, r, K):
    f = synth.dbf_factors(seed, N, r, K)
    xb, _ = synth.activations(seed, M, K)
    return {
        "X": _cuda(xb.view(np.int16)).view(torch.bfloat16),
        "SB": ops.ob_pack_signs(_cuda(f["S_B"].astype(np.float32))),
        "SA": ops.ob_pack_signs(_cuda(f["S_A"].astype(np.float32))),
        "m": _cuda(f["m"]), "a": _cuda(f["a"]), "b": _cuda(f["b"]),
        "M": M, "N": N, "r": r, "K": K,
    }


def _call_both(lib, p, stream):
    """The existing entry point (caller-owned workspace) and the static-scratch one, via the C ABI."""
    M, N, r, K = p["M"], p["N"], p["r"], p["K"]
    y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y_new = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws_bytes = lib.dbf_workspace_size(M, r)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    args = (p["X"].data_ptr(), M, K, p["SB"].data_ptr(), r, p["m"].data_ptr(), p["SA"].data_ptr(), N,
            p["a"].data_ptr(), p["b"].data_ptr())
    st = lib.dbf_linear(*args, y_ref.data_ptr(), 0, ws.data_ptr(), ws.numel(), stream)
    assert st == 0, st
    st = lib.dbf_linear_noalloc(*args, y_new.data_ptr(), 0, stream)
    assert st == 0, st
    torch.cuda.synchronize()
    return y_ref, y_new


def test_noalloc_matches_dbf_linear_two_calls_in_a_row():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import _lib, ops
    lib = _lib.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # Two different problems back to back: the second call finds the first one's
    # intermediate in the shared array and must not be affected by it.
    p1 = _problem(ops, 41, 512, 4096, 2048, 4096)   # the DBF prefill workload: 2 MiB intermediate
    p2 = _problem(ops, 42, 3, 200, 96, 160)          # small, ragged
    for p in (p1, p2):
        y_ref, y_new = _call_both(lib, p, stream)
        assert_gemm_close(y_new, y_ref.float().cpu().numpy().astype(np.float64),
                          what=f"noalloc M={p['M']} N={p['N']} r={p['r']} K={p['K']}")
    assert ops.ob_last_device_error() == 0


def test_noalloc_rejects_intermediate_beyond_static_scratch():
    from binary_weight_gemm_b200 import build
    build.build()
    from binary_weight_gemm_b200 import _lib
    lib = _lib.lib()
    # M * r * 2 bytes one row over the limit: refused before anything is launched.
    r = 2048
    M = _lib.DBF_NOALLOC_SCRATCH_BYTES // (2 * r) + 1
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    st = lib.dbf_linear_noalloc(p, M, 4096, p, r, p, p, 4096, p, p, p, 0,
                                torch.cuda.current_stream().cuda_stream)
    assert st == 6  # OB_ERR_WORKSPACE
