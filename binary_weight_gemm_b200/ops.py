"""Python binding of libobgemm: the C-ABI calls, by the same names, on torch CUDA tensors.

Argument marshalling only.  Every step of the computation runs in the library's
CUDA kernels; torch supplies device memory and the current stream.  There is no
CPU fallback: without the built library the calls raise.

Layouts (see include/obgemm.h): X bf16 [M, K]; packed signs int32 [R, C/32]
(uint32 bit patterns, bit i of word w <-> column 32w+i, set bit = -1); scale
vectors fp32; Y bf16 or fp32 [M, N].
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (OB_FLAG_STATIC_WEIGHTS, OB_PATH_STACK, OB_PATH_TC1, OB_OUT_BF16, OB_OUT_F32, OB_PATH_AUTO, OB_PATH_I8, OB_PATH_MMA_DECODE, OB_PATH_SIMT,  # noqa: F401
                   OB_PATH_TC, ObError)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple | None = None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _out_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return OB_OUT_BF16
    if dtype == torch.float32:
        return OB_OUT_F32
    raise TypeError("output dtype must be torch.bfloat16 or torch.float32")


def ob_pack_signs(W: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Packed W_sign (int32 [N, K/32]) of fp32 W [N, K]; K % 32 == 0."""
    N, K = W.shape
    _need(W, "W", torch.float32)
    if out is None:
        out = torch.empty((N, K // 32), dtype=torch.int32, device=W.device)
    _need(out, "out", torch.int32, (N, K // 32))
    _lib.check("ob_pack_signs", _lib.lib().ob_pack_signs(_ptr(W), N, K, _ptr(out), _stream(stream)))
    return out


def ob_last_device_error(stream=None) -> int:
    """Synchronise, then read and clear the device error word (returns an ob_status code)."""
    return int(_lib.lib().ob_last_device_error(_stream(stream)))


def ob_svid_workspace_size(N: int, K: int) -> int:
    return int(_lib.lib().ob_svid_workspace_size(N, K))


def ob_svid_rank1(W: torch.Tensor, max_iters: int = 0, tol: float = 0.0, workspace: torch.Tensor | None = None,
                  stream=None, check: bool = True):
    """Rank-1 SVID of |W|: returns (a [N], b [K], sigma1 [1], iterations, status)."""
    N, K = W.shape
    _need(W, "W", torch.float32)
    a = torch.empty(N, dtype=torch.float32, device=W.device)
    b = torch.empty(K, dtype=torch.float32, device=W.device)
    sigma = torch.empty(1, dtype=torch.float32, device=W.device)
    ws_bytes = ob_svid_workspace_size(N, K)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=W.device)
    iters = ctypes.c_int(0)
    st = int(_lib.lib().ob_svid_rank1(_ptr(W), N, K, _ptr(a), _ptr(b), _ptr(sigma), int(max_iters),
                                      float(tol), ctypes.byref(iters), _ptr(workspace), workspace.numel(),
                                      _stream(stream)))
    if check:
        _lib.check("ob_svid_rank1", st)
    return a, b, sigma, iters.value, st


def ob_linear_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.lib().ob_linear_workspace_size(M, N, K))


def ob_linear(X: torch.Tensor, W_packed: torch.Tensor, a: torch.Tensor, b: torch.Tensor,
              out_dtype: torch.dtype = torch.bfloat16, path: int = OB_PATH_AUTO, out: torch.Tensor | None = None,
              stream=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """OneBit layer Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T; X bf16 [M, K], W_packed int32 [N, K/32].

    workspace (uint8, optional): lets a few-tile tcgen05 problem split over K (ob_linear_ws).
    """
    M, K = X.shape
    N = W_packed.shape[0]
    _need(X, "X", torch.bfloat16)
    _need(W_packed, "W_packed", torch.int32, (N, K // 32))
    _need(a, "a", torch.float32, (N,))
    _need(b, "b", torch.float32, (K,))
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=X.device)
    _need(out, "out", out_dtype, (M, N))
    if workspace is None:
        st = _lib.lib().ob_linear_ex(_ptr(X), M, K, _ptr(W_packed), N, _ptr(a), _ptr(b), _ptr(out),
                                     _out_code(out_dtype), int(path), _stream(stream))
    else:
        st = _lib.lib().ob_linear_ws(_ptr(X), M, K, _ptr(W_packed), N, _ptr(a), _ptr(b), _ptr(out),
                                     _out_code(out_dtype), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     int(path), _stream(stream))
    _lib.check("ob_linear", st)
    return out


def ob_linear_ln(X: torch.Tensor, W_packed: torch.Tensor, a: torch.Tensor, b: torch.Tensor, eps: float = 1e-5,
                 out_dtype: torch.dtype = torch.bfloat16, path: int = OB_PATH_AUTO, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """OneBit layer then LayerNorm over each token's N outputs: Z = LayerNorm(Y), no affine, biased variance."""
    M, K = X.shape
    N = W_packed.shape[0]
    _need(X, "X", torch.bfloat16)
    _need(W_packed, "W_packed", torch.int32, (N, K // 32))
    _need(a, "a", torch.float32, (N,))
    _need(b, "b", torch.float32, (K,))
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=X.device)
    _need(out, "out", out_dtype, (M, N))
    st = _lib.lib().ob_linear_ln(_ptr(X), M, K, _ptr(W_packed), N, _ptr(a), _ptr(b), _ptr(out),
                                 _out_code(out_dtype), float(eps), int(path), _stream(stream))
    _lib.check("ob_linear_ln", st)
    return out


def ob_stack_workspace_size() -> int:
    return int(_lib.lib().ob_stack_workspace_size())


def _stack_array(layers, M: int):
    arr = (_lib.ObLayer * max(1, len(layers)))()
    dev = None
    for i, (X, P, a, b, Y, after) in enumerate(layers):
        K = X.shape[1]
        N = P.shape[0]
        _need(X, "X", torch.bfloat16, (M, K))
        _need(P, "W_packed", torch.int32, (N, K // 32))
        _need(a, "a", torch.float32, (N,))
        if b is not None:
            _need(b, "b", torch.float32, (K,))
        _need(Y, "Y", Y.dtype, (M, N))
        arr[i] = _lib.ObLayer(_ptr(X), _ptr(P), _ptr(a), _ptr(b), _ptr(Y), K, N, _out_code(Y.dtype),
                              1 if after else 0)
        dev = X.device
    return arr, dev


def ob_linear_stack_workspace_size(layers, M: int) -> int:
    """Workspace bytes with which ob_linear_stack runs this list in its dataflow form (tagged
    outputs instead of grid barriers; int8 form, one token, every layer writing its own
    buffer), or ob_stack_workspace_size() where that form does not apply."""
    arr, _ = _stack_array(layers, M)
    return int(_lib.lib().ob_linear_stack_workspace_size(arr, len(layers), M))


def ob_linear_stack(layers, M: int, workspace: torch.Tensor | None = None, stream=None,
                    path: int = OB_PATH_AUTO) -> None:
    """Run a list of OneBit layers (M <= 16 tokens) in one persistent launch.

    layers: sequence of (X, W_packed, a, b, Y, after_previous); X bf16 [M, K], W_packed int32
    [N, K/32], a fp32 [N], b fp32 [K] or None, Y bf16/fp32 [M, N] (written), after_previous:
    True if X is an output of an earlier layer of the list.  path: OB_PATH_AUTO,
    OB_PATH_MMA_DECODE or OB_PATH_I8 (M <= 2).  workspace: at least ob_stack_workspace_size()
    bytes; ob_linear_stack_workspace_size(layers, M) bytes enable the dataflow form.
    """
    arr, dev = _stack_array(layers, M)
    if workspace is None:
        workspace = torch.zeros(ob_stack_workspace_size(), dtype=torch.uint8, device=dev or "cuda")
    st = _lib.lib().ob_linear_stack_ex(arr, len(layers), M, _ptr(workspace), workspace.numel(), int(path),
                                       _stream(stream))
    _lib.check("ob_linear_stack_ex", st)


def dbf_workspace_size(M: int, r: int) -> int:
    return int(_lib.lib().dbf_workspace_size(M, r))


def dbf_linear(X: torch.Tensor, SB_packed: torch.Tensor, m: torch.Tensor, SA_packed: torch.Tensor,
               a: torch.Tensor, b: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16,
               path: int = OB_PATH_AUTO, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """DBF layer Y = ((((X ⊙ b^T) S_B^T) ⊙ m^T) S_A^T) ⊙ a^T.

    X bf16 [M, K]; SB_packed int32 [r, K/32]; m fp32 [r]; SA_packed int32 [N, r/32].
    """
    M, K = X.shape
    r = SB_packed.shape[0]
    N = SA_packed.shape[0]
    _need(X, "X", torch.bfloat16)
    _need(SB_packed, "SB_packed", torch.int32, (r, K // 32))
    _need(SA_packed, "SA_packed", torch.int32, (N, r // 32))
    _need(m, "m", torch.float32, (r,))
    _need(a, "a", torch.float32, (N,))
    _need(b, "b", torch.float32, (K,))
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=X.device)
    _need(out, "out", out_dtype, (M, N))
    ws_bytes = dbf_workspace_size(M, r)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=X.device)
    st = _lib.lib().dbf_linear_ex(_ptr(X), M, K, _ptr(SB_packed), r, _ptr(m), _ptr(SA_packed), N, _ptr(a),
                                  _ptr(b), _ptr(out), _out_code(out_dtype), _ptr(workspace), workspace.numel(),
                                  int(path), _stream(stream))
    _lib.check("dbf_linear", st)
    return out


def dbf_factorize_workspace_size(N: int, K: int, r: int) -> int:
    return int(_lib.lib().dbf_factorize_workspace_size(N, K, r))


def dbf_factorize(W: torch.Tensor, r: int, omega: torch.Tensor, sweeps: int = 20, admm_iters: int = 3,
                  cg_iters: int = 5, rho_rel: float = 1.0, refit_rounds: int = 2,
                  workspace: torch.Tensor | None = None, stream=None) -> dict:
    """DBF factorisation W ≈ diag(a) S_A diag(m) S_B diag(b) (synchronous).

    W fp32 [N, K]; omega fp32 [K, r] (the start's random matrix).  Returns a dict with
    SA_packed int32 [N, r/32], SB_packed int32 [r, K/32], a [N], m [r], b [K] (fp32, on
    W's device), "history" (list of sweeps floats), "best" and "error" (floats).
    """
    N, K = W.shape
    _need(W, "W", torch.float32)
    _need(omega, "omega", torch.float32, (K, r))
    dev = W.device
    SA = torch.empty((N, r // 32), dtype=torch.int32, device=dev)
    SB = torch.empty((r, K // 32), dtype=torch.int32, device=dev)
    a = torch.empty(N, dtype=torch.float32, device=dev)
    m = torch.empty(r, dtype=torch.float32, device=dev)
    b = torch.empty(K, dtype=torch.float32, device=dev)
    ws_bytes = dbf_factorize_workspace_size(N, K, r)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    hist = (ctypes.c_float * max(sweeps, 1))()
    best, err = ctypes.c_float(0.0), ctypes.c_float(0.0)
    st = _lib.lib().dbf_factorize(_ptr(W), N, K, r, _ptr(omega), int(sweeps), int(admm_iters), int(cg_iters),
                                  float(rho_rel), int(refit_rounds), _ptr(SA), _ptr(SB), _ptr(a), _ptr(m), _ptr(b),
                                  ctypes.cast(hist, ctypes.c_void_p), ctypes.cast(ctypes.pointer(best), ctypes.c_void_p),
                                  ctypes.cast(ctypes.pointer(err), ctypes.c_void_p), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _lib.check("dbf_factorize", st)
    return {"SA_packed": SA, "SB_packed": SB, "a": a, "m": m, "b": b, "history": list(hist)[:sweeps],
            "best": best.value, "error": err.value}


def ob_selftest_timeout(limit_ns: int = 2_000_000, stream=None) -> int:
    """Run the bounded-wait self-test; returns the ob_status it reports (8 = timeout recorded)."""
    return int(_lib.lib().ob_selftest_timeout(int(limit_ns), _stream(stream)))
