"""Python binding of libsru.so, the B200 (sm_100a) SRU layer library.

Argument marshalling only: every call forwards torch tensors' device pointers
and the current CUDA stream to the C ABI declared in ``include/sru.h``; all of
the arithmetic runs in the library's CUDA kernels.  There is no fallback: if
the shared library is missing or a tensor is not on a CUDA device, the call
raises.

Layer: the SRU cell of "When Attention Meets Fast Recurrence: Training Language
Models with Reduced Compute" (T. Lei), background section on SRU -- Eq. (1)
(the grouped projection U = X [W; W_f; W_r]^T) and Eqs. (2)-(5) (the
element-wise recurrence), with a highway scale alpha.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsru.so")

SRU_OK, SRU_ERR_INVALID, SRU_ERR_CUDA, SRU_ERR_TIMEOUT, SRU_ERR_UNSUPPORTED = 0, 1, 2, 3, 4
SRU_F32, SRU_BF16 = 0, 1
SRU_FLAG_V_ZERO = 0x1
SRU_FLAG_FORCE_SCAN = 0x2
SRU_FLAG_FORCE_SEQUENTIAL = 0x4
SRU_FLAG_TEST_WITHHOLD_CARRY = 0x8

# every symbol include/sru.h declares
EXPORTED = ("sru_status_string", "sru_get_last_cuda_error", "sru_version", "sru_workspace_bytes",
            "sru_project", "sru_project_backward", "sru_forward", "sru_backward", "sru_forward_scan_noalloc",
            "sru_forward_fused",
            "sru_project_factored", "sru_project_factored_backward", "sru_project_factored_backward_workspace_bytes",
            "sru_attention_workspace_bytes",
            "sru_attention_project", "sru_attention_backward_workspace_bytes", "sru_attention_project_backward",
            "sru_decode_workspace_bytes", "sru_decode_step", "sru_sync_status")


class SRUError(RuntimeError):
    def __init__(self, status: int, where: str, lib=None):
        self.status = status
        msg = f"{where}: status {status}"
        if lib is not None:
            msg += " (" + lib.sru_status_string(status).decode() + ")"
            if status == SRU_ERR_CUDA:
                msg += f" cudaError={lib.sru_get_last_cuda_error()}"
        super().__init__(msg)


_lib = None
_vp, _i64, _int, _f32, _u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_uint


def load_library(path: str = LIB_PATH):
    """Load libsru.so (built by parallelizable_recurrence_b200/build.py); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libsru.so not found at {path}: build it with "
                           "`python parallelizable_recurrence_b200/build.py` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    lib.sru_status_string.restype = ctypes.c_char_p
    lib.sru_status_string.argtypes = [_int]
    lib.sru_get_last_cuda_error.restype = _int
    lib.sru_get_last_cuda_error.argtypes = []
    lib.sru_version.restype = _int
    lib.sru_version.argtypes = []
    lib.sru_workspace_bytes.restype = ctypes.c_size_t
    lib.sru_workspace_bytes.argtypes = [_i64, _i64, _i64, _int, _u32]
    lib.sru_project.restype = _int
    lib.sru_project.argtypes = [_vp, _int, _vp, _int, _vp, _int, _i64, _i64, _i64, _vp]
    lib.sru_project_backward.restype = _int
    lib.sru_project_backward.argtypes = [_vp, _vp, _vp, _int, _vp, _int, _vp, _i64, _i64, _i64, _vp]
    lib.sru_forward.restype = _int
    lib.sru_forward.argtypes = [_vp, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _f32, _int, _u32,
                                _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.sru_backward.restype = _int
    lib.sru_backward.argtypes = [_vp, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _f32, _int, _u32,
                                 _vp, _vp, _vp, ctypes.c_size_t, _vp, _int, _vp, _vp, _vp, _vp, _vp]
    lib.sru_forward_scan_noalloc.restype = _int
    lib.sru_forward_scan_noalloc.argtypes = [_vp, _int, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _f32, _int,
                                             _vp, _vp, _vp]
    lib.sru_forward_fused.restype = _int
    lib.sru_forward_fused.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _f32, _int,
                                      _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.sru_project_factored.restype = _int
    lib.sru_project_factored.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _i64, _i64, _vp]
    lib.sru_project_factored_backward.restype = _int
    lib.sru_project_factored_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp, _i64, _i64,
                                                  _i64, _i64, _vp, ctypes.c_size_t, _vp]
    lib.sru_project_factored_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.sru_project_factored_backward_workspace_bytes.argtypes = [_i64, _i64, _i64, _i64]
    lib.sru_attention_workspace_bytes.restype = ctypes.c_size_t
    lib.sru_attention_workspace_bytes.argtypes = [_i64, _i64, _i64]
    lib.sru_attention_project.restype = _int
    lib.sru_attention_project.argtypes = [_vp, _vp, _vp, _vp, _f32, _vp, _vp, _int, _vp, _int, _i64, _i64, _i64,
                                          _i64, _i64, _vp, ctypes.c_size_t, _vp]
    lib.sru_attention_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.sru_attention_backward_workspace_bytes.argtypes = [_i64, _i64, _i64, _i64, _i64]
    lib.sru_attention_project_backward.restype = _int
    lib.sru_attention_project_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _int, _vp, ctypes.c_size_t,
                                                   _vp, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64,
                                                   _vp, ctypes.c_size_t, _vp]
    lib.sru_decode_step.restype = _int
    lib.sru_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _f32, _vp, ctypes.c_size_t, _vp]
    lib.sru_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.sru_decode_workspace_bytes.argtypes = [_i64, _i64]
    lib.sru_sync_status.restype = _int
    lib.sru_sync_status.argtypes = [_vp]
    _lib = lib
    return lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SRU_F32
    if t.dtype == torch.bfloat16:
        return SRU_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor], dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != SRU_OK:
        raise SRUError(status, where, _lib)


def sru_workspace_bytes(L: int, B: int, d: int, bidirectional: bool = False, flags: int = 0) -> int:
    return int(load_library().sru_workspace_bytes(L, B, d, int(bool(bidirectional)), flags))


def alloc_workspace(L: int, B: int, d: int, bidirectional: bool = False, flags: int = 0,
                    device="cuda") -> torch.Tensor:
    """A byte tensor of sru_workspace_bytes(...) bytes (torch owns the memory)."""
    n = sru_workspace_bytes(L, B, d, bidirectional, flags)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def sru_project(X: torch.Tensor, W: torch.Tensor, U: torch.Tensor, stream=None) -> torch.Tensor:
    """U[M, N] = X[M, K] @ W[N, K]^T (Eq. (1)); U is written in place and returned."""
    lib = load_library()
    K = X.shape[-1]
    M = X.numel() // K
    N = W.shape[0]
    assert W.shape[-1] == K and U.numel() == M * N
    _check(lib.sru_project(_ptr(X), _dtype_code(X), _ptr(W), _dtype_code(W), _ptr(U), _dtype_code(U),
                           M, N, K, _stream(stream)), "sru_project")
    return U


def sru_project_backward(dU: torch.Tensor, X: torch.Tensor, W: torch.Tensor,
                         dX: Optional[torch.Tensor] = None, dW: Optional[torch.Tensor] = None,
                         accumulate: bool = False, stream=None):
    """dX (+)= dU @ W and dW = dU^T @ X (fp32 outputs, written in place)."""
    lib = load_library()
    K = W.shape[-1]
    N = W.shape[0]
    M = dU.numel() // N
    t = _dtype_code(dU)
    assert X.dtype == dU.dtype and W.dtype == dU.dtype
    _check(lib.sru_project_backward(_ptr(dU), _ptr(X), _ptr(W), t, _ptr(dX, torch.float32), int(bool(accumulate)),
                                    _ptr(dW, torch.float32), M, N, K, _stream(stream)), "sru_project_backward")
    return dX, dW


def sru_forward(U, x, v, b, h, c_T, c0=None, mask=None, alpha: float = 1.0, bidirectional: bool = False,
                flags: int = 0, workspace=None, stream=None):
    """Eqs. (2)-(5).  U (L,B,n_dir,3,d) f32/bf16; x (L,B,d); v, b (n_dir,2,d);
    outputs h (L,B,n_dir,d) and c_T (B,n_dir,d) written in place."""
    lib = load_library()
    L, B, d = x.shape
    _check(lib.sru_forward(_ptr(U), _dtype_code(U), _ptr(x, torch.float32), _ptr(v, torch.float32),
                           _ptr(b, torch.float32), _ptr(c0, torch.float32), _ptr(mask, torch.uint8),
                           L, B, d, float(alpha), int(bool(bidirectional)), flags,
                           _ptr(h, torch.float32), _ptr(c_T, torch.float32), _ptr(workspace),
                           _nbytes(workspace), _stream(stream)),
           "sru_forward")
    return h, c_T


def sru_backward(U, x, v, b, dh, workspace, dU, dx, dv, db, dc0, c0=None, mask=None, dc_T=None,
                 alpha: float = 1.0, bidirectional: bool = False, flags: int = 0, stream=None):
    """Backward of sru_forward (same inputs and workspace); outputs written in place."""
    lib = load_library()
    L, B, d = x.shape
    _check(lib.sru_backward(_ptr(U), _dtype_code(U), _ptr(x, torch.float32), _ptr(v, torch.float32),
                            _ptr(b, torch.float32), _ptr(c0, torch.float32), _ptr(mask, torch.uint8),
                            L, B, d, float(alpha), int(bool(bidirectional)), flags,
                            _ptr(dh, torch.float32), _ptr(dc_T, torch.float32), _ptr(workspace),
                            _nbytes(workspace), _ptr(dU), _dtype_code(dU), _ptr(dx, torch.float32), _ptr(dv, torch.float32),
                            _ptr(db, torch.float32), _ptr(dc0, torch.float32), _stream(stream)),
           "sru_backward")
    return dU, dx, dv, db, dc0


def sru_forward_scan_noalloc(U, x, b, h, c_T, c0=None, mask=None, alpha: float = 1.0,
                             bidirectional: bool = False, stream=None):
    """Forward for v = 0 with no workspace, for callers that cannot allocate
    device memory: the scan's scratch is an 8 MiB static array inside libsru.so
    (shared by every call on a device, so calls must not overlap on the GPU).
    Inference only (no checkpoints).  Outputs h and c_T are written in place;
    a request larger than the static scratch raises SRUError (SRU_ERR_UNSUPPORTED)."""
    lib = load_library()
    L, B, d = x.shape
    _check(lib.sru_forward_scan_noalloc(_ptr(U), _dtype_code(U), _ptr(x, torch.float32), _ptr(b, torch.float32),
                                        _ptr(c0, torch.float32), _ptr(mask, torch.uint8), L, B, d, float(alpha),
                                        int(bool(bidirectional)), _ptr(h, torch.float32),
                                        _ptr(c_T, torch.float32), _stream(stream)),
           "sru_forward_scan_noalloc")
    return h, c_T


def sru_forward_fused(X, W, x, v, b, h, c_T, workspace, c0=None, mask=None, alpha: float = 1.0,
                      bidirectional: bool = False, U=None, stream=None):
    """Eq. (1) and Eqs. (2)-(5) in one kernel: X (L*B, d) bf16, W (n_dir*3d, d)
    bf16, x (L, B, d) fp32, v and b (n_dir, 2, d); h (L, B, n_dir, d) and c_T
    (B, n_dir, d) written in place.  With U ((L, B, n_dir, 3, d) bf16) the
    projection and the checkpoints are stored for sru_backward (same workspace)."""
    lib = load_library()
    L, B, d = x.shape
    _check(lib.sru_forward_fused(_ptr(X, torch.bfloat16), _ptr(W, torch.bfloat16), _ptr(x, torch.float32),
                                 _ptr(v, torch.float32), _ptr(b, torch.float32), _ptr(c0, torch.float32),
                                 _ptr(mask, torch.uint8), L, B, d, float(alpha), int(bool(bidirectional)),
                                 _ptr(h, torch.float32), _ptr(c_T, torch.float32), _ptr(U, torch.bfloat16),
                                 _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "sru_forward_fused")
    return h, c_T


def sru_project_factored(X, Wq, Wo, P, U, stream=None):
    """P = X Wq^T (bf16, written to P), U = P Wo^T.  X (M, K), Wq (Kp, K), Wo (N, Kp) bf16."""
    lib = load_library()
    M, K = X.shape
    Kp, N = Wq.shape[0], Wo.shape[0]
    if Wq.shape[1] != K or Wo.shape[1] != Kp or tuple(P.shape) != (M, Kp) or U.numel() != M * N:
        raise ValueError("shape mismatch")
    _check(lib.sru_project_factored(_ptr(X, torch.bfloat16), _ptr(Wq, torch.bfloat16), _ptr(Wo, torch.bfloat16),
                                    _ptr(P, torch.bfloat16), _ptr(U), _dtype_code(U), M, N, K, Kp,
                                    _stream(stream)), "sru_project_factored")
    return U


def sru_project_factored_backward(dU, X, Wq, Wo, P, dP, dX=None, accumulate: bool = False, dWq=None, dWo=None,
                                  workspace=None, stream=None):
    """dWo = dU^T P, dP = dU Wo (bf16, into dP), dWq = dP^T X, dX (+)= dP Wq (fp32 outputs).
    A workspace of sru_project_factored_backward_workspace_bytes bytes (the
    split weight gradients' slabs) is allocated when none is given; an empty
    tensor runs without one."""
    lib = load_library()
    M, K = X.shape
    Kp, N = Wq.shape[0], Wo.shape[0]
    if workspace is None:
        n = int(lib.sru_project_factored_backward_workspace_bytes(M, N, K, Kp))
        workspace = torch.empty(n, dtype=torch.uint8, device=dU.device)
    ws_ptr = _ptr(workspace) if workspace.numel() > 0 else None
    _check(lib.sru_project_factored_backward(_ptr(dU, torch.bfloat16), _ptr(X, torch.bfloat16),
                                             _ptr(Wq, torch.bfloat16), _ptr(Wo, torch.bfloat16),
                                             _ptr(P, torch.bfloat16), _ptr(dP, torch.bfloat16),
                                             _ptr(dX, torch.float32), int(bool(accumulate)),
                                             _ptr(dWq, torch.float32), _ptr(dWo, torch.float32), M, N, K, Kp,
                                             ws_ptr, _nbytes(workspace) if ws_ptr is not None else 0,
                                             _stream(stream)), "sru_project_factored_backward")
    return dX, dWq, dWo


def sru_attention_project(X, Wq, Wkv, Wo, U, L: int, B: int, alpha: float, ln_gamma=None, ln_beta=None,
                          causal: bool = True, workspace=None, stream=None):
    """SRU++ attention producer of U (see sru.h).  X (L*B, d) bf16 time-major,
    Wq (d', d), Wkv (2d', d') = [Wk; Wv], Wo (N, d') bf16; U (L*B, N) bf16 or
    fp32.  A workspace of sru_attention_workspace_bytes bytes is allocated when
    none is given."""
    lib = load_library()
    M, d = X.shape
    dp, N = Wq.shape[0], Wo.shape[0]
    if M != L * B or Wq.shape[1] != d or tuple(Wkv.shape) != (2 * dp, dp) or Wo.shape[1] != dp:
        raise ValueError("shape mismatch")
    if workspace is None:
        n = int(lib.sru_attention_workspace_bytes(L, B, dp))
        if n == 0:
            raise SRUError(SRU_ERR_UNSUPPORTED, "sru_attention_workspace_bytes", lib)
        workspace = torch.empty(n, dtype=torch.uint8, device=X.device)
    _check(lib.sru_attention_project(_ptr(X, torch.bfloat16), _ptr(Wq, torch.bfloat16), _ptr(Wkv, torch.bfloat16),
                                     _ptr(Wo, torch.bfloat16), float(alpha), _ptr(ln_gamma, torch.float32),
                                     _ptr(ln_beta, torch.float32), int(bool(causal)), _ptr(U), _dtype_code(U),
                                     L, B, d, dp, N, _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "sru_attention_project")
    return U


def sru_attention_project_backward(dU, X, Wq, Wkv, Wo, L: int, B: int, alpha: float, fwd_workspace, dX, dWq, dWkv,
                                   dWo, accumulate: bool = False, ln_gamma=None, ln_beta=None, dgamma=None,
                                   dbeta=None, causal: bool = True, workspace=None, stream=None):
    """Backward of sru_attention_project (see sru.h).  dU (L*B, N) bf16; X, Wq,
    Wkv, Wo, alpha, ln_gamma, ln_beta and causal as given to the forward, whose
    workspace (unchanged since) is fwd_workspace.  Writes dX (L*B, d) fp32 (or
    adds onto it with accumulate), dWq (d', d), dWkv (2d', d'), dWo (N, d') and,
    with the norm, dgamma, dbeta (d',), all fp32.  A workspace of
    sru_attention_backward_workspace_bytes bytes is allocated when none is given."""
    lib = load_library()
    M, d = X.shape
    dp, N = Wq.shape[0], Wo.shape[0]
    if M != L * B or tuple(dU.shape) != (M, N) or Wq.shape[1] != d or tuple(Wkv.shape) != (2 * dp, dp) \
            or Wo.shape[1] != dp:
        raise ValueError("shape mismatch")
    if tuple(dX.shape) != (M, d) or tuple(dWq.shape) != (dp, d) or tuple(dWkv.shape) != (2 * dp, dp) \
            or tuple(dWo.shape) != (N, dp):
        raise ValueError("gradient shape mismatch")
    if workspace is None:
        n = int(lib.sru_attention_backward_workspace_bytes(L, B, d, dp, N))
        if n == 0:
            raise SRUError(SRU_ERR_UNSUPPORTED, "sru_attention_backward_workspace_bytes", lib)
        workspace = torch.empty(n, dtype=torch.uint8, device=X.device)
    _check(lib.sru_attention_project_backward(
        _ptr(dU, torch.bfloat16), _ptr(X, torch.bfloat16), _ptr(Wq, torch.bfloat16), _ptr(Wkv, torch.bfloat16),
        _ptr(Wo, torch.bfloat16), float(alpha), _ptr(ln_gamma, torch.float32), _ptr(ln_beta, torch.float32),
        int(bool(causal)), _ptr(fwd_workspace), _nbytes(fwd_workspace), _ptr(dX, torch.float32),
        int(bool(accumulate)), _ptr(dWq, torch.float32), _ptr(dWkv, torch.float32), _ptr(dWo, torch.float32),
        _ptr(dgamma, torch.float32), _ptr(dbeta, torch.float32), L, B, d, dp, N, _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "sru_attention_project_backward")
    return dX, dWq, dWkv, dWo


def sru_decode_step(X_t, W, x_t, v, b, c, h_t, alpha: float = 1.0, workspace=None, stream=None):
    """One inference step of a unidirectional layer: u = X_t W^T (fp32), then
    Eqs. (2)-(5).  X_t (B, d) bf16, W (3d, d) bf16, x_t (B, d) fp32, v and b
    (2, d) fp32 (a (1, 2, d) slice is fine), c (B, d) fp32 state updated in
    place, h_t (B, d) fp32 output.  One fused kernel, except for batches of
    8, 16, 24, ... rows, whose product runs on the tensor cores in a workspace
    of sru_decode_workspace_bytes bytes (allocated when none is given)."""
    lib = load_library()
    B, d = X_t.shape
    if W.shape[0] != 3 * d or W.shape[1] != d:
        raise ValueError("W must be (3*d, d)")
    if workspace is None:
        n = int(lib.sru_decode_workspace_bytes(B, d))
        if n:
            workspace = torch.empty(n, dtype=torch.uint8, device=X_t.device)
    _check(lib.sru_decode_step(_ptr(X_t, torch.bfloat16), _ptr(W, torch.bfloat16), _ptr(x_t, torch.float32),
                               _ptr(v, torch.float32), _ptr(b, torch.float32), _ptr(c, torch.float32),
                               _ptr(h_t, torch.float32), B, d, float(alpha), _ptr(workspace), _nbytes(workspace),
                               _stream(stream)),
           "sru_decode_step")
    return h_t, c


def sru_sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side status code."""
    return int(load_library().sru_sync_status(_stream(stream)))
