"""Plain fp64 CPU oracle of the SRU layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never does, and this package imports nothing from it.

The arithmetic lives in ``sru_oracle.c`` (plain C loops in double precision,
one (direction, batch row, channel) stream at a time); this module only builds
that file with gcc and marshals numpy arrays into it.

Source of the method: "When Attention Meets Fast Recurrence: Training Language
Models with Reduced Compute" (T. Lei), background section on SRU, Eq. (1)
(grouped projection) and Eqs. (2)-(5) (element-wise recurrence).  The backward
pass is the reverse-mode derivative of those equations.

Layouts (time-major, last index fastest):
  U (L, B, n_dir, 3, d) with gate blocks [candidate | forget | reset]
  x (L, B, d); h (L, B, n_dir, d); v, bias (n_dir, 2, d) rows [forget, reset]
  c0, cT (B, n_dir, d); mask (L, B) uint8 with 1 = padded position.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sru_oracle.c")
_LIB = os.path.join(_HERE, "libsru_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile sru_oracle.c into libsru_oracle.so (plain -O2, IEEE arithmetic)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.sru_oracle_forward.restype = ctypes.c_int
        lib.sru_oracle_forward.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_double,
                                           _dp, _dp, _dp, _dp, _dp, ctypes.c_void_p,
                                           _dp, _dp]
        lib.sru_oracle_backward.restype = ctypes.c_int
        lib.sru_oracle_backward.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_double,
                                            _dp, _dp, _dp, _dp, _dp, ctypes.c_void_p,
                                            _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        gemm_args = [ctypes.c_void_p, ctypes.c_int, _i64, _i64,
                     ctypes.c_void_p, ctypes.c_int, _i64, _i64, _dp]
        lib.sru_oracle_gemm.restype = ctypes.c_int
        lib.sru_oracle_gemm.argtypes = [_i64, _i64, _i64] + gemm_args
        lib.sru_oracle_gemm_entries.restype = ctypes.c_int
        lib.sru_oracle_gemm_entries.argtypes = [_i64, ctypes.c_void_p, ctypes.c_void_p, _i64] + gemm_args
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _mask_ptr(mask, L, B):
    if mask is None:
        return None, None
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    assert m.shape == (L, B)
    return m, ctypes.c_void_p(m.ctypes.data)


def forward(U, x, v, bias, c0=None, mask=None, alpha=1.0):
    """Eqs. (2)-(5) for every channel.  Returns (h, cT) in float64.

    U: (L, B, n_dir, 3, d); x: (L, B, d); v, bias: (n_dir, 2, d);
    c0: (B, n_dir, d) or None; mask: (L, B) or None.
    """
    U = _f64(U)
    L, B, n_dir, three, d = U.shape
    assert three == 3
    x, v, bias = _f64(x), _f64(v), _f64(bias)
    assert x.shape == (L, B, d) and v.shape == (n_dir, 2, d) and bias.shape == (n_dir, 2, d)
    c0 = None if c0 is None else _f64(c0)
    m, mp = _mask_ptr(mask, L, B)
    h = np.empty((L, B, n_dir, d))
    cT = np.empty((B, n_dir, d))
    rc = _load().sru_oracle_forward(L, B, d, n_dir, float(alpha), _ptr(U), _ptr(x), _ptr(v),
                                    _ptr(bias), _ptr(c0), mp, _ptr(h), _ptr(cT))
    if rc != 0:
        raise RuntimeError(f"sru_oracle_forward failed ({rc})")
    return h, cT


def backward(U, x, v, bias, dh, c0=None, mask=None, dcT=None, alpha=1.0):
    """Reverse-mode derivative of forward() for Loss = sum(dh*h) + sum(dcT*cT).

    Returns dict with dU (L,B,n_dir,3,d), dx (L,B,d) (highway part, summed over
    directions), dv and dbias (n_dir,2,d), dc0 (B,n_dir,d); all float64.
    """
    U = _f64(U)
    L, B, n_dir, _, d = U.shape
    x, v, bias, dh = _f64(x), _f64(v), _f64(bias), _f64(dh)
    assert dh.shape == (L, B, n_dir, d)
    c0 = None if c0 is None else _f64(c0)
    dcT = None if dcT is None else _f64(dcT)
    m, mp = _mask_ptr(mask, L, B)
    out = dict(dU=np.empty((L, B, n_dir, 3, d)), dx=np.empty((L, B, d)),
               dv=np.empty((n_dir, 2, d)), dbias=np.empty((n_dir, 2, d)),
               dc0=np.empty((B, n_dir, d)))
    rc = _load().sru_oracle_backward(L, B, d, n_dir, float(alpha), _ptr(U), _ptr(x), _ptr(v),
                                     _ptr(bias), _ptr(c0), mp, _ptr(dh), _ptr(dcT),
                                     _ptr(out["dU"]), _ptr(out["dx"]), _ptr(out["dv"]),
                                     _ptr(out["dbias"]), _ptr(out["dc0"]))
    if rc != 0:
        raise RuntimeError(f"sru_oracle_backward failed ({rc})")
    return out


def _operand(a):
    """(contiguous array, dtype code) for a GEMM operand: fp32, bf16 bits (uint16) or fp64."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.uint16:
        return a, 1
    if a.dtype == np.float64:
        return a, 2
    raise TypeError(f"unsupported operand dtype {a.dtype}")


def gemm(A, a_rs, a_ks, Bm, b_rs, b_ks, R, C, K):
    """out[r, c] = sum_k A(r, k) * Bm(c, k) with explicit element strides (float64 result)."""
    A, at = _operand(A)
    Bm, bt = _operand(Bm)
    out = np.empty((R, C))
    rc = _load().sru_oracle_gemm(R, C, K, ctypes.c_void_p(A.ctypes.data), at, a_rs, a_ks,
                                 ctypes.c_void_p(Bm.ctypes.data), bt, b_rs, b_ks, _ptr(out))
    if rc != 0:
        raise RuntimeError("sru_oracle_gemm failed")
    return out


def gemm_entries(rows, cols, K, A, a_rs, a_ks, Bm, b_rs, b_ks):
    """The gemm() sum evaluated only at the listed (rows[i], cols[i]) entries."""
    A, at = _operand(A)
    Bm, bt = _operand(Bm)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    assert rows.shape == cols.shape
    out = np.empty(rows.shape[0])
    rc = _load().sru_oracle_gemm_entries(rows.shape[0], ctypes.c_void_p(rows.ctypes.data),
                                         ctypes.c_void_p(cols.ctypes.data), K,
                                         ctypes.c_void_p(A.ctypes.data), at, a_rs, a_ks,
                                         ctypes.c_void_p(Bm.ctypes.data), bt, b_rs, b_ks, _ptr(out))
    if rc != 0:
        raise RuntimeError("sru_oracle_gemm_entries failed")
    return out


# --- the three products of Eq. (1) and its gradients, named -----------------

def project(X, W):
    """U = X W^T (Eq. (1)): X (M, K), W (N, K) -> (M, N) float64."""
    M, K = X.shape
    N = W.shape[0]
    return gemm(X, K, 1, W, K, 1, M, N, K)


def project_dX(dU, W):
    """dX = dU W: dU (M, N), W (N, K) -> (M, K) float64."""
    M, N = dU.shape
    K = W.shape[1]
    return gemm(dU, N, 1, W, 1, K, M, K, N)


def project_dW(dU, X):
    """dW = dU^T X: dU (M, N), X (M, K) -> (N, K) float64."""
    M, N = dU.shape
    K = X.shape[1]
    return gemm(dU, 1, N, X, 1, K, N, K, M)


def project_entries(X, W, rows, cols):
    """Selected entries U[rows[i], cols[i]] of X W^T."""
    K = X.shape[1]
    return gemm_entries(rows, cols, K, X, K, 1, W, K, 1)


def project_dX_entries(dU, W, rows, cols):
    """Selected entries dX[rows[i], cols[i]] of dU W."""
    N = dU.shape[1]
    K = W.shape[1]
    return gemm_entries(rows, cols, N, dU, N, 1, W, 1, K)


def project_dW_entries(dU, X, rows, cols):
    """Selected entries dW[rows[i], cols[i]] of dU^T X."""
    M, N = dU.shape
    K = X.shape[1]
    return gemm_entries(rows, cols, M, dU, 1, N, X, 1, K)


def _as_f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:  # bf16 bits, widened exactly
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def attention_project(X, Wq, Wk, Wv, Wo, alpha, L, B, causal=True, ln_gamma=None, ln_beta=None, ln_eps=1e-5):
    """SRU++'s producer of U ("When Attention Meets Fast Recurrence", SRU++
    section: attention replaces the linear map of Eq. (1)), in fp64:

      Q = X Wq^T, K = Q Wk^T, V = Q Wv^T         (rows = tokens; Wq (d', d), Wk, Wv (d', d'))
      per batch row b, over its L tokens:
        A_b = softmax(Q_b K_b^T / sqrt(d')) V_b   (scaled dot-product attention;
                                                   with causal=True token t sees tokens <= t)
      R = Q + alpha A, or layernorm(Q + alpha A) over the d' features
          (ln_gamma, ln_beta given; the page's post-attention normalisation)
      U = R Wo^T                                  (Wo (N, d'))

    X is (L*B, d) time-major (row t*B + b), bf16 bits or floats; returns U
    (L*B, N) float64.  Every product is a plain matrix product; the softmax
    subtracts the row maximum before exponentiating (the same value).
    """
    X, Wq, Wk, Wv, Wo = (_as_f64(a) for a in (X, Wq, Wk, Wv, Wo))
    Q = X @ Wq.T
    K = Q @ Wk.T
    V = Q @ Wv.T
    dp = Q.shape[1]
    A = np.zeros_like(Q)
    for b in range(B):
        rows = np.arange(L) * B + b
        Qb, Kb, Vb = Q[rows], K[rows], V[rows]
        for t in range(L):
            n = t + 1 if causal else L
            s = Kb[:n] @ Qb[t] / np.sqrt(dp)
            p = np.exp(s - s.max())
            A[rows[t]] = (p / p.sum()) @ Vb[:n]
    R = Q + alpha * A
    if ln_gamma is not None:
        mu = R.mean(axis=1, keepdims=True)
        var = ((R - mu) ** 2).mean(axis=1, keepdims=True)
        R = (R - mu) / np.sqrt(var + ln_eps) * _as_f64(ln_gamma) + _as_f64(ln_beta)
    return R @ Wo.T


def attention_project_backward(dU, X, Wq, Wk, Wv, Wo, alpha, L, B, causal=True, ln_gamma=None, ln_beta=None,
                               ln_eps=1e-5):
    """Reverse-mode derivative of attention_project for Loss = sum(dU * U), in
    fp64, taking the forward's steps backwards one at a time (the chain rule on
    each line of attention_project; the forward values are recomputed here):

      U = R Wo^T                     dWo = dU^T R,  dR = dU Wo
      R = layernorm(Z) g + b         dg = sum_m dR * Zhat,  db = sum_m dR,
                                     dZ = (dZhat - mean(dZhat) - Zhat mean(dZhat * Zhat)) / sigma,
                                     dZhat = dR g   (or dZ = dR without the norm)
      Z = Q + alpha A                dQ = dZ,  dA = alpha dZ
      A_t = sum_s p_ts V_s           dV_s += p_ts dA_t,  dp_ts = V_s . dA_t
      p_t = softmax(q_t K^T / sqrt(d'))
                                     ds_ts = p_ts (dp_ts - sum_s' p_ts' dp_ts') / sqrt(d')
                                     dQ_t += sum_s ds_ts K_s,  dK_s += ds_ts Q_t
      K = Q Wk^T, V = Q Wv^T         dQ += dK Wk + dV Wv,  dWk = dK^T Q,  dWv = dV^T Q
      Q = X Wq^T                     dWq = dQ^T X,  dX = dQ Wq

    Returns a dict with dX (L*B, d), dWq, dWk, dWv, dWo and, with the norm,
    dgamma and dbeta (d',), all float64.
    """
    dU, X, Wq, Wk, Wv, Wo = (_as_f64(a) for a in (dU, X, Wq, Wk, Wv, Wo))
    Q = X @ Wq.T
    K = Q @ Wk.T
    V = Q @ Wv.T
    dp = Q.shape[1]
    A = np.zeros_like(Q)
    probs = {}
    for b in range(B):
        rows = np.arange(L) * B + b
        Qb, Kb, Vb = Q[rows], K[rows], V[rows]
        for t in range(L):
            n = t + 1 if causal else L
            s = Kb[:n] @ Qb[t] / np.sqrt(dp)
            p = np.exp(s - s.max())
            p = p / p.sum()
            probs[(b, t)] = p
            A[rows[t]] = p @ Vb[:n]
    Z = Q + alpha * A
    out = {}
    if ln_gamma is not None:
        g = _as_f64(ln_gamma)
        mu = Z.mean(axis=1, keepdims=True)
        sigma = np.sqrt(((Z - mu) ** 2).mean(axis=1, keepdims=True) + ln_eps)
        Zhat = (Z - mu) / sigma
        R = Zhat * g + _as_f64(ln_beta)
    else:
        R = Z
    out["dWo"] = dU.T @ R
    dR = dU @ Wo
    if ln_gamma is not None:
        out["dgamma"] = (dR * Zhat).sum(axis=0)
        out["dbeta"] = dR.sum(axis=0)
        dZhat = dR * g
        dZ = (dZhat - dZhat.mean(axis=1, keepdims=True) - Zhat * (dZhat * Zhat).mean(axis=1, keepdims=True)) / sigma
    else:
        dZ = dR
    dQ = dZ.copy()
    dA = alpha * dZ
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for b in range(B):
        rows = np.arange(L) * B + b
        Qb, Kb, Vb = Q[rows], K[rows], V[rows]
        for t in range(L):
            n = t + 1 if causal else L
            p = probs[(b, t)]
            dV[rows[:n]] += np.outer(p, dA[rows[t]])
            dpt = Vb[:n] @ dA[rows[t]]
            ds = p * (dpt - p @ dpt) / np.sqrt(dp)
            dQ[rows[t]] += ds @ Kb[:n]
            dK[rows[:n]] += np.outer(ds, Qb[t])
    dQ += dK @ Wk + dV @ Wv
    out["dWk"] = dK.T @ Q
    out["dWv"] = dV.T @ Q
    out["dWq"] = dQ.T @ X
    out["dX"] = dQ @ Wq
    return out
