"""Helpers shared by the GPU parity tests: move seeded inputs to the device, run
the CUDA path through the C-ABI binding, run the fp64 oracle on the same inputs
(or on a sampled sub-problem), and compare with the stated tolerances.

Tolerances:
  recurrence outputs (h, c_T, dU, highway dx, dv, db, dc0), fp32 arithmetic:
      |gpu - ref| <= 1e-5 * (1 + |ref|)
  a bf16-stored dU additionally gets one bf16 unit in the last place of ref
  outputs that go through a bf16 projection (U, end-to-end h):
      |gpu - ref| <= 2e-2 * (1 + |ref|)
  fp32 outputs of long products (dX, dW):
      |gpu - ref| <= 1e-5 * (1 + |ref|) + 1e-5 * sum_k |a_k b_k|
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from synthetic import bf16_bits_to_f32

REC_TOL = 1e-5
BF16_TOL = 2e-2


def to_dev_f32(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_dev_u8(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_U(inp):
    """U on the device in its storage type (bf16 from bit patterns, or fp32)."""
    U = inp["U"]
    return to_dev_bf16(U) if U.dtype == np.uint16 else to_dev_f32(U)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def U_values(inp) -> np.ndarray:
    U = inp["U"]
    return bf16_bits_to_f32(U) if U.dtype == np.uint16 else U


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 2.0 ** -133)


def abs_operand(a: np.ndarray) -> np.ndarray:
    """|a| in the same storage type (bf16 bit patterns: clear the sign bit)."""
    return (a & np.uint16(0x7FFF)) if a.dtype == np.uint16 else np.abs(a)


def assert_close_sum(name, got, ref, absref, tol=1e-5, sum_tol=1e-5):
    """For a product computed as a long fp32 sum: |gpu - ref| <= tol*(1+|ref|) + sum_tol*sum_k|a_k b_k|.

    absref is the same sum over |a| and |b|; rounding error of an fp32 sum grows
    with it, not with |ref| (which cancellation can make small)."""
    assert_close(name, got, ref, tol, extra=sum_tol * np.asarray(absref, dtype=np.float64))


def assert_close(name, got, ref, tol, extra=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    bound = tol * (1.0 + np.abs(ref))
    if extra is not None:
        bound = bound + extra
    err = np.abs(got - ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), err.shape)
        raise AssertionError(f"{name}: {bad.sum()} of {err.size} outside tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} |d|={err[i]:.3e} bound={bound[i]:.3e}")


def run_gpu_recurrence(sru, inp, n_dir, alpha, du_dtype=torch.float32, flags=0, backward=True, dc_T=None):
    """Run sru_forward (+ sru_backward) on the device; returns host numpy outputs."""
    x = inp["x"]
    L, B, d = x.shape
    U = dev_U(inp)
    xd = to_dev_f32(x)
    v, b = to_dev_f32(inp["v"]), to_dev_f32(inp["bias"])
    c0 = to_dev_f32(inp["c0"])
    mask = to_dev_u8(inp["mask"])
    h = torch.full((L, B, n_dir, d), float("nan"), device="cuda")
    cT = torch.full((B, n_dir, d), float("nan"), device="cuda")
    ws = sru.alloc_workspace(L, B, d, n_dir == 2, flags)
    sru.sru_forward(U, xd, v, b, h, cT, c0=c0, mask=mask, alpha=alpha, bidirectional=n_dir == 2,
                    flags=flags, workspace=ws)
    out = {}
    if backward:
        dh = to_dev_f32(inp["dh"])
        dcT = to_dev_f32(dc_T)
        dU = torch.full((L, B, n_dir, 3, d), float("nan"), device="cuda", dtype=du_dtype)
        dx = torch.full((L, B, d), float("nan"), device="cuda")
        dv = torch.full((n_dir, 2, d), float("nan"), device="cuda")
        db = torch.full((n_dir, 2, d), float("nan"), device="cuda")
        dc0 = torch.full((B, n_dir, d), float("nan"), device="cuda")
        sru.sru_backward(U, xd, v, b, dh, ws, dU, dx, dv, db, dc0, c0=c0, mask=mask, dc_T=dcT, alpha=alpha,
                         bidirectional=n_dir == 2, flags=flags)
        out.update(dU=dU, dx=dx, dv=dv, db=db, dc0=dc0)
    status = sru.sru_sync_status()
    assert status == 0, f"device status {status}"
    out.update(h=h, cT=cT)
    return {k: host_f64(t) for k, t in out.items()}


def oracle_recurrence(inp, alpha, bs=None, js=None, backward=True, dc_T=None):
    """Oracle forward/backward on all channels, or on batch rows bs x channels js."""
    U = U_values(inp)
    x, v, bias, c0, mask = inp["x"], inp["v"], inp["bias"], inp["c0"], inp["mask"]
    dh = inp.get("dh")
    if bs is not None:
        bs = np.asarray(bs)
        js = np.asarray(js)
        U = U[:, bs][:, :, :, :, js]
        x = x[:, bs][:, :, js]
        v, bias = v[:, :, js], bias[:, :, js]
        c0 = None if c0 is None else c0[bs][:, :, js]
        mask = None if mask is None else mask[:, bs]
        dh = None if dh is None else dh[:, bs][:, :, :, js]
        dc_T = None if dc_T is None else dc_T[bs][:, :, js]
    h, cT = oracle.forward(U, x, v, bias, c0=c0, mask=mask, alpha=alpha)
    out = dict(h=h, cT=cT)
    if backward:
        out.update(oracle.backward(U, x, v, bias, dh, c0=c0, mask=mask, dcT=dc_T, alpha=alpha))
    return out


def compare_recurrence(gpu, ref, du_bf16=False, bs=None, js=None, backward=True):
    sel = (lambda a, nb: a) if bs is None else None
    if bs is not None:
        bs = np.asarray(bs)
        js = np.asarray(js)

        def sel(a, kind):
            if kind == "LBD":      # (L, B, n_dir, d)
                return a[:, bs][:, :, :, js]
            if kind == "LBD3":     # (L, B, n_dir, 3, d)
                return a[:, bs][:, :, :, :, js]
            if kind == "LBd":      # (L, B, d)
                return a[:, bs][:, :, js]
            if kind == "BD":       # (B, n_dir, d)
                return a[bs][:, :, js]
            if kind == "V":        # (n_dir, 2, d) -- needs every b in bs
                return a[:, :, js]
            raise ValueError(kind)
    assert_close("h", sel(gpu["h"], "LBD"), ref["h"], REC_TOL)
    assert_close("c_T", sel(gpu["cT"], "BD"), ref["cT"], REC_TOL)
    if not backward:
        return
    extra = bf16_ulp(ref["dU"]) if du_bf16 else None
    assert_close("dU", sel(gpu["dU"], "LBD3"), ref["dU"], REC_TOL, extra=extra)
    assert_close("dx", sel(gpu["dx"], "LBd"), ref["dx"], REC_TOL)
    assert_close("dc0", sel(gpu["dc0"], "BD"), ref["dc0"], REC_TOL)
    assert_close("dv", sel(gpu["dv"], "V"), ref["dv"], REC_TOL)
    assert_close("db", sel(gpu["db"], "V"), ref["dbias"], REC_TOL)
