"""GPU parity of sru_decode_step (one inference step with the projection fused)
against the fp64 oracle: oracle.project (Eq. (1)) then oracle.forward with
L = 1 (Eqs. (2)-(5)), from the same state c the GPU step started from.

Tolerance: the kernel forms u in fp32 (sums of d products), so each u carries
an error below 1e-5 * sum_k |X_k W_gk| (S_g); through one cell step an error
in u moves c and h by at most its size times (1 + |c - u_c| + |c' - alpha x|)
(the gates' slopes are <= 1/4, the candidate's <= 1).  On top of that the
fp32 cell itself: 1e-5 * (1 + |ref|).
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sru():
    import parallelizable_recurrence_b200 as m
    m.load_library()
    return m


def _inputs(B, d, seed):
    rng = np.random.default_rng(seed)
    Xb = f32_to_bf16_bits(rng.standard_normal((B, d)).astype(np.float32))
    lim = np.sqrt(3.0 / d)
    Wb = f32_to_bf16_bits(rng.uniform(-lim, lim, (3 * d, d)).astype(np.float32))
    x = bf16_bits_to_f32(Xb)  # the highway input is the layer input
    v = rng.uniform(-0.5, 0.5, (1, 2, d)).astype(np.float32)
    bias = rng.normal(0.0, 0.1, (1, 2, d)).astype(np.float32)
    c = rng.standard_normal((B, d)).astype(np.float32)
    return Xb, Wb, x, v, bias, c


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _oracle_step(Xb, Wb, x, v, bias, c, alpha):
    B, d = x.shape
    U = oracle.project(Xb, Wb).reshape(1, B, 1, 3, d)
    h, cT = oracle.forward(U, x.reshape(1, B, d), v, bias, c0=c.reshape(B, 1, d), alpha=alpha)
    Xf = bf16_bits_to_f32(Xb).astype(np.float64)
    Wf = bf16_bits_to_f32(Wb).astype(np.float64)
    S = np.abs(Xf) @ np.abs(Wf).T  # (B, 3d): sum_k |X_k W_gk|
    S = S[:, :d] + S[:, d:2 * d] + S[:, 2 * d:]
    U = U.reshape(B, 3, d)
    slope = 1.0 + np.abs(c - U[:, 0]) + np.abs(cT.reshape(B, d) - alpha * x)
    return h.reshape(B, d), cT.reshape(B, d), 1e-5 * S * slope


def _check(name, got, ref, extra):
    err = np.abs(got - ref)
    tol = 1e-5 * (1.0 + np.abs(ref)) + extra
    bad = err > tol
    assert not bad.any(), f"{name}: {bad.sum()} of {bad.size} beyond tolerance, worst {np.max(err - tol):.3g}"


# B = 8, 16, 24 take the tensor-core product (a multiple of 8, at least 8); the rest the fused kernel
@pytest.mark.parametrize("B,d", [(1, 8), (1, 2048), (3, 136), (16, 512), (21, 264), (2, 4096), (8, 2048),
                                 (24, 1024), (16, 4096)])
def test_decode_step_matches_oracle(sru, B, d):
    alpha = 1.0 if B != 3 else 0.5
    Xb, Wb, x, v, bias, c = _inputs(B, d, seed=B * 1000 + d)
    cd = torch.from_numpy(c).cuda()
    hd = torch.full((B, d), float("nan"), device="cuda")
    sru.sru_decode_step(_dev_bf16(Xb), _dev_bf16(Wb), torch.from_numpy(x).cuda(), torch.from_numpy(v).cuda(),
                        torch.from_numpy(bias).cuda(), cd, hd, alpha=alpha)
    assert sru.sru_sync_status() == 0
    h_ref, c_ref, extra = _oracle_step(Xb, Wb, x, v, bias, c, alpha)
    _check("h", hd.cpu().numpy().astype(np.float64), h_ref, extra)
    _check("c", cd.cpu().numpy().astype(np.float64), c_ref, extra)


def test_decode_steps_chain_the_state(sru):
    """Six steps in a row: each matches the oracle step from the state the GPU held."""
    B, d = 4, 1024
    _, Wb, _, v, bias, c = _inputs(B, d, seed=7)
    Wd, vd, bd = _dev_bf16(Wb), torch.from_numpy(v).cuda(), torch.from_numpy(bias).cuda()
    cd = torch.from_numpy(c).cuda()
    hd = torch.empty(B, d, device="cuda")
    rng = np.random.default_rng(8)
    for step in range(6):
        Xb = f32_to_bf16_bits(rng.standard_normal((B, d)).astype(np.float32))
        x = bf16_bits_to_f32(Xb)
        c_before = cd.cpu().numpy()
        sru.sru_decode_step(_dev_bf16(Xb), Wd, torch.from_numpy(x).cuda(), vd, bd, cd, hd)
        assert sru.sru_sync_status() == 0
        h_ref, c_ref, extra = _oracle_step(Xb, Wb, x, v, bias, c_before, 1.0)
        _check(f"h step {step}", hd.cpu().numpy().astype(np.float64), h_ref, extra)
        _check(f"c step {step}", cd.cpu().numpy().astype(np.float64), c_ref, extra)


def test_decode_step_agrees_with_forward_on_the_same_u(sru):
    """Given u that is exact in bf16 (so the forward's U holds it exactly), a
    decode step and sru_forward over L = 1 run the same cell arithmetic: with X
    one-hot rows, u = a single W entry, and the results agree bit for bit."""
    B, d = 3, 64
    _, Wb, _, v, bias, c = _inputs(B, d, seed=11)
    X = np.zeros((B, d), np.float32)
    for b in range(B):
        X[b, 5 * b + 1] = 1.0
    Xb = f32_to_bf16_bits(X)
    x = np.random.default_rng(12).standard_normal((B, d)).astype(np.float32)
    cd = torch.from_numpy(c).cuda()
    hd = torch.empty(B, d, device="cuda")
    xd = torch.from_numpy(x).cuda()
    vd, bd = torch.from_numpy(v).cuda(), torch.from_numpy(bias).cuda()
    sru.sru_decode_step(_dev_bf16(Xb), _dev_bf16(Wb), xd, vd, bd, cd, hd, alpha=0.75)
    Wf = bf16_bits_to_f32(Wb)
    U = (X @ Wf.T).reshape(1, B, 1, 3, d)  # exact: one nonzero product per entry
    h2 = torch.empty(1, B, 1, d, device="cuda")
    c2 = torch.empty(B, 1, d, device="cuda")
    sru.sru_forward(_dev_bf16(f32_to_bf16_bits(U)), xd.view(1, B, d), vd, bd, h2, c2,
                    c0=torch.from_numpy(c).cuda().view(B, 1, d), alpha=0.75, flags=sru.SRU_FLAG_FORCE_SEQUENTIAL)
    assert sru.sru_sync_status() == 0
    assert torch.equal(hd, h2.view(B, d))
    assert torch.equal(cd, c2.view(B, d))
