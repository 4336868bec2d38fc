"""GPU parity of the factorised projection (P = X Wq^T, U = P Wo^T) and its
gradients against the fp64 oracle's plain products.

The oracle keeps every intermediate in fp64; the GPU rounds P, dP (and a bf16
U) to bf16 (relative error <= 2^-9 each) and accumulates in fp32.  So each
output may differ by 2^-8 of the sum of the magnitudes of the products that
passed through a rounded operand, 2^-8 of itself when it is stored in bf16,
and 1e-5 of the sum of product magnitudes for the fp32 accumulation.  A
dropped k-slice, a transposed operand or a wrong block moves outputs by
O(1) of those sums, far outside these bounds.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

R8 = 2.0 ** -8


@pytest.fixture(scope="module")
def sru():
    import parallelizable_recurrence_b200 as m
    m.load_library()
    return m


def _bits(rng, shape, scale):
    return f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _host_bf16(t):
    return bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def _check(name, got, ref, tol):
    err = np.abs(got - ref)
    bad = err > tol
    assert not bad.any(), f"{name}: {bad.sum()} of {bad.size} beyond tolerance, worst {np.max(err - tol):.3g}"


@pytest.mark.parametrize("M,K,Kp,N", [(111, 256, 64, 768), (256, 2048, 512, 6144), (9, 64, 16, 192),
                                       (4100, 512, 128, 1536)])  # few output tiles, long reduction: split
def test_factored_projection_and_gradients(sru, M, K, Kp, N):
    rng = np.random.default_rng(M + K)
    Xb = _bits(rng, (M, K), 1.0)
    Wqb = _bits(rng, (Kp, K), K ** -0.5)
    Wob = _bits(rng, (N, Kp), Kp ** -0.5)
    dUb = _bits(rng, (M, N), 1.0)
    X, Wq, Wo, dU = (bf16_bits_to_f32(a).astype(np.float64) for a in (Xb, Wqb, Wob, dUb))
    aX, aWq, aWo, adU = np.abs(X), np.abs(Wq), np.abs(Wo), np.abs(dU)

    Xd, Wqd, Wod = _dev(Xb), _dev(Wqb), _dev(Wob)
    P = torch.empty(M, Kp, device="cuda", dtype=torch.bfloat16)
    U = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    sru.sru_project_factored(Xd, Wqd, Wod, P, U)
    Uf = torch.empty(M, N, device="cuda")
    sru.sru_project_factored(Xd, Wqd, Wod, torch.empty_like(P), Uf)
    assert sru.sru_sync_status() == 0

    P_ref = oracle.project(Xb, Wqb)          # fp64, never rounded
    U_ref = oracle.project(P_ref, Wob)
    aP = np.abs(P_ref)
    sP = aX @ aWq.T                          # magnitudes summed into each P
    _check("P", _host_bf16(P), P_ref, R8 * aP + 1e-5 * sP)
    tolU = R8 * (aP @ aWo.T) + 1e-5 * (sP @ aWo.T) + 1e-5 * (aP @ aWo.T)
    _check("U fp32", Uf.cpu().numpy().astype(np.float64), U_ref, tolU)
    _check("U bf16", _host_bf16(U), U_ref, tolU + R8 * np.abs(U_ref))

    dUd = _dev(dUb)
    dP = torch.empty(M, Kp, device="cuda", dtype=torch.bfloat16)
    dX = torch.full((M, K), 0.5, device="cuda")
    dWq = torch.empty(Kp, K, device="cuda")
    dWo = torch.empty(N, Kp, device="cuda")
    sru.sru_project_factored_backward(dUd, Xd, Wqd, Wod, P, dP, dX=dX, accumulate=True, dWq=dWq, dWo=dWo)
    assert sru.sru_sync_status() == 0

    dWo_ref = oracle.project_dW(dUb, P_ref)                 # dU^T P
    dP_ref = oracle.project_dX(dUb, Wob)                    # dU Wo
    dWq_ref = oracle.project_dW(dP_ref, Xb)                 # dP^T X
    dX_ref = oracle.project_dX(dP_ref, Wqb) + 0.5           # dP Wq, onto the 0.5 already there
    adP = np.abs(dP_ref)
    s_dP = adU @ aWo
    _check("dWo", dWo.cpu().numpy().astype(np.float64), dWo_ref,
           R8 * (adU.T @ aP) + 1e-5 * (adU.T @ sP) + 1e-5 * (adU.T @ aP))
    _check("dP", _host_bf16(dP), dP_ref, R8 * adP + 1e-5 * s_dP)
    _check("dWq", dWq.cpu().numpy().astype(np.float64), dWq_ref,
           R8 * (adP.T @ aX) + 1e-5 * (s_dP.T @ aX) + 1e-5 * (adP.T @ aX))
    _check("dX", dX.cpu().numpy().astype(np.float64), dX_ref,
           R8 * (adP @ aWq) + 1e-5 * (s_dP @ aWq) + 1e-5 * (adP @ aWq) + 1e-6)


def test_factored_equals_two_plain_projections(sru):
    """The factored call is exactly the two sru_project calls it chains."""
    rng = np.random.default_rng(3)
    M, K, Kp, N = 200, 512, 128, 1536
    Xd, Wqd, Wod = _dev(_bits(rng, (M, K), 1.0)), _dev(_bits(rng, (Kp, K), 0.05)), _dev(_bits(rng, (N, Kp), 0.1))
    P1 = torch.empty(M, Kp, device="cuda", dtype=torch.bfloat16)
    U1 = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    sru.sru_project_factored(Xd, Wqd, Wod, P1, U1)
    P2 = torch.empty_like(P1)
    U2 = torch.empty_like(U1)
    sru.sru_project(Xd, Wqd, P2)
    sru.sru_project(P2, Wod, U2)
    assert sru.sru_sync_status() == 0
    assert torch.equal(P1.view(torch.int16), P2.view(torch.int16))
    assert torch.equal(U1.view(torch.int16), U2.view(torch.int16))


def test_split_weight_gradients_are_deterministic_and_match_the_single_product(sru):
    """dWq and dWo of a narrow d' over many tokens are cut along the tokens
    into workspace slabs summed in a fixed order: the same bits on every run,
    and the single product (no workspace) within fp32 summation-order error."""
    rng = np.random.default_rng(5)
    M, K, Kp, N = 8192, 256, 64, 768
    Xd, Wqd, Wod = _dev(_bits(rng, (M, K), 1.0)), _dev(_bits(rng, (Kp, K), 0.06)), _dev(_bits(rng, (N, Kp), 0.1))
    dUd = _dev(_bits(rng, (M, N), 1.0))
    P = torch.empty(M, Kp, device="cuda", dtype=torch.bfloat16)
    sru.sru_project_factored(Xd, Wqd, Wod, P, torch.empty(M, N, device="cuda", dtype=torch.bfloat16))
    runs = []
    for ws in (None, None, torch.empty(0, dtype=torch.uint8, device="cuda")):
        dP = torch.empty(M, Kp, device="cuda", dtype=torch.bfloat16)
        dWq, dWo = torch.empty(Kp, K, device="cuda"), torch.empty(N, Kp, device="cuda")
        sru.sru_project_factored_backward(dUd, Xd, Wqd, Wod, P, dP, dWq=dWq, dWo=dWo, workspace=ws)
        assert sru.sru_sync_status() == 0
        runs.append((dWq, dWo))
    assert sru.load_library().sru_project_factored_backward_workspace_bytes(M, N, K, Kp) > 0
    for a, b in zip(runs[0], runs[1]):
        assert torch.equal(a, b)
    for a, b in zip(runs[0], runs[2]):
        scale = b.abs().max().item()
        assert (a - b).abs().max().item() <= 1e-5 * scale * 8
