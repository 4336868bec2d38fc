"""GPU parity of the projection of Eq. (1) and of its gradients against the fp64
oracle (plain sums over the same bf16 / fp32 operands).

Shapes are ragged in every dimension of the 128 x 256 x 64 tensor-core tile
(M = 300, N = 600, K = 200) and also span several tiles and k-blocks.
"""
import numpy as np
import pytest
import torch

import oracle
import sru_testlib as tl
from synthetic import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

# Products with fp32 outputs (dX, dW, fp32 U) are long sums: their rounding
# error grows with sum_k |a_k b_k|, not with |ref| (which cancellation can make
# arbitrarily small), so they are checked against
#   |gpu - ref| <= 1e-5 * (1 + |ref|) + 1e-5 * sum_k |a_k b_k|,
# a bound that a dropped or misplaced k-slice exceeds by orders of magnitude.
# bf16 outputs (U) are also checked within one bf16 ulp and in the 2e-2 class.


@pytest.fixture(scope="module")
def sru():
    import parallelizable_recurrence_b200 as m
    m.load_library()
    return m


def _bf16(rng, shape, scale=1.0):
    return f32_to_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))


SHAPES = [(300, 600, 200), (128, 256, 64), (1000, 1536, 512), (64, 24, 8), (4096, 768, 256)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_project_bf16(sru, M, N, K):
    rng = np.random.default_rng(M + N + K)
    Xb, Wb = _bf16(rng, (M, K)), _bf16(rng, (N, K), 1.0 / np.sqrt(K))
    ref = oracle.project(Xb, Wb)
    X, W = tl.to_dev_bf16(Xb), tl.to_dev_bf16(Wb)
    U32 = torch.full((M, N), float("nan"), device="cuda")
    sru.sru_project(X, W, U32)
    U16 = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    sru.sru_project(X, W, U16)
    assert sru.sru_sync_status() == 0
    tl.assert_close_sum("U(f32 out)", tl.host_f64(U32), ref, oracle.project(tl.abs_operand(Xb), tl.abs_operand(Wb)))
    tl.assert_close("U(bf16 out)", tl.host_f64(U16), ref, tl.BF16_TOL)
    # the bf16 output is the fp32 accumulator rounded to nearest: within one bf16 ulp of ref
    tl.assert_close("U(bf16 out, ulp)", tl.host_f64(U16), ref, 1e-5, extra=tl.bf16_ulp(ref))


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("accumulate", [False, True])
def test_project_backward_bf16(sru, M, N, K, accumulate):
    rng = np.random.default_rng(7 * M + N + K)
    Xb, Wb, dUb = _bf16(rng, (M, K)), _bf16(rng, (N, K), 0.1), _bf16(rng, (M, N))
    base = rng.standard_normal((M, K)).astype(np.float32)
    ref_dX = oracle.project_dX(dUb, Wb) + (base if accumulate else 0.0)
    ref_dW = oracle.project_dW(dUb, Xb)
    dX = tl.to_dev_f32(base) if accumulate else torch.full((M, K), float("nan"), device="cuda")
    dW = torch.full((N, K), float("nan"), device="cuda")
    sru.sru_project_backward(tl.to_dev_bf16(dUb), tl.to_dev_bf16(Xb), tl.to_dev_bf16(Wb), dX=dX, dW=dW,
                             accumulate=accumulate)
    assert sru.sru_sync_status() == 0
    abs_dX = oracle.project_dX(tl.abs_operand(dUb), tl.abs_operand(Wb)) + (np.abs(base) if accumulate else 0.0)
    abs_dW = oracle.project_dW(tl.abs_operand(dUb), tl.abs_operand(Xb))
    tl.assert_close_sum("dX", tl.host_f64(dX), ref_dX, abs_dX)
    tl.assert_close_sum("dW", tl.host_f64(dW), ref_dW, abs_dW)


@pytest.mark.parametrize("M,N,K", [(32, 96, 32), (300, 600, 200), (77, 40, 16)])
def test_project_fp32(sru, M, N, K):
    rng = np.random.default_rng(3 * M + K)
    X = rng.standard_normal((M, K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32)
    dU = rng.standard_normal((M, N)).astype(np.float32)
    U = torch.empty(M, N, device="cuda")
    sru.sru_project(tl.to_dev_f32(X), tl.to_dev_f32(W), U)
    dX = torch.empty(M, K, device="cuda")
    dW = torch.empty(N, K, device="cuda")
    sru.sru_project_backward(tl.to_dev_f32(dU), tl.to_dev_f32(X), tl.to_dev_f32(W), dX=dX, dW=dW)
    assert sru.sru_sync_status() == 0
    aX, aW, adU = np.abs(X), np.abs(W), np.abs(dU)
    tl.assert_close_sum("U", tl.host_f64(U), oracle.project(X, W), oracle.project(aX, aW))
    tl.assert_close_sum("dX", tl.host_f64(dX), oracle.project_dX(dU, W), oracle.project_dX(adU, aW))
    tl.assert_close_sum("dW", tl.host_f64(dW), oracle.project_dW(dU, X), oracle.project_dW(adU, aX))


def test_project_large_k_sampled(sru):
    """dW at a training-step-like reduction length (K_red = M = 16384), sampled entries."""
    rng = np.random.default_rng(99)
    M, N, K = 16384, 512, 256
    Xb, dUb = _bf16(rng, (M, K)), _bf16(rng, (M, N))
    dW = torch.empty(N, K, device="cuda")
    sru.sru_project_backward(tl.to_dev_bf16(dUb), tl.to_dev_bf16(Xb), tl.to_dev_bf16(_bf16(rng, (N, K))), dW=dW)
    assert sru.sru_sync_status() == 0
    rows, cols = rng.integers(0, N, 2048), rng.integers(0, K, 2048)
    ref = oracle.project_dW_entries(dUb, Xb, rows, cols)
    absref = oracle.project_dW_entries(tl.abs_operand(dUb), tl.abs_operand(Xb), rows, cols)
    tl.assert_close_sum("dW sampled", tl.host_f64(dW)[rows, cols], ref, absref)


@pytest.mark.parametrize("N,K", [(6144, 2048), (3072, 2048), (4096, 2048)])
def test_tail_split_dw_matches_oracle_and_is_deterministic(sru, N, K):
    """dW whose output tiles do not fill whole rounds of the 74 CTA pairs: the
    tiles of the last, partial round are cut in two k-pieces that add onto a
    zeroed region (192 tiles: pieces of K/3 and 2K/3, some pairs taking two short
    pieces; 96 tiles: halves).  At 128 tiles the partial round holds 54 of the
    74 pairs, more than two thirds, and no tail is split.  Entries of those tiles and of whole tiles match
    the oracle's plain sums, and with two addends per element the fp32 result is
    the same whichever piece lands first: repeated calls agree bit for bit."""
    rng = np.random.default_rng(5)
    M = 1024                          # 16 k-blocks: pieces of 5 and 11, or 8 and 8
    Xb, dUb = _bf16(rng, (M, K)), _bf16(rng, (M, N))
    Xd, dUd, Wd = tl.to_dev_bf16(Xb), tl.to_dev_bf16(dUb), tl.to_dev_bf16(_bf16(rng, (N, K)))
    outs = []
    for _ in range(3):
        dW = torch.full((N, K), float("nan"), device="cuda")
        sru.sru_project_backward(dUd, Xd, Wd, dW=dW)
        outs.append(dW)
    assert sru.sru_sync_status() == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    got = tl.host_f64(outs[0])
    # sampled entries anywhere, and every entry of one row and one column of the last tiles
    rows = np.concatenate([rng.integers(0, N, 2048), np.full(K, N - 1), np.arange(N - 256, N)])
    cols = np.concatenate([rng.integers(0, K, 2048), np.arange(K), np.full(256, K - 1)])
    ref = oracle.project_dW_entries(dUb, Xb, rows, cols)
    absref = oracle.project_dW_entries(tl.abs_operand(dUb), tl.abs_operand(Xb), rows, cols)
    tl.assert_close_sum("dW sampled", got[rows, cols], ref, absref)


@pytest.mark.parametrize("M,K", [(16384, 512), (15360, 512), (12288, 512)])
def test_tail_split_dx_matches_oracle_and_is_deterministic(sru, M, K):
    """dX written (not accumulated) whose output tiles do not fill whole rounds
    of the 74 CTA pairs: 128 tiles (a partial round of 54 pairs, more than two
    thirds: no split), 120 tiles (pieces of a third and two thirds of the
    reduction) and 96 tiles (halves) of 256 x 256.  The pieces add onto a zeroed
    region, two addends per element, so repeated calls agree bit for bit; sampled
    entries, and every entry of the last row and column, match the oracle."""
    rng = np.random.default_rng(11)
    N = 1024                          # the reduction: 16 k-blocks
    dUb, Wb = _bf16(rng, (M, N)), _bf16(rng, (N, K), 0.1)
    dUd, Wd = tl.to_dev_bf16(dUb), tl.to_dev_bf16(Wb)
    Xd = tl.to_dev_bf16(_bf16(rng, (M, K)))
    outs = []
    for _ in range(3):
        dX = torch.full((M, K), float("nan"), device="cuda")
        sru.sru_project_backward(dUd, Xd, Wd, dX=dX, accumulate=False)
        outs.append(dX)
    assert sru.sru_sync_status() == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    got = tl.host_f64(outs[0])
    rows = np.concatenate([rng.integers(0, M, 2048), np.full(K, M - 1), np.arange(M - 256, M)])
    cols = np.concatenate([rng.integers(0, K, 2048), np.arange(K), np.full(256, K - 1)])
    ref = oracle.project_dX_entries(dUb, Wb, rows, cols)
    absref = oracle.project_dX_entries(tl.abs_operand(dUb), tl.abs_operand(Wb), rows, cols)
    tl.assert_close_sum("dX sampled", got[rows, cols], ref, absref)
