"""GPU parity of the SRU++ attention producer's backward
(sru_attention_project_backward) against the fp64 oracle
(oracle.attention_project_backward, itself pinned to central differences of
the forward oracle) on the same bf16 inputs.

The GPU rounds dA, the softmax gradient dS, [dK | dV] and dQ to bf16 where they
become tensor-core operands, on top of the forward's bf16 Q, K, V, P and R
(the oracle keeps every intermediate in fp64).  Each rounding moves a value by
at most 2^-9 relative, and a gradient passes through at most five of them.
  * Every gradient: relative Frobenius error under 1e-2 (measured 0.1-0.5 %).
  * Elementwise, every entry is a sum (dX over the d' features, the weight
    gradients over all L*B tokens) and can cancel to near zero while the
    rounding error of its summands stays at their scale, so the bound adds to
    the bf16 class 2e-2 * (1 + |ref|) the term 5e-2 * rms(ref): the largest
    entry of a relative error of 1e-2 spread over thousands of entries (about
    4.5 times its rms).
A dropped 1/sqrt(d'), a transposed operand, a causal range off by a tile or a
wrong batch stride moves a gradient by O(1) and fails the last check.
"""
import numpy as np
import pytest
import torch

import oracle
import sru_testlib as tl
from synthetic import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sru():
    import parallelizable_recurrence_b200 as m
    m.load_library()
    return m


def _bits(rng, shape, scale):
    return f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _run(sru, L, B, d, dp, alpha, causal, ln, seed, accumulate=False):
    rng = np.random.default_rng(seed)
    N = 3 * d
    Xb = _bits(rng, (L * B, d), 1.0)
    Wqb = _bits(rng, (dp, d), d ** -0.5)
    Wkvb = _bits(rng, (2 * dp, dp), dp ** -0.5)
    Wob = _bits(rng, (N, dp), dp ** -0.5)
    dUb = _bits(rng, (L * B, N), 1.0)
    g = (1.0 + 0.1 * rng.standard_normal(dp)).astype(np.float32) if ln else None
    be = (0.1 * rng.standard_normal(dp)).astype(np.float32) if ln else None
    X, Wq, Wkv, Wo, dU = (_dev(a) for a in (Xb, Wqb, Wkvb, Wob, dUb))
    gd = None if g is None else torch.from_numpy(g).cuda()
    bd = None if be is None else torch.from_numpy(be).cuda()
    fws = torch.empty(int(sru.load_library().sru_attention_workspace_bytes(L, B, dp)), dtype=torch.uint8,
                      device="cuda")
    U = torch.empty(L * B, N, device="cuda", dtype=torch.bfloat16)
    sru.sru_attention_project(X, Wq, Wkv, Wo, U, L, B, alpha, ln_gamma=gd, ln_beta=bd, causal=causal, workspace=fws)
    x0 = torch.from_numpy(rng.standard_normal((L * B, d)).astype(np.float32)).cuda()
    out = dict(dX=x0.clone() if accumulate else torch.full((L * B, d), float("nan"), device="cuda"),
               dWq=torch.full((dp, d), float("nan"), device="cuda"),
               dWkv=torch.full((2 * dp, dp), float("nan"), device="cuda"),
               dWo=torch.full((N, dp), float("nan"), device="cuda"))
    if ln:
        out["dgamma"] = torch.full((dp,), float("nan"), device="cuda")
        out["dbeta"] = torch.full((dp,), float("nan"), device="cuda")
    sru.sru_attention_project_backward(dU, X, Wq, Wkv, Wo, L, B, alpha, fws, out["dX"], out["dWq"], out["dWkv"],
                                       out["dWo"], accumulate=accumulate, ln_gamma=gd, ln_beta=bd,
                                       dgamma=out.get("dgamma"), dbeta=out.get("dbeta"), causal=causal)
    assert sru.sru_sync_status() == 0
    ref = oracle.attention_project_backward(dUb, Xb, Wqb, Wkvb[:dp], Wkvb[dp:], Wob, alpha, L, B, causal=causal,
                                            ln_gamma=g, ln_beta=be)
    ref["dWkv"] = np.concatenate([ref.pop("dWk"), ref.pop("dWv")], axis=0)
    if accumulate:
        ref["dX"] = ref["dX"] + x0.cpu().numpy().astype(np.float64)
    return out, ref


def _compare(out, ref):
    assert sorted(out) == sorted(ref)
    for k in out:
        got = tl.host_f64(out[k])
        tl.assert_close(k, got, ref[k], tl.BF16_TOL, extra=5e-2 * np.sqrt(np.mean(ref[k] ** 2)))
        rel = np.linalg.norm(got - ref[k]) / max(np.linalg.norm(ref[k]), 1e-30)
        assert rel < 1e-2, (k, rel)


@pytest.mark.parametrize("L,B,d,dp,alpha,causal,ln", [
    (40, 3, 64, 16, 0.5, True, False),
    (40, 3, 64, 16, 0.5, False, True),
    (128, 2, 256, 64, 1.0, True, True),
    (256, 3, 128, 64, 0.25, True, False),    # one full score tile
    (600, 2, 128, 32, 0.5, True, True),      # causal over 3 score tiles, the last one ragged
    (600, 2, 128, 32, -0.7, False, False),   # the same without the mask: every tile computed
    (2048, 5, 64, 16, 0.5, True, False),     # every batch row's probabilities kept by the forward (one group)
    (4096, 3, 64, 16, 0.5, True, True),      # long rows in groups of 2: the probabilities are recomputed
    (72, 3, 96, 40, 0.9, True, True),        # widths that are not multiples of a tile or a k-block
    (48, 2, 64, 1024, 0.5, True, True),      # d' = 1024: the widest norm row held in registers
    (48, 2, 64, 1152, 0.5, False, True),     # d' past that: the norm's row-loop kernels
    (80, 5, 64, 200, 0.5, True, True),       # norm slices of 32 tokens ending mid-slice
])
def test_attention_backward_matches_oracle(sru, L, B, d, dp, alpha, causal, ln):
    out, ref = _run(sru, L, B, d, dp, alpha, causal, ln, seed=L + B + d + dp)
    _compare(out, ref)


def test_attention_backward_accumulates_dx(sru):
    out, ref = _run(sru, 64, 2, 128, 32, 0.75, True, True, seed=7, accumulate=True)
    _compare(out, ref)


def test_attention_backward_is_deterministic(sru):
    a, _ = _run(sru, 304, 3, 64, 32, 0.5, True, True, seed=9)
    b, _ = _run(sru, 304, 3, 64, 32, 0.5, True, True, seed=9)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_attention_backward_alpha_zero_leaves_the_attention_weights_without_gradient(sru):
    # alpha = 0: the attention does not reach U, so dWkv is exactly zero
    out, ref = _run(sru, 64, 2, 128, 32, 0.0, True, False, seed=11)
    assert torch.count_nonzero(out["dWkv"]).item() == 0
    _compare(out, ref)


def test_attention_backward_at_the_training_layer_width(sru):
    """d = 2048, d' = 512, N = 6144 as in the training layer, with the batch cut
    to 2 rows so that the fp64 oracle finishes in seconds: every product at
    its full width, the split weight gradients at their full reduction plans'
    shapes (dWo 6144 x 512, dWkv 1024 x 512, dWq 512 x 2048)."""
    out, ref = _run(sru, 1024, 2, 2048, 512, 0.5, True, True, seed=31)
    _compare(out, ref)
