"""GPU parity of SRU++'s attention producer of U (sru_attention_project)
against the fp64 oracle (oracle.attention_project) on the same bf16 inputs.

The GPU rounds Q, K, V, the probabilities and R to bf16 (they feed the
tensor cores), so U is a bf16-projection output: the bound is
|gpu - ref| <= 2e-2 * (1 + |ref|), the class every bf16-projection output of
this library is held to.  A wrong mask, a missing 1/sqrt(d'), a transposed
V or a wrong batch stride moves U by O(1).
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


@pytest.mark.parametrize("L,B,d,dp,alpha,causal,ln", [
    (40, 3, 64, 16, 0.5, True, False),
    (40, 3, 64, 16, 0.5, False, True),
    (128, 2, 256, 64, 1.0, True, True),
    (256, 4, 512, 128, 0.25, True, False),
    (64, 2, 128, 32, 0.0, True, False),
    (4096, 3, 64, 16, 0.5, True, False),   # long rows: batch rows go in groups of 2 (score buffer bound)
    (600, 2, 128, 32, 0.5, True, True),    # causal over 3 score tiles, the last one ragged
    (600, 2, 128, 32, 0.5, False, False),  # the same without the mask: every tile computed
    (72, 3, 96, 40, 0.9, True, True),      # widths that are not multiples of a tile or a k-block
])
def test_attention_producer_matches_oracle(sru, L, B, d, dp, alpha, causal, ln):
    rng = np.random.default_rng(L + B + d + dp)
    N = 3 * d
    Xb = _bits(rng, (L * B, d), 1.0)
    Wqb = _bits(rng, (dp, d), d ** -0.5)
    Wkvb = _bits(rng, (2 * dp, dp), dp ** -0.5)
    Wob = _bits(rng, (N, dp), dp ** -0.5)
    g = (1.0 + 0.1 * rng.standard_normal(dp)).astype(np.float32) if ln else None
    be = (0.1 * rng.standard_normal(dp)).astype(np.float32) if ln else None
    ref = oracle.attention_project(Xb, Wqb, Wkvb[:dp], Wkvb[dp:], Wob, alpha, L, B, causal=causal,
                                   ln_gamma=g, ln_beta=be)
    U32 = torch.full((L * B, N), float("nan"), device="cuda")
    U16 = torch.full((L * B, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    gd = None if g is None else torch.from_numpy(g).cuda()
    bd = None if be is None else torch.from_numpy(be).cuda()
    for U in (U32, U16):
        sru.sru_attention_project(_dev(Xb), _dev(Wqb), _dev(Wkvb), _dev(Wob), U, L, B, alpha, ln_gamma=gd,
                                  ln_beta=bd, causal=causal)
    assert sru.sru_sync_status() == 0
    tl.assert_close("U fp32", tl.host_f64(U32), ref, tl.BF16_TOL)
    tl.assert_close("U bf16", tl.host_f64(U16), ref, tl.BF16_TOL)
    # the error is far inside the class bound on average, not only at the maximum
    assert np.mean(np.abs(tl.host_f64(U32) - ref)) < 2e-3 * (1.0 + np.mean(np.abs(ref)))


def test_alpha_zero_equals_the_factorised_projection(sru):
    """With alpha = 0 the producer is the factorised projection Wo (Wq X) (the
    page's initial state); on the GPU the two paths share Q and the last
    product, so they agree exactly."""
    rng = np.random.default_rng(1)
    L, B, d, dp = 64, 2, 128, 32
    N = 3 * d
    X, Wq, Wo = _dev(_bits(rng, (L * B, d), 1.0)), _dev(_bits(rng, (dp, d), 0.1)), _dev(_bits(rng, (N, dp), 0.2))
    Wkv = _dev(_bits(rng, (2 * dp, dp), 0.2))
    U1 = torch.empty(L * B, N, device="cuda", dtype=torch.bfloat16)
    sru.sru_attention_project(X, Wq, Wkv, Wo, U1, L, B, 0.0)
    U2 = torch.empty_like(U1)
    sru.sru_project_factored(X, Wq, Wo, torch.empty(L * B, dp, device="cuda", dtype=torch.bfloat16), U2)
    assert sru.sru_sync_status() == 0
    assert torch.equal(U1.view(torch.int16), U2.view(torch.int16))
