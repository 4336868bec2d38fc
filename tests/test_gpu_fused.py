"""sru_forward_fused (Eq. (1) and Eqs. (2)-(5) in one kernel, the page's
Figure 2(a) with its two boxes fused) against the fp64 oracle and against the
two-call path, through the C ABI.

Checks per case:
  * end to end: h and c_T vs the oracle projecting from X itself (fp64 of the
    bf16 X and W), tolerance 2e-2 * (1 + |ref|) (the bf16-projection class);
  * U (stored when asked for) vs the oracle's projection, same class;
  * recurrence on the stored U: h, c_T vs the oracle run on exactly those bf16
    U values, tolerance 1e-5 * (1 + |ref|) (the recurrence class);
  * the fused h, c_T equal sru_forward's on the fused U bit for bit (the same
    cell arithmetic on the same values), and a following sru_backward gives
    bit-identical gradients (the checkpoints are the same).
Cases span several time tiles (32 steps), ragged L, B (not a multiple of the
8 rows of a CTA pair) and d (not a multiple of the 64-channel slice), masks
with holes, both directions, c0 given or not, alpha != 1, and widths from one
64-channel slice to 32 slices per direction.
"""
import numpy as np
import pytest
import torch

import oracle
import sru_testlib as tl
from synthetic import CONFIGS, SRUConfig, bf16_bits_to_f32, generate

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sru():
    import parallelizable_recurrence_b200 as m
    m.load_library()
    return m


def _inputs(L, B, d, nd, seed, masked, c0, hole=True):
    cfg = SRUConfig(name="fused", L=L, B=B, d=d, n_dir=nd, seed=seed, proj_dtype="bf16", bias="normal0.1",
                    c0="normal" if c0 else "zero", masked=masked)
    inp = generate(cfg, with_grad=True)
    if masked and hole and L > 5:
        inp["mask"][min(5, L - 1), 0] = 1  # a hole inside the first row, besides the padded tails
    return cfg, inp


def _run_fused(sru, cfg, inp, alpha, want_u=True):
    L, B, d, nd = cfg.L, cfg.B, cfg.d, cfg.n_dir
    X, W = tl.to_dev_bf16(inp["X"]), tl.to_dev_bf16(inp["W"])
    x, v, b = tl.to_dev_f32(inp["x"]), tl.to_dev_f32(inp["v"]), tl.to_dev_f32(inp["bias"])
    c0, mask = tl.to_dev_f32(inp["c0"]), tl.to_dev_u8(inp["mask"])
    h = torch.full((L, B, nd, d), float("nan"), device="cuda")
    cT = torch.full((B, nd, d), float("nan"), device="cuda")
    U = torch.full((L, B, nd, 3, d), float("nan"), device="cuda", dtype=torch.bfloat16) if want_u else None
    ws = sru.alloc_workspace(L, B, d, nd == 2)
    sru.sru_forward_fused(X, W, x, v, b, h, cT, ws, c0=c0, mask=mask, alpha=alpha, bidirectional=nd == 2, U=U)
    assert sru.sru_sync_status() == 0
    return dict(X=X, W=W, x=x, v=v, b=b, c0=c0, mask=mask, h=h, cT=cT, U=U, ws=ws)


CASES = [  # L, B, d, n_dir, seed, masked, c0, alpha
    (70, 3, 72, 1, 11, False, False, 1.0),      # one CTA pair, a lone batch group, ragged d and L
    (96, 8, 128, 1, 12, False, True, 1.0),      # whole tiles, c0
    (130, 12, 200, 2, 13, True, True, 0.5),     # ragged everything, both directions, mask with a hole
    (257, 16, 64, 2, 14, True, False, 1.0),     # many time tiles handed between CTAs
    (33, 9, 512, 1, 15, True, True, -2.0),      # L one past a tile, B one past a pair
    (40, 5, 1088, 2, 18, True, True, 0.75),     # 17 slices, the last one 64 wide; both directions
    (70, 8, 1024, 1, 19, False, False, 1.0),    # 16 whole slices
    (100, 3, 2048, 1, 20, True, True, 1.0),     # 32 slices over several time tiles, a lone batch group
]


@pytest.mark.parametrize("L,B,d,nd,seed,masked,c0,alpha", CASES)
def test_fused_forward_matches_oracle(sru, L, B, d, nd, seed, masked, c0, alpha):
    cfg, inp = _inputs(L, B, d, nd, seed, masked, c0)
    out = _run_fused(sru, cfg, inp, alpha)
    # end to end, the oracle projecting from X itself
    U_ref = oracle.project(inp["X"], inp["W"]).reshape(L, B, nd, 3, d)
    h_ref, cT_ref = oracle.forward(U_ref, inp["x"], inp["v"], inp["bias"], c0=inp["c0"], mask=inp["mask"],
                                   alpha=alpha)
    tl.assert_close("h end to end", tl.host_f64(out["h"]), h_ref, tl.BF16_TOL)
    tl.assert_close("c_T end to end", tl.host_f64(out["cT"]), cT_ref, tl.BF16_TOL)
    # the stored projection
    Ub = out["U"].view(torch.int16).cpu().numpy().view(np.uint16)
    U_got = bf16_bits_to_f32(Ub).astype(np.float64)
    tl.assert_close("U", U_got, U_ref, tl.BF16_TOL)
    # the recurrence on exactly the stored bf16 U
    h_r, cT_r = oracle.forward(U_got, inp["x"], inp["v"], inp["bias"], c0=inp["c0"], mask=inp["mask"], alpha=alpha)
    tl.assert_close("h on the stored U", tl.host_f64(out["h"]), h_r, tl.REC_TOL)
    tl.assert_close("c_T on the stored U", tl.host_f64(out["cT"]), cT_r, tl.REC_TOL)


@pytest.mark.parametrize("L,B,d,nd,seed,masked,c0,alpha", CASES[2:4])
def test_fused_equals_two_call_path_bitwise_and_feeds_the_backward(sru, L, B, d, nd, seed, masked, c0, alpha):
    cfg, inp = _inputs(L, B, d, nd, seed, masked, c0)
    f = _run_fused(sru, cfg, inp, alpha)
    # the two-call path on the fused kernel's own U
    h2 = torch.full_like(f["h"], float("nan"))
    cT2 = torch.full_like(f["cT"], float("nan"))
    ws2 = sru.alloc_workspace(L, B, d, nd == 2)
    sru.sru_forward(f["U"], f["x"], f["v"], f["b"], h2, cT2, c0=f["c0"], mask=f["mask"], alpha=alpha,
                    bidirectional=nd == 2, workspace=ws2)
    assert sru.sru_sync_status() == 0
    assert torch.equal(f["h"], h2), "fused h differs from sru_forward on the same U"
    assert torch.equal(f["cT"], cT2)
    dh = tl.to_dev_f32(inp["dh"])
    grads = []
    for ws in (f["ws"], ws2):
        g = dict(dU=torch.empty(L, B, nd, 3, d, device="cuda", dtype=torch.bfloat16),
                 dx=torch.empty(L, B, d, device="cuda"), dv=torch.empty(nd, 2, d, device="cuda"),
                 db=torch.empty(nd, 2, d, device="cuda"), dc0=torch.empty(B, nd, d, device="cuda"))
        sru.sru_backward(f["U"], f["x"], f["v"], f["b"], dh, ws, g["dU"], g["dx"], g["dv"], g["db"], g["dc0"],
                         c0=f["c0"], mask=f["mask"], alpha=alpha, bidirectional=nd == 2)
        assert sru.sru_sync_status() == 0
        grads.append(g)
    for k in grads[0]:
        assert torch.equal(grads[0][k], grads[1][k]), k


def test_fused_without_u_is_inference_only_and_equal(sru):
    cfg, inp = _inputs(100, 10, 136, 2, 16, True, True)
    a = _run_fused(sru, cfg, inp, 1.0, want_u=True)
    b = _run_fused(sru, cfg, inp, 1.0, want_u=False)
    assert torch.equal(a["h"], b["h"]) and torch.equal(a["cT"], b["cT"])


def test_fused_repeated_calls_reuse_the_workspace(sru):
    """The carry words are cleared before every launch: a second call on
    the same workspace gives the same result."""
    cfg, inp = _inputs(200, 8, 256, 1, 17, False, True)
    f = _run_fused(sru, cfg, inp, 1.0)
    h1, c1 = f["h"].clone(), f["cT"].clone()
    sru.sru_forward_fused(f["X"], f["W"], f["x"], f["v"], f["b"], f["h"], f["cT"], f["ws"], c0=f["c0"], U=f["U"])
    assert sru.sru_sync_status() == 0
    assert torch.equal(h1, f["h"]) and torch.equal(c1, f["cT"])


def test_fused_no_steps_and_no_rows(sru):
    B, d = 3, 64
    X = torch.empty(0, d, device="cuda", dtype=torch.bfloat16)
    W = torch.zeros(3 * d, d, device="cuda", dtype=torch.bfloat16)
    x = torch.empty(0, B, d, device="cuda")
    v, b = torch.zeros(1, 2, d, device="cuda"), torch.zeros(1, 2, d, device="cuda")
    h = torch.empty(0, B, 1, d, device="cuda")
    c0 = torch.randn(B, 1, d, device="cuda")
    cT = torch.full((B, 1, d), float("nan"), device="cuda")
    ws = sru.alloc_workspace(1, B, d)
    sru.sru_forward_fused(X, W, x, v, b, h, cT, ws, c0=c0)
    assert sru.sru_sync_status() == 0
    assert torch.equal(cT, c0)


@pytest.mark.parametrize("name", ["lm_fwd", "lm_train", "bidir_masked"])
def test_fused_full_size_sampled(sru, name):
    """The workloads' full sizes, in the launch configuration the benchmark
    times; sampled batch rows and channels against the oracle projecting from X."""
    cfg = CONFIGS[name]
    inp = generate(cfg, with_grad=False)
    L, B, d, nd = cfg.L, cfg.B, cfg.d, cfg.n_dir
    out = _run_fused(sru, cfg, inp, cfg.alpha, want_u=cfg.backward)
    rng = np.random.default_rng(4000 + cfg.seed)
    js = np.sort(rng.choice(d, size=4, replace=False))
    bs = np.sort(rng.choice(B, size=min(3, B), replace=False))
    m_idx = (np.arange(L)[:, None] * B + bs[None, :]).reshape(-1)
    n_idx = np.array([(dr * 3 + g) * d + j for dr in range(nd) for g in range(3) for j in js])
    rr = np.repeat(m_idx, n_idx.size)
    cc = np.tile(n_idx, m_idx.size)
    U_sub = oracle.project_entries(inp["X"], inp["W"], rr, cc).reshape(L, bs.size, nd, 3, js.size)
    h_ref, cT_ref = oracle.forward(U_sub, inp["x"][:, bs][:, :, js], inp["v"][:, :, js], inp["bias"][:, :, js],
                                   c0=None if inp["c0"] is None else inp["c0"][bs][:, :, js],
                                   mask=None if inp["mask"] is None else inp["mask"][:, bs], alpha=cfg.alpha)
    tl.assert_close("h end to end", tl.host_f64(out["h"])[:, bs][:, :, :, js], h_ref, tl.BF16_TOL)
    tl.assert_close("c_T end to end", tl.host_f64(out["cT"])[bs][:, :, js], cT_ref, tl.BF16_TOL)
    if out["U"] is not None:
        Ub = out["U"].view(torch.int16).cpu().numpy().view(np.uint16)
        got = bf16_bits_to_f32(Ub.reshape(L * B, nd * 3 * d)[rr, cc]).astype(np.float64)
        tl.assert_close("U sampled", got, U_sub.reshape(-1), tl.BF16_TOL)
