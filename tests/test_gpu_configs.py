"""GPU parity at the full sizes of the five layer workloads, in the launch
configuration the benchmark times.

For each workload:
  * recurrence: the inputs of the workload with U drawn directly (bf16 N(0,1),
    the distribution of X W^T here), GPU vs oracle on every batch row of a
    random sample of channels (all t), which also fixes dv and db for those
    channels exactly; tolerance 1e-5 * (1 + |ref|);
  * projection: >= 4096 sampled entries of U = X W^T vs the oracle's plain sum;
  * end to end: h from X (projection then recurrence) vs the oracle projecting
    from X itself, on sampled channels; tolerance 2e-2 * (1 + |ref|) (bf16 U);
  * projection gradients: dX, dW from a drawn bf16 dU, sampled entries.
The tiny fp32 workload is compared in full, end to end, at 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
import sru_testlib as tl
from synthetic import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, generate

pytestmark = pytest.mark.gpu

N_CHANNELS = 16
N_ENTRIES = 4096


@pytest.fixture(scope="module")
def sru():
    import parallelizable_recurrence_b200 as m
    m.load_library()
    return m


def _sample_channels(rng, d, n=N_CHANNELS):
    return np.sort(rng.choice(d, size=min(n, d), replace=False))


@pytest.mark.parametrize("name,force_scan", [("lm_fwd", False), ("lm_train", False), ("bidir_masked", False),
                                             ("rec_only", False), ("rec_only_v0", False), ("rec_only_v0", True)])
def test_recurrence_full_size(sru, name, force_scan):
    cfg = CONFIGS[name]
    inp = generate(cfg, u_direct=True)
    flags = sru.SRU_FLAG_V_ZERO if cfg.v_zero else 0
    if force_scan:
        flags |= sru.SRU_FLAG_FORCE_SCAN
    gpu = tl.run_gpu_recurrence(sru, inp, cfg.n_dir, cfg.alpha, du_dtype=torch.bfloat16, flags=flags,
                                backward=cfg.backward)
    rng = np.random.default_rng(1000 + cfg.seed)
    js = _sample_channels(rng, cfg.d)
    bs = np.arange(cfg.B)
    ref = tl.oracle_recurrence(inp, cfg.alpha, bs=bs, js=js, backward=cfg.backward)
    tl.compare_recurrence(gpu, ref, du_bf16=True, bs=bs, js=js, backward=cfg.backward)


@pytest.mark.parametrize("name", ["lm_fwd", "lm_train", "bidir_masked"])
def test_projection_and_end_to_end_full_size(sru, name):
    cfg = CONFIGS[name]
    inp = generate(cfg, with_grad=False)
    L, B, d, nd = cfg.L, cfg.B, cfg.d, cfg.n_dir
    M, N = L * B, cfg.N
    X, W = tl.to_dev_bf16(inp["X"]), tl.to_dev_bf16(inp["W"])
    U = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    sru.sru_project(X, W, U)
    x = tl.to_dev_f32(inp["x"])
    h = torch.empty(L, B, nd, d, device="cuda")
    cT = torch.empty(B, nd, d, device="cuda")
    sru.sru_forward(U.view(L, B, nd, 3, d), x, tl.to_dev_f32(inp["v"]), tl.to_dev_f32(inp["bias"]), h, cT,
                    c0=tl.to_dev_f32(inp["c0"]), mask=tl.to_dev_u8(inp["mask"]), alpha=cfg.alpha,
                    bidirectional=nd == 2)
    assert sru.sru_sync_status() == 0
    rng = np.random.default_rng(2000 + cfg.seed)
    # sampled entries of U
    rows, cols = rng.integers(0, M, N_ENTRIES), rng.integers(0, N, N_ENTRIES)
    ref_u = oracle.project_entries(inp["X"], inp["W"], rows, cols)
    Uh = U.view(torch.int16).cpu().numpy().view(np.uint16)
    tl.assert_close("U sampled", bf16_bits_to_f32(Uh[rows, cols]), ref_u, tl.BF16_TOL)
    # end to end on sampled channels, all rows and steps: oracle projects from X itself
    js = _sample_channels(rng, d, 4)
    bs = np.sort(rng.choice(B, size=min(4, B), replace=False))
    m_idx = (np.arange(L)[:, None] * B + bs[None, :]).reshape(-1)          # (L*|bs|)
    n_idx = np.array([(dr * 3 + g) * d + j for dr in range(nd) for g in range(3) for j in js])
    rr = np.repeat(m_idx, n_idx.size)
    cc = np.tile(n_idx, m_idx.size)
    U_sub = oracle.project_entries(inp["X"], inp["W"], rr, cc).reshape(L, bs.size, nd, 3, js.size)
    sub = dict(U=U_sub, x=inp["x"][:, bs][:, :, js], v=inp["v"][:, :, js], bias=inp["bias"][:, :, js],
               c0=None if inp["c0"] is None else inp["c0"][bs][:, :, js],
               mask=None if inp["mask"] is None else inp["mask"][:, bs])
    h_ref, cT_ref = oracle.forward(sub["U"], sub["x"], sub["v"], sub["bias"], c0=sub["c0"], mask=sub["mask"],
                                   alpha=cfg.alpha)
    h_gpu = tl.host_f64(h)[:, bs][:, :, :, js]
    tl.assert_close("h end to end", h_gpu, h_ref, tl.BF16_TOL)
    tl.assert_close("c_T end to end", tl.host_f64(cT)[bs][:, :, js], cT_ref, tl.BF16_TOL)


@pytest.mark.parametrize("name", ["lm_train", "bidir_masked"])
def test_projection_backward_full_size(sru, name):
    cfg = CONFIGS[name]
    inp = generate(cfg, with_grad=False)
    L, B, d = cfg.L, cfg.B, cfg.d
    M, N = L * B, cfg.N
    rng = np.random.default_rng(3000 + cfg.seed)
    dUb = f32_to_bf16_bits(rng.standard_normal((M, N), dtype=np.float32))
    hw = rng.standard_normal((M, d), dtype=np.float32)  # stands in for the highway part of dx
    dX = tl.to_dev_f32(hw)
    dW = torch.empty(N, d, device="cuda")
    sru.sru_project_backward(tl.to_dev_bf16(dUb), tl.to_dev_bf16(inp["X"]), tl.to_dev_bf16(inp["W"]), dX=dX, dW=dW,
                             accumulate=True)
    assert sru.sru_sync_status() == 0
    rows, cols = rng.integers(0, M, N_ENTRIES), rng.integers(0, d, N_ENTRIES)
    adU = tl.abs_operand(dUb)
    ref = oracle.project_dX_entries(dUb, inp["W"], rows, cols) + hw[rows, cols]
    absref = oracle.project_dX_entries(adU, tl.abs_operand(inp["W"]), rows, cols) + np.abs(hw[rows, cols])
    tl.assert_close_sum("dX sampled", tl.host_f64(dX)[rows, cols], ref, absref)
    rows, cols = rng.integers(0, N, N_ENTRIES), rng.integers(0, d, N_ENTRIES)
    ref = oracle.project_dW_entries(dUb, inp["X"], rows, cols)
    absref = oracle.project_dW_entries(adU, tl.abs_operand(inp["X"]), rows, cols)
    tl.assert_close_sum("dW sampled", tl.host_f64(dW)[rows, cols], ref, absref)


def test_tiny_fp32_end_to_end(sru):
    """Projection + forward + backward + projection gradients, fp32 throughout, every element."""
    cfg = CONFIGS["tiny_fp32"]
    inp = generate(cfg)
    L, B, d = cfg.L, cfg.B, cfg.d
    M, N = L * B, cfg.N
    X, W = tl.to_dev_f32(inp["X"]), tl.to_dev_f32(inp["W"])
    U = torch.empty(L, B, 1, 3, d, device="cuda")
    sru.sru_project(X, W, U)
    x, v, b = tl.to_dev_f32(inp["x"]), tl.to_dev_f32(inp["v"]), tl.to_dev_f32(inp["bias"])
    h = torch.empty(L, B, 1, d, device="cuda")
    cT = torch.empty(B, 1, d, device="cuda")
    ws = sru.alloc_workspace(L, B, d)
    sru.sru_forward(U, x, v, b, h, cT, workspace=ws)
    dh = tl.to_dev_f32(inp["dh"])
    dU = torch.empty_like(U)
    dx = torch.empty(L, B, d, device="cuda")
    dv, db = torch.empty(1, 2, d, device="cuda"), torch.empty(1, 2, d, device="cuda")
    dc0 = torch.empty(B, 1, d, device="cuda")
    sru.sru_backward(U, x, v, b, dh, ws, dU, dx, dv, db, dc0)
    dW = torch.empty(N, d, device="cuda")
    sru.sru_project_backward(dU, X, W, dX=dx, dW=dW, accumulate=True)
    assert sru.sru_sync_status() == 0
    # oracle, from X itself
    U_ref = oracle.project(inp["X"], inp["W"]).reshape(L, B, 1, 3, d)
    h_ref, cT_ref = oracle.forward(U_ref, inp["x"], inp["v"], inp["bias"])
    g = oracle.backward(U_ref, inp["x"], inp["v"], inp["bias"], inp["dh"])
    dU_ref = g["dU"].reshape(M, N)
    dx_ref = g["dx"].reshape(M, d) + oracle.project_dX(dU_ref, inp["W"].astype(np.float64))
    dW_ref = oracle.project_dW(dU_ref, inp["X"].astype(np.float64))
    tl.assert_close("U", tl.host_f64(U).reshape(M, N), U_ref.reshape(M, N), tl.REC_TOL)
    tl.assert_close("h", tl.host_f64(h), h_ref, tl.REC_TOL)
    tl.assert_close("c_T", tl.host_f64(cT), cT_ref, tl.REC_TOL)
    tl.assert_close("dU", tl.host_f64(dU).reshape(M, N), dU_ref, tl.REC_TOL)
    tl.assert_close("dx total", tl.host_f64(dx).reshape(M, d), dx_ref, tl.REC_TOL)
    tl.assert_close("dW", tl.host_f64(dW), dW_ref, tl.REC_TOL)
    tl.assert_close("dv", tl.host_f64(dv), g["dv"], tl.REC_TOL)
    tl.assert_close("db", tl.host_f64(db), g["dbias"], tl.REC_TOL)
    tl.assert_close("dc0", tl.host_f64(dc0), g["dc0"], tl.REC_TOL)
