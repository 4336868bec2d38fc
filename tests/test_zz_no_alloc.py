"""The allocation-free entry point sru_forward_scan_noalloc, through the C ABI.

Callers such as an inference plugin whose host framework owns all device
memory, or a latency-critical loop that must not call cudaMalloc, cannot pass
a workspace; this entry point keeps the scan's scratch in a static device
array inside libsru.so instead.  On two calls in a row (the second reuses the
scratch the first one left behind) its results must equal
  - the fp64 oracle's, within the recurrence tolerance 1e-5 * (1 + |ref|), and
  - those of the existing entry point (sru_forward with the scan forced and a
    caller-provided workspace), within the same tolerance.
Cases: bidirectional with bf16 U, c0 given, padded tails and a hole; and
unidirectional with fp32 U and no c0.  L = 0 returns c_T = c0 (0 without c0).

This file is collected last so that a failure here cannot hide another test;
it passes alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import sru_testlib as tl
from synthetic import SRUConfig, generate

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sru():
    import parallelizable_recurrence_b200 as m
    m.load_library()
    return m


def _workload(seed, L, B, d, n_dir=2, proj_dtype="bf16", c0="normal", masked=True):
    cfg = SRUConfig(name="noalloc", L=L, B=B, d=d, n_dir=n_dir, seed=seed, proj_dtype=proj_dtype,
                    bias="normal0.1", c0=c0, masked=masked, v_zero=True, backward=False)
    inp = generate(cfg, u_direct=True, with_grad=False)
    if masked:
        inp["mask"][3, 0] = 1  # a hole inside a row as well as padded tails
    return cfg, inp


def _reference_forward(sru, cfg, inp):
    """The existing entry point: sru_forward, scan forced, caller-provided workspace."""
    L, B, d, nd = cfg.L, cfg.B, cfg.d, cfg.n_dir
    flags = sru.SRU_FLAG_V_ZERO | sru.SRU_FLAG_FORCE_SCAN
    h = torch.full((L, B, nd, d), float("nan"), device="cuda")
    cT = torch.full((B, nd, d), float("nan"), device="cuda")
    ws = sru.alloc_workspace(L, B, d, nd == 2, flags)
    sru.sru_forward(tl.dev_U(inp), tl.to_dev_f32(inp["x"]), tl.to_dev_f32(inp["v"]), tl.to_dev_f32(inp["bias"]),
                    h, cT, c0=tl.to_dev_f32(inp["c0"]), mask=tl.to_dev_u8(inp["mask"]), bidirectional=nd == 2,
                    flags=flags, workspace=ws)
    assert sru.sru_sync_status() == 0
    return tl.host_f64(h), tl.host_f64(cT)


def _noalloc_forward(sru, cfg, inp):
    L, B, d, nd = cfg.L, cfg.B, cfg.d, cfg.n_dir
    h = torch.full((L, B, nd, d), float("nan"), device="cuda")
    cT = torch.full((B, nd, d), float("nan"), device="cuda")
    sru.sru_forward_scan_noalloc(tl.dev_U(inp), tl.to_dev_f32(inp["x"]), tl.to_dev_f32(inp["bias"]), h, cT,
                                 c0=tl.to_dev_f32(inp["c0"]), mask=tl.to_dev_u8(inp["mask"]), bidirectional=nd == 2)
    assert sru.sru_sync_status() == 0
    return tl.host_f64(h), tl.host_f64(cT)


CASES = [  # (seed, L, B, d, n_dir, U type, c0, masked); the first call is the larger one
    (41, 300, 4, 200, 2, "bf16", "normal", True),
    (42, 130, 3, 72, 2, "bf16", "normal", True),
    (43, 150, 2, 96, 1, "fp32", "zero", False),
]


def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls_in_a_row(sru):
    for seed, L, B, d, nd, ut, c0, masked in CASES:
        cfg, inp = _workload(seed, L, B, d, nd, ut, c0, masked)
        ref = tl.oracle_recurrence(inp, 1.0, backward=False)
        h_ws, cT_ws = _reference_forward(sru, cfg, inp)
        for call in range(2):
            h, cT = _noalloc_forward(sru, cfg, inp)
            tl.assert_close(f"h (no-alloc vs oracle, call {call})", h, ref["h"], tl.REC_TOL)
            tl.assert_close(f"c_T (no-alloc vs oracle, call {call})", cT, ref["cT"], tl.REC_TOL)
            tl.assert_close(f"h (no-alloc vs workspace, call {call})", h, h_ws, tl.REC_TOL)
            tl.assert_close(f"c_T (no-alloc vs workspace, call {call})", cT, cT_ws, tl.REC_TOL)


def test_noalloc_with_no_steps_returns_the_initial_state(sru):
    B, d = 3, 64
    x = torch.empty(0, B, d, device="cuda")
    U = torch.empty(0, B, 1, 3, d, device="cuda")
    b = torch.zeros(1, 2, d, device="cuda")
    h = torch.empty(0, B, 1, d, device="cuda")
    c0 = torch.randn(B, 1, d, device="cuda")
    cT = torch.full((B, 1, d), float("nan"), device="cuda")
    sru.sru_forward_scan_noalloc(U, x, b, h, cT, c0=c0)
    assert sru.sru_sync_status() == 0
    assert torch.equal(cT, c0)
    cT.fill_(float("nan"))
    sru.sru_forward_scan_noalloc(U, x, b, h, cT)
    assert sru.sru_sync_status() == 0
    assert torch.count_nonzero(cT).item() == 0


def test_noalloc_rejects_requests_beyond_its_scratch(sru):
    lib = sru.load_library()
    fake = ctypes.c_void_p(0x10000)
    # ceil(4096/128) * ceil(1024/64) * 64 rows * 2 directions = 65536 work items >> the scratch
    status = lib.sru_forward_scan_noalloc(fake, sru.SRU_BF16, fake, fake, None, None, 4096, 64, 1024, 1.0, 1,
                                          fake, fake, None)
    assert status == sru.SRU_ERR_UNSUPPORTED
