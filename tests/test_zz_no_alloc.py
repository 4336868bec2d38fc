"""The allocation-free entry point sru_forward_scan_noalloc, through the C ABI.

Callers such as an inference plugin whose host framework owns all device
memory, or a latency-critical loop that must not call cudaMalloc, cannot pass
a workspace; this entry point keeps the scan's scratch in a static device
array inside libsru.so instead.  Its results must equal those of the existing
entry point (sru_forward with the scan forced and a caller-provided
workspace), within the recurrence tolerance 1e-5 * (1 + |ref|), on two calls
in a row -- the second call reuses the scratch the first one left behind.

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


def _workload(seed, L, B, d):
    cfg = SRUConfig(name="noalloc", L=L, B=B, d=d, n_dir=2, seed=seed, proj_dtype="bf16", bias="normal0.1",
                    c0="normal", masked=True, v_zero=True, backward=False)
    inp = generate(cfg, u_direct=True, with_grad=False)
    inp["mask"][3, 0] = 1  # a hole inside a row as well as padded tails
    return cfg, inp


def _reference_forward(sru, cfg, inp):
    """The existing entry point: sru_forward, scan forced, caller-provided workspace."""
    L, B, d = cfg.L, cfg.B, cfg.d
    flags = sru.SRU_FLAG_V_ZERO | sru.SRU_FLAG_FORCE_SCAN
    h = torch.full((L, B, 2, d), float("nan"), device="cuda")
    cT = torch.full((B, 2, d), float("nan"), device="cuda")
    ws = sru.alloc_workspace(L, B, d, True, flags)
    sru.sru_forward(tl.dev_U(inp), tl.to_dev_f32(inp["x"]), tl.to_dev_f32(inp["v"]), tl.to_dev_f32(inp["bias"]),
                    h, cT, c0=tl.to_dev_f32(inp["c0"]), mask=tl.to_dev_u8(inp["mask"]), bidirectional=True,
                    flags=flags, workspace=ws)
    assert sru.sru_sync_status() == 0
    return tl.host_f64(h), tl.host_f64(cT)


def _noalloc_forward(sru, cfg, inp):
    L, B, d = cfg.L, cfg.B, cfg.d
    h = torch.full((L, B, 2, d), float("nan"), device="cuda")
    cT = torch.full((B, 2, d), float("nan"), device="cuda")
    sru.sru_forward_scan_noalloc(tl.dev_U(inp), tl.to_dev_f32(inp["x"]), tl.to_dev_f32(inp["bias"]), h, cT,
                                 c0=tl.to_dev_f32(inp["c0"]), mask=tl.to_dev_u8(inp["mask"]), bidirectional=True)
    assert sru.sru_sync_status() == 0
    return tl.host_f64(h), tl.host_f64(cT)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(sru):
    # the first call is the larger one, so the second runs on scratch the first left behind
    for seed, (L, B, d) in [(41, (300, 4, 200)), (42, (130, 3, 72))]:
        cfg, inp = _workload(seed, L, B, d)
        h_ref, cT_ref = _reference_forward(sru, cfg, inp)
        h, cT = _noalloc_forward(sru, cfg, inp)
        tl.assert_close("h (no-alloc vs workspace)", h, h_ref, tl.REC_TOL)
        tl.assert_close("c_T (no-alloc vs workspace)", cT, cT_ref, tl.REC_TOL)


def test_noalloc_rejects_requests_beyond_its_scratch(sru):
    lib = sru.load_library()
    fake = ctypes.c_void_p(0x10000)
    # ceil(4096/64) * ceil(1024/64) * 64 rows * 2 directions = 131072 work items >> the scratch
    status = lib.sru_forward_scan_noalloc(fake, sru.SRU_BF16, fake, fake, None, None, 4096, 64, 1024, 1.0, 1,
                                          fake, fake, None)
    assert status == sru.SRU_ERR_UNSUPPORTED
