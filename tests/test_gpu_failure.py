"""The device-side failure path, exercised without a fault, a trap or a hang.

A chunked-scan CTA finds the state entering its chunk by waiting for its
predecessors' published carries.  With SRU_FLAG_TEST_WITHHOLD_CARRY the first
work item never publishes, so the waits that look back to it run out after
their bounded limit (about 2 s), publish an abort that releases every
successor, and return.  The host must then read SRU_ERR_TIMEOUT from
sru_sync_status(), the status must be cleared by that read, and the context
must still run a clean call that matches the oracle.
"""
import time

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


# 4 scan chunks x 1 channel tile: every work item is resident at once.
CFG = SRUConfig(name="fail", L=256, B=1, d=64, seed=31, proj_dtype="bf16", bias="normal0.1", c0="normal",
                v_zero=True)
SCAN = 0x1 | 0x2  # SRU_FLAG_V_ZERO | SRU_FLAG_FORCE_SCAN


def _tensors(inp):
    L, B, d = inp["x"].shape
    t = dict(U=tl.dev_U(inp), x=tl.to_dev_f32(inp["x"]), v=tl.to_dev_f32(inp["v"]), b=tl.to_dev_f32(inp["bias"]),
             c0=tl.to_dev_f32(inp["c0"]), dh=tl.to_dev_f32(inp["dh"]))
    t.update(h=torch.empty(L, B, 1, d, device="cuda"), cT=torch.empty(B, 1, d, device="cuda"),
             dU=torch.empty(L, B, 1, 3, d, device="cuda"), dx=torch.empty(L, B, d, device="cuda"),
             dv=torch.empty(1, 2, d, device="cuda"), db=torch.empty(1, 2, d, device="cuda"),
             dc0=torch.empty(B, 1, d, device="cuda"))
    return t


def _expect_timeout(sru):
    t0 = time.monotonic()
    status = sru.sru_sync_status()
    waited = time.monotonic() - t0
    assert status == sru.SRU_ERR_TIMEOUT, f"status {status}"
    assert waited < 30.0
    assert sru.sru_sync_status() == sru.SRU_OK  # the read cleared it


def test_withheld_forward_carry_reports_timeout_then_recovers(sru):
    inp = generate(CFG, u_direct=True, with_grad=True)
    t = _tensors(inp)
    assert sru.sru_sync_status() == sru.SRU_OK
    ws = sru.alloc_workspace(CFG.L, CFG.B, CFG.d, False, SCAN)
    sru.sru_forward(t["U"], t["x"], t["v"], t["b"], t["h"], t["cT"], c0=t["c0"], workspace=ws,
                    flags=SCAN | sru.SRU_FLAG_TEST_WITHHOLD_CARRY)
    _expect_timeout(sru)
    gpu = tl.run_gpu_recurrence(sru, inp, 1, 1.0, flags=SCAN)
    tl.compare_recurrence(gpu, tl.oracle_recurrence(inp, 1.0))


def test_withheld_backward_carry_reports_timeout_then_recovers(sru):
    inp = generate(CFG, u_direct=True, with_grad=True)
    t = _tensors(inp)
    assert sru.sru_sync_status() == sru.SRU_OK
    ws = sru.alloc_workspace(CFG.L, CFG.B, CFG.d, False, SCAN)
    sru.sru_forward(t["U"], t["x"], t["v"], t["b"], t["h"], t["cT"], c0=t["c0"], workspace=ws, flags=SCAN)
    assert sru.sru_sync_status() == sru.SRU_OK
    sru.sru_backward(t["U"], t["x"], t["v"], t["b"], t["dh"], ws, t["dU"], t["dx"], t["dv"], t["db"], t["dc0"],
                     c0=t["c0"], flags=SCAN | sru.SRU_FLAG_TEST_WITHHOLD_CARRY)
    _expect_timeout(sru)
    gpu = tl.run_gpu_recurrence(sru, inp, 1, 1.0, flags=SCAN)
    tl.compare_recurrence(gpu, tl.oracle_recurrence(inp, 1.0))
    assert np.isfinite(gpu["dv"]).all()
