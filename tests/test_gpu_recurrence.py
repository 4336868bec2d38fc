"""GPU parity of the recurrence kernels (sru_forward / sru_backward) against the
fp64 oracle, on the same seeded inputs, element by element.

Sizes span several 64-channel tiles and several 16-step chunks with ragged
tails in both (d = 200 = 3*64 + 8, L = 37 = 2*16 + 5).
"""
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


def _cfg(**kw):
    base = dict(name="t", L=37, B=3, d=200, seed=21, proj_dtype="bf16", bias="normal0.1", c0="normal")
    base.update(kw)
    return SRUConfig(**base)


@pytest.mark.parametrize("u_dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("n_dir,masked", [(1, False), (1, True), (2, False), (2, True)])
@pytest.mark.parametrize("du_dtype", [torch.float32, torch.bfloat16])
def test_recurrence_matches_oracle(sru, u_dtype, n_dir, masked, du_dtype):
    cfg = _cfg(n_dir=n_dir, masked=masked, proj_dtype=u_dtype)
    inp = generate(cfg, u_direct=True)
    if masked:
        inp["mask"][5, 1] = 1        # a hole inside a row as well as the padded tail
    alpha = 0.5 if masked else 1.0
    dcT = np.random.default_rng(5).standard_normal((cfg.B, n_dir, cfg.d)).astype(np.float32)
    gpu = tl.run_gpu_recurrence(sru, inp, n_dir, alpha, du_dtype=du_dtype, dc_T=dcT)
    ref = tl.oracle_recurrence(inp, alpha, dc_T=dcT)
    tl.compare_recurrence(gpu, ref, du_bf16=du_dtype == torch.bfloat16)


@pytest.mark.parametrize("L,B,d", [(1, 1, 8), (16, 1, 64), (17, 2, 8), (64, 5, 136), (2, 7, 512)])
def test_recurrence_edge_sizes(sru, L, B, d):
    cfg = _cfg(L=L, B=B, d=d, n_dir=2, masked=False)
    inp = generate(cfg, u_direct=True)
    gpu = tl.run_gpu_recurrence(sru, inp, 2, 1.0)
    ref = tl.oracle_recurrence(inp, 1.0)
    tl.compare_recurrence(gpu, ref)


def test_fully_padded_rows_and_zero_c0(sru):
    cfg = _cfg(L=40, B=4, d=72, n_dir=2, masked=True, c0="zero")
    inp = generate(cfg, u_direct=True)
    inp["mask"][:, 2] = 1            # one row entirely padded
    inp["mask"][:, 0] = 0            # one row not padded at all
    gpu = tl.run_gpu_recurrence(sru, inp, 2, 1.0)
    ref = tl.oracle_recurrence(inp, 1.0)
    tl.compare_recurrence(gpu, ref)
    assert np.all(gpu["h"][:, 2] == 0.0) and np.all(gpu["dU"][:, 2] == 0.0)


def test_zero_length_sequence(sru):
    B, d = 3, 16
    c0 = torch.randn(B, 1, d, device="cuda")
    cT = torch.full((B, 1, d), float("nan"), device="cuda")
    x = torch.empty(0, B, d, device="cuda")
    U = torch.empty(0, B, 1, 3, d, device="cuda")
    v = torch.zeros(1, 2, d, device="cuda")
    sru.sru_forward(U, x, v, v, torch.empty(0, B, 1, d, device="cuda"), cT, c0=c0)
    torch.cuda.synchronize()
    assert torch.equal(cT, c0)


def test_forward_state_chaining(sru):
    """forward(L1 + L2) == forward(L2) started from c_T of forward(L1)."""
    cfg = _cfg(L=50, B=2, d=64, n_dir=1, masked=False)
    inp = generate(cfg, u_direct=True)
    U = tl.dev_U(inp)
    x, v, b, c0 = tl.to_dev_f32(inp["x"]), tl.to_dev_f32(inp["v"]), tl.to_dev_f32(inp["bias"]), tl.to_dev_f32(inp["c0"])
    h = torch.empty(50, 2, 1, 64, device="cuda")
    cT = torch.empty(2, 1, 64, device="cuda")
    sru.sru_forward(U, x, v, b, h, cT, c0=c0)
    h1 = torch.empty(21, 2, 1, 64, device="cuda")
    c1 = torch.empty(2, 1, 64, device="cuda")
    sru.sru_forward(U[:21].contiguous(), x[:21].contiguous(), v, b, h1, c1, c0=c0)
    h2 = torch.empty(29, 2, 1, 64, device="cuda")
    c2 = torch.empty(2, 1, 64, device="cuda")
    sru.sru_forward(U[21:].contiguous(), x[21:].contiguous(), v, b, h2, c2, c0=c1)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([h1, h2]), h) and torch.equal(c2, cT)


def test_mask_equals_truncated_rows_on_gpu(sru):
    cfg = _cfg(L=48, B=3, d=64, n_dir=2, masked=False)
    inp = generate(cfg, u_direct=True)
    lengths = [48, 20, 33]
    mask = np.zeros((48, 3), np.uint8)
    for bb, lb in enumerate(lengths):
        mask[lb:, bb] = 1
    inp["mask"] = mask
    full = tl.run_gpu_recurrence(sru, inp, 2, 1.0)
    for bb, lb in enumerate(lengths):
        sub = {k: (None if inp[k] is None else inp[k]) for k in inp}
        sub["U"] = inp["U"][:lb, bb:bb + 1].copy()
        sub["x"] = inp["x"][:lb, bb:bb + 1].copy()
        sub["dh"] = inp["dh"][:lb, bb:bb + 1].copy()
        sub["c0"] = inp["c0"][bb:bb + 1].copy()
        sub["mask"] = None
        part = tl.run_gpu_recurrence(sru, sub, 2, 1.0)
        np.testing.assert_array_equal(full["h"][:lb, bb], part["h"][:, 0])
        np.testing.assert_array_equal(full["cT"][bb], part["cT"][0])
        np.testing.assert_array_equal(full["dU"][:lb, bb], part["dU"][:, 0])
        np.testing.assert_array_equal(full["dc0"][bb], part["dc0"][0])


def test_reverse_direction_equals_forward_on_flipped_input(sru):
    """Direction 1 walks t = L-1 .. 0: given direction 0's inputs mirrored in
    time (its U block, dh, and a palindromic x, which both directions read),
    and the same v, b and c0, it produces direction 0's outputs mirrored in
    time.  L is a multiple of the 16-step chunk, so the two walks perform the
    same operations in mirrored order."""
    L, B, d = 64, 3, 200
    cfg = _cfg(L=L, B=B, d=d, n_dir=2, masked=False)
    inp = generate(cfg, u_direct=True)
    inp["U"][:, :, 1] = inp["U"][::-1, :, 0]
    x = inp["x"]
    inp["x"] = np.ascontiguousarray(np.concatenate([x[: L // 2], x[: L // 2][::-1]]))  # x[t] == x[L-1-t]
    inp["dh"][:, :, 1] = inp["dh"][::-1, :, 0]
    inp["v"][1], inp["bias"][1] = inp["v"][0], inp["bias"][0]
    inp["c0"][:, 1] = inp["c0"][:, 0]
    gpu = tl.run_gpu_recurrence(sru, inp, 2, 0.75)
    np.testing.assert_array_equal(gpu["h"][:, :, 1], gpu["h"][::-1, :, 0])
    np.testing.assert_array_equal(gpu["cT"][:, 1], gpu["cT"][:, 0])
    np.testing.assert_array_equal(gpu["dU"][:, :, 1], gpu["dU"][::-1, :, 0])
    np.testing.assert_array_equal(gpu["dc0"][:, 1], gpu["dc0"][:, 0])
    np.testing.assert_array_equal(gpu["dv"][1], gpu["dv"][0])
    np.testing.assert_array_equal(gpu["db"][1], gpu["db"][0])


def test_invalid_arguments_are_rejected(sru):
    x = torch.zeros(4, 2, 12, device="cuda")  # d = 12 is not a multiple of 8
    U = torch.zeros(4, 2, 1, 3, 12, device="cuda")
    v = torch.zeros(1, 2, 12, device="cuda")
    with pytest.raises(sru.SRUError) as e:
        sru.sru_forward(U, x, v, v, torch.zeros(4, 2, 1, 12, device="cuda"), torch.zeros(2, 1, 12, device="cuda"))
    assert e.value.status == sru.SRU_ERR_UNSUPPORTED


@pytest.mark.parametrize("n_dir,masked", [(1, False), (2, True), (1, True)])
@pytest.mark.parametrize("L", [1, 37, 200])
@pytest.mark.parametrize("du_dtype", [torch.float32, torch.bfloat16])
def test_scan_path_matches_oracle(sru, n_dir, masked, L, du_dtype):
    """v = 0 through the chunked associative scan (forced), against the oracle."""
    cfg = _cfg(L=L, B=3, d=200, n_dir=n_dir, masked=masked, v_zero=True)
    inp = generate(cfg, u_direct=True)
    if masked and L > 5:
        inp["mask"][5, 1] = 1
    dcT = np.random.default_rng(6).standard_normal((cfg.B, n_dir, cfg.d)).astype(np.float32)
    flags = sru.SRU_FLAG_V_ZERO | sru.SRU_FLAG_FORCE_SCAN
    gpu = tl.run_gpu_recurrence(sru, inp, n_dir, 0.75, du_dtype=du_dtype, flags=flags, dc_T=dcT)
    ref = tl.oracle_recurrence(inp, 0.75, dc_T=dcT)
    tl.compare_recurrence(gpu, ref, du_bf16=du_dtype == torch.bfloat16)


def test_scan_equals_sequential_many_chunks(sru):
    """Scan and sequential paths agree at v = 0 over many scan chunks (L = 1000, 16 chunks)."""
    cfg = _cfg(L=1000, B=2, d=128, n_dir=2, masked=True, v_zero=True)
    inp = generate(cfg, u_direct=True)
    seq = tl.run_gpu_recurrence(sru, inp, 2, 1.0, flags=sru.SRU_FLAG_V_ZERO | sru.SRU_FLAG_FORCE_SEQUENTIAL)
    scan = tl.run_gpu_recurrence(sru, inp, 2, 1.0, flags=sru.SRU_FLAG_V_ZERO | sru.SRU_FLAG_FORCE_SCAN)
    for k in seq:
        tl.assert_close(k, scan[k], seq[k], tl.REC_TOL)
    ref = tl.oracle_recurrence(inp, 1.0, bs=np.arange(2), js=np.arange(0, 128, 9))
    tl.compare_recurrence(scan, ref, bs=np.arange(2), js=np.arange(0, 128, 9))


@pytest.mark.parametrize("n_dir,masked", [(1, False), (2, True)])
@pytest.mark.parametrize("L", [1, 37, 200])
def test_backward_scan_any_v_matches_oracle(sru, n_dir, masked, L):
    """The backward's chunked scan is exact for v != 0 too (affine state-gradient
    recurrence with coefficients recomputed from the forward checkpoints)."""
    cfg = _cfg(L=L, B=3, d=200, n_dir=n_dir, masked=masked)
    inp = generate(cfg, u_direct=True)
    if masked and L > 5:
        inp["mask"][5, 1] = 1
    dcT = np.random.default_rng(8).standard_normal((cfg.B, n_dir, cfg.d)).astype(np.float32)
    gpu = tl.run_gpu_recurrence(sru, inp, n_dir, 0.5, flags=sru.SRU_FLAG_FORCE_SCAN, dc_T=dcT)
    ref = tl.oracle_recurrence(inp, 0.5, dc_T=dcT)
    tl.compare_recurrence(gpu, ref)


def test_small_batch_takes_the_backward_scan_by_itself(sru):
    """B*d = 128 channels cannot fill the GPU: the library's own dispatch picks the
    backward scan (no flag) and the result still matches the oracle."""
    cfg = _cfg(L=700, B=2, d=64, n_dir=2, masked=True)
    inp = generate(cfg, u_direct=True)
    gpu = tl.run_gpu_recurrence(sru, inp, 2, 1.0)
    ref = tl.oracle_recurrence(inp, 1.0)
    tl.compare_recurrence(gpu, ref)
    seq = tl.run_gpu_recurrence(sru, inp, 2, 1.0, flags=sru.SRU_FLAG_FORCE_SEQUENTIAL)
    for k in ("dU", "dx", "dv", "db", "dc0"):
        tl.assert_close(k + " scan vs sequential", gpu[k], seq[k], tl.REC_TOL)


def test_padded_layer_taken_longest_rows_first(sru):
    """A padded bidirectional layer whose grid needs several waves of resident
    CTAs runs its batch rows longest first (a launch order computed from the
    mask on the device): the results do not depend on the order, so they match
    the oracle element by element, and equal the results of the same rows run
    in the natural order (a layer of few rows, which fits in one wave)."""
    cfg = _cfg(L=70, B=48, d=1024, n_dir=2, masked=True, seed=23)
    inp = generate(cfg, u_direct=True)
    inp["mask"][7, 3] = 1            # a hole inside a row
    inp["mask"][:, 5] = 1            # a row entirely padded
    gpu = tl.run_gpu_recurrence(sru, inp, 2, 1.0, du_dtype=torch.bfloat16)
    ref = tl.oracle_recurrence(inp, 1.0)
    tl.compare_recurrence(gpu, ref, du_bf16=True)
    # rows 0..3 alone (one wave, natural order) give the same bits per row
    sub = {k: (v[:, :4] if k in ("x", "U", "dh", "mask") and v is not None else v) for k, v in inp.items()}
    sub["c0"] = None if inp["c0"] is None else inp["c0"][:4]
    g4 = tl.run_gpu_recurrence(sru, sub, 2, 1.0, du_dtype=torch.bfloat16)
    for k in ("h", "cT", "dU", "dx", "dc0"):
        a = g4[k]
        b = gpu[k][:, :4] if k in ("h", "dU", "dx") else gpu[k][:4]
        assert np.array_equal(a, b), k
