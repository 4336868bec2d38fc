"""Pins of the fp64 CPU oracle against facts the SRU equations fix.

The oracle must not be trusted because it agrees with itself: each test below
checks it against something independent of its code -- hand-derived values,
closed forms of special cases, central finite differences, invariants that the
equations imply, and numpy's matrix product.

Equations: "When Attention Meets Fast Recurrence: Training Language Models with
Reduced Compute" (T. Lei), background section on SRU, Eq. (1) and Eqs. (2)-(5).
"""
import math
import os

import numpy as np
import pytest

import oracle
from synthetic import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, generate, lengths_to_mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sru_hand_cases.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=")
            vals[k.strip()] = float(v)
    return vals


def _rand_problem(rng, L, B, d, n_dir, mask=False, v_scale=0.5):
    U = rng.standard_normal((L, B, n_dir, 3, d))
    x = rng.standard_normal((L, B, d))
    v = rng.uniform(-v_scale, v_scale, (n_dir, 2, d))
    bias = 0.1 * rng.standard_normal((n_dir, 2, d))
    c0 = rng.standard_normal((B, n_dir, d))
    m = None
    if mask:
        lengths = rng.integers(L // 2, L, size=B, endpoint=True)
        m = lengths_to_mask(lengths, L)
    return U, x, v, bias, c0, m


# ---------------------------------------------------------------- hand cases

@pytest.mark.parametrize("n_dir,dir_", [(1, 0), (2, 0), (2, 1)])
def test_one_step_hand_worked(n_dir, dir_):
    g = _golden()
    d = 1
    U = np.zeros((1, 1, n_dir, 3, d))
    v = np.zeros((n_dir, 2, d))
    bias = np.zeros((n_dir, 2, d))
    c0 = np.zeros((1, n_dir, d))
    # the other direction (if any) gets unrelated values, so a direction mix-up shows
    U[0, 0, :, :, 0] = 0.3
    v[:, :, 0] = 0.1
    U[0, 0, dir_, 0, 0] = g["L1.u_c"]
    U[0, 0, dir_, 1, 0] = math.log(3.0) - 1.25
    U[0, 0, dir_, 2, 0] = g["L1.u_r"]
    v[dir_, 0, 0], v[dir_, 1, 0] = g["L1.v_f"], g["L1.v_r"]
    bias[dir_, 0, 0], bias[dir_, 1, 0] = g["L1.b_f"], g["L1.b_r"]
    c0[0, dir_, 0] = g["L1.c0"]
    x = np.full((1, 1, d), g["L1.x"])
    alpha = g["L1.alpha"]
    h, cT = oracle.forward(U, x, v, bias, c0=c0, alpha=alpha)
    assert h[0, 0, dir_, 0] == pytest.approx(g["L1.h"], abs=1e-12)
    assert cT[0, dir_, 0] == pytest.approx(g["L1.cT"], abs=1e-12)
    dh = np.zeros((1, 1, n_dir, d))
    dh[0, 0, dir_, 0] = 1.0
    gr = oracle.backward(U, x, v, bias, dh, c0=c0, alpha=alpha)
    assert gr["dU"][0, 0, dir_, 0, 0] == pytest.approx(g["L1.dU_c"], abs=1e-12)
    assert gr["dU"][0, 0, dir_, 1, 0] == pytest.approx(g["L1.dU_f"], abs=1e-12)
    assert gr["dU"][0, 0, dir_, 2, 0] == pytest.approx(g["L1.dU_r"], abs=1e-12)
    assert gr["dx"][0, 0, 0] == pytest.approx(g["L1.dx"], abs=1e-12)
    assert gr["dv"][dir_, 0, 0] == pytest.approx(g["L1.dv_f"], abs=1e-12)
    assert gr["dv"][dir_, 1, 0] == pytest.approx(g["L1.dv_r"], abs=1e-12)
    assert gr["dbias"][dir_, 0, 0] == pytest.approx(g["L1.db_f"], abs=1e-12)
    assert gr["dbias"][dir_, 1, 0] == pytest.approx(g["L1.db_r"], abs=1e-12)
    assert gr["dc0"][0, dir_, 0] == pytest.approx(g["L1.dc0"], abs=1e-12)
    if n_dir == 2:
        other = 1 - dir_
        assert np.all(gr["dU"][0, 0, other] == 0.0)
        assert gr["dc0"][0, other, 0] == 0.0


def test_two_steps_time_order_of_directions():
    g = _golden()
    U = np.zeros((2, 1, 2, 3, 1))
    U[0, 0, :, 0, 0] = g["L2.u_c_t0"]
    U[1, 0, :, 0, 0] = g["L2.u_c_t1"]
    U[:, 0, :, 2, 0] = 1e4              # r = 1 exactly in fp64
    v = np.zeros((2, 2, 1))
    bias = np.zeros((2, 2, 1))
    x = np.full((2, 1, 1), 123.0)       # must not leak into h when r = 1
    h, cT = oracle.forward(U, x, v, bias)
    assert h[0, 0, 0, 0] == g["L2.dir0.h_t0"] and h[1, 0, 0, 0] == g["L2.dir0.h_t1"]
    assert h[0, 0, 1, 0] == g["L2.dir1.h_t0"] and h[1, 0, 1, 0] == g["L2.dir1.h_t1"]
    assert cT[0, 0, 0] == g["L2.dir0.cT"] and cT[0, 1, 0] == g["L2.dir1.cT"]


# ------------------------------------------------------------- closed forms

def test_constant_forget_gate_is_an_exponential_moving_average():
    """v = 0 and constant u_f: c_t = f^(t+1) c0 + (1-f) sum_{k<=t} f^(t-k) u_k."""
    rng = np.random.default_rng(11)
    L, B, d = 40, 3, 5
    U, x, v, bias, c0, _ = _rand_problem(rng, L, B, d, 1)
    v[:] = 0.0
    zf = rng.standard_normal(d)
    U[:, :, 0, 1, :] = zf[None, None, :] - bias[0, 0][None, None, :]
    U[:, :, 0, 2, :] = 1e4                   # r = 1: h = c
    f = 1.0 / (1.0 + np.exp(-zf))            # (d,)
    h, cT = oracle.forward(U, x, v, bias, c0=c0)
    uc = U[:, :, 0, 0, :]                    # (L, B, d)
    expected = np.empty((L, B, d))
    for tt in range(L):
        k = np.arange(tt + 1)
        w = (1.0 - f)[None, :] * f[None, :] ** (tt - k)[:, None]          # (tt+1, d)
        expected[tt] = f ** (tt + 1) * c0[:, 0, :] + np.einsum("kd,kbd->bd", w, uc[: tt + 1])
    np.testing.assert_allclose(h[:, :, 0, :], expected, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(cT[:, 0, :], expected[-1], rtol=1e-12, atol=1e-12)


def test_constant_input_relaxes_geometrically():
    """v = 0, constant f and u: c_t = u + f^(t+1) (c0 - u)."""
    L, d = 30, 4
    f_target = np.array([0.1, 0.5, 0.9, 0.99])
    zf = np.log(f_target / (1.0 - f_target))
    u = np.array([1.0, -2.0, 0.5, 3.0])
    c0 = np.array([[[-1.0, 4.0, 2.0, 0.0]]])
    U = np.zeros((L, 1, 1, 3, d))
    U[:, 0, 0, 0, :] = u
    U[:, 0, 0, 1, :] = zf
    U[:, 0, 0, 2, :] = 1e4
    h, _ = oracle.forward(U, np.zeros((L, 1, d)), np.zeros((1, 2, d)), np.zeros((1, 2, d)), c0=c0)
    t = np.arange(L)[:, None]
    np.testing.assert_allclose(h[:, 0, 0, :], u + f_target ** (t + 1) * (c0[0, 0] - u), rtol=1e-12, atol=1e-12)


def test_forget_gate_closed_copies_candidate():
    """f = 0 (u_f = -1e4, v_f = 0): c_t = u_c[t] exactly."""
    rng = np.random.default_rng(2)
    U, x, v, bias, c0, _ = _rand_problem(rng, 9, 2, 6, 2)
    v[:, 0, :] = 0.0
    U[:, :, :, 1, :] = -1e4
    U[:, :, :, 2, :] = 1e4
    h, cT = oracle.forward(U, x, v, bias, c0=c0)
    assert np.array_equal(h, U[:, :, :, 0, :])
    assert np.array_equal(cT[:, 0, :], U[-1, :, 0, 0, :])
    assert np.array_equal(cT[:, 1, :], U[0, :, 1, 0, :])


def test_forget_gate_open_keeps_initial_state():
    """f = 1 (u_f = +1e4, v_f = 0): c_t = c0 for all t."""
    rng = np.random.default_rng(3)
    U, x, v, bias, c0, _ = _rand_problem(rng, 7, 2, 5, 2)
    v[:, 0, :] = 0.0
    U[:, :, :, 1, :] = 1e4
    U[:, :, :, 2, :] = 1e4
    h, cT = oracle.forward(U, x, v, bias, c0=c0)
    assert np.array_equal(h, np.broadcast_to(c0[None], h.shape))
    assert np.array_equal(cT, c0)


@pytest.mark.parametrize("alpha", [1.0, 0.5, -2.0])
def test_reset_gate_limits(alpha):
    """r = 1 gives h = c; r = 0 gives h = alpha * x exactly (Eq. (5))."""
    rng = np.random.default_rng(4)
    U, x, v, bias, c0, _ = _rand_problem(rng, 8, 3, 4, 1)
    v[:, 1, :] = 0.0
    U1 = U.copy()
    U1[:, :, :, 2, :] = 1e4
    h1, _ = oracle.forward(U1, x, v, bias, c0=c0, alpha=alpha)
    U0 = U.copy()
    U0[:, :, :, 2, :] = -1e4
    h0, _ = oracle.forward(U0, x, v, bias, c0=c0, alpha=alpha)
    assert np.array_equal(h0[:, :, 0, :], alpha * x)
    # with r = 1 the output is the state, which does not depend on the reset gate or x
    h1b, _ = oracle.forward(U1, 5.0 * x, v, bias, c0=c0, alpha=alpha)
    assert np.array_equal(h1, h1b)
    # and the state itself follows Eq. (4): check one step by hand
    f0 = 1.0 / (1.0 + np.exp(-(U[0, :, 0, 1, :] + v[0, 0] * c0[:, 0, :] + bias[0, 0])))
    np.testing.assert_allclose(h1[0, :, 0, :], f0 * c0[:, 0, :] + (1 - f0) * U[0, :, 0, 0, :], rtol=1e-14)


# -------------------------------------------------------- finite differences

def _loss(U, x, v, bias, c0, mask, dh, dcT, alpha):
    h, cT = oracle.forward(U, x, v, bias, c0=c0, mask=mask, alpha=alpha)
    return float(np.sum(dh * h) + np.sum(dcT * cT))


@pytest.mark.parametrize("L,B,d,n_dir,masked", [
    (16, 2, 32, 1, False),   # the tiny fp32 workload's size, every element
    (6, 3, 3, 2, True),      # bidirectional with padding
    (5, 2, 4, 1, True),
])
def test_backward_matches_central_differences(L, B, d, n_dir, masked):
    rng = np.random.default_rng(100 + L)
    U, x, v, bias, c0, mask = _rand_problem(rng, L, B, d, n_dir, mask=masked)
    if masked:
        mask[L - 1, 0] = 1          # at least one padded position
        mask[1, B - 1] = 1          # and one hole inside a row
    alpha = 0.7
    dh = rng.standard_normal((L, B, n_dir, d))
    dcT = rng.standard_normal((B, n_dir, d))
    gr = oracle.backward(U, x, v, bias, dh, c0=c0, mask=mask, dcT=dcT, alpha=alpha)
    eps = 1e-6
    args = dict(U=U, x=x, v=v, bias=bias, c0=c0)
    grads = dict(U=gr["dU"], x=gr["dx"], v=gr["dv"], bias=gr["dbias"], c0=gr["dc0"])
    for name, arr in args.items():
        fd = np.empty(arr.size)
        flat = arr.reshape(-1)
        for i in range(arr.size):
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(mask=mask, dh=dh, dcT=dcT, alpha=alpha, **args)
            flat[i] = old - eps
            lm = _loss(mask=mask, dh=dh, dcT=dcT, alpha=alpha, **args)
            flat[i] = old
            fd[i] = (lp - lm) / (2 * eps)
        an = grads[name].reshape(-1)
        err = np.abs(fd - an)
        assert np.all(err <= 1e-6 * (1.0 + np.abs(an))), (name, err.max())


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("n_dir", [1, 2])
def test_mask_equals_truncated_rows(n_dir):
    """A suffix-padded row gives exactly the run on that row cut to its length."""
    rng = np.random.default_rng(7)
    L, B, d = 12, 4, 3
    U, x, v, bias, c0, _ = _rand_problem(rng, L, B, d, n_dir)
    lengths = np.array([12, 6, 9, 1])
    mask = lengths_to_mask(lengths, L)
    dh = rng.standard_normal((L, B, n_dir, d))
    dcT = rng.standard_normal((B, n_dir, d))
    h, cT = oracle.forward(U, x, v, bias, c0=c0, mask=mask)
    gr = oracle.backward(U, x, v, bias, dh, c0=c0, mask=mask, dcT=dcT)
    for b, lb in enumerate(lengths):
        sl = (slice(0, lb), slice(b, b + 1))
        hb, cTb = oracle.forward(U[sl], x[sl], v, bias, c0=c0[b:b + 1])
        grb = oracle.backward(U[sl], x[sl], v, bias, dh[sl], c0=c0[b:b + 1], dcT=dcT[b:b + 1])
        np.testing.assert_array_equal(h[:lb, b], hb[:, 0])
        assert np.all(h[lb:, b] == 0.0)
        np.testing.assert_array_equal(cT[b], cTb[0])
        np.testing.assert_array_equal(gr["dU"][:lb, b], grb["dU"][:, 0])
        assert np.all(gr["dU"][lb:, b] == 0.0) and np.all(gr["dx"][lb:, b] == 0.0)
        np.testing.assert_array_equal(gr["dx"][:lb, b], grb["dx"][:, 0])
        np.testing.assert_array_equal(gr["dc0"][b], grb["dc0"][0])


def test_masked_hole_is_a_deleted_step():
    """A padded position inside a row acts as if that time step were removed."""
    rng = np.random.default_rng(8)
    L, B, d = 10, 1, 4
    U, x, v, bias, c0, _ = _rand_problem(rng, L, B, d, 1)
    mask = np.zeros((L, B), np.uint8)
    mask[4, 0] = 1
    h, cT = oracle.forward(U, x, v, bias, c0=c0, mask=mask)
    keep = [t for t in range(L) if t != 4]
    h2, cT2 = oracle.forward(U[keep], x[keep], v, bias, c0=c0)
    np.testing.assert_array_equal(h[keep], h2)
    assert np.all(h[4] == 0.0)
    np.testing.assert_array_equal(cT, cT2)


def test_reverse_direction_is_forward_on_flipped_time():
    rng = np.random.default_rng(9)
    L, B, d = 11, 3, 5
    U, x, v, bias, c0, _ = _rand_problem(rng, L, B, d, 2)
    dh = rng.standard_normal((L, B, 2, d))
    dcT = rng.standard_normal((B, 2, d))
    h, cT = oracle.forward(U, x, v, bias, c0=c0, alpha=0.5)
    gr = oracle.backward(U, x, v, bias, dh, c0=c0, dcT=dcT, alpha=0.5)
    Uf = U[::-1, :, 1:2]
    hf, cTf = oracle.forward(Uf, x[::-1], v[1:2], bias[1:2], c0=c0[:, 1:2], alpha=0.5)
    np.testing.assert_array_equal(h[::-1, :, 1:2], hf)
    np.testing.assert_array_equal(cT[:, 1:2], cTf)
    grf = oracle.backward(Uf, x[::-1], v[1:2], bias[1:2], dh[::-1, :, 1:2], c0=c0[:, 1:2],
                          dcT=dcT[:, 1:2], alpha=0.5)
    np.testing.assert_array_equal(gr["dU"][::-1, :, 1:2], grf["dU"])
    gr0 = oracle.backward(U[:, :, 0:1], x, v[0:1], bias[0:1], dh[:, :, 0:1], c0=c0[:, 0:1],
                          dcT=dcT[:, 0:1], alpha=0.5)
    np.testing.assert_allclose(gr["dx"], gr0["dx"] + grf["dx"][::-1], rtol=1e-15, atol=1e-15)


def test_state_chaining():
    """forward over L1+L2 steps == forward over L2 steps started from cT of the first L1."""
    rng = np.random.default_rng(10)
    L, B, d = 14, 2, 3
    U, x, v, bias, c0, _ = _rand_problem(rng, L, B, d, 1)
    dh = rng.standard_normal((L, B, 1, d))
    h, cT = oracle.forward(U, x, v, bias, c0=c0)
    h1, c1 = oracle.forward(U[:5], x[:5], v, bias, c0=c0)
    h2, c2 = oracle.forward(U[5:], x[5:], v, bias, c0=c1)
    np.testing.assert_array_equal(h, np.concatenate([h1, h2]))
    np.testing.assert_array_equal(cT, c2)
    gr = oracle.backward(U, x, v, bias, dh, c0=c0)
    g2 = oracle.backward(U[5:], x[5:], v, bias, dh[5:], c0=c1)
    g1 = oracle.backward(U[:5], x[:5], v, bias, dh[:5], c0=c0, dcT=g2["dc0"])
    np.testing.assert_allclose(gr["dU"], np.concatenate([g1["dU"], g2["dU"]]), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(gr["dc0"], g1["dc0"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(gr["dv"], g1["dv"] + g2["dv"], rtol=1e-12, atol=1e-12)


def test_channels_are_independent():
    """Each (b, j) channel depends only on its own inputs: a sub-problem gives the same values."""
    rng = np.random.default_rng(12)
    L, B, d = 9, 4, 6
    U, x, v, bias, c0, mask = _rand_problem(rng, L, B, d, 2, mask=True)
    h, cT = oracle.forward(U, x, v, bias, c0=c0, mask=mask)
    bs, js = [1, 3], [0, 4, 5]
    ix = np.ix_(range(L), bs)
    hs, cTs = oracle.forward(U[:, bs][:, :, :, :, js], x[:, bs][:, :, js], v[:, :, js], bias[:, :, js],
                             c0=c0[bs][:, :, js], mask=mask[ix])
    np.testing.assert_array_equal(h[:, bs][:, :, :, js], hs)
    np.testing.assert_array_equal(cT[bs][:, :, js], cTs)


# -------------------------------------------------------------- projection

def test_projection_and_gradients_match_numpy():
    rng = np.random.default_rng(13)
    M, N, K = 37, 21, 19
    X = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    dU = rng.standard_normal((M, N))
    np.testing.assert_allclose(oracle.project(X, W), X @ W.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.project_dX(dU, W), dU @ W, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.project_dW(dU, X), dU.T @ X, rtol=1e-12, atol=1e-12)
    rows = rng.integers(0, M, 50)
    cols = rng.integers(0, N, 50)
    np.testing.assert_allclose(oracle.project_entries(X, W, rows, cols), (X @ W.T)[rows, cols], rtol=1e-12)
    colsk = rng.integers(0, K, 50)
    np.testing.assert_allclose(oracle.project_dX_entries(dU, W, rows, colsk), (dU @ W)[rows, colsk], rtol=1e-12)
    rowsn = rng.integers(0, N, 50)
    np.testing.assert_allclose(oracle.project_dW_entries(dU, X, rowsn, colsk), (dU.T @ X)[rowsn, colsk], rtol=1e-12)


def test_projection_reads_bf16_and_fp32_operands_exactly():
    rng = np.random.default_rng(14)
    M, N, K = 9, 7, 33
    Xb = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    Wf = rng.standard_normal((N, K)).astype(np.float32)
    ref = bf16_bits_to_f32(Xb).astype(np.float64) @ Wf.astype(np.float64).T
    np.testing.assert_allclose(oracle.project(Xb, Wf), ref, rtol=1e-13, atol=1e-13)


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e38], np.float32)
    back = bf16_bits_to_f32(f32_to_bf16_bits(vals))
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1); 1 + 3*2^-8 is a tie -> 1 + 2^-6
    np.testing.assert_array_equal(back[:4], np.array([1.0, 1.0, 1.0 + 2 ** -6, 1.0], np.float32))
    assert back[4] == -2.5


def test_generated_workloads_have_the_stated_shapes():
    cfg = CONFIGS["tiny_fp32"]
    inp = generate(cfg)
    assert inp["x"].shape == (16, 2, 32) and inp["W"].shape == (96, 32)
    assert inp["dh"].shape == (16, 2, 1, 32)
    a = math.sqrt(3.0 / 32)
    assert np.all(np.abs(inp["W"]) <= a) and np.all(np.abs(inp["v"]) <= 0.5)
    assert np.all(inp["bias"] == 0) and inp["c0"] is None
    small = CONFIGS["bidir_masked"].replace(L=64, B=8, d=16)
    s = generate(small)
    assert s["W"].dtype == np.uint16 and s["W"].shape == (2 * 3 * 16, 16)
    assert np.all((s["lengths"] >= 32) & (s["lengths"] <= 64))
    assert s["mask"].shape == (64, 8)
    # reproducible from the seed
    assert np.array_equal(generate(small)["x"], s["x"])
