"""Pins of the oracle's SRU++ attention producer (oracle.attention_project),
each against a fact the page or the mathematics fixes, not against the
oracle's own formula."""
import numpy as np

import oracle


def _w(rng, *shape):
    return rng.standard_normal(shape) / np.sqrt(shape[-1])


def _case(seed=0, L=5, B=3, d=12, dp=4, N=18):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((L * B, d)), _w(rng, dp, d), _w(rng, dp, dp), _w(rng, dp, dp), _w(rng, N, dp), L, B)


def test_alpha_zero_is_the_factorised_linear_map():
    # the page: with alpha = 0, U = Wo Q = (Wo Wq) X^T, the attention is skipped
    X, Wq, Wk, Wv, Wo, L, B = _case()
    U = oracle.attention_project(X, Wq, Wk, Wv, Wo, 0.0, L, B)
    np.testing.assert_allclose(U, X @ (Wo @ Wq).T, rtol=1e-12, atol=1e-12)


def test_single_token_attends_only_to_itself():
    # L = 1: the softmax of one score is 1, so A = V = Q Wv^T and U = Wo (Q + alpha V)
    X, Wq, Wk, Wv, Wo, _, B = _case(L=1)
    alpha = 0.7
    Q = X @ Wq.T
    U = oracle.attention_project(X, Wq, Wk, Wv, Wo, alpha, 1, B)
    np.testing.assert_allclose(U, (Q + alpha * (Q @ Wv.T)) @ Wo.T, rtol=1e-12, atol=1e-12)


def test_constant_sequence_averages_identical_values():
    # every token of a row equal: all V_t equal, so any convex weights give A_t = V_t
    X, Wq, Wk, Wv, Wo, L, B = _case(L=6)
    X = np.repeat(X[:B][None], L, axis=0).reshape(L * B, -1)
    alpha = -1.3
    Q = X @ Wq.T
    for causal in (True, False):
        U = oracle.attention_project(X, Wq, Wk, Wv, Wo, alpha, L, B, causal=causal)
        np.testing.assert_allclose(U, (Q + alpha * (Q @ Wv.T)) @ Wo.T, rtol=1e-12, atol=1e-12)


def test_causal_output_ignores_later_tokens_and_rows():
    X, Wq, Wk, Wv, Wo, L, B = _case(L=7, B=2)
    U = oracle.attention_project(X, Wq, Wk, Wv, Wo, 0.9, L, B)
    Y = X.copy()
    Y[4 * B + 1] += 3.0                      # token t = 4 of batch row 1
    V = oracle.attention_project(Y, Wq, Wk, Wv, Wo, 0.9, L, B)
    rows_b1 = np.arange(L) * B + 1
    np.testing.assert_array_equal(U[:4 * B], V[:4 * B])              # earlier tokens: unchanged
    np.testing.assert_array_equal(U[np.arange(L) * B], V[np.arange(L) * B])  # other batch row: unchanged
    assert np.abs(U[rows_b1[4:]] - V[rows_b1[4:]]).max() > 1e-3       # this and later tokens move


def test_last_token_is_the_same_with_or_without_the_causal_mask():
    X, Wq, Wk, Wv, Wo, L, B = _case(L=6)
    U = oracle.attention_project(X, Wq, Wk, Wv, Wo, 1.1, L, B, causal=True)
    V = oracle.attention_project(X, Wq, Wk, Wv, Wo, 1.1, L, B, causal=False)
    last = (L - 1) * B + np.arange(B)
    np.testing.assert_allclose(U[last], V[last], rtol=1e-12, atol=1e-12)
    assert np.abs(U[:B] - V[:B]).max() > 1e-6


def test_two_token_softmax_by_hand():
    # L = 2, d = d' = 1, N = 1, every weight 1 except Wv: scores are q_t q_s, A_1 mixes V_0, V_1
    X = np.array([[0.5], [2.0]])             # B = 1: tokens 0 and 1
    one = np.ones((1, 1))
    Wv = np.array([[3.0]])
    U = oracle.attention_project(X, one, one, Wv, one, 1.0, 2, 1)
    q0, q1 = 0.5, 2.0
    w0, w1 = np.exp(q1 * q0), np.exp(q1 * q1)   # sqrt(d') = 1
    a1 = (w0 * 3 * q0 + w1 * 3 * q1) / (w0 + w1)
    np.testing.assert_allclose(U[:, 0], [q0 + 3 * q0, q1 + a1], rtol=1e-12)


def test_layernorm_single_token_closed_form():
    X, Wq, Wk, Wv, Wo, _, B = _case(L=1, dp=6)
    g = np.linspace(0.5, 1.5, 6)
    be = np.linspace(-0.2, 0.3, 6)
    Q = X @ Wq.T
    R = Q + 0.4 * (Q @ Wv.T)
    Rn = (R - R.mean(1, keepdims=True)) / np.sqrt(R.var(1, keepdims=True) + 1e-5) * g + be
    U = oracle.attention_project(X, Wq, Wk, Wv, Wo, 0.4, 1, B, ln_gamma=g, ln_beta=be)
    np.testing.assert_allclose(U, Rn @ Wo.T, rtol=1e-11, atol=1e-12)


def test_two_token_softmax_scaled_by_sqrt_dprime():
    # d = d' = N = 4, Wq = Wk = Wo = I, Wv = 3 I: Q = K = X, V = 3 X; only feature 0 is nonzero.
    # Token 1's scores are q1.k0 / sqrt(4) and q1.k1 / sqrt(4) (the 1/sqrt(d') matters here).
    a, b = 0.5, 2.0
    X = np.zeros((2, 4))
    X[0, 0], X[1, 0] = a, b                  # B = 1: tokens 0 and 1
    eye = np.eye(4)
    U = oracle.attention_project(X, eye, eye, 3 * eye, eye, 1.0, 2, 1)
    w0, w1 = np.exp(b * a / 2.0), np.exp(b * b / 2.0)
    a1 = (w0 * 3 * a + w1 * 3 * b) / (w0 + w1)
    np.testing.assert_allclose(U[:, 0], [a + 3 * a, b + a1], rtol=1e-12)
    np.testing.assert_array_equal(U[:, 1:], 0.0)


# ------------------------------------------------------------ the backward
def _loss(dU, *args, **kw):
    return float((dU * oracle.attention_project(*args, **kw)).sum())


def _central(f, arr, idx, h=1e-6):
    old = arr[idx]
    arr[idx] = old + h
    up = f()
    arr[idx] = old - h
    dn = f()
    arr[idx] = old
    return (up - dn) / (2 * h)


def _check_backward_against_differences(causal, with_ln, alpha, seed):
    # every input element's gradient against a central difference of the
    # forward oracle's loss sum(dU * U): pins each step of the chain rule
    X, Wq, Wk, Wv, Wo, L, B = _case(seed=seed, L=4, B=2, d=6, dp=4, N=5)
    rng = np.random.default_rng(100 + seed)
    dU = rng.standard_normal((L * B, Wo.shape[0]))
    g = 1.0 + 0.3 * rng.standard_normal(Wq.shape[0]) if with_ln else None
    be = 0.2 * rng.standard_normal(Wq.shape[0]) if with_ln else None
    kw = dict(causal=causal, ln_gamma=g, ln_beta=be)
    got = oracle.attention_project_backward(dU, X, Wq, Wk, Wv, Wo, alpha, L, B, **kw)
    named = {"dX": X, "dWq": Wq, "dWk": Wk, "dWv": Wv, "dWo": Wo}
    if with_ln:
        named.update(dgamma=g, dbeta=be)
    else:
        assert "dgamma" not in got and "dbeta" not in got
    for name, arr in named.items():
        assert got[name].shape == arr.shape, name
        for idx in np.ndindex(arr.shape):
            fd = _central(lambda: _loss(dU, X, Wq, Wk, Wv, Wo, alpha, L, B, **kw), arr, idx)
            assert abs(got[name][idx] - fd) <= 1e-6 * (1 + abs(fd)), (name, idx, got[name][idx], fd)


def test_backward_matches_central_differences_causal():
    _check_backward_against_differences(True, False, 0.8, 1)


def test_backward_matches_central_differences_full_attention_with_norm():
    _check_backward_against_differences(False, True, -0.6, 2)


def test_backward_matches_central_differences_causal_with_norm():
    _check_backward_against_differences(True, True, 1.3, 3)


def test_backward_at_alpha_zero_is_the_factorised_maps_gradient():
    # alpha = 0: U = X (Wo Wq)^T, so dX = dU Wo Wq, dWo = dU^T Q, dWq = (dU Wo)^T X,
    # and the attention weights receive nothing
    X, Wq, Wk, Wv, Wo, L, B = _case(seed=4)
    dU = np.random.default_rng(5).standard_normal((L * B, Wo.shape[0]))
    got = oracle.attention_project_backward(dU, X, Wq, Wk, Wv, Wo, 0.0, L, B)
    Q = X @ Wq.T
    np.testing.assert_allclose(got["dX"], dU @ Wo @ Wq, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dWo"], dU.T @ Q, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dWq"], (dU @ Wo).T @ X, rtol=1e-12, atol=1e-12)
    assert np.abs(got["dWk"]).max() == 0 and np.abs(got["dWv"]).max() == 0
