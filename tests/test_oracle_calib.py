"""Pins of the oracle's head-map calibration (least squares of receiver maps on sender maps
over causal positions; the pages say the head-mapping weights are learned offline with both
models frozen, without stating the objective).

Each check holds for a reason outside the oracle's own code: a Gram written with numpy's
einsum on the explicitly masked maps, exact recovery of a planted linear map, numpy's lstsq
on the explicit design matrix, the residual summed directly, ridge limits, and the
invariance to bytes outside the causal triangle.
"""
import numpy as np
import pytest
import torch

import oracle


def _maps(rng, h, L, Lp, garbage=True):
    a = rng.standard_normal((h, Lp, Lp)).astype(np.float32)
    if not garbage:
        i, j = np.indices((Lp, Lp))
        a[:, (j > i) | (i >= L) | (j >= L)] = 0.0
    return a


def _features(X, Y, L):
    """Design matrix: one row per causal position (i < L, j <= i), columns = heads."""
    i, j = np.tril_indices(L)
    return np.concatenate([X[:, i, j], Y[:, i, j]], axis=0).T.astype(np.float64)


def test_gram_equals_einsum_over_causal_positions():
    rng = np.random.default_rng(1)
    L, Lp, h_s, h_r = 37, 40, 3, 2
    X, Y = _maps(rng, h_s, L, Lp), _maps(rng, h_r, L, Lp)
    g = oracle.calib_gram(torch.from_numpy(X), torch.from_numpy(Y), L)
    f = _features(X, Y, L)
    np.testing.assert_allclose(g, np.einsum("pa,pb->ab", f, f), rtol=1e-12, atol=1e-9)
    assert np.allclose(g, g.T) and np.linalg.eigvalsh(g).min() > -1e-9


def test_bytes_outside_the_causal_triangle_do_not_count():
    rng = np.random.default_rng(2)
    L, Lp = 29, 32
    X, Y = _maps(rng, 2, L, Lp, garbage=False), _maps(rng, 2, L, Lp, garbage=False)
    g0 = oracle.calib_gram(torch.from_numpy(X), torch.from_numpy(Y), L)
    i, j = np.indices((Lp, Lp))
    out = (j > i) | (i >= L) | (j >= L)
    X[:, out], Y[:, out] = 7.0, -3.0
    g1 = oracle.calib_gram(torch.from_numpy(X), torch.from_numpy(Y), L)
    np.testing.assert_array_equal(g0, g1)


def test_accumulates_over_sequences():
    rng = np.random.default_rng(3)
    X1, Y1 = _maps(rng, 2, 20, 24), _maps(rng, 3, 20, 24)
    X2, Y2 = _maps(rng, 2, 11, 16), _maps(rng, 3, 11, 16)
    g = oracle.calib_gram(torch.from_numpy(X1), torch.from_numpy(Y1), 20)
    oracle.calib_gram(torch.from_numpy(X2), torch.from_numpy(Y2), 11, gram=g)
    f = np.concatenate([_features(X1, Y1, 20), _features(X2, Y2, 11)])
    np.testing.assert_allclose(g, f.T @ f, rtol=1e-12, atol=1e-9)


def test_planted_linear_map_is_recovered_with_zero_residual():
    rng = np.random.default_rng(4)
    h_s, h_r, L, Lp = 5, 3, 48, 48
    X = _maps(rng, h_s, L, Lp)
    W_true = rng.standard_normal((h_r, h_s))
    Y = np.einsum("rs,sij->rij", W_true, X.astype(np.float64)).astype(np.float32)
    W, res = oracle.calib_solve(oracle.calib_gram(torch.from_numpy(X), torch.from_numpy(Y), L), h_s, h_r)
    np.testing.assert_allclose(W, W_true, rtol=0, atol=1e-6)  # Y was rounded to float32
    syy = np.sum(Y.astype(np.float64)[:, np.tril_indices(L)[0], np.tril_indices(L)[1]] ** 2, axis=1)
    assert np.all(np.abs(res) <= 1e-9 * syy)


def test_solve_matches_lstsq_and_direct_residual():
    rng = np.random.default_rng(5)
    h_s, h_r, L = 4, 3, 30
    X, Y = _maps(rng, h_s, L, L), _maps(rng, h_r, L, L)
    g = oracle.calib_gram(torch.from_numpy(X), torch.from_numpy(Y), L)
    W, res = oracle.calib_solve(g, h_s, h_r)
    f = _features(X, Y, L)
    A, B = f[:, :h_s], f[:, h_s:]
    W_ls = np.linalg.lstsq(A, B, rcond=None)[0].T
    np.testing.assert_allclose(W, W_ls, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(res, np.sum((B - A @ W.T) ** 2, axis=0), rtol=1e-8)


def test_ridge_limits():
    rng = np.random.default_rng(6)
    h_s, h_r, L = 3, 2, 25
    X, Y = _maps(rng, h_s, L, L), _maps(rng, h_r, L, L)
    g = oracle.calib_gram(torch.from_numpy(X), torch.from_numpy(Y), L)
    norms = [np.linalg.norm(oracle.calib_solve(g, h_s, h_r, lam)[0]) for lam in (0.0, 1.0, 1e2, 1e4, 1e12)]
    assert all(a > b for a, b in zip(norms, norms[1:])) and norms[-1] < 1e-8
    # ridge solve = the normal equations of the augmented system
    lam = 3.0
    W = oracle.calib_solve(g, h_s, h_r, lam)[0]
    np.testing.assert_allclose(W.T, np.linalg.solve(g[:h_s, :h_s] + lam * np.eye(h_s), g[:h_s, h_s:]),
                               rtol=1e-10)


def test_singular_sender_gram_is_refused_without_ridge():
    rng = np.random.default_rng(7)
    X = _maps(rng, 2, 16, 16)
    X[1] = 0.0  # a silent sender head
    Y = _maps(rng, 1, 16, 16)
    g = oracle.calib_gram(torch.from_numpy(X), torch.from_numpy(Y), 16)
    with pytest.raises(ValueError):
        oracle.calib_solve(g, 2, 1)
    W, _ = oracle.calib_solve(g, 2, 1, ridge=1e-3)
    assert W[0, 1] == 0.0


def test_bf16_inputs_are_read_exactly():
    rng = np.random.default_rng(8)
    X, Y = _maps(rng, 2, 12, 16), _maps(rng, 2, 12, 16)
    Xb, Yb = torch.from_numpy(X).to(torch.bfloat16), torch.from_numpy(Y).to(torch.bfloat16)
    g = oracle.calib_gram(Xb, Yb, 12)
    f = _features(Xb.float().numpy(), Yb.float().numpy(), 12)
    np.testing.assert_allclose(g, f.T @ f, rtol=1e-12, atol=1e-9)
