"""Pins for the oracle's error-feedback (LDLQ) driver, against facts that do not
come from the oracle.

* the three-weight toy of the 2-bit post (values the page prints): correlated
  inputs give [0, 1, 0], a diagonal H gives plain rounding [0, 0, 0];
* a diagonal H (U = I) reduces the driver to independent coding blocks;
* the loss identity: with feedback through U's off-diagonal blocks and a U
  whose within-block part is the identity, the proxy loss sum_r e_r H e_r^T
  (e = w - q, H = U diag(d) U^T) equals the sum of the blocks' Viterbi costs
  exactly, whatever the codebook.  A dropped feedback term, a wrong sign, a
  transposed U or feedback of the target error instead of the weight error
  each break it;
* the first coding block of every row is an ordinary encode of w.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle_decode, oracle_encode, oracle_ldlq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def udu_factor(H):
    """H = U diag(d) U^T with U unit upper triangular, via a Cholesky factor of
    the index-reversed matrix (numpy's routine, an independent computation)."""
    n = H.shape[0]
    J = np.eye(n)[::-1]
    C = np.linalg.cholesky(J @ H @ J)  # lower
    R = J @ C @ J  # upper, H = R R^T
    diag = np.diag(R).copy()
    U = R / diag[None, :]
    return U, diag**2


def block_free_u(rng, cols, T, scale=0.3):
    """Unit upper U whose T x T diagonal blocks are the identity."""
    U = np.triu(rng.standard_normal((cols, cols)) * scale, 1)
    for j in range(cols // T):
        U[j * T:(j + 1) * T, j * T:(j + 1) * T] = 0.0
    return U + np.eye(cols)


def test_udu_factor_reconstructs():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((9, 30))
    H = A @ A.T / 30 + 0.1 * np.eye(9)
    U, d = udu_factor(H)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.allclose(np.diag(U), 1.0)
    assert np.allclose(U @ np.diag(d) @ U.T, H, atol=1e-12)


def test_page_three_weight_toy():
    with open(os.path.join(GOLDEN, "page_error_feedback_toy.json")) as f:
        g = json.load(f)
    w = np.array([g["w"]])
    n = w.shape[1]
    cb = np.array(g["codebook"])
    # correlated inputs: H = 1 1^T + eps I
    H = np.ones((n, n)) + g["eps"] * np.eye(n)
    U, d = udu_factor(H)
    q, _, _, _, _ = oracle_ldlq(w, U, d, cb, g["L"], g["k"], g["T"])
    assert q[0].tolist() == g["printed_feedback_rounding"]
    assert abs(q.sum() - w.sum()) == pytest.approx(0.2)
    # uncorrelated inputs: diagonal H is plain rounding
    Hd = np.diag([1.0, 2.0, 0.5])
    Ud, dd = udu_factor(Hd)
    assert np.allclose(Ud, np.eye(n))
    q0, _, _, _, _ = oracle_ldlq(w, Ud, dd, cb, g["L"], g["k"], g["T"])
    assert q0[0].tolist() == g["printed_plain_rounding"]


@pytest.mark.parametrize("L,k,T,rows,cols", [(4, 2, 8, 3, 32), (6, 1, 5, 2, 20), (8, 2, 16, 2, 64)])
def test_diagonal_hessian_is_independent_blocks(L, k, T, rows, cols):
    rng = np.random.default_rng(100 + L + T)
    w = rng.standard_normal((rows, cols))
    d = rng.lognormal(0.0, 0.5, cols)
    cb = rng.standard_normal(1 << L)
    q, xt, start, bits, cost = oracle_ldlq(w, np.eye(cols), d, cb, L, k, T)
    assert np.array_equal(xt, w)
    nb = cols // T
    for r in range(rows):
        for j in range(nb):
            s1, b1, c1 = oracle_encode(w[r, j * T:(j + 1) * T], d[j * T:(j + 1) * T], cb, L, k)
            assert cost[r * nb + j] == pytest.approx(c1[0], rel=1e-12, abs=1e-300)
            y = oracle_decode(bits[r * nb + j][None, :], start[r * nb + j:r * nb + j + 1], cb, L, k, T)
            assert np.array_equal(y[0], q[r, j * T:(j + 1) * T])


@pytest.mark.parametrize("L,k,T,rows,cols", [(4, 2, 8, 3, 32), (6, 2, 4, 4, 24), (5, 1, 6, 2, 30), (8, 3, 8, 2, 48)])
def test_loss_identity(L, k, T, rows, cols):
    rng = np.random.default_rng(7 * L + 13 * T + cols)
    w = rng.standard_normal((rows, cols))
    d = rng.lognormal(0.0, 0.7, cols)
    cb = rng.standard_normal(1 << L)
    U = block_free_u(rng, cols, T)
    H = U @ np.diag(d) @ U.T
    q, xt, start, bits, cost = oracle_ldlq(w, U, d, cb, L, k, T)
    e = w - q
    loss = float(np.einsum("ri,ij,rj->", e, H, e))
    assert loss == pytest.approx(float(cost.sum()), rel=1e-10)
    # the feedback is not trivial on these inputs
    assert not np.allclose(xt, w)


def test_loss_identity_detects_a_wrong_feedback():
    """The identity is a real check: plain blockwise coding of w under the same H
    misses it by a wide margin."""
    rng = np.random.default_rng(77)
    L, k, T, rows, cols = 4, 2, 8, 3, 32
    w = rng.standard_normal((rows, cols))
    d = rng.lognormal(0.0, 0.7, cols)
    cb = rng.standard_normal(1 << L)
    U = block_free_u(rng, cols, T)
    H = U @ np.diag(d) @ U.T
    q, _, _, _, cost = oracle_ldlq(w, np.eye(cols), d, cb, L, k, T)
    e = w - q
    loss = float(np.einsum("ri,ij,rj->", e, H, e))
    assert abs(loss - float(cost.sum())) > 1e-3 * float(cost.sum())


def test_first_block_is_plain_encode_and_costs_reproduce():
    rng = np.random.default_rng(31)
    L, k, T, rows, cols = 6, 2, 8, 3, 40
    w = rng.standard_normal((rows, cols))
    A = rng.standard_normal((cols, 3 * cols))
    H = A @ A.T / (3 * cols) + 0.05 * np.eye(cols)
    U, d = udu_factor(H)
    cb = rng.standard_normal(1 << L)
    q, xt, start, bits, cost = oracle_ldlq(w, U, d, cb, L, k, T)
    nb = cols // T
    assert np.array_equal(xt[:, :T], w[:, :T])
    for r in range(rows):
        for j in range(nb):
            sl = slice(j * T, (j + 1) * T)
            # every block's cost is its weighted error against its target
            assert cost[r * nb + j] == pytest.approx(float(np.sum(d[sl] * (xt[r, sl] - q[r, sl]) ** 2)), rel=1e-10)


def test_rejects_bad_shapes():
    cb = np.zeros(16)
    with pytest.raises(ValueError):
        oracle_ldlq(np.zeros((2, 10)), np.eye(10), np.ones(10), cb, 4, 2, 4)  # cols % T != 0


def test_feedback_targets_match_the_driver():
    """The standalone feedback step, fed the driver's own reconstruction,
    reproduces the driver's targets for every block."""
    from oracle import oracle_feedback_targets

    rng = np.random.default_rng(53)
    L, k, T, rows, cols = 5, 1, 6, 3, 36
    w = rng.standard_normal((rows, cols))
    d = rng.lognormal(0.0, 0.5, cols)
    cb = rng.standard_normal(1 << L)
    U = np.triu(rng.standard_normal((cols, cols)) * 0.2, 1) + np.eye(cols)
    q, xt, _, _, _ = oracle_ldlq(w, U, d, cb, L, k, T)
    assert np.array_equal(oracle_feedback_targets(w, U, q, T), xt)
