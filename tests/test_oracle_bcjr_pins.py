"""Pins for the oracle's soft (forward-backward) trellis quantizer.

* exhaustive enumeration: the Boltzmann average over every path, summed
  directly (``bruteforce.py``, no recursion), for tiny trellises and three
  temperatures;
* the limits the BCJR-QAT abstract names: as tau -> 0 the soft code returns to
  the hard Viterbi code and F -> J_min; at any tau, J_min - tau log N <= F <= J_min
  (N paths); as tau -> infinity every state is equally likely at every step, so
  y_t is the codebook mean;
* no trellis memory (L = k): the path distribution factorises and y_t is a
  per-weight softmax average, log Z a sum of per-weight log-sum-exps;
* the derivative identity dF/dx_t = 2 d_t (x_t - y_t), checked by central
  differences of F alone, so the marginals are pinned to the partition function;
* scaling (d, tau) -> (a d, a tau) leaves y unchanged and scales F by a.
"""
import numpy as np
import pytest

from oracle import oracle_bcjr, oracle_encode
from tests.bruteforce import boltzmann_brute_force, path_table

BF = [(2, 1, 5), (3, 1, 6), (4, 2, 4), (5, 2, 3), (6, 2, 4), (6, 3, 3), (4, 1, 8)]


@pytest.mark.parametrize("L,k,T", BF)
@pytest.mark.parametrize("tau", [0.05, 0.5, 5.0])
@pytest.mark.parametrize("weighted", [False, True])
def test_bcjr_matches_path_enumeration(L, k, T, tau, weighted):
    rng = np.random.default_rng(100 * L + 10 * k + T + (3 if weighted else 0))
    x = rng.standard_normal(T)
    d = rng.lognormal(0.0, 0.7, T) if weighted else None
    cb = rng.standard_normal(1 << L)
    y_bf, F_bf = boltzmann_brute_force(x, d, cb, L, k, tau)
    y, F = oracle_bcjr(x, d, cb, L, k, tau)
    np.testing.assert_allclose(y[0], y_bf, rtol=1e-10, atol=1e-12)
    assert F[0] == pytest.approx(F_bf, rel=1e-11, abs=1e-12)


@pytest.mark.parametrize("L,k,T", [(4, 2, 4), (6, 2, 4), (5, 1, 8)])
def test_zero_temperature_limit_is_viterbi(L, k, T):
    rng = np.random.default_rng(7 + L + T)
    x = rng.standard_normal(T)
    d = rng.lognormal(0.0, 0.5, T)
    cb = rng.standard_normal(1 << L)
    st, J = path_table(x, d, cb, L, k)
    order = np.argsort(J)
    gap = J[order[1]] - J[order[0]]
    assert gap > 1e-6
    start, bits, Jv = oracle_encode(x, d, cb, L, k)
    assert Jv[0] == pytest.approx(J[order[0]], rel=1e-12)
    n_paths = len(J)
    tau = gap / (np.log(n_paths) + 40.0)
    y, F = oracle_bcjr(x, d, cb, L, k, tau)
    # all but a 1e-17 share of the mass sits on the Viterbi path
    np.testing.assert_allclose(y[0], cb[st[order[0]]], atol=1e-12)
    assert Jv[0] - tau * np.log(n_paths) <= F[0] <= Jv[0] + 1e-12


@pytest.mark.parametrize("tau", [1e-3, 0.1, 1.0, 30.0])
def test_free_energy_bounds(tau):
    rng = np.random.default_rng(11)
    L, k, T = 8, 2, 40
    x = rng.standard_normal((3, T))
    d = rng.lognormal(0.0, 1.0, (3, T))
    cb = rng.standard_normal(1 << L)
    _, _, Jv = oracle_encode(x, d, cb, L, k)
    _, F = oracle_bcjr(x, d, cb, L, k, tau)
    log_n = (L + k * (T - 1)) * np.log(2.0)
    assert np.all(F <= Jv + 1e-9 * Jv)
    assert np.all(F >= Jv - tau * log_n - 1e-9 * Jv)


def test_infinite_temperature_is_codebook_mean():
    rng = np.random.default_rng(12)
    L, k, T = 6, 2, 20
    x = rng.standard_normal(T)
    cb = rng.standard_normal(1 << L)
    y, _ = oracle_bcjr(x, None, cb, L, k, 1e9)
    np.testing.assert_allclose(y[0], np.full(T, cb.mean()), atol=1e-7)


@pytest.mark.parametrize("L", [1, 3, 5])
def test_no_memory_is_per_weight_softmax(L):
    rng = np.random.default_rng(13 + L)
    T, tau = 12, 0.3
    x = rng.standard_normal(T)
    d = rng.lognormal(0.0, 0.5, T)
    cb = rng.standard_normal(1 << L)
    y, F = oracle_bcjr(x, d, cb, L, L, tau)
    a = -d[:, None] * (x[:, None] - cb[None, :]) ** 2 / tau  # [T, 2^L]
    m = a.max(axis=1, keepdims=True)
    p = np.exp(a - m)
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(y[0], p @ cb, rtol=1e-12, atol=1e-14)
    logz = (m[:, 0] + np.log(np.exp(a - m).sum(axis=1))).sum()
    assert F[0] == pytest.approx(-tau * logz, rel=1e-12)


def test_marginals_are_the_gradient_of_the_free_energy():
    rng = np.random.default_rng(14)
    L, k, T, tau = 6, 2, 10, 0.4
    x = rng.standard_normal(T)
    d = rng.lognormal(0.0, 0.5, T)
    cb = rng.standard_normal(1 << L)
    y, _ = oracle_bcjr(x, d, cb, L, k, tau)
    h = 1e-5
    for t in range(T):
        xp, xm = x.copy(), x.copy()
        xp[t] += h
        xm[t] -= h
        dF = (oracle_bcjr(xp, d, cb, L, k, tau)[1][0] - oracle_bcjr(xm, d, cb, L, k, tau)[1][0]) / (2 * h)
        assert dF == pytest.approx(2 * d[t] * (x[t] - y[0, t]), rel=1e-6, abs=1e-9)


def test_scaling_weight_and_temperature():
    rng = np.random.default_rng(15)
    L, k, T = 6, 2, 16
    x = rng.standard_normal((2, T))
    d = rng.lognormal(0.0, 0.5, (2, T))
    cb = rng.standard_normal(1 << L)
    y1, F1 = oracle_bcjr(x, d, cb, L, k, 0.2)
    y2, F2 = oracle_bcjr(x, 4.0 * d, cb, L, k, 0.8)
    np.testing.assert_allclose(y2, y1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(F2, 4.0 * F1, rtol=1e-12)


def test_soft_code_within_codebook_range_and_rejections():
    rng = np.random.default_rng(16)
    cb = rng.standard_normal(256)
    y, _ = oracle_bcjr(rng.standard_normal((4, 30)) * 3, None, cb, 8, 2, 0.7)
    assert np.all(y >= cb.min() - 1e-12) and np.all(y <= cb.max() + 1e-12)
    for bad_tau in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(ValueError):
            oracle_bcjr(np.zeros(4), None, cb, 8, 2, bad_tau)


def test_zero_weights_are_uniform_over_paths():
    """d = 0: every path has J = 0, so P is uniform over the 2^(L + k(T-1))
    paths, every state equally likely at every step (y_t = mean c) and
    F = -tau (L + k (T - 1)) ln 2."""
    rng = np.random.default_rng(17)
    L, k, T, tau = 6, 2, 9, 0.7
    cb = rng.standard_normal(1 << L)
    y, F = oracle_bcjr(rng.standard_normal(T), np.zeros(T), cb, L, k, tau)
    np.testing.assert_allclose(y[0], np.full(T, cb.mean()), rtol=1e-12, atol=1e-14)
    assert F[0] == pytest.approx(-tau * (L + k * (T - 1)) * np.log(2.0), rel=1e-12)
