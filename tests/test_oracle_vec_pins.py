"""Pins for the oracle's vector trellis (V weights per step).

* exhaustive enumeration (``bruteforce.py``, the window reading with kV-bit
  symbols, independent of the oracle) for tiny trellises, and the returned path
  decoded by that window reading reaches the minimum;
* V = 1 is the scalar trellis bit for bit;
* L = kV (no memory) is per-step nearest vector codeword;
* a codebook of repeated pairs (c, c) turns the V = 2 search into the scalar
  search with kV bits per weight on the pair means with doubled weights, plus the
  pairs' fixed spread;
* the decode of the encode reproduces the cost.
"""
import numpy as np
import pytest

from oracle import oracle_decode_vec, oracle_encode, oracle_encode_vec
from tests.bruteforce import brute_force_vec, decode_window_vec

BF = [(2, 1, 2, 4), (3, 1, 2, 6), (4, 1, 2, 8), (4, 2, 2, 4), (5, 1, 3, 6), (6, 2, 2, 6), (6, 1, 4, 8), (4, 1, 4, 8)]


@pytest.mark.parametrize("L,k,V,T", BF)
@pytest.mark.parametrize("weighted", [False, True])
def test_vec_matches_bruteforce(L, k, V, T, weighted):
    rng = np.random.default_rng(300 + 17 * L + 5 * k + V + T)
    for _ in range(2):
        x = rng.standard_normal(T)
        d = rng.lognormal(0.0, 0.8, T) if weighted else None
        cb = rng.standard_normal((1 << L, V))
        J_bf, _, _ = brute_force_vec(x, d, cb, L, k, V)
        start, bits, cost = oracle_encode_vec(x, d, cb, L, k, V)
        assert abs(cost[0] - J_bf) <= 1e-12 * max(1.0, J_bf)
        y = decode_window_vec(bits[0], int(start[0]), cb, L, k, V, T)
        dd = np.ones(T) if d is None else d
        assert abs(float(np.sum(dd * (x - y) ** 2)) - J_bf) <= 1e-12 * max(1.0, J_bf)
        assert start[0] < (1 << (L - k * V))


def test_v1_is_the_scalar_trellis():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((4, 20))
    d = rng.lognormal(0.0, 1.0, (4, 20))
    cb = rng.standard_normal(1 << 8)
    a = oracle_encode(x, d, cb, 8, 2)
    b = oracle_encode_vec(x, d, cb, 8, 2, 1)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("L,k,V", [(4, 2, 2), (6, 2, 3), (4, 1, 4)])
def test_no_memory_is_nearest_vector(L, k, V):
    rng = np.random.default_rng(41 + L)
    T = 6 * V
    x = rng.standard_normal(T)
    d = rng.lognormal(0.0, 0.5, T)
    cb = rng.standard_normal((1 << L, V))
    _, _, cost = oracle_encode_vec(x, d, cb, L, k, V)
    xs, ds = x.reshape(-1, V), d.reshape(-1, V)
    per_step = ((ds[:, None, :] * (xs[:, None, :] - cb[None, :, :]) ** 2).sum(-1)).min(axis=1)
    assert cost[0] == pytest.approx(per_step.sum(), rel=1e-12)


def test_repeated_pairs_reduce_to_the_scalar_trellis():
    rng = np.random.default_rng(51)
    L, k, T = 8, 1, 24
    x = rng.standard_normal((3, T))
    c = rng.standard_normal(1 << L)
    cbv = np.stack([c, c], axis=1)
    _, _, J_vec = oracle_encode_vec(x, None, cbv, L, k, 2)
    pairs = x.reshape(3, -1, 2)
    mean, spread = pairs.mean(-1), ((pairs[..., 0] - pairs[..., 1]) ** 2).sum(-1) / 2
    _, _, J_1 = oracle_encode(mean, np.full(mean.shape, 2.0), c, L, 2 * k)
    np.testing.assert_allclose(J_vec, J_1 + spread, rtol=1e-12)


def test_round_trip_and_rejections():
    rng = np.random.default_rng(61)
    L, k, V, T = 10, 2, 2, 40
    x = rng.standard_normal((5, T))
    d = rng.lognormal(0.0, 1.0, (5, T))
    cb = rng.standard_normal((1 << L, V))
    start, bits, cost = oracle_encode_vec(x, d, cb, L, k, V)
    y = oracle_decode_vec(bits, start, cb, L, k, V, T)
    np.testing.assert_allclose((d * (x - y) ** 2).sum(1), cost, rtol=1e-12)
    with pytest.raises(ValueError):
        oracle_encode_vec(x[:, :39], None, cb, L, k, V)     # V does not divide T
    with pytest.raises(ValueError):
        oracle_encode_vec(x, None, np.zeros((16, 3)), 4, 2, 3)  # kV > L
