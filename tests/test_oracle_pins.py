"""Pins for the fp64 CPU oracle, against facts that do not come from the oracle.

* exhaustive enumeration on tiny trellises (``bruteforce.py``, independent code);
* the 1-bit two-coset toy of the Pingala-8 post (values the page prints, and
  costs worked by hand from the page's own numbers);
* closed forms: no trellis memory (L = k) is per-weight nearest-codeword
  rounding; T = 1 is nearest codeword over the whole table; a codebook that
  depends only on the last symbol removes the memory; scaling d scales J;
  x on a trellis path costs 0;
* invariants: optimum <= greedy, free start = min over fixed starts, the
  decode-of-encode round trip reproduces J, decode ignores the start's bits
  above L - k, costs are non-negative.
"""
import json
import os

import numpy as np
import pytest

from oracle import (
    oracle_decode,
    oracle_encode,
    oracle_greedy,
    oracle_path_cost,
    oracle_words_per_block,
)
from tests.bruteforce import brute_force, decode_window, unpack_symbols

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# exhaustive enumeration
# --------------------------------------------------------------------------
BF_CASES = [
    (L, k, T)
    for L in range(1, 7)
    for k in (1, 2, 3)
    if k <= L
    for T in {1: (1, 2, 3, 5, 8), 2: (1, 2, 4, 6), 3: (1, 3, 4)}[k]
]


@pytest.mark.parametrize("L,k,T", BF_CASES)
@pytest.mark.parametrize("weighted", [False, True])
def test_oracle_matches_bruteforce(L, k, T, weighted):
    rng = _rng(1000 * L + 100 * k + T + (7 if weighted else 0))
    for _ in range(2):
        x = rng.standard_normal(T)
        d = rng.lognormal(0.0, 1.0, T) if weighted else None
        cb = rng.standard_normal(1 << L)
        J_bf, _, _ = brute_force(x, d, cb, L, k)
        start, bits, cost = oracle_encode(x, d, cb, L, k)
        assert abs(cost[0] - J_bf) <= 1e-12 * max(1.0, J_bf)
        # the returned path, decoded by the independent window reading, reaches J_min
        y = decode_window(bits[0], int(start[0]), cb, L, k, T)
        dd = np.ones(T) if d is None else d
        assert abs(float(np.sum(dd * (x - y) ** 2)) - J_bf) <= 1e-12 * max(1.0, J_bf)
        assert int(start[0]) < (1 << (L - k)), "stored start is canonical (s_1 >> k)"
        # fixed start: the oracle matches enumeration over bitstreams alone
        s0 = int(rng.integers(0, 1 << L))
        J_bf_fixed, _, _ = brute_force(x, d, cb, L, k, fixed_start=s0)
        _, _, cost_fixed = oracle_encode(x, d, cb, L, k, fixed_start=s0)
        assert abs(cost_fixed[0] - J_bf_fixed) <= 1e-12 * max(1.0, J_bf_fixed)


@pytest.mark.parametrize("L,k,T", [(3, 1, 6), (4, 2, 5), (5, 3, 4), (6, 2, 4)])
def test_oracle_decode_matches_window_reading(L, k, T):
    rng = _rng(L * 31 + k * 7 + T)
    n = 20
    W = oracle_words_per_block(k, T)
    assert W == (T * k + 31) // 32
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    # unused bits of the last word are zero in a well-formed stream
    used = T * k - 32 * (W - 1)
    bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used)) if used < 32 else np.uint32(0xFFFFFFFF)
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)  # non-canonical
    cb = rng.standard_normal(1 << L)
    y = oracle_decode(bits, start, cb, L, k, T)
    for i in range(n):
        np.testing.assert_array_equal(y[i], decode_window(bits[i], int(start[i]), cb, L, k, T))


# --------------------------------------------------------------------------
# the page's worked toy
# --------------------------------------------------------------------------
def _toy():
    with open(os.path.join(GOLDEN, "page_toy_trellis.json")) as f:
        return json.load(f)


def test_page_toy_fixed_start():
    g = _toy()
    L, k, x, cb = g["L"], g["k"], np.array(g["x"]), np.array(g["codebook"])
    # plain rounding to {-1, 1}: the page prints 1.42
    levels = np.array(g["plain_rounding_levels"])
    plain = float(np.sum(np.min((x[:, None] - levels[None, :]) ** 2, axis=1)))
    assert plain == pytest.approx(g["printed_plain_rounding_cost"], abs=1e-12)

    start, bits, cost = oracle_encode(x, None, cb, L, k, fixed_start=g["start_state"])
    _, greedy = oracle_greedy(x, None, cb, L, k, [g["start_state"]])
    # the page: greedy loses to plain rounding, the searched path beats it
    assert greedy[0] > plain > cost[0]
    # by hand from the page's numbers: bits 0,1,1 give -1.5, 0.5, 1.5, errors
    # 1.1^2 + 0.4^2 + 0^2 = 1.37; greedy takes 0.5, -0.5, 0.5: 0.81 + 0.36 + 1.0 = 2.17
    assert cost[0] == pytest.approx(1.1**2 + 0.4**2, abs=1e-12)
    assert greedy[0] == pytest.approx(0.9**2 + 0.6**2 + 1.0**2, abs=1e-12)
    assert list(unpack_symbols(bits[0], k, 3)) == [0, 1, 1]
    y = oracle_decode(bits, np.array([g["start_state"]]), cb, L, k, 3)
    np.testing.assert_array_equal(y[0], [-1.5, 0.5, 1.5])


def test_page_toy_free_start():
    g = _toy()
    L, k, x, cb = g["L"], g["k"], np.array(g["x"]), np.array(g["codebook"])
    start, bits, cost = oracle_encode(x, None, cb, L, k)
    # a stored start state of 1 opens the coset {-0.5, 1.5}: -0.5, 0.5, 1.5,
    # errors 0.1^2 + 0.4^2 + 0 = 0.17
    assert int(start[0]) == 1
    assert cost[0] == pytest.approx(0.1**2 + 0.4**2, abs=1e-12)
    assert list(unpack_symbols(bits[0], k, 3)) == [0, 1, 1]


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
@pytest.mark.parametrize("L", [1, 2, 3, 4])
def test_no_memory_is_nearest_codeword_rounding(L):
    rng = _rng(40 + L)
    T, n = 37, 6
    x = rng.standard_normal((n, T))
    d = rng.lognormal(0.0, 1.0, (n, T))
    cb = rng.standard_normal(1 << L)
    _, bits, cost = oracle_encode(x, d, cb, L, L)
    expect = np.sum(d * np.min((x[..., None] - cb[None, None, :]) ** 2, axis=-1), axis=1)
    np.testing.assert_allclose(cost, expect, rtol=1e-12, atol=0)
    for i in range(n):
        sym = unpack_symbols(bits[i], L, T)
        np.testing.assert_array_equal(sym, np.argmin((x[i, :, None] - cb[None, :]) ** 2, axis=1))


@pytest.mark.parametrize("L,k", [(4, 1), (6, 2), (8, 2), (9, 3), (12, 2)])
def test_single_step_is_global_nearest(L, k):
    rng = _rng(L * 3 + k)
    x = rng.standard_normal((9, 1))
    d = rng.lognormal(0.0, 1.0, (9, 1))
    cb = rng.standard_normal(1 << L)
    start, bits, cost = oracle_encode(x, d, cb, L, k)
    sq = d * (x - cb[None, :]) ** 2
    np.testing.assert_allclose(cost, sq.min(axis=1), rtol=1e-12)
    s1 = np.argmin(sq, axis=1)
    np.testing.assert_array_equal(start, s1 >> k)
    np.testing.assert_array_equal(bits[:, 0] >> np.uint32(32 - k), s1 & ((1 << k) - 1))


@pytest.mark.parametrize("L,k", [(5, 1), (6, 2), (8, 3)])
def test_codebook_of_last_symbol_only_removes_memory(L, k):
    rng = _rng(70 + L)
    T = 25
    v = rng.standard_normal(1 << k)
    cb = v[np.arange(1 << L) & ((1 << k) - 1)]
    x = rng.standard_normal((4, T))
    d = rng.lognormal(0.0, 1.0, (4, T))
    _, _, cost = oracle_encode(x, d, cb, L, k)
    expect = np.sum(d * np.min((x[..., None] - v) ** 2, axis=-1), axis=1)
    np.testing.assert_allclose(cost, expect, rtol=1e-12)


def test_scaling_d_scales_cost():
    rng = _rng(5)
    L, k, T = 6, 2, 40
    x = rng.standard_normal((5, T))
    d = rng.lognormal(0.0, 1.0, (5, T))
    cb = rng.standard_normal(1 << L)
    s1, b1, c1 = oracle_encode(x, d, cb, L, k)
    s2, b2, c2 = oracle_encode(x, 4.0 * d, cb, L, k)  # power of two: exact scaling
    np.testing.assert_array_equal(c2, 4.0 * c1)
    np.testing.assert_array_equal(b1, b2)
    np.testing.assert_array_equal(s1, s2)


@pytest.mark.parametrize("L,k", [(4, 1), (6, 2), (9, 3), (10, 2)])
def test_input_on_a_trellis_path_costs_zero(L, k):
    rng = _rng(90 + L + k)
    T = 31
    cb = rng.standard_normal(1 << L)
    s = int(rng.integers(0, 1 << L))
    x = np.empty(T)
    for t in range(T):
        s = ((s << k) | int(rng.integers(0, 1 << k))) & ((1 << L) - 1)
        x[t] = cb[s]
    start, bits, cost = oracle_encode(x, None, cb, L, k)
    assert cost[0] == 0.0
    np.testing.assert_array_equal(oracle_decode(bits, start, cb, L, k, T)[0], x)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------
@pytest.mark.parametrize("L,k,T", [(4, 1, 30), (6, 2, 50), (8, 2, 64), (7, 3, 33), (10, 2, 20)])
def test_invariants(L, k, T):
    rng = _rng(L * 100 + k * 10 + T)
    n = 8
    x = rng.standard_normal((n, T))
    d = rng.lognormal(0.0, 1.0, (n, T))
    cb = rng.standard_normal(1 << L)
    start, bits, cost = oracle_encode(x, d, cb, L, k)
    assert np.all(cost >= 0)
    # round trip: decode(encode(x)) reproduces the reported cost
    y = oracle_decode(bits, start, cb, L, k, T)
    np.testing.assert_allclose(oracle_path_cost(x, d, y), cost, rtol=1e-12)
    # decode reads only the low L-k bits of the start state
    noisy = start | (rng.integers(0, 1 << (32 - (L - k)), size=n, dtype=np.uint64).astype(np.uint32)
                     << np.uint32(L - k))
    np.testing.assert_array_equal(oracle_decode(bits, noisy, cb, L, k, T), y)
    # optimum never loses to greedy, from any start
    for s0 in (0, int(start[0]), (1 << L) - 1):
        _, greedy = oracle_greedy(x, d, cb, L, k, [s0] * n)
        assert np.all(cost <= greedy + 1e-12)
    # a free start is the best of all fixed starts
    best_fixed = np.full(n, np.inf)
    for s0 in range(1 << (L - k)):
        _, _, cf = oracle_encode(x, d, cb, L, k, fixed_start=s0)
        assert np.all(cost <= cf + 1e-12)
        best_fixed = np.minimum(best_fixed, cf)
    np.testing.assert_allclose(cost, best_fixed, rtol=1e-12)


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle_encode(np.zeros((1, 4)), None, np.zeros(8), 3, 4)  # k > L
    with pytest.raises(ValueError):
        oracle_encode(np.zeros((1, 4)), None, np.zeros(7), 3, 1)  # codebook size


# --------------------------------------------------------------------------
# decode-in-matvec: the oracle GEMV is decode followed by a dense product
# --------------------------------------------------------------------------
@pytest.mark.parametrize("L,k,T,rows,nb", [(4, 2, 8, 5, 3), (6, 3, 4, 3, 4), (8, 2, 16, 4, 2)])
@pytest.mark.parametrize("scaled", [False, True])
def test_oracle_gemv_is_decode_then_dense_product(L, k, T, rows, nb, scaled):
    from oracle import oracle_gemv

    rng = _rng(L * 13 + k + T)
    cols = nb * T
    W = oracle_words_per_block(k, T)
    n = rows * nb
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    used = T * k - 32 * (W - 1)
    if used < 32:
        bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    cb = rng.standard_normal(1 << L)
    scale = rng.lognormal(0.0, 0.5, n) if scaled else None
    x = rng.standard_normal(cols)
    dense = np.zeros((rows, cols))
    for r in range(rows):
        for j in range(nb):
            b = r * nb + j
            vals = decode_window(bits[b], int(start[b]), cb, L, k, T)
            dense[r, j * T:(j + 1) * T] = vals * (scale[b] if scaled else 1.0)
    y = oracle_gemv(bits, start, scale, cb, L, k, T, rows, cols, x)
    np.testing.assert_allclose(y, dense @ x, rtol=1e-12, atol=1e-12)
