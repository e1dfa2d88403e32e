"""Pins of the oracle's 8-state set-partitioned trellis (oracle_ub8_encode,
oracle_ub8_decode) against what the pages and the mathematics fix.

The 2-bit post (Pingala-8 section) names Ungerboeck's 8-state set-partitioned
trellis over symbols of several weights at about 2 bits per weight, and its
section on trellis-coded quantization says what a state does: it selects the
subset the next symbol may use, the bits pick a value inside that subset and
set the next state, and the format holds twice as many values as its bits
address.  The reading (Marcellin and Fischer's TCQ on Ungerboeck's 8-state
one-dimensional code, parity-check polynomials 13 and 04 octal) is pinned
here by an enumeration that uses the code's parity-check equation alone, not
the oracle's state machine, and by closed forms.
"""
import itertools

import numpy as np
import pytest

from oracle import oracle_ub8_decode, oracle_ub8_encode
from tests.bruteforce import (ub8_brute_force, ub8_decode_parity, ub8_first_parities,
                              ub8_parities)


def _case(V, m, S, weighted, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((1, S * V))
    d = rng.lognormal(0.0, 1.0, (1, S * V)) if weighted else None
    cb = rng.standard_normal((4 << m) * V)
    return x, d, cb


def _path_cost(x, d, y):
    d = np.ones_like(x) if d is None else d
    return float((d * (x - y) ** 2).sum())


# --------------------------------------------------------------------------
# exhaustive enumeration through the parity-check equation
# --------------------------------------------------------------------------
CASES = [(V, m, S, w) for V in (1, 2) for m in (0, 1, 2) for S in (1, 2, 3, 4, 5) for w in (False, True)
         if 3 + S * (1 + m) <= 14]


@pytest.mark.parametrize("V,m,S,weighted", CASES)
def test_encode_equals_enumeration_of_code_sequences(V, m, S, weighted):
    x, d, cb = _case(V, m, S, weighted, seed=100 * V + 10 * m + S + (7 if weighted else 0))
    J_bf, _ = ub8_brute_force(x[0], None if d is None else d[0], cb, V, m)
    start, bits, J = oracle_ub8_encode(x, d, cb, V, m)
    assert J[0] == pytest.approx(J_bf, rel=1e-12, abs=1e-12)
    assert 0 <= start[0] < 8
    # the returned path, decoded through the parity equation, reaches J
    y = ub8_decode_parity(bits[0], start[0], cb, V, m, S * V)
    assert _path_cost(x[0], None if d is None else d[0], y) == pytest.approx(J[0], rel=1e-12, abs=1e-12)


@pytest.mark.parametrize("start", range(8))
@pytest.mark.parametrize("V,m,S", [(1, 1, 4), (2, 0, 5), (1, 2, 3)])
def test_fixed_start_equals_enumeration(start, V, m, S):
    x, d, cb = _case(V, m, S, True, seed=900 + start + 10 * S)
    J_bf, _ = ub8_brute_force(x[0], d[0], cb, V, m, fixed_start=start)
    s, bits, J = oracle_ub8_encode(x, d, cb, V, m, fixed_start=start)
    assert J[0] == pytest.approx(J_bf, rel=1e-12, abs=1e-12)
    assert s[0] == start
    y = ub8_decode_parity(bits[0], s[0], cb, V, m, S * V)
    assert _path_cost(x[0], d[0], y) == pytest.approx(J[0], rel=1e-12, abs=1e-12)


def test_free_start_is_the_best_fixed_start():
    x, d, cb = _case(2, 2, 6, True, seed=77)
    _, _, J = oracle_ub8_encode(x, d, cb, 2, 2)
    fixed = [oracle_ub8_encode(x, d, cb, 2, 2, fixed_start=s)[2][0] for s in range(8)]
    assert J[0] == pytest.approx(min(fixed), rel=1e-14)


# --------------------------------------------------------------------------
# decoder: the state machine against the parity equation
# --------------------------------------------------------------------------
@pytest.mark.parametrize("V,m,S", [(1, 0, 9), (1, 3, 17), (4, 7, 64), (2, 5, 33), (3, 2, 11)])
def test_decode_matches_parity_equation_on_random_streams(V, m, S):
    rng = np.random.default_rng(V * 1000 + m * 10 + S)
    n = 12
    K = 1 + m
    W = (S * K + 31) // 32
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    used = S * K - 32 * (W - 1)
    if used < 32:
        bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)  # high bits ignored
    cb = rng.standard_normal((4 << m) * V)
    y = oracle_ub8_decode(bits, start, cb, V, m, S * V)
    for b in range(n):
        np.testing.assert_array_equal(y[b], ub8_decode_parity(bits[b], start[b], cb, V, m, S * V))
    y7 = oracle_ub8_decode(bits, start & np.uint32(7), cb, V, m, S * V)
    np.testing.assert_array_equal(y, y7)


def test_round_trip_reproduces_cost():
    rng = np.random.default_rng(5)
    V, m, S = 4, 7, 64
    x = rng.standard_normal((6, S * V))
    d = rng.lognormal(0.0, 1.0, (6, S * V))
    cb = rng.standard_normal((4 << m) * V)
    start, bits, J = oracle_ub8_encode(x, d, cb, V, m)
    y = oracle_ub8_decode(bits, start, cb, V, m, S * V)
    np.testing.assert_allclose((d * (x - y) ** 2).sum(axis=1), J, rtol=1e-12)
    assert np.all(J >= 0)


# --------------------------------------------------------------------------
# the trellis structure the pages state
# --------------------------------------------------------------------------
def _branches():
    """(state, branch bit) -> (subset, next state), read off the parity equation:
    a path from state s with first branch bit z uses subset 2 z + z0_1 and, one
    step later, is in the state whose first parities continue the sequence."""
    out = {}
    for s in range(8):
        for z in (0, 1):
            z0 = ub8_first_parities(s, z)
            sub = 2 * z + z0[0]
            # the next state s2 is the one whose first parities, for every next
            # branch bit, continue (z0_2, z0_3, z0_4) of this path
            nxt = [s2 for s2 in range(8)
                   if all(ub8_first_parities(s2, z2) ==
                          tuple(ub8_parities([z, z2, 0, 0], z0)[1:4]) for z2 in (0, 1))]
            assert len(nxt) == 1
            out[(s, z)] = (sub, nxt[0])
    return out


def test_each_state_offers_the_two_subsets_of_one_half():
    br = _branches()
    for s in range(8):
        subs = {br[(s, z)][0] for z in (0, 1)}
        assert subs in ({0, 2}, {1, 3})          # one half of the partition
        assert br[(s, 0)][1] != br[(s, 1)][1]    # the bits set the next state
    incoming = {s2: [(s, z) for (s, z), (_, n2) in br.items() if n2 == s2] for s2 in range(8)}
    for s2, ins in incoming.items():
        assert len(ins) == 2
        assert len({br[i][0] % 2 for i in ins}) == 1  # both from the same half
        assert {br[i][0] for i in ins} in ({0, 2}, {1, 3})


def test_union_holds_twice_the_values_the_bits_address():
    for V, m in [(1, 1), (4, 7), (2, 3)]:
        x, _, cb = _case(V, m, 2, False, seed=3)
        bits_per_step = 1 + m
        assert cb.size // V == 2 * (1 << bits_per_step)
        # and the oracle accepts exactly that size
        oracle_ub8_encode(x, None, cb, V, m)
        with pytest.raises(ValueError):
            oracle_ub8_encode(x, None, cb[:-V], V, m)


# --------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------
def test_identical_subsets_remove_the_memory():
    """With D_0 = D_1 = D_2 = D_3 every symbol may take any value: J is the sum of
    per-step nearest codewords (plain vector rounding)."""
    rng = np.random.default_rng(11)
    V, m, S = 2, 3, 40
    base = rng.standard_normal(((1 << m), V))
    cb = np.repeat(base, 4, axis=0).reshape(-1)  # row 4 i + j = base[i]
    x = rng.standard_normal((3, S * V))
    d = rng.lognormal(0.0, 1.0, (3, S * V))
    _, _, J = oracle_ub8_encode(x, d, cb, V, m)
    xs, ds = x.reshape(3, S, 1, V), d.reshape(3, S, 1, V)
    per = (ds * (xs - base[None, None]) ** 2).sum(axis=-1).min(axis=-1)
    np.testing.assert_allclose(J, per.sum(axis=1), rtol=1e-12)


def test_single_step_is_nearest_in_the_union():
    rng = np.random.default_rng(12)
    V, m = 3, 4
    cb = rng.standard_normal((4 << m) * V)
    x = rng.standard_normal((20, V))
    _, _, J = oracle_ub8_encode(x, None, cb, V, m)
    rows = cb.reshape(-1, V)
    np.testing.assert_allclose(J, ((x[:, None, :] - rows[None]) ** 2).sum(-1).min(-1), rtol=1e-12)


def test_memoryless_lower_bound_and_weight_scaling():
    rng = np.random.default_rng(13)
    V, m, S = 1, 2, 200
    cb = np.sort(rng.standard_normal(4 << m))
    x = rng.standard_normal((4, S))
    d = rng.lognormal(0.0, 1.0, (4, S))
    s1, b1, J = oracle_ub8_encode(x, d, cb, V, m)
    lower = (d[:, :, None] * (x[:, :, None] - cb[None, None]) ** 2).min(-1).sum(-1)
    assert np.all(J >= lower - 1e-12)
    s4, b4, J4 = oracle_ub8_encode(x, 4.0 * d, cb, V, m)
    np.testing.assert_array_equal(s1, s4)
    np.testing.assert_array_equal(b1, b4)
    np.testing.assert_allclose(J4, 4.0 * J, rtol=1e-14)


def test_values_on_a_path_cost_nothing():
    rng = np.random.default_rng(14)
    V, m, S = 2, 3, 30
    cb = rng.standard_normal((4 << m) * V)
    K = 1 + m
    W = (S * K + 31) // 32
    bits = rng.integers(0, 2**32, size=(1, W), dtype=np.uint64).astype(np.uint32)
    used = S * K - 32 * (W - 1)
    if used < 32:
        bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
    y = oracle_ub8_decode(bits, np.array([5], dtype=np.uint32), cb, V, m, S * V)
    _, _, J = oracle_ub8_encode(y, None, cb, V, m)
    assert J[0] == 0.0


def test_scalar_tcq_gain_on_uniform_data():
    """Marcellin and Fischer's setting: R bits per sample from a doubled uniform
    alphabet of 2^(R+1) levels, against plain R-bit rounding to the 2^R-level
    alphabet on uniform data.  The searched trellis code must gain, more as the
    rate grows (the alphabet's ends matter less), and never reach 10 log10(pi e
    / 6) = 1.53 dB, the granular gain no quantizer can exceed.  A trellis with
    a broken branch rule (wrong next state or subset) gains far less."""
    rng = np.random.default_rng(15)
    n = 20000
    x = rng.uniform(-1, 1, (1, n))
    gains = []
    for R in (2, 3, 4, 5):
        lv2 = (np.arange(2 ** (R + 1)) + 0.5) / 2 ** (R + 1) * 2 - 1
        lv1 = (np.arange(2 ** R) + 0.5) / 2 ** R * 2 - 1
        _, _, J = oracle_ub8_encode(x, None, lv2, 1, R - 1)
        plain = ((x[0][:, None] - lv1[None]) ** 2).min(-1).sum()
        gains.append(10 * np.log10(plain / J[0]))
    assert all(a < b for a, b in zip(gains, gains[1:])), gains
    assert 0.9 < gains[-1] < 10 * np.log10(np.pi * np.e / 6), gains


def test_enumeration_helper_self_check():
    """The parity recursion generates 8 * 2^S distinct label sequences from the
    8 start states (the realisation is one-to-one), as a rate-1/2 code with
    three memory bits must."""
    S = 6
    seqs = set()
    for s in range(8):
        for z1 in itertools.product((0, 1), repeat=S):
            z0 = ub8_parities(list(z1), ub8_first_parities(s, z1[0]))
            seqs.add(tuple(zip(z1, z0)))
    assert len(seqs) == 8 * 2 ** S
