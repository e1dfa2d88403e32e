"""Pins for the oracle's computed (lookup-free) code.

* values worked by hand for a few states (``golden/mad_code_values.json``);
* every codeword is a multiple of 1/128 within [-255/128, 255/128], so it is
  exact in binary16 and fp32;
* over all 2^16 states the distribution is that of the sum of two near-uniform
  bytes: mean 0 and standard deviation sqrt(2 (256^2 - 1) / 12) / 128 within 1 %;
* the top byte of A s mod 2^32 is a function of every state bit: flipping any
  single bit of s changes the codeword of most states.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle_mad_codebook

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_worked_values():
    with open(os.path.join(GOLDEN, "mad_code_values.json")) as f:
        g = json.load(f)
    cb = oracle_mad_codebook(16)
    for e in g["worked_by_hand"]:
        assert cb[e["s"]] == e["c"]
        assert e["c"] == (e["byte2"] + e["byte3"] - 255) / 128


@pytest.mark.parametrize("L", [2, 8, 12, 16])
def test_exact_in_binary16(L):
    cb = oracle_mad_codebook(L)
    assert cb.shape == (1 << L,)
    q = cb * 128
    assert np.all(q == np.round(q)) and np.all(np.abs(q) <= 255)
    assert np.array_equal(cb.astype(np.float16).astype(np.float64), cb)


def test_distribution_and_mixing():
    cb = oracle_mad_codebook(16)
    assert abs(cb.mean()) < 0.01
    sd = np.sqrt(2 * (256 ** 2 - 1) / 12) / 128
    assert cb.std() == pytest.approx(sd, rel=0.01)
    s = np.arange(1 << 16)
    for bit in range(16):
        changed = np.mean(cb[s] != cb[s ^ (1 << bit)])
        assert changed > 0.9
    # a smaller L is the prefix of the same code
    np.testing.assert_array_equal(oracle_mad_codebook(10), cb[:1 << 10])
