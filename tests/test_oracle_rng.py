"""Pins for the oracle's counter RNG (CPU only).

The mix function is pinned by the published SplitMix64 test vector; the
uniform's range and resolution by its definition (24 bits, exactly
representable in float32 and double); its quality by a Kolmogorov-Smirnov
test against U[0, 1).
"""
import os

import numpy as np
import pytest
from scipy import stats

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splitmix64_seed0.txt")
GAMMA = 0x9E3779B97F4A7C15
MASK = (1 << 64) - 1


def _vector():
    with open(GOLDEN) as f:
        return [int(line, 16) for line in f if line.strip() and not line.startswith("#")]


def test_splitmix64_known_answer():
    want = _vector()
    got = [oracle.splitmix64_mix((k * GAMMA) & MASK) for k in range(len(want))]
    assert got == want


def test_uniform_is_24_bit_and_in_range():
    for seq in range(50):
        for row in range(9):
            for purpose in (0, 1):
                u = oracle.uniform(7, seq, 3, row, purpose)
                assert 0.0 <= u <= 1.0 - 2.0 ** -24
                k = u * 2 ** 24
                assert k == int(k)
                assert float(np.float32(u)) == u


def test_uniform_is_top_24_bits_of_hash():
    for args in [(0, 0, 0, 0, 0), (1, 2, 3, 4, 1), (2**63 + 5, 17, 2**40, 31, 0)]:
        h = oracle.counter_hash(*args)
        assert oracle.uniform(*args) == (h >> 40) / 2.0 ** 24


def test_every_counter_changes_the_stream():
    base = (11, 22, 33, 4, 0)
    h0 = oracle.counter_hash(*base)
    for pos in range(5):
        args = list(base)
        args[pos] ^= 1
        assert oracle.counter_hash(*args) != h0


def test_uniforms_pass_ks():
    us = oracle.uniforms(5, range(4000), 9, 8, 0).ravel()
    assert stats.kstest(us, "uniform").pvalue > 1e-3
    # the two purposes are not the same stream
    ur = oracle.uniforms(5, range(4000), 9, 8, 1).ravel()
    assert abs(np.corrcoef(us, ur)[0, 1]) < 0.02


def test_chain_composition():
    """The counter hash is a definition of this library (the pages fix no
    RNG): five chained SplitMix64 steps over seed, seq, step, row, purpose.
    The mix itself is pinned above by the published vector."""
    mix = oracle.splitmix64_mix
    for s, q, t, r, p in [(0, 0, 0, 0, 0), (1, 2, 3, 4, 1), (2**64 - 1, 9, 2**33, 16, 0)]:
        want = mix(mix(mix(mix(mix(s) ^ q) ^ t) ^ r) ^ p)
        assert oracle.counter_hash(s, q, t, r, p) == want
