"""The table learner's prefix codes (CPU): the library's package-merge
(ecco_huffman_lengths, host code, no device needed) gives complete prefix codes
with lengths <= 8 whose total length equals the optimum found by exhaustive
dynamic programming (oracle/huffman.py), and the same lengths as the host
learner's package-merge.

Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression" (review page: 4 Huffman codebooks per
pattern; referee comment 1: lengths limited to 8 bits).
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle.huffman import optimal_cost
import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200 import _lib
from entropy_coded_kv_b200.build import build
from entropy_coded_kv_b200.calib import package_merge


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()


def _weights(rng, kind):
    if kind == 0:
        return rng.integers(1, 1000, 16).astype(np.float64)
    if kind == 1:  # very skewed: an unlimited Huffman code would exceed 8 bits
        return np.array([2.0 ** (k + 1) for k in range(16)])
    if kind == 2:  # many ties
        return rng.integers(1, 4, 16).astype(np.float64)
    return (rng.geometric(0.3, 16) ** 3).astype(np.float64) + 1


@pytest.mark.parametrize("kind", [0, 1, 2, 3])
def test_lengths_optimal_complete_and_limited(kind):
    rng = np.random.default_rng(10 + kind)
    for _ in range(25):
        w = _weights(rng, kind)
        L = ecco.huffman_lengths(w, 8).astype(np.int64)
        assert L.min() >= 1 and L.max() <= 8
        assert sum(2.0 ** -int(l) for l in L) == 1.0
        assert float((w * L).sum()) == pytest.approx(optimal_cost(w, 8), rel=1e-12)
        np.testing.assert_array_equal(L, package_merge(w, 8))


def test_small_limits_and_alphabets():
    for n, lmax in ((2, 1), (3, 2), (4, 2), (5, 3), (16, 4)):
        w = np.arange(1, n + 1, dtype=np.float64) ** 2
        L = ecco.huffman_lengths(w, lmax).astype(np.int64)
        assert L.max() <= lmax and sum(2.0 ** -int(l) for l in L) == 1.0
        assert float((w * L).sum()) == pytest.approx(optimal_cost(w, lmax), rel=1e-12)
    assert list(ecco.huffman_lengths([5.0], 8)) == [1]


def test_argument_errors():
    lib = _lib.load()
    w = np.ones(17)
    out = np.zeros(17, dtype=np.uint8)
    P = lambda a: a.ctypes.data  # noqa: E731
    assert lib.ecco_huffman_lengths(P(w), 17, 4, P(out)) == _lib.ECCO_ERR_ARG  # 17 > 2^4
    assert lib.ecco_huffman_lengths(P(w), 0, 8, P(out)) == _lib.ECCO_ERR_ARG
    w[3] = 0.0
    assert lib.ecco_huffman_lengths(P(w), 16, 8, P(out)) == _lib.ECCO_ERR_ARG
    assert lib.ecco_learn_tables(None, 10, 128, 64, 0, None, 7952, None) == _lib.ECCO_ERR_ARG
