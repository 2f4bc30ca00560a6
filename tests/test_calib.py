"""Host logic of the offline table learner (CPU)."""
import itertools

import numpy as np
import pytest

import oracle
import workloads as W
from entropy_coded_kv_b200.calib import learn_tables, package_merge


def brute_force_cost(w, lmax):
    best = None
    for ls in itertools.product(range(1, lmax + 1), repeat=len(w)):
        if sum(2.0 ** -l for l in ls) <= 1.0:
            c = sum(a * b for a, b in zip(w, ls))
            best = c if best is None or c < best else best
    return best


@pytest.mark.parametrize("n,lmax", [(2, 1), (3, 2), (4, 2), (5, 3), (6, 3), (7, 3), (5, 4), (7, 5)])
def test_package_merge_is_optimal_under_the_length_limit(n, lmax):
    rng = np.random.default_rng(n * 10 + lmax)
    for _ in range(6):
        w = list(rng.integers(1, 60, n))
        lens = package_merge(w, lmax)
        assert lens.max() <= lmax and lens.min() >= 1
        assert sum(2.0 ** -int(l) for l in lens) == 1.0
        assert sum(a * int(b) for a, b in zip(w, lens)) == brute_force_cost(w, lmax)


def test_package_merge_equals_huffman_cost_when_limit_does_not_bind():
    import heapq
    rng = np.random.default_rng(3)
    for _ in range(20):
        w = list(rng.integers(1, 1000, 16))
        h = [(x, i) for i, x in enumerate(w)]
        heapq.heapify(h)
        cost, k = 0, 16
        while len(h) > 1:
            a, b = heapq.heappop(h), heapq.heappop(h)
            cost += a[0] + b[0]
            heapq.heappush(h, (a[0] + b[0], k)); k += 1
        lens = package_merge(w, 15)
        assert sum(a * int(b) for a, b in zip(w, lens)) == cost


def test_package_merge_skewed_hits_the_8_bit_limit():
    w = [2 ** 20 >> i for i in range(16)]  # geometric: unrestricted Huffman needs 15 bits
    lens = package_merge(w, 8)
    assert lens.max() == 8 and sum(2.0 ** -int(l) for l in lens) == 1.0


@pytest.mark.parametrize("kind", ["c1", "kv", "weight"])
def test_learned_tables_are_valid(kind):
    if kind == "c1":
        x = W.c1_matrix()
    elif kind == "kv":
        x = W.c2_calibration(shape=(1, 2, 512, 128))[0]
    else:
        x = W.c3_weight(rows=256, cols=1024)
    blob = learn_tables(x, seed=1, max_groups=2048)
    assert oracle.tables_check(blob) == 0
    _, _, st, C, lens = W.unpack_tables(blob)
    assert np.all(np.diff(C, axis=1) > 0) and lens.max() <= 8
