"""Table learner on the GPU (ecco_learn_tables) (needs a B200).

A learner is a heuristic, so it is checked by what must hold rather than by
bit-equality with another learner: the blob is valid (sorted centroids,
complete codes, lengths <= 8; checked by the oracle), S_t is exactly
absmax / 448 of the sample, the same sample and seed give the same blob, a
pattern-limited blob repeats row 0, and the tables code held-out data about
as well as the host learner's (entropy_coded_kv_b200/calib.py) -- squared
error and payload bits within 10%.

Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression" (review page: patterns and codebooks learned
once, offline, per tensor; free parameters S = 64, H = 4).
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200.calib import learn_tables as host_learn
from test_gpu_parity import bits

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _quality(blob, x, group=128):
    t = ecco.Tables(blob, DEV)
    st = ecco.new_stats(DEV)
    if group == 128:
        y = ecco.decode(ecco.encode(x, t, stats=st), t)
    else:
        y = ecco.decode_act(ecco.encode_act(x, t, stats=st), t)
    xf, yf = x.float().reshape(-1), y.float().reshape(-1)
    s = ecco.read_stats(st)
    return float(((yf - xf) ** 2).sum() / (xf ** 2).sum()), s["payload_bits"] / max(1, s["n_groups"])


@pytest.mark.parametrize("what", ["kv", "weight", "act"])
def test_learned_tables_valid_deterministic_and_as_good_as_host(what):
    if what == "kv":
        calib, _ = W.c2_calibration(device=DEV)
        held, _ = W.c2_kv(device=DEV, shape=(2, 8, 4096, 128))
        group = 128
    elif what == "weight":
        calib = W.c3_weight(device=DEV, rows=4096, cols=4096, seed=30)
        held = W.c3_weight(device=DEV, rows=2048, cols=4096, seed=31)
        group = 128
    else:
        calib = W.hidden_states(4096, seed=40, device=DEV)
        held = W.hidden_states(4096, seed=41, device=DEV)
        group = 64
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    blob = ecco.learn_tables(calib, seed=3, group=group)
    t_gpu = time.perf_counter() - t0
    assert len(blob) == oracle.TABLES_BYTES and oracle.tables_check(blob) == 0
    assert blob == ecco.learn_tables(calib, seed=3, group=group)
    _, _, S_t, _, _ = W.unpack_tables(blob)
    xb = bits(calib).reshape(-1)
    finite = xb[(xb & 0x7F80) != 0x7F80]
    amax = float((((finite & 0x7FFF).max().astype(np.uint32)) << 16).view(np.float32))
    assert np.float32(S_t) == np.float32(np.float32(amax) / np.float32(448.0))
    t0 = time.perf_counter()
    ref = host_learn(calib, seed=3, group=group)
    t_host = time.perf_counter() - t0
    e_gpu, b_gpu = _quality(blob, held, group)
    e_host, b_host = _quality(ref, held, group)
    print(f"{what}: gpu learner {t_gpu * 1e3:.1f} ms, host {t_host * 1e3:.0f} ms; rel sq error {e_gpu:.4e} vs "
          f"{e_host:.4e}; payload bits {b_gpu:.1f} vs {b_host:.1f}")
    assert e_gpu <= e_host * 1.10
    assert abs(b_gpu - b_host) <= 0.10 * b_host


def test_pattern_limited_learning_and_encoding():
    calib, _ = W.c2_calibration(device=DEV, shape=(1, 8, 2048, 128))
    blob = ecco.learn_tables(calib, seed=1, n_patterns=16)
    assert oracle.tables_check(blob) == 0
    _, _, _, C, lens = W.unpack_tables(blob)
    for q in range(16, 64):
        np.testing.assert_array_equal(C[q], C[0])
        np.testing.assert_array_equal(lens[q], lens[0])
    x = calib.reshape(-1, 128)[:3000].contiguous()
    t = ecco.Tables(blob, DEV)
    got = ecco.encode(x, t, n_patterns=16).cpu().numpy()
    want, _ = oracle.encode(blob, bits(x), nthreads=8, npat=16)
    np.testing.assert_array_equal(got, want)


def test_tiny_and_degenerate_samples():
    # fewer groups than patterns, and an all-zero sample
    x = W.hidden_states(5, hidden=128, seed=2, device=DEV)
    blob = ecco.learn_tables(x, seed=0)
    assert oracle.tables_check(blob) == 0
    z = torch.zeros(40, 128, dtype=torch.bfloat16, device=DEV)
    blob = ecco.learn_tables(z, seed=0)
    assert oracle.tables_check(blob) == 0
    _, _, S_t, _, _ = W.unpack_tables(blob)
    assert S_t == 1.0
