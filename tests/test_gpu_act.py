"""Activation format (64-value groups in 512-bit blocks) through the C ABI vs
the oracle: encoded blocks and decoded bf16 bit-identical (needs a B200).

Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression" (review page free parameters: group size 64
and a 2x ratio for activations; Fig. 9 text: the low-ratio compressor reuses
the high-ratio compressor's components).
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200 import _lib
from entropy_coded_kv_b200.calib import learn_tables
from test_gpu_parity import bits, inputs, table_set, to_dev_bf16, sample_rows

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
GA = 64

_ACT_TABLES = {}


def act_tables(name):
    if name not in _ACT_TABLES:
        if name == "learned_act":
            _ACT_TABLES[name] = learn_tables(W.hidden_states(512, seed=60), seed=0, group=GA)
        else:
            _ACT_TABLES[name] = table_set(name)
    return _ACT_TABLES[name]


@pytest.mark.parametrize("tname", ["random0", "random1", "random2", "random3", "learned_kv", "learned_act"])
@pytest.mark.parametrize("kind", ["gauss", "t5", "kv", "special"])
def test_act_encode_decode_bit_exact(tname, kind):
    blob = act_tables(tname)
    t = ecco.Tables(blob, DEV)
    n = 3001  # 64-value groups
    xb = inputs(kind, (n + 1) // 2, seed=7)[: n * GA]
    got = ecco.encode_act(to_dev_bf16(xb), t)
    want, _ = oracle.encode(blob, xb, nthreads=8, gs=GA)
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    y = ecco.decode_act(got, t)
    np.testing.assert_array_equal(bits(y).reshape(-1, GA), oracle.decode(blob, want, nthreads=8, gs=GA))


@pytest.mark.parametrize("n", [1, 2, 3, 31, 257, 4097, 70001])
def test_act_ragged_sizes_and_stats(n):
    blob = act_tables("learned_act")
    t = ecco.Tables(blob, DEV)
    xb = bits(W.hidden_states(n, hidden=GA, seed=n)).reshape(-1)
    st = ecco.new_stats(DEV)
    got = ecco.encode_act(to_dev_bf16(xb), t, stats=st)
    want, ost = oracle.encode(blob, xb, nthreads=8, gs=GA)
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    s = ecco.read_stats(st)
    for k in ("n_groups", "n_zero", "n_clipped", "n_padded", "n_records", "n_nonfinite", "payload_bits"):
        assert s[k] == getattr(ost, k), k


def test_act_garbage_blocks_and_strided_descriptor():
    blob = act_tables("random1")
    t = ecco.Tables(blob, DEV)
    rng = np.random.default_rng(3)
    blk = rng.integers(0, 256, (5000, 64), dtype=np.uint8)
    y = ecco.decode_act(torch.from_numpy(blk).to(DEV), t)
    np.testing.assert_array_equal(bits(y).reshape(-1, GA), oracle.decode(blob, blk, nthreads=8, gs=GA))
    # rows of 40 groups written into rows of 100 at offset 7
    rows, gpr, dst_stride, off = 30, 40, 100, 7
    xb = inputs("kv", rows * gpr // 2, seed=9)
    cache = torch.zeros(rows * dst_stride + off, 64, dtype=torch.uint8, device=DEV)
    d = _lib.Desc(rows, gpr, gpr, dst_stride, 0, off)
    ecco.encode_act(to_dev_bf16(xb), t, out=cache, desc=d)
    want, _ = oracle.encode(blob, xb, nthreads=8, gs=GA)
    c = cache.cpu().numpy()
    for r in range(rows):
        np.testing.assert_array_equal(c[off + r * dst_stride: off + r * dst_stride + gpr], want[r * gpr:(r + 1) * gpr])


def test_full_size_hidden_states_sampled():
    """[8192, 4096] activations (Llama-3-8B hidden size), 524,288 groups of 64."""
    x = W.hidden_states(8192, device=DEV)
    blob = learn_tables(W.hidden_states(2048, seed=61), seed=0, group=GA)
    t = ecco.Tables(blob, DEV)
    blocks = ecco.encode_act(x, t)
    y = ecco.decode_act(blocks, t)
    n = x.numel() // GA
    idx = torch.from_numpy(sample_rows(n, 4000, 13)).to(DEV)
    want, _ = oracle.encode(blob, bits(x.view(n, GA)[idx]), nthreads=8, gs=GA)
    np.testing.assert_array_equal(blocks[idx].cpu().numpy(), want)
    np.testing.assert_array_equal(bits(y.view(n, GA)[idx]), oracle.decode(blob, want, nthreads=8, gs=GA))
