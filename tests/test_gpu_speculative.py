"""The warp-parallel speculative decoder (ecco_decode_speculative) against the
CPU oracle, through the C ABI (needs a B200): the same bf16 bits as the
oracle's decoder on encoded, clipped, garbage and hand-made golden blocks,
ragged sizes and strided descriptors, and on the full KV cache."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200 import _lib
from test_gpu_parity import DEV, KINDS, TABLES, bits, inputs, table_set, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tname", TABLES)
@pytest.mark.parametrize("kind", KINDS)
def test_speculative_decode_bit_exact(tname, kind):
    blob = table_set(tname)
    n = 4096 + 37
    xb = inputs(kind, n, seed=(hash((tname, kind)) + 1) & 0xFFFF)
    blocks, _ = oracle.encode(blob, xb, nthreads=8)
    t = ecco.Tables(blob, DEV)
    y = ecco.decode(torch.from_numpy(blocks).to(DEV), t, speculative=True)
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(blob, blocks, nthreads=8))


@pytest.mark.parametrize("tname", ["random0", "random1", "crowded", "learned_kv"])
def test_speculative_decode_garbage_blocks(tname):
    blob = table_set(tname)
    rng = np.random.default_rng(7)
    blocks = rng.integers(0, 256, (3000, 64), dtype=np.uint8)
    blocks[::7, 0] = 0x00   # zero scale code
    blocks[1::7, 0] = 0x7F  # NaN scale code
    blocks[2::7, 0] = 0xFE
    t = ecco.Tables(blob, DEV)
    y = ecco.decode(torch.from_numpy(blocks).to(DEV), t, speculative=True)
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(blob, blocks, nthreads=8))


def test_speculative_decode_golden_blocks():
    import test_oracle_pins as P
    blob, spec = P.golden_tables()
    t = ecco.Tables(blob, DEV)
    cases = [c for c in spec["cases"] if c.get("group", 128) == 128]
    want = np.stack([P.assemble_stream(c["stream"]) for c in cases])
    y = ecco.decode(torch.from_numpy(want).to(DEV), t, speculative=True)
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), np.stack([P.expand(c["decoded"], 128) for c in cases]))


@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 1023, 148 * 32 - 1, 148 * 32 + 1, 3 * 148 * 32 + 5])
def test_speculative_decode_ragged_sizes(n):
    blob = table_set("learned_kv")
    xb = inputs("kv", n, seed=100 + n)
    blocks, _ = oracle.encode(blob, xb, nthreads=8)
    t = ecco.Tables(blob, DEV)
    y = ecco.decode(torch.from_numpy(blocks).to(DEV), t, speculative=True)
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(blob, blocks, nthreads=8))


def test_speculative_decode_strided_descriptor():
    blob = table_set("learned_kv")
    t = ecco.Tables(blob, DEV)
    rows, S = 6, 40
    xb = inputs("kv", rows * S, seed=11)
    blocks, _ = oracle.encode(blob, xb, nthreads=4)
    cache = torch.from_numpy(blocks).to(DEV)
    src = ecco.Desc(4, 20, S, 25, S + 10, 3)   # rows 1..4, tokens [10, 30), into an offset output
    out = torch.full((4 * 25 + 3, 128), -1.0, dtype=torch.bfloat16, device=DEV)
    ecco.decode(cache, t, out=out, desc=src, speculative=True)
    o = bits(out)
    for r in range(4):
        first = S + 10 + r * S
        np.testing.assert_array_equal(o[3 + r * 25: 3 + r * 25 + 20],
                                      oracle.decode(blob, blocks[first: first + 20], nthreads=2))
        assert (o[3 + r * 25 + 20: 3 + (r + 1) * 25] == 0xBF80).all()
    assert (o[:3] == 0xBF80).all()


def test_speculative_decode_argument_errors():
    t = ecco.Tables(table_set("random0"), DEV)
    lib = _lib.load()
    blk = torch.zeros((4, 64), dtype=torch.uint8, device=DEV)
    y = torch.zeros((4, 128), dtype=torch.bfloat16, device=DEV)
    d = ecco.flat_desc(4)
    P = ctypes.c_void_p
    assert lib.ecco_decode_speculative(None, P(blk.data_ptr()), d, P(y.data_ptr()), None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_decode_speculative(t.handle, None, d, P(y.data_ptr()), None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_decode_speculative(t.handle, P(blk.data_ptr() + 4), d, P(y.data_ptr()), None) == _lib.ECCO_ERR_ALIGN
    assert lib.ecco_decode_speculative(t.handle, P(blk.data_ptr()), ecco.flat_desc(0), P(y.data_ptr()), None) == 0


def test_speculative_decode_full_kv_cache():
    """The KV cache [8, 8, 4096, 128]'s K (262,144 blocks): equal to the
    thread-per-block decoder on every block, and to the oracle on a sample."""
    from entropy_coded_kv_b200.calib import learn_tables
    calib = W.c2_calibration(device="cpu")[0]
    blob = learn_tables(calib, seed=0)
    t = ecco.Tables(blob, DEV)
    k = W.c2_kv(device=DEV)[0]
    blocks = ecco.encode(k, t)
    y_serial = ecco.decode(blocks, t)
    y_spec = ecco.decode(blocks, t, speculative=True)
    assert torch.equal(y_serial.view(torch.int16), y_spec.view(torch.int16))
    idx = np.sort(np.random.default_rng(3).choice(blocks.shape[0], 4096, replace=False))
    sel = torch.from_numpy(idx).to(DEV)
    np.testing.assert_array_equal(bits(y_spec[sel]), oracle.decode(blob, blocks[sel].cpu().numpy(), nthreads=8))
