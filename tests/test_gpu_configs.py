"""The five benchmark workloads at full size, through bench.py's own workload
classes (the same tensors, tables and launches the bench times), against the
CPU oracle (needs a B200).

- 256 x 1024 matrix, the one-layer KV cache [8, 8, 4096, 128] x K,V and the
  14336 x 4096 MLP weight: every encoded block and every decoded bf16 value.
- The 32-layer, 224-tensor Llama-3-8B-shaped weight set (one encode_multi and
  one decode_multi call, 64 segments per launch): every block and value of
  layers 0 and 31 (all 7 shapes), 512 sampled groups of every other tensor.
- The long-context cache, 32 layers x K,V x [1, 8, 131072, 128] (17.2 GB of
  bf16): one bench step (the one-token append of every layer and the decode of
  the whole cache, both multi-segment); every block and value of layers 0, 1,
  16 and 31, sampled groups of the others, and the appended token's blocks
  against the oracle's encoding of that token.

Blocks and bf16 values must be identical; the fused GEMV must lie within
|y - y64| <= 1e-3 * sum_k |W~ x| + 1e-30 of the oracle's fp64 product (R19).
"""
from __future__ import annotations

import gc
import os

import numpy as np
import pytest
import torch

import bench
import oracle
import workloads as W

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
NT = os.cpu_count() or 1
GEMV_RTOL = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return W.bf16_bits(t)


def check_tensor(blob, x: torch.Tensor, blocks: torch.Tensor, y: torch.Tensor, what: str):
    """Every block and every decoded value of one tensor."""
    xb = bits(x).reshape(-1, 128)
    want, _ = oracle.encode(blob, xb, nthreads=NT)
    got = blocks.view(-1, 64).cpu().numpy()
    bad = np.flatnonzero((got != want).any(1))
    assert bad.size == 0, f"{what}: {bad.size} of {len(want)} blocks differ, first {bad[:5]}"
    wy = oracle.decode(blob, want, nthreads=NT)
    gy = bits(y).reshape(-1, 128)
    bad = np.flatnonzero((gy != wy).any(1))
    assert bad.size == 0, f"{what}: {bad.size} of {len(wy)} decoded groups differ, first {bad[:5]}"


def check_sampled(blob, x: torch.Tensor, blocks: torch.Tensor, y: torch.Tensor, k: int, seed: int, what: str):
    """k sampled groups (and the first and last) of one tensor."""
    n = x.numel() // 128
    rng = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([rng.choice(n, min(k, n), replace=False), [0, n - 1]]))
    sel = torch.from_numpy(idx).to(DEV)
    want, _ = oracle.encode(blob, bits(x.reshape(-1, 128)[sel]), nthreads=NT)
    np.testing.assert_array_equal(blocks.view(-1, 64)[sel].cpu().numpy(), want, err_msg=what)
    np.testing.assert_array_equal(bits(y.reshape(-1, 128)[sel]), oracle.decode(blob, want, nthreads=NT),
                                  err_msg=what)


def release():
    """Returns the freed device memory of a finished workload to the driver."""
    gc.collect()
    torch.cuda.empty_cache()


def test_matrix_256x1024_every_block():
    wl = bench.C1Workload(DEV)
    wl.step()
    torch.cuda.synchronize()
    check_tensor(wl.tables.blob, wl.x, wl.blocks, wl.out, "256x1024")


def test_kv_cache_layer_every_block():
    """Both caches after one bench step: the 64-token append re-encodes tokens
    4032..4095 from separate tensors into the cache, then the whole cache is
    decoded; the result must be the oracle's encoding of the whole cache."""
    wl = bench.KVWorkload(DEV)
    before = [b.clone() for b in wl.blocks]
    wl.step()
    torch.cuda.synchronize()
    for i, name in enumerate("KV"):
        assert torch.equal(before[i], wl.blocks[i]), f"{name}: the append changed the cache"
        check_tensor(wl.tables[i].blob, wl.caches[i], wl.blocks[i], wl.out[i], f"KV cache {name}")
    del wl
    release()


def test_mlp_weight_every_block_and_every_gemv_row():
    wl = bench.MLPWorkload(DEV)
    wl.step()
    torch.cuda.synchronize()
    check_tensor(wl.tables.blob, wl.w, wl.blocks, wl.out, "14336x4096")
    blk = wl.blocks.cpu().numpy()
    for x, y in ((wl.x1, wl.y1), (wl.x16, wl.y16)):
        want, absum = oracle.gemv(wl.tables.blob, blk, wl.rows, wl.cols, bits(x))
        err = np.abs(y.cpu().numpy().astype(np.float64) - want)
        lim = GEMV_RTOL * absum + 1e-30
        assert (err <= lim).all(), f"batch {x.shape[0]}: max excess {(err - lim).max()}"
    del wl
    release()


def test_model_weights_224_tensors():
    wl = bench.ModelWorkload(DEV)
    wl.step()
    torch.cuda.synchronize()
    names = [n for n, _, _ in W.C4_SHAPES]
    per_layer = len(names)
    assert len(wl.w) == W.C4_LAYERS * per_layer
    for i, (x, tb, b, y) in enumerate(zip(wl.w, wl.tables, wl.blocks, wl.out)):
        layer, name = divmod(i, per_layer)
        what = f"layer {layer} {names[name]}"
        if layer in (0, W.C4_LAYERS - 1):
            check_tensor(tb.blob, x, b, y, what)
        else:
            check_sampled(tb.blob, x, b, y, 512, i, what)
    del wl
    release()


def test_long_context_cache_step():
    wl = bench.LongCtxWorkload(DEV)
    S = wl.S
    # the appended token's blocks, from the oracle's encoding of that token
    want_new = [oracle.encode(tb.blob, bits(nw).reshape(-1, 128), nthreads=NT)[0]
                for tb, nw in zip(wl.tables, wl.new)]
    wl.step()
    torch.cuda.synchronize()
    for i, (tb, c, b, y) in enumerate(zip(wl.tables, wl.caches, wl.blocks, wl.out)):
        layer, kv = divmod(i, 2)
        what = f"layer {layer} {'KV'[kv]}"
        np.testing.assert_array_equal(b.view(8, S, 64)[:, S - 1].cpu().numpy(), want_new[i], err_msg=what)
        if layer in (0, 1, 16, 31):
            check_tensor(tb.blob, c, b, y, what)
        else:
            check_sampled(tb.blob, c, b, y, 2048, i, what)
    del wl
    release()
