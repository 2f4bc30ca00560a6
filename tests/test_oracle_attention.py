"""Pins of the oracle's decode-phase attention over a compressed KV cache (CPU).

The oracle decodes K and V with its own (separately pinned) block decoder and
then applies softmax attention in float64.  These tests tie that second part
to things other than itself:

* one token: the softmax weight is exactly 1, so the output is that token's
  decoded V row, bit for bit;
* a zero query: all weights are equal, so the output is the plain mean;
* torch's scaled_dot_product_attention in float64, with the grouped-query
  mapping written as repeat_interleave (query head j reads KV head j // G);
* permuting the tokens (K and V together) leaves the output unchanged.

Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression" (review page: "If this is right", Fig. 11
caption: decode-phase attention reads the compressed KV cache).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as W


def _kv_blocks(B, H, S, seed):
    kt = W.random_tables(11, S_t=None)
    vt = W.random_tables(12, S_t=None)
    g = torch.Generator().manual_seed(seed)
    K = (torch.randn(B, H, S, 128, generator=g) * 0.5).to(torch.bfloat16)
    V = (torch.randn(B, H, S, 128, generator=g) * 0.5).to(torch.bfloat16)
    kb, _ = oracle.encode(kt, W.bf16_bits(K))
    vb, _ = oracle.encode(vt, W.bf16_bits(V))
    return kt, vt, kb.reshape(B, H, S, 64), vb.reshape(B, H, S, 64)


def _q(B, Hq, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return W.bf16_bits((torch.randn(B, Hq, 128, generator=g) * scale).to(torch.bfloat16))


def _decoded(tables, blocks):
    B, H, S, _ = blocks.shape
    y = oracle.decode(tables, blocks.reshape(-1, 64)).astype(np.uint32) << 16
    return y.view(np.float32).astype(np.float64).reshape(B, H, S, 128)


def test_single_token_returns_its_value_row():
    kt, vt, kb, vb = _kv_blocks(1, 2, 3, seed=1)
    q = _q(1, 4, seed=2)
    out, aw = oracle.attention(kt, vt, kb, vb, q, seq_len=1, scale=0.1)
    Vd = _decoded(vt, vb)
    for j in range(4):
        np.testing.assert_array_equal(out[0, j], Vd[0, j // 2, 0])
        np.testing.assert_array_equal(aw[0, j], np.abs(Vd[0, j // 2, 0]))


def test_zero_query_gives_the_mean_of_the_values():
    kt, vt, kb, vb = _kv_blocks(2, 1, 37, seed=3)
    q = np.zeros((2, 3, 128), dtype=np.uint16)
    out, _ = oracle.attention(kt, vt, kb, vb, q, seq_len=29, scale=0.3)
    Vd = _decoded(vt, vb)
    for b in range(2):
        for j in range(3):
            np.testing.assert_allclose(out[b, j], Vd[b, 0, :29].mean(axis=0), rtol=1e-13, atol=1e-15)


def test_matches_torch_sdpa_in_float64_with_grouped_queries():
    B, H, G, S, n = 2, 3, 4, 50, 41
    kt, vt, kb, vb = _kv_blocks(B, H, S, seed=5)
    q = _q(B, H * G, seed=6)
    scale = 1.0 / np.sqrt(128.0)
    out, aw = oracle.attention(kt, vt, kb, vb, q, seq_len=n, scale=scale)
    Kd = torch.from_numpy(_decoded(kt, kb)[:, :, :n]).repeat_interleave(G, dim=1)
    Vd = torch.from_numpy(_decoded(vt, vb)[:, :, :n]).repeat_interleave(G, dim=1)
    qf = torch.from_numpy((q.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(qf.unsqueeze(2), Kd, Vd, scale=scale).squeeze(2)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)
    ref_aw = torch.nn.functional.scaled_dot_product_attention(qf.unsqueeze(2), Kd, Vd.abs(), scale=scale).squeeze(2)
    np.testing.assert_allclose(aw, ref_aw.numpy(), rtol=1e-10, atol=1e-12)


def test_token_order_does_not_matter():
    kt, vt, kb, vb = _kv_blocks(1, 2, 64, seed=7)
    q = _q(1, 2, seed=8, scale=2.0)
    out, _ = oracle.attention(kt, vt, kb, vb, q, seq_len=64, scale=0.2)
    perm = np.random.default_rng(9).permutation(64)
    out2, _ = oracle.attention(kt, vt, kb[:, :, perm].copy(), vb[:, :, perm].copy(), q, seq_len=64, scale=0.2)
    np.testing.assert_allclose(out, out2, rtol=1e-12, atol=1e-14)
