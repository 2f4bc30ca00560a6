"""Decode-phase attention over compressed K and V (CUDA, through the C ABI) vs
the oracle, for both entry points: ecco_decode_attention (the blocks decoded
inside the attention kernel) and ecco_decode_attention_staged (each chunk of
tokens decoded by the block decoder into a scratch, then attended).

The oracle decodes the K and V blocks and applies softmax attention in
float64.  The kernel decodes the same blocks bit-exactly (the block decoder's
own parity tests) but computes scores, softmax and the weighted sum in fp32.
Tolerance per output element: |out - ref| <= 1e-3 * sum_s p_s |v~_s|.  The
largest fp32 effect is the 128-term score dot product, whose absolute error
(<= 128 u sum_i |q_i k_i| * scale, u = 2^-24) moves every weight p_s by about
that relative amount; for these inputs that is below 1e-4.

Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression" (review page: "If this is right", Fig. 11
caption).
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
from test_gpu_parity import inputs, table_set, to_dev_bf16

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
RTOL = 1e-3


def q_bits(B, Hq, seed):
    g = torch.Generator().manual_seed(seed)
    return W.bf16_bits(torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16))


def check(out, ref, aw):
    err = np.abs(out.astype(np.float64) - ref)
    bad = err > RTOL * aw + 1e-30
    assert not bad.any(), (f"{bad.sum()} elements out of tolerance; worst excess "
                           f"{(err - RTOL * aw).max():.3e}")


PATHS = {"fused": (ecco.decode_attention, ecco.attention_workspace_bytes),
         "staged": (ecco.decode_attention_staged, ecco.attention_staged_workspace_bytes)}


def run(kt, vt, kb, vb, q, seq_len, scale, ws=None, path="fused"):
    B, H, S, _ = kb.shape
    return PATHS[path][0](torch.from_numpy(kb).to(DEV), torch.from_numpy(vb).to(DEV),
                          ecco.Tables(kt, DEV), ecco.Tables(vt, DEV), to_dev_bf16(q), seq_len,
                          scale, workspace=ws).cpu().numpy()


CASES = [
    # B, H, G, S_cap, seq_len, K tables, V tables, K kind, V kind
    (2, 2, 4, 1300, 1237, "learned_kv", "random1", "kv", "kv"),
    (1, 1, 1, 1, 1, "learned_kv", "learned_kv", "kv", "kv"),
    (1, 3, 3, 600, 512, "random0", "learned_kv", "gauss", "kv"),
    (1, 2, 8, 1100, 1025, "learned_kv", "learned_kv", "kv", "kv"),
    (3, 1, 5, 40, 33, "random3", "random2", "t5", "special"),
    (1, 1, 7, 2048, 2048, "random1", "random3", "special", "t5"),
    (1, 2, 2, 700, 513, "learned_c1", "learned_w", "c1", "t5"),
    (2, 1, 6, 3000, 2999, "learned_w", "learned_kv", "t5", "kv"),
]


@pytest.mark.parametrize("path", ["fused", "staged"])
@pytest.mark.parametrize("B,H,G,S_cap,n,ktn,vtn,kk,vk", CASES)
def test_attention_matches_oracle(B, H, G, S_cap, n, ktn, vtn, kk, vk, path):
    kt, vt = table_set(ktn), table_set(vtn)
    kb, _ = oracle.encode(kt, inputs(kk, B * H * S_cap, seed=S_cap), nthreads=8)
    vb, _ = oracle.encode(vt, inputs(vk, B * H * S_cap, seed=S_cap + 1), nthreads=8)
    kb = kb.reshape(B, H, S_cap, 64)
    vb = vb.reshape(B, H, S_cap, 64)
    q = q_bits(B, H * G, seed=n)
    scale = 1.0 / np.sqrt(128.0)
    ref, aw = oracle.attention(kt, vt, kb, vb, q, n, scale)
    out = run(kt, vt, kb, vb, q, n, scale, path=path)
    check(out, ref, aw)


def test_staged_chunks():
    """4096 (batch, KV head) rows make the staged chunk 512 tokens (1 GiB of
    decoded rows), so 1237 tokens run as chunks of 512, 512 and 213 tokens
    through the same scratch; the partials hold five 256-token splits."""
    B, H, G, S_cap, n = 512, 8, 1, 1240, 1237
    assert _lib.load().ecco_decode_attention_staged_workspace_bytes(B, H, G, n) == (
        4 * 130 * B * H * G * 5 + 256 + 2 * B * H * 512 * 256)
    kt, vt = table_set("learned_kv"), table_set("random2")
    rng = np.random.default_rng(31)  # every 64-byte pattern is a block (clips, records, null scales)
    kb = rng.integers(0, 256, (B, H, S_cap, 64), dtype=np.uint8)
    vb = rng.integers(0, 256, (B, H, S_cap, 64), dtype=np.uint8)
    q = q_bits(B, H * G, seed=33)
    ref, aw = oracle.attention(kt, vt, kb, vb, q, n, 1e-3, nthreads=8)
    assert np.isfinite(ref).all()
    check(run(kt, vt, kb, vb, q, n, 1e-3, path="staged"), ref, aw)


@pytest.mark.parametrize("path", ["fused", "staged"])
def test_blocks_past_seq_len_are_never_used(path):
    """Garbage after seq_len (random bytes) must not change the result."""
    B, H, G, S_cap, n = 1, 2, 4, 1500, 1111
    kt = vt = table_set("learned_kv")
    kb, _ = oracle.encode(kt, inputs("kv", B * H * S_cap, seed=1), nthreads=8)
    vb, _ = oracle.encode(vt, inputs("kv", B * H * S_cap, seed=2), nthreads=8)
    kb, vb = kb.reshape(B, H, S_cap, 64), vb.reshape(B, H, S_cap, 64)
    rng = np.random.default_rng(3)
    kb2, vb2 = kb.copy(), vb.copy()
    kb2[:, :, n:] = rng.integers(0, 256, kb2[:, :, n:].shape, dtype=np.uint8)
    vb2[:, :, n:] = rng.integers(0, 256, vb2[:, :, n:].shape, dtype=np.uint8)
    q = q_bits(B, H * G, seed=4)
    ref, aw = oracle.attention(kt, vt, kb, vb, q, n, 0.1)
    check(run(kt, vt, kb2, vb2, q, n, 0.1, path=path), ref, aw)


@pytest.mark.parametrize("path", ["fused", "staged"])
def test_workspace_reused_across_two_calls(path):
    B, H, G, S_cap, n = 2, 2, 4, 1024, 1000
    kt = vt = table_set("learned_kv")
    kb, _ = oracle.encode(kt, inputs("kv", B * H * S_cap, seed=5), nthreads=8)
    vb, _ = oracle.encode(vt, inputs("kv", B * H * S_cap, seed=6), nthreads=8)
    kb, vb = kb.reshape(B, H, S_cap, 64), vb.reshape(B, H, S_cap, 64)
    # garbage in the workspace (partials and scratch) must not matter
    ws = torch.full((PATHS[path][1](B, H, G, n),), 0xff, dtype=torch.uint8, device=DEV)
    for seed in (7, 8):
        q = q_bits(B, H * G, seed=seed)
        ref, aw = oracle.attention(kt, vt, kb, vb, q, n, 0.09)
        check(run(kt, vt, kb, vb, q, n, 0.09, ws=ws, path=path), ref, aw)


def test_full_size_kv_cache_attention_sampled():
    """[8, 8, 4096, 128] K and V (Llama-3-8B layer shape), 32 query heads
    (group 4): the whole batch on the GPU, sampled (batch, KV head) pairs
    against the oracle (whose blocks are the oracle's own encoding)."""
    K, V = W.c2_kv(device=DEV)
    Kc, Vc = W.c2_calibration(device=DEV)
    kt, vt = learn_tables(Kc, seed=0), learn_tables(Vc, seed=0)
    tk, tv = ecco.Tables(kt, DEV), ecco.Tables(vt, DEV)
    B, H, S, _ = K.shape
    G = 4
    kb = ecco.encode(K, tk).view(B, H, S, 64)
    vb = ecco.encode(V, tv).view(B, H, S, 64)
    q = q_bits(B, H * G, seed=21)
    scale = 1.0 / np.sqrt(128.0)
    out = ecco.decode_attention(kb, vb, tk, tv, to_dev_bf16(q), S, scale).cpu().numpy()
    # staged: 64 rows make 1024-token chunks, so four chunks through the scratch
    outs = ecco.decode_attention_staged(kb, vb, tk, tv, to_dev_bf16(q), S, scale).cpu().numpy()
    for b, h in ((0, 0), (3, 5), (7, 7), (5, 2)):
        kbo, _ = oracle.encode(kt, W.bf16_bits(K[b, h]), nthreads=8)
        vbo, _ = oracle.encode(vt, W.bf16_bits(V[b, h]), nthreads=8)
        np.testing.assert_array_equal(kb[b, h].cpu().numpy(), kbo)
        np.testing.assert_array_equal(vb[b, h].cpu().numpy(), vbo)
        ref, aw = oracle.attention(kt, vt, kbo.reshape(1, 1, S, 64), vbo.reshape(1, 1, S, 64),
                                   q[b:b + 1, h * G:(h + 1) * G], S, scale)
        check(out[b:b + 1, h * G:(h + 1) * G], ref, aw)
        check(outs[b:b + 1, h * G:(h + 1) * G], ref, aw)


def test_long_context_layer_attention_sampled():
    """One long-context layer, K and V [1, 8, 131072, 128], 32 query heads:
    the merge combines 256 splits (fused) and 512 (staged) per head.  Two KV
    heads against the oracle, whose blocks are its own encoding."""
    K, V = W.c5_layer(0, device=DEV)
    Kc, Vc = W.c5_calibration(0, device=DEV)
    kt, vt = learn_tables(Kc, seed=0), learn_tables(Vc, seed=0)
    tk, tv = ecco.Tables(kt, DEV), ecco.Tables(vt, DEV)
    B, H, S, _ = K.shape
    G = 4
    kb = ecco.encode(K, tk).view(B, H, S, 64)
    vb = ecco.encode(V, tv).view(B, H, S, 64)
    q = q_bits(B, H * G, seed=41)
    scale = 1.0 / np.sqrt(128.0)
    out = ecco.decode_attention(kb, vb, tk, tv, to_dev_bf16(q), S, scale).cpu().numpy()
    outs = ecco.decode_attention_staged(kb, vb, tk, tv, to_dev_bf16(q), S, scale).cpu().numpy()
    for h in (0, 6):
        kbo, _ = oracle.encode(kt, W.bf16_bits(K[0, h]), nthreads=8)
        vbo, _ = oracle.encode(vt, W.bf16_bits(V[0, h]), nthreads=8)
        np.testing.assert_array_equal(kb[0, h].cpu().numpy(), kbo)
        np.testing.assert_array_equal(vb[0, h].cpu().numpy(), vbo)
        ref, aw = oracle.attention(kt, vt, kbo.reshape(1, 1, S, 64), vbo.reshape(1, 1, S, 64),
                                   q[:, h * G:(h + 1) * G], S, scale, nthreads=8)
        check(out[:, h * G:(h + 1) * G], ref, aw)
        check(outs[:, h * G:(h + 1) * G], ref, aw)


def test_attention_argument_errors():
    lib = _lib.load()
    t = ecco.Tables(table_set("learned_kv"), DEV)
    kb = torch.zeros(1, 1, 64, 64, dtype=torch.uint8, device=DEV)
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(1, 4, 128, dtype=torch.float32, device=DEV)
    ws = torch.empty(1 << 16, dtype=torch.uint8, device=DEV)
    P = ctypes.c_void_p

    def call(kptr=kb.data_ptr(), s_cap=64, group=4, n=64, ws_bytes=ws.numel()):
        return lib.ecco_decode_attention(t.handle, t.handle, P(kptr), P(kb.data_ptr()), s_cap, 1, 1, group, n,
                                         P(q.data_ptr()), 1.0, P(out.data_ptr()), P(ws.data_ptr()), ws_bytes,
                                         None)

    assert call() == _lib.ECCO_OK
    torch.cuda.synchronize()
    assert call(group=9) == _lib.ECCO_ERR_ARG
    assert call(group=0) == _lib.ECCO_ERR_ARG
    assert call(n=65) == _lib.ECCO_ERR_ARG
    assert call(n=0) == _lib.ECCO_ERR_ARG
    assert call(ws_bytes=4 * 130 * 4 - 1) == _lib.ECCO_ERR_ARG
    assert call(kptr=kb.data_ptr() + 8) == _lib.ECCO_ERR_ALIGN

    need = lib.ecco_decode_attention_staged_workspace_bytes(1, 1, 4, 64)
    wss = torch.empty(need, dtype=torch.uint8, device=DEV)

    def staged(kptr=kb.data_ptr(), group=4, n=64, ws_bytes=need):
        return lib.ecco_decode_attention_staged(t.handle, t.handle, P(kptr), P(kb.data_ptr()), 64, 1, 1, group,
                                                n, P(q.data_ptr()), 1.0, P(out.data_ptr()), P(wss.data_ptr()),
                                                ws_bytes, None)

    assert staged() == _lib.ECCO_OK
    torch.cuda.synchronize()
    assert staged(group=9) == _lib.ECCO_ERR_ARG
    assert staged(n=65) == _lib.ECCO_ERR_ARG
    assert staged(ws_bytes=need - 1) == _lib.ECCO_ERR_ARG
    assert staged(kptr=kb.data_ptr() + 8) == _lib.ECCO_ERR_ALIGN


def test_attention_on_garbage_blocks():
    """Random K and V blocks (clipped streams, duplicate record indexes, null
    scale codes) against the oracle's attention over its own decoding."""
    B, H, G, S_cap, n = 1, 2, 4, 777, 700
    kt, vt = table_set("learned_kv"), table_set("random1")
    rng = np.random.default_rng(9)
    kb = rng.integers(0, 256, (B, H, S_cap, 64), dtype=np.uint8)
    vb = rng.integers(0, 256, (B, H, S_cap, 64), dtype=np.uint8)
    q = q_bits(B, H * G, seed=10)
    scale = 1e-3  # random scales make huge scores; keep the softmax finite
    ref, aw = oracle.attention(kt, vt, kb, vb, q, n, scale)
    assert np.isfinite(ref).all()
    check(run(kt, vt, kb, vb, q, n, scale), ref, aw)
    check(run(kt, vt, kb, vb, q, n, scale, path="staged"), ref, aw)
