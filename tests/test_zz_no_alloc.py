"""ecco_decode_attention_static (the partials in the library's static device
workspace, nothing allocated by the call) against ecco_decode_attention with
a caller workspace, on the same inputs (needs a B200).

Both run the same kernels; only the order of fp32 shared-memory additions can
differ between launches, so results agree to a few fp32 ulps of the output's
scale.  The static workspace is shared state, so each case runs the static
call twice in a row and must not depend on what earlier tests left in it.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import workloads as W
import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200 import _lib
from test_gpu_parity import table_set

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _case(B, H, G, S_cap, seed):
    K, V = W.kv_cache((B, H, S_cap, 128), seed, device=DEV)
    tk, tv = ecco.Tables(table_set("learned_kv"), DEV), ecco.Tables(table_set("random1"), DEV)
    kb = ecco.encode(K, tk).view(B, H, S_cap, 64)
    vb = ecco.encode(V, tv).view(B, H, S_cap, 64)
    g = torch.Generator(device=DEV).manual_seed(seed + 2)
    q = torch.randn(B, H * G, 128, generator=g, device=DEV).to(torch.bfloat16)
    return tk, tv, kb, vb, q


def _close(a, b):
    a, b = a.cpu().numpy(), b.cpu().numpy()
    np.testing.assert_allclose(a, b, rtol=1e-5, atol=1e-6 * float(np.abs(b).max()))


def _device_allocations():
    """(caching-allocator allocations so far, bytes free on the device)."""
    torch.cuda.synchronize()
    return torch.cuda.memory_stats(DEV).get("allocation.all.allocated", 0), torch.cuda.mem_get_info(DEV)[0]


@pytest.mark.parametrize("B,H,G,S_cap,n", [(2, 2, 4, 1300, 1237), (1, 3, 8, 700, 513), (8, 8, 4, 4096, 4096)])
def test_static_workspace_matches_caller_workspace(B, H, G, S_cap, n):
    tk, tv, kb, vb, q = _case(B, H, G, S_cap, seed=n)
    want = ecco.decode_attention(kb, vb, tk, tv, q, n, 0.0884)
    out = torch.empty_like(want)
    for i in range(2):
        out.fill_(float("nan"))
        before = _device_allocations()
        ecco.decode_attention_static(kb, vb, tk, tv, q, n, 0.0884, out=out)
        # the call itself allocates nothing: no caching-allocator block and,
        # after the first call's one-time set-up, no device memory at all
        after = _device_allocations()
        assert after[0] == before[0]
        if i == 1:
            assert after[1] == before[1]
        _close(out, want)


def test_largest_request_that_fits_and_first_that_does_not():
    # workspace = 4 * 130 * B * H * G * ceil(seq_len / 512) bytes; with G = 8 the
    # static 4 MiB holds 1008 splits of 512 tokens, not 1009
    per_split = 4 * 130 * 8
    fits, over = 1008 * 512, 1009 * 512
    assert fits // 512 * per_split <= _lib.ATTENTION_STATIC_WS_BYTES < over // 512 * per_split
    tk, tv, kb, vb, q = _case(1, 1, 8, over, seed=5)
    want = ecco.decode_attention(kb, vb, tk, tv, q, fits, 0.0884)
    _close(ecco.decode_attention_static(kb, vb, tk, tv, q, fits, 0.0884), want)
    out = torch.zeros(1, 8, 128, dtype=torch.float32, device=DEV)
    rc = _lib.load().ecco_decode_attention_static(
        tk.handle, tv.handle, ctypes.c_void_p(kb.data_ptr()), ctypes.c_void_p(vb.data_ptr()), over, 1, 1, 8, over,
        ctypes.c_void_p(q.data_ptr()), 0.0884, ctypes.c_void_p(out.data_ptr()), None)
    assert rc == _lib.ECCO_ERR_WORKSPACE
    assert "static" in _lib.strerror(rc)
    # argument errors come first, as in ecco_decode_attention: an oversized
    # request with a null table handle or a misaligned q is an argument error
    L = _lib.load()
    rc = L.ecco_decode_attention_static(None, tv.handle, ctypes.c_void_p(kb.data_ptr()), ctypes.c_void_p(vb.data_ptr()),
                                        over, 1, 1, 8, over, ctypes.c_void_p(q.data_ptr()), 0.0884,
                                        ctypes.c_void_p(out.data_ptr()), None)
    assert rc == _lib.ECCO_ERR_ARG
    rc = L.ecco_decode_attention_static(tk.handle, tv.handle, ctypes.c_void_p(kb.data_ptr()),
                                        ctypes.c_void_p(vb.data_ptr()), over, 1, 1, 8, over,
                                        ctypes.c_void_p(q.data_ptr() + 1), 0.0884, ctypes.c_void_p(out.data_ptr()),
                                        None)
    assert rc == _lib.ECCO_ERR_ALIGN
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0  # nothing was enqueued
