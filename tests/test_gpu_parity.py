"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Encoded blocks and decoded bf16 must be bit-identical to the oracle's; the
fused decode+GEMV must satisfy |y - y64| <= 1e-3 * sum_k |W~ x| (+1e-30) per
element against the oracle's fp64 product of the decoded matrix (a bf16
result alone would already exceed 1e-3; fp32 accumulation of 4096 exact
products stays orders of magnitude inside it).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200 import _lib
from entropy_coded_kv_b200.calib import learn_tables

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
GEMV_RTOL = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return W.bf16_bits(t)


def to_dev_bf16(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(DEV)


_TABLE_CACHE = {}


def table_set(name: str) -> bytes:
    if name not in _TABLE_CACHE:
        if name.startswith("random"):
            seed = int(name[6:])
            st = {0: 0.02 * 4 / 448, 1: None, 2: 2.0 ** -40, 3: 1.0}.get(seed)
            _TABLE_CACHE[name] = W.random_tables(seed, S_t=st)
        elif name == "crowded":
            # every other pattern with 8 centroids 1e-5 apart: several of its
            # thresholds share one bucket of the encoder's threshold map, so
            # those patterns take the bisection search
            blob = W.random_tables(11)
            S_t = float(np.frombuffer(blob, np.float32, 1, 8)[0])
            C = np.frombuffer(blob, np.float32, 64 * 15, 16).reshape(64, 15).copy()
            lens = np.frombuffer(blob, np.uint8, 64 * 4 * 16, 16 + 64 * 15 * 4).reshape(64, 4, 16)
            for p in range(0, 64, 2):
                C[p, 3:11] = C[p, 3] + np.arange(8, dtype=np.float32) * np.float32(1e-5)
            assert np.all(np.diff(C, axis=1) > 0)
            _TABLE_CACHE[name] = W.pack_tables(S_t, C, lens)
        elif name == "learned_c1":
            _TABLE_CACHE[name] = learn_tables(W.c1_matrix(), seed=0)
        elif name == "learned_kv":
            _TABLE_CACHE[name] = learn_tables(W.c2_calibration(shape=(1, 8, 512, 128))[0], seed=0)
        elif name == "learned_w":
            _TABLE_CACHE[name] = learn_tables(W.c3_weight(rows=512, cols=4096), seed=0)
        else:
            raise KeyError(name)
    return _TABLE_CACHE[name]


def inputs(kind: str, n_groups: int, seed: int) -> np.ndarray:
    g = torch.Generator().manual_seed(seed)
    if kind == "gauss":
        x = torch.randn(n_groups * 128, generator=g) * 0.02
    elif kind == "t5":
        x = W.student_t((n_groups * 128,), 5, g, "cpu") * 0.02
    elif kind == "kv":
        z = torch.randn(n_groups, 128, generator=g)
        sc = torch.exp(torch.randn(128, generator=g) * 0.5)
        sc[torch.randperm(128, generator=g)[:4]] *= 15
        x = (z * sc).reshape(-1)
    elif kind == "c1":
        x = W.c1_matrix().float().reshape(-1)
        x = x.repeat((n_groups * 128 + x.numel() - 1) // x.numel())[: n_groups * 128]
    elif kind == "special":
        x = torch.randn(n_groups * 128, generator=g) * 0.02
        xr = x.view(n_groups, 128)
        xr[0] = 0.0                           # all-zero group
        xr[1] = 1e-30                         # rounds to a zero scale
        xr[2, 5] = float("nan")               # non-finite elements
        xr[3, 7] = float("inf")
        xr[3, 9] = float("-inf")
        xr[4] = 3e38                          # saturating scale, huge values
        xr[5] = -7.0
        xr[6, :] = torch.linspace(-1, 1, 128)  # many ties and exact values
        xr[7, :] = 0.25
        xr[8, 0] = -1.0
    else:
        raise KeyError(kind)
    return bits(x.to(torch.bfloat16))


TABLES = ["random0", "random1", "random2", "random3", "crowded", "learned_c1", "learned_kv", "learned_w"]
KINDS = ["gauss", "t5", "kv", "c1", "special"]


@pytest.mark.parametrize("tname", TABLES)
@pytest.mark.parametrize("kind", KINDS)
def test_encode_and_decode_bit_exact(tname, kind):
    blob = table_set(tname)
    n = 4096 + 37  # several CTAs' worth plus a ragged tail
    xb = inputs(kind, n, seed=hash((tname, kind)) & 0xFFFF)
    want_blocks, want_st = oracle.encode(blob, xb, nthreads=8)
    t = ecco.Tables(blob, DEV)
    st = ecco.new_stats(DEV)
    got = ecco.encode(to_dev_bf16(xb), t, stats=st)
    got_np = got.cpu().numpy()
    bad = np.flatnonzero((got_np != want_blocks).any(1))
    assert bad.size == 0, f"{bad.size} blocks differ, first {bad[:5]}"
    s = ecco.read_stats(st)
    for k in ("n_groups", "n_zero", "n_clipped", "n_padded", "n_records", "n_nonfinite", "payload_bits"):
        assert s[k] == getattr(want_st, k), k
    y = ecco.decode(got, t)
    want_y = oracle.decode(blob, want_blocks, nthreads=8)
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), want_y)


@pytest.mark.parametrize("tname", ["random0", "random1", "learned_kv"])
def test_decode_garbage_blocks_bit_exact(tname):
    blob = table_set(tname)
    rng = np.random.default_rng(1)
    blocks = rng.integers(0, 256, (3000, 64), dtype=np.uint8)
    blocks[::7, 0] = 0x00   # zero scale code
    blocks[1::7, 0] = 0x7F  # NaN scale code
    blocks[2::7, 0] = 0xFE
    t = ecco.Tables(blob, DEV)
    y = ecco.decode(torch.from_numpy(blocks).to(DEV), t)
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(blob, blocks, nthreads=8))


@pytest.mark.parametrize("gs", [128, 64])
def test_golden_blocks_on_gpu(gs):
    import test_oracle_pins as P
    blob, spec = P.golden_tables()
    t = ecco.Tables(blob, DEV)
    cases = [c for c in spec["cases"] if c.get("group", 128) == gs]
    enc, dec = (ecco.encode, ecco.decode) if gs == 128 else (ecco.encode_act, ecco.decode_act)
    xs = np.stack([P.expand(c["x"], gs) for c in cases])
    want = np.stack([P.assemble_stream(c["stream"]) for c in cases])
    got = enc(to_dev_bf16(xs), t).cpu().numpy()
    np.testing.assert_array_equal(got, want)
    y = dec(torch.from_numpy(want).to(DEV), t)
    np.testing.assert_array_equal(bits(y).reshape(-1, gs), np.stack([P.expand(c["decoded"], gs) for c in cases]))


@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 255, 257, 1023, 1025, 148 * 1024 + 5])
def test_ragged_sizes(n):
    blob = table_set("learned_kv")
    xb = inputs("kv", n, seed=n)
    t = ecco.Tables(blob, DEV)
    got = ecco.encode(to_dev_bf16(xb), t).cpu().numpy()
    want, _ = oracle.encode(blob, xb, nthreads=8)
    np.testing.assert_array_equal(got, want)
    y = ecco.decode(torch.from_numpy(want).to(DEV), t)
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(blob, want, nthreads=8))


def test_decode_into_16_byte_aligned_output():
    """Outputs aligned to 16 but not 32 bytes take the 16-byte-store variant."""
    blob = table_set("learned_kv")
    xb = inputs("kv", 700, seed=4)
    blocks, _ = oracle.encode(blob, xb, nthreads=8)
    t = ecco.Tables(blob, DEV)
    flat = torch.zeros(700 * 128 + 8, dtype=torch.bfloat16, device=DEV)
    out = flat[8:].view(700, 128)
    assert out.data_ptr() % 32 == 16
    ecco.decode(torch.from_numpy(blocks).to(DEV), t, out=out)
    np.testing.assert_array_equal(bits(out), oracle.decode(blob, blocks, nthreads=8))
    assert (bits(flat[:8]) == 0).all()


def test_decode_from_16_byte_aligned_blocks():
    """Blocks aligned to 16 but not 32 bytes take the 16-byte-load variant."""
    blob = table_set("learned_kv")
    xb = inputs("kv", 700, seed=5)
    blocks, _ = oracle.encode(blob, xb, nthreads=8)
    t = ecco.Tables(blob, DEV)
    flat = torch.zeros(700 * 64 + 16, dtype=torch.uint8, device=DEV)
    blk = flat[16:].view(700, 64)
    blk.copy_(torch.from_numpy(blocks).to(DEV))
    assert blk.data_ptr() % 32 == 16
    for dec in (ecco.decode, lambda b, tt: ecco.decode(b, tt, speculative=True)):
        y = dec(blk, t)
        np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(blob, blocks, nthreads=8))
    y = torch.empty((700, 128), dtype=torch.bfloat16, device=DEV)
    ecco.decode_multi([ecco.Seg(t, blk, y)])
    np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(blob, blocks, nthreads=8))


def test_empty_inputs_enqueue_nothing():
    t = ecco.Tables(table_set("random0"), DEV)
    x = torch.empty(0, dtype=torch.bfloat16, device=DEV)
    assert ecco.encode(x, t).numel() == 0
    assert ecco.decode(torch.empty((0, 64), dtype=torch.uint8, device=DEV), t).numel() == 0
    y = ecco.decode_gemv(torch.empty(0, dtype=torch.uint8, device=DEV), t, 0, 128,
                         torch.zeros(1, 128, dtype=torch.bfloat16, device=DEV))
    assert y.numel() == 0


def test_kv_append_and_strided_decode_descriptors():
    blob = table_set("learned_kv")
    t = ecco.Tables(blob, DEV)
    B, H, S, T, D = 2, 3, 40, 8, 128
    cache = torch.full((B * H * S, 64), 0xA5, dtype=torch.uint8, device=DEV)
    newkv = to_dev_bf16(inputs("kv", B * H * T, seed=3))
    d = ecco.kv_append_desc(B * H, T, S, S - T)
    ecco.encode(newkv, t, out=cache, desc=d)
    c = cache.view(B * H, S, 64).cpu().numpy()
    want, _ = oracle.encode(blob, bits(newkv), nthreads=4)
    np.testing.assert_array_equal(c[:, S - T:].reshape(-1, 64), want)
    assert (c[:, : S - T] == 0xA5).all()
    # decode rows 1..4 of the cache, token window [10, 30), into an offset output
    src = ecco.Desc(4, 20, S, 25, S + 10, 3)
    out = torch.full((4 * 25 + 3, 128), -1.0, dtype=torch.bfloat16, device=DEV)
    ecco.decode(cache, t, out=out, desc=src)
    o = bits(out)
    allblk = cache.cpu().numpy()
    for r in range(4):
        want_rows = oracle.decode(blob, allblk[S + 10 + r * S: S + 10 + r * S + 20], nthreads=2)
        np.testing.assert_array_equal(o[3 + r * 25: 3 + r * 25 + 20], want_rows)
        assert (o[3 + r * 25 + 20: 3 + (r + 1) * 25] == 0xBF80).all()
    assert (o[:3] == 0xBF80).all()


def test_argument_errors_return_codes_and_launch_nothing():
    t = ecco.Tables(table_set("random0"), DEV)
    lib = _lib.load()
    x = torch.zeros(4 * 128 + 8, dtype=torch.bfloat16, device=DEV)
    out = torch.zeros(5 * 64 + 16, dtype=torch.uint8, device=DEV)
    d = _lib.Desc(1, 4, 4, 4, 0, 0)
    import ctypes
    mis = ctypes.c_void_p(x.data_ptr() + 2)
    assert lib.ecco_select_encode(t.handle, mis, d, ctypes.c_void_p(out.data_ptr()), None, None) == _lib.ECCO_ERR_ALIGN
    assert lib.ecco_decode(t.handle, ctypes.c_void_p(out.data_ptr() + 8), d, ctypes.c_void_p(x.data_ptr()),
                           None) == _lib.ECCO_ERR_ALIGN
    bad = _lib.Desc(2, 4, 4, 3, 0, 0)  # overlapping destination rows
    assert lib.ecco_decode(t.handle, ctypes.c_void_p(out.data_ptr()), bad, ctypes.c_void_p(x.data_ptr()),
                           None) == _lib.ECCO_ERR_ARG
    neg = _lib.Desc(1, -4, 4, 4, 0, 0)
    assert lib.ecco_decode(t.handle, ctypes.c_void_p(out.data_ptr()), neg, ctypes.c_void_p(x.data_ptr()),
                           None) == _lib.ECCO_ERR_ARG
    # more than 2^31 - 2048 groups in one call (the kernels' 32-bit group index)
    huge = _lib.Desc(1 << 20, 1 << 11, 1 << 11, 1 << 11, 0, 0)
    for fn in (lib.ecco_decode, lib.ecco_decode_speculative):
        assert fn(t.handle, ctypes.c_void_p(out.data_ptr()), huge, ctypes.c_void_p(x.data_ptr()),
                  None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_select_encode(t.handle, ctypes.c_void_p(x.data_ptr()), huge, ctypes.c_void_p(out.data_ptr()),
                                  None, None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_decode_gemv(t.handle, ctypes.c_void_p(out.data_ptr()), 1, 100, ctypes.c_void_p(x.data_ptr()),
                                1, ctypes.c_void_p(x.data_ptr()), None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_decode_gemv(t.handle, ctypes.c_void_p(out.data_ptr()), 1, 128, ctypes.c_void_p(x.data_ptr()),
                                17, ctypes.c_void_p(x.data_ptr()), None) == _lib.ECCO_ERR_ARG
    with pytest.raises(ecco.EccoError):
        ecco.Tables(b"\0" * 7952, DEV)
    torch.cuda.synchronize()
    assert (out == 0).all()


def gemv_check(blob, blocks_np, rows, cols, xb, y):
    want, absum = oracle.gemv(blob, blocks_np, rows, cols, xb)
    err = np.abs(y.astype(np.float64) - want)
    lim = GEMV_RTOL * absum + 1e-30
    assert (err <= lim).all(), f"max excess {(err - lim).max()}"


@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 16])
@pytest.mark.parametrize("rows,cols", [(700, 384), (64, 1024), (1030, 512), (5, 8192), (33, 4224)])
def test_gemv_within_tolerance(batch, rows, cols):
    blob = table_set("learned_w")
    wb = inputs("t5", rows * cols // 128, seed=rows + cols)
    blocks, _ = oracle.encode(blob, wb, nthreads=8)
    t = ecco.Tables(blob, DEV)
    xb = bits(torch.randn(batch, cols, generator=torch.Generator().manual_seed(batch)).to(torch.bfloat16))
    y = ecco.decode_gemv(torch.from_numpy(blocks).to(DEV), t, rows, cols, to_dev_bf16(xb)).cpu().numpy()
    gemv_check(blob, blocks, rows, cols, xb, y)


@pytest.mark.parametrize("batch", [1, 3])
def test_gemv_restages_x_windows(batch):
    """A matrix so wide (5,000 column groups, one strip of rows) that a CTA's
    items span more than one 32-group window of x: the CUDA-core product runs
    its items in rounds and restages x as they move on."""
    blob = table_set("learned_w")
    rows, cols = 7, 128 * 5000
    wb = inputs("t5", rows * cols // 128, seed=12)
    blocks, _ = oracle.encode(blob, wb, nthreads=8)
    t = ecco.Tables(blob, DEV)
    xb = bits(torch.randn(batch, cols, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16))
    y = ecco.decode_gemv(torch.from_numpy(blocks).to(DEV), t, rows, cols, to_dev_bf16(xb)).cpu().numpy()
    gemv_check(blob, blocks, rows, cols, xb, y)


def test_gemv_one_hot_selects_a_decoded_column_exactly():
    blob = table_set("learned_w")
    rows, cols = 300, 256
    wb = inputs("t5", rows * cols // 128, seed=5)
    blocks, _ = oracle.encode(blob, wb, nthreads=8)
    Wd = oracle.decode(blob, blocks).reshape(rows, cols)
    t = ecco.Tables(blob, DEV)
    for col in (0, 129, 255):
        x = np.zeros((1, cols), dtype=np.uint16)
        x[0, col] = 0x3F80
        y = ecco.decode_gemv(torch.from_numpy(blocks).to(DEV), t, rows, cols, to_dev_bf16(x)).cpu().numpy()
        want = (Wd[:, col].astype(np.uint32) << 16).view(np.float32)
        np.testing.assert_array_equal(y[0], want)


def test_multi_segment_decode_and_encode():
    names = ["learned_kv", "random1", "learned_w"]
    tabs = [ecco.Tables(table_set(n), DEV) for n in names]
    xs = [inputs(k, n, seed=i) for i, (k, n) in enumerate([("kv", 1000), ("gauss", 77), ("t5", 3000)])]
    segs, outs = [], []
    for t, xb in zip(tabs, xs):
        o = torch.empty((xb.size // 128, 64), dtype=torch.uint8, device=DEV)
        segs.append(ecco.Seg(t, to_dev_bf16(xb), o))
        outs.append(o)
    st = ecco.new_stats(DEV)
    ecco.encode_multi(segs, st)
    ys = []
    dsegs = []
    for t, o in zip(tabs, outs):
        yy = torch.empty((o.shape[0], 128), dtype=torch.bfloat16, device=DEV)
        dsegs.append(ecco.Seg(t, o, yy))
        ys.append(yy)
    ecco.decode_multi(dsegs)
    tot = 0
    for n, xb, o, yy in zip(names, xs, outs, ys):
        want, wst = oracle.encode(table_set(n), xb, nthreads=8)
        np.testing.assert_array_equal(o.cpu().numpy(), want)
        np.testing.assert_array_equal(bits(yy).reshape(-1, 128), oracle.decode(table_set(n), want, nthreads=8))
        tot += wst.n_groups
    assert ecco.read_stats(st)["n_groups"] == tot


# ------------------------------------------------------------------ full sizes, sampled
def sample_rows(n, k, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(n, k, replace=False), [0, n - 1]]))


def test_full_size_kv_cache_sampled():
    """The full KV cache workload: [8, 8, 4096, 128] K and V, online encode of
    the last 64 tokens plus full-cache decode, sampled against the oracle."""
    K, V = W.c2_kv(device=DEV)
    Kc, Vc = W.c2_calibration(device=DEV)
    for cache, calib in ((K, Kc), (V, Vc)):
        blob = learn_tables(calib, seed=0)
        t = ecco.Tables(blob, DEV)
        n = cache.numel() // 128
        blocks = ecco.encode(cache, t)
        # re-encode the last 64 tokens from a separate contiguous tensor
        new = cache.view(64, 4096, 128)[:, 4032:].contiguous()
        blocks2 = blocks.clone()
        ecco.encode(new, t, out=blocks2, desc=ecco.kv_append_desc(64, 64, 4096, 4032))
        assert torch.equal(blocks, blocks2)
        y = ecco.decode(blocks, t)
        idx = sample_rows(n, 4000, 11)
        xb = bits(cache.view(n, 128)[torch.from_numpy(idx).to(DEV)])
        want, _ = oracle.encode(blob, xb, nthreads=8)
        np.testing.assert_array_equal(blocks[torch.from_numpy(idx).to(DEV)].cpu().numpy(), want)
        np.testing.assert_array_equal(bits(y[torch.from_numpy(idx).to(DEV)]), oracle.decode(blob, want, nthreads=8))


def test_full_size_mlp_weight_sampled():
    """14336 x 4096 Student-t weight: decode and fused GEMV (batch 1 and 16)."""
    Wt = W.c3_weight(device=DEV)
    rows, cols = Wt.shape
    blob = learn_tables(Wt, seed=0)
    t = ecco.Tables(blob, DEV)
    blocks = ecco.encode(Wt, t)
    y = ecco.decode(blocks, t)
    n = rows * cols // 128
    idx = sample_rows(n, 4000, 5)
    sel = torch.from_numpy(idx).to(DEV)
    want, _ = oracle.encode(blob, bits(Wt.view(n, 128)[sel]), nthreads=8)
    np.testing.assert_array_equal(blocks[sel].cpu().numpy(), want)
    np.testing.assert_array_equal(bits(y[sel]), oracle.decode(blob, want, nthreads=8))
    for batch in (1, 16):
        x = W.activations(cols, batch, device=DEV)
        yv = ecco.decode_gemv(blocks, t, rows, cols, x).cpu().numpy()
        rsel = sample_rows(rows, 96, batch)
        bl = blocks.view(rows, cols // 128, 64)[torch.from_numpy(rsel).to(DEV)].cpu().numpy()
        gemv_check(blob, bl, len(rsel), cols, bits(x), yv[:, rsel])


def test_multi_segment_many_small_segments_cross_launches():
    """70 segments (more than one launch's worth), some empty, mixed tables and
    sizes, so CTA shares cross segment boundaries mid-round."""
    names = ["learned_kv", "random1", "learned_w", "random0"]
    tabs = {n: ecco.Tables(table_set(n), DEV) for n in names}
    rng = np.random.default_rng(70)
    plan = []
    for i in range(70):
        n = int(rng.choice([0, 1, 7, 33, 130, 1500]))
        plan.append((names[i % 4], n, i))
    segs, outs, xs = [], [], []
    for name, n, i in plan:
        xb = inputs(["kv", "gauss", "t5", "c1"][i % 4], max(n, 1), seed=1000 + i)[: n * 128]
        x = to_dev_bf16(xb) if n else torch.empty(0, dtype=torch.bfloat16, device=DEV)
        o = torch.empty((n, 64), dtype=torch.uint8, device=DEV)
        segs.append(ecco.Seg(tabs[name], x, o))
        outs.append(o)
        xs.append(xb)
    st = ecco.new_stats(DEV)
    ecco.encode_multi(segs, st)
    ys = [torch.empty((o.shape[0], 128), dtype=torch.bfloat16, device=DEV) for o in outs]
    ecco.decode_multi([ecco.Seg(tabs[name], o, y) for (name, _, _), o, y in zip(plan, outs, ys)])
    tot = 0
    for (name, n, _), xb, o, y in zip(plan, xs, outs, ys):
        if n == 0:
            continue
        want, wst = oracle.encode(table_set(name), xb, nthreads=4)
        np.testing.assert_array_equal(o.cpu().numpy(), want)
        np.testing.assert_array_equal(bits(y).reshape(-1, 128), oracle.decode(table_set(name), want, nthreads=4))
        tot += wst.n_groups
    assert ecco.read_stats(st)["n_groups"] == tot


def test_prepared_segments_one_token_append_over_64_segments():
    """A one-token append into 64 caches of 16 rows (one CTA per segment),
    through a prepared segment list called twice with new token contents:
    bit-exact with the oracle, the other tokens untouched; a prepared decode
    of the caches; a list prepared for decode is refused by encode_multi."""
    names = ["learned_kv", "random1"]
    tabs = [ecco.Tables(table_set(n), DEV) for n in names]
    S, n = 5, 64
    H = 16  # rows (KV heads) per cache: the "special" inputs need 9 groups or more
    caches = [torch.zeros((H * S, 64), dtype=torch.uint8, device=DEV) for _ in range(n)]
    new = [torch.empty((H, 128), dtype=torch.bfloat16, device=DEV) for _ in range(n)]
    app = ecco.kv_append_desc(H, 1, S, S - 1)
    prep = ecco.prepare_encode([ecco.Seg(tabs[i % 2], new[i], caches[i], app) for i in range(n)])
    for rep in range(2):
        xbs = [inputs(KINDS[(i + rep) % len(KINDS)], H, seed=100 * rep + i) for i in range(n)]
        for nw, xb in zip(new, xbs):
            nw.copy_(to_dev_bf16(xb).view(H, 128))
        ecco.encode_multi(prep)
        for i in range(n):
            want, _ = oracle.encode(table_set(names[i % 2]), xbs[i], nthreads=2)
            c = caches[i].view(H, S, 64).cpu().numpy()
            np.testing.assert_array_equal(c[:, S - 1], want, err_msg=f"segment {i}, call {rep}")
            assert not c[:, :S - 1].any()
    ys = [torch.empty((H * S, 128), dtype=torch.bfloat16, device=DEV) for _ in range(n)]
    dprep = ecco.prepare_decode([ecco.Seg(tabs[i % 2], caches[i], ys[i]) for i in range(n)])
    ecco.decode_multi(dprep)
    for i in (0, 1, n - 1):
        blk = caches[i].cpu().numpy()
        np.testing.assert_array_equal(bits(ys[i]).reshape(-1, 128), oracle.decode(table_set(names[i % 2]), blk,
                                                                                 nthreads=2))
    with pytest.raises(ValueError):
        ecco.encode_multi(dprep)


@pytest.mark.parametrize("batch", [5, 16])
def test_tensor_core_gemv_one_hot_columns_are_exact(batch):
    """Batch > 4 runs on tcgen05 tensor cores.  With x[b] one-hot at column c_b,
    y[b] must be decoded column c_b bit for bit (one exact product per row)."""
    blob = table_set("learned_w")
    rows, cols = 700, 384
    wb = inputs("t5", rows * cols // 128, seed=9)
    blocks, _ = oracle.encode(blob, wb, nthreads=8)
    Wd = oracle.decode(blob, blocks).reshape(rows, cols)
    t = ecco.Tables(blob, DEV)
    cs = [0, 17, 127, 128, 200, 255, 256, 383, 64, 300, 5, 130, 260, 99, 333, 1][:batch]
    x = np.zeros((batch, cols), dtype=np.uint16)
    for b, c in enumerate(cs):
        x[b, c] = 0x3F80
    y = ecco.decode_gemv(torch.from_numpy(blocks).to(DEV), t, rows, cols, to_dev_bf16(x)).cpu().numpy()
    for b, c in enumerate(cs):
        np.testing.assert_array_equal(y[b], (Wd[:, c].astype(np.uint32) << 16).view(np.float32))


@pytest.mark.parametrize("batch", [5, 16])
@pytest.mark.parametrize("rows,cols", [(1536, 9728), (58268, 256)])
def test_tensor_core_gemv_leftover_units(batch, rows, cols):
    """Shapes whose units (768 rows x one column group) do not divide evenly
    over the SMs (152 units on 148, so a few CTAs take one unit more), the
    extra units inside one row tile and across two row tiles with a ragged
    last one.  One-hot columns come out bit for bit; random x stays within
    the product tolerance."""
    blob = table_set("learned_w")
    wb = inputs("t5", rows * cols // 128, seed=rows)
    blocks, _ = oracle.encode(blob, wb, nthreads=8)
    Wd = oracle.decode(blob, blocks, nthreads=8).reshape(rows, cols)
    t = ecco.Tables(blob, DEV)
    dblocks = torch.from_numpy(blocks).to(DEV)
    cs = [(37 * b + 5) % cols for b in range(batch - 1)] + [cols - 1]
    x = np.zeros((batch, cols), dtype=np.uint16)
    for b, c in enumerate(cs):
        x[b, c] = 0x3F80
    y = ecco.decode_gemv(dblocks, t, rows, cols, to_dev_bf16(x)).cpu().numpy()
    for b, c in enumerate(cs):
        np.testing.assert_array_equal(y[b], (Wd[:, c].astype(np.uint32) << 16).view(np.float32))
    xb = bits(torch.randn(batch, cols, generator=torch.Generator().manual_seed(batch)).to(torch.bfloat16))
    y = ecco.decode_gemv(dblocks, t, rows, cols, to_dev_bf16(xb)).cpu().numpy()
    gemv_check(blob, blocks, rows, cols, xb, y)


def test_no_device_wait_gave_up():
    """Tensor-core GEMV launches leave the timeout count where it was."""
    import ctypes
    lib = _lib.load()
    before, after = ctypes.c_uint(123), ctypes.c_uint(456)
    assert lib.ecco_device_timeouts(ctypes.byref(before)) == 0
    blob = table_set("learned_w")
    t = ecco.Tables(blob, DEV)
    blocks = torch.from_numpy(oracle.encode(blob, inputs("t5", 700 * 3, seed=2), nthreads=8)[0]).to(DEV)
    for batch in (5, 16):
        ecco.decode_gemv(blocks, t, 700, 384, W.activations(384, batch, device=DEV))
    torch.cuda.synchronize()
    assert lib.ecco_device_timeouts(ctypes.byref(after)) == 0
    assert after.value == before.value


def test_offsets_past_4_gib():
    """Descriptors that address groups more than 2^32 bytes into the buffers
    (row stride 2^25 groups = 8 GiB of bf16): every index is 64-bit."""
    blob = table_set("learned_kv")
    t = ecco.Tables(blob, DEV)
    gpr, stride = 300, 1 << 25
    xb = inputs("kv", 2 * gpr, seed=77)
    src = torch.empty((stride + gpr, 128), dtype=torch.bfloat16, device=DEV)  # ~8.6 GB, not written
    src[:gpr] = to_dev_bf16(xb[: gpr * 128]).view(gpr, 128)
    src[stride:] = to_dev_bf16(xb[gpr * 128:]).view(gpr, 128)
    blocks = torch.empty((2 * gpr, 64), dtype=torch.uint8, device=DEV)
    ecco.encode(src, t, out=blocks, desc=_lib.Desc(2, gpr, stride, gpr, 0, 0))
    want, _ = oracle.encode(blob, xb, nthreads=8)
    np.testing.assert_array_equal(blocks.cpu().numpy(), want)
    out = torch.empty_like(src)
    ecco.decode(blocks, t, out=out, desc=_lib.Desc(2, gpr, gpr, stride, 0, 0))
    wy = oracle.decode(blob, want, nthreads=8)
    np.testing.assert_array_equal(bits(out[:gpr]).reshape(-1, 128), wy[:gpr])
    np.testing.assert_array_equal(bits(out[stride:]).reshape(-1, 128), wy[gpr:])
    del src, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("batch", [1, 3, 8, 16])
def test_gemv_on_garbage_blocks(batch):
    """Random 64-byte blocks (clipped streams, duplicate record indexes, null
    and NaN scale codes) through the fused GEMV on CUDA cores and tcgen05: the
    result must match the fp64 product of the oracle's decoding."""
    blob = table_set("random1")
    t = ecco.Tables(blob, DEV)
    rng = np.random.default_rng(100 + batch)
    rows, cols = 700, 512
    blk = rng.integers(0, 256, (rows * cols // 128, 64), dtype=np.uint8)
    xb = bits(W.activations(cols, batch=batch, seed=batch))
    y = ecco.decode_gemv(torch.from_numpy(blk).to(DEV), t, rows, cols, to_dev_bf16(xb)).cpu().numpy()
    want, absum = oracle.gemv(blob, blk, rows, cols, xb)
    ok = np.isfinite(want)  # decoded values can be huge but stay finite for this table set
    err = np.abs(y.astype(np.float64) - want)
    assert (err[ok] <= GEMV_RTOL * absum[ok] + 1e-30).all()
