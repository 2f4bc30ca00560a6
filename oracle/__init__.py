"""CPU oracle for the Ecco 512-bit block codec -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no source with it: the arithmetic lives in ``ecco_oracle.c`` (plain C,
compiled with ``-ffp-contract=off`` so every fp32 operation is rounded on its
own, as the format specifies) and this module only marshals numpy arrays.

Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression" (review page sections "What carries the
argument", "Core claim", Fig. 4 caption, free-parameter list).  The readings
R1-R21 that fix what the page leaves open are listed in ``ecco_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ecco_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libecco_oracle.so")
_lock = threading.Lock()
_lib = None

G = 128
NPAT = 64
NCENT = 15
NBOOK = 4
NSYM = 16
LMAX = 8
BLOCK_BYTES = 64
TABLES_BYTES = 16 + NPAT * NCENT * 4 + NPAT * NBOOK * NSYM


class Stats(ctypes.Structure):
    _fields_ = [
        ("n_groups", ctypes.c_uint64),
        ("n_zero", ctypes.c_uint64),
        ("n_clipped", ctypes.c_uint64),
        ("n_padded", ctypes.c_uint64),
        ("n_records", ctypes.c_uint64),
        ("n_nonfinite", ctypes.c_uint64),
        ("payload_bits", ctypes.c_uint64),
        ("n_mse_differs", ctypes.c_uint64),
        ("mse_minmax", ctypes.c_double),
        ("mse_full", ctypes.c_double),
    ]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class GroupInfo(ctypes.Structure):
    _fields_ = [
        ("m", ctypes.c_int32),
        ("zero", ctypes.c_int32),
        ("code", ctypes.c_uint8),
        ("p", ctypes.c_uint8),
        ("h", ctypes.c_uint8),
        ("clipped", ctypes.c_uint8),
        ("s", ctypes.c_float),
        ("inv", ctypes.c_float),
        ("umin", ctypes.c_float),
        ("umax", ctypes.c_float),
        ("L", ctypes.c_int32),
        ("k_clip", ctypes.c_int32),
        ("n_rec", ctypes.c_int32),
        ("sym", ctypes.c_uint8 * G),
        ("rec_pos", ctypes.c_uint8 * 16),
        ("rec_q", ctypes.c_int8 * 16),
        ("u", ctypes.c_float * G),
        ("e", ctypes.c_float * NPAT),
        ("Lh", ctypes.c_int32 * NBOOK),
        ("nonfinite", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc into oracle/_build (idempotent)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fno-builtin", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            L.or_bf16_to_f32.restype = ctypes.c_float
            L.or_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.or_f32_to_bf16.restype = ctypes.c_uint16
            L.or_f32_to_bf16.argtypes = [ctypes.c_float]
            L.or_e4m3_value.restype = ctypes.c_double
            L.or_e4m3_value.argtypes = [ctypes.c_uint8]
            L.or_e4m3_from_f32.restype = ctypes.c_uint8
            L.or_e4m3_from_f32.argtypes = [ctypes.c_float]
            L.or_tables_check.restype = ctypes.c_int
            L.or_tables_check.argtypes = [P]
            L.or_canonical_codes.restype = None
            L.or_canonical_codes.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
            L.or_encode_group_ex.restype = None
            L.or_encode_group_ex.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int]
            L.or_encode_group_sel.restype = None
            L.or_encode_group_sel.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
            L.or_decode_block.restype = ctypes.c_int
            L.or_decode_block.argtypes = [P, P, P]
            L.or_encode.restype = None
            L.or_encode.argtypes = [P, P, I64, P, P, ctypes.c_int, ctypes.c_int]
            L.or_encode_group_gs.restype = None
            L.or_encode_group_gs.argtypes = [P, P, P, P] + [ctypes.c_int] * 5
            L.or_decode_block_gs.restype = ctypes.c_int
            L.or_decode_block_gs.argtypes = [P, P, P, ctypes.c_int]
            L.or_encode_gs.restype = None
            L.or_encode_gs.argtypes = [P, P, I64, P, P] + [ctypes.c_int] * 5
            L.or_decode_gs.restype = None
            L.or_decode_gs.argtypes = [P, P, I64, P, ctypes.c_int, ctypes.c_int]
            L.or_encode_sel.restype = None
            L.or_encode_sel.argtypes = [P, P, I64, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
            L.or_decode.restype = None
            L.or_decode.argtypes = [P, P, I64, P, ctypes.c_int]
            L.or_gemv.restype = None
            L.or_gemv.argtypes = [P, P, I64, I64, P, ctypes.c_int, P, P]
            for fn in ("or_sizeof_tables", "or_sizeof_group_info", "or_sizeof_stats"):
                getattr(L, fn).restype = ctypes.c_int
            assert L.or_sizeof_tables() == TABLES_BYTES
            assert L.or_sizeof_group_info() == ctypes.sizeof(GroupInfo)
            assert L.or_sizeof_stats() == ctypes.sizeof(Stats)
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _blob(tables) -> np.ndarray:
    b = np.frombuffer(bytes(tables), dtype=np.uint8) if not isinstance(tables, np.ndarray) else tables
    b = np.ascontiguousarray(b, dtype=np.uint8)
    assert b.size == TABLES_BYTES, b.size
    return b


def _bits(x) -> np.ndarray:
    """Accepts uint16 bf16 bit patterns (numpy) or a torch bf16 tensor."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint16))


# ---------------------------------------------------------------- formats
def bf16_to_f32(h: int) -> float:
    return float(lib().or_bf16_to_f32(int(h)))


def f32_to_bf16(f: float) -> int:
    return int(lib().or_f32_to_bf16(float(f)))


def e4m3_value(code: int) -> float:
    return float(lib().or_e4m3_value(int(code)))


def e4m3_from_f32(r: float) -> int:
    return int(lib().or_e4m3_from_f32(float(r)))


# ---------------------------------------------------------------- tables
def tables_check(tables) -> int:
    b = _blob(tables)
    return int(lib().or_tables_check(_ptr(b)))


def canonical_codes(tables, p: int, h: int) -> np.ndarray:
    b = _blob(tables)
    out = np.zeros(NSYM, dtype=np.uint32)
    lib().or_canonical_codes(_ptr(b), p, h, _ptr(out))
    return out


# ---------------------------------------------------------------- codec
G_ACT = 64          # R25: activation groups (2x format)
SELECT_MINMAX = 0   # R8: min/max squared error (the method)
SELECT_MSE = 1      # R23: full squared error, pairwise fp32 sum


def encode_group(tables, x, force_p: int = -1, force_h: int = -1, select: int = SELECT_MINMAX,
                 npat: int = NPAT, gs: int = G):
    """One group: returns (block bytes [64] uint8, GroupInfo).  `select` and
    `npat` (patterns searched, R24) pick the selection variant; gs = 64 is
    the activation format (R25)."""
    b = _blob(tables)
    xb = _bits(x).reshape(-1)
    assert gs in (G, G_ACT) and xb.size == gs and 1 <= npat <= NPAT
    blk = np.zeros(BLOCK_BYTES, dtype=np.uint8)
    info = GroupInfo()
    lib().or_encode_group_gs(_ptr(b), _ptr(xb), _ptr(blk), ctypes.byref(info), gs, select, npat, force_p, force_h)
    return blk, info


def decode_block(tables, blk, gs: int = G) -> tuple[np.ndarray, int]:
    b = _blob(tables)
    bb = np.ascontiguousarray(np.asarray(blk, dtype=np.uint8).reshape(-1))
    assert bb.size == BLOCK_BYTES and gs in (G, G_ACT)
    y = np.zeros(gs, dtype=np.uint16)
    k = lib().or_decode_block_gs(_ptr(b), _ptr(bb), _ptr(y), gs)
    return y, int(k)


def encode(tables, x, with_mse: bool = False, nthreads: int = 1, select: int = SELECT_MINMAX,
           npat: int = NPAT, gs: int = G):
    """x: [..., 128*k] bf16 bits, contiguous groups.  Returns (blocks [n,64], Stats).
    With with_mse, Stats.mse_minmax is the fp64 squared error of the chosen
    patterns (whatever `select`), mse_full that of the fp64-best of all 64."""
    b = _blob(tables)
    xb = _bits(x).reshape(-1)
    assert gs in (G, G_ACT) and xb.size % gs == 0 and 1 <= npat <= NPAT
    n = xb.size // gs
    blocks = np.zeros((n, BLOCK_BYTES), dtype=np.uint8)
    st = Stats()
    lib().or_encode_gs(_ptr(b), _ptr(xb), n, _ptr(blocks), ctypes.byref(st), int(with_mse), nthreads,
                       select, npat, gs)
    return blocks, st


def decode(tables, blocks, nthreads: int = 1, gs: int = G) -> np.ndarray:
    """blocks: [n, 64] uint8.  Returns bf16 bits [n, gs] uint16."""
    b = _blob(tables)
    bb = np.ascontiguousarray(np.asarray(blocks, dtype=np.uint8).reshape(-1, BLOCK_BYTES))
    assert gs in (G, G_ACT)
    n = bb.shape[0]
    y = np.zeros((n, gs), dtype=np.uint16)
    lib().or_decode_gs(_ptr(b), _ptr(bb), n, _ptr(y), nthreads, gs)
    return y


def gemv(tables, blocks, rows: int, cols: int, x):
    """y[b, r] = sum_k W~[r, k] x[b, k] in fp64; also returns sum_k |W~ x|."""
    b = _blob(tables)
    bb = np.ascontiguousarray(np.asarray(blocks, dtype=np.uint8).reshape(-1))
    assert bb.size == rows * (cols // G) * BLOCK_BYTES
    xb = _bits(x).reshape(-1, cols)
    batch = xb.shape[0]
    y = np.zeros((batch, rows), dtype=np.float64)
    ya = np.zeros((batch, rows), dtype=np.float64)
    lib().or_gemv(_ptr(b), _ptr(bb), rows, cols, _ptr(xb), batch, _ptr(y), _ptr(ya))
    return y, ya


def attention(k_tables, v_tables, k_blocks, v_blocks, q, seq_len: int, scale: float, nthreads: int = 1):
    """Decode-phase attention over a compressed KV cache, in fp64.

    k_blocks / v_blocks: [B, Hkv, S_cap, 64] uint8 (token s of head h at [b, h, s]);
    q: bf16 bits [B, Hkv * G, 128] (query head j uses KV head j // G).
    K~, V~ are this oracle's decoded bf16 values; then, per query head,
    softmax over the first seq_len tokens of (q . k~) * scale, and out = sum p v~.
    Returns (out [B, Hq, 128] fp64, abs_weighted [B, Hq, 128] = sum_s p_s |v~_s|).
    nthreads: threads for the block decoding (the attention itself is numpy)."""
    kb = np.ascontiguousarray(np.asarray(k_blocks, dtype=np.uint8))
    vb = np.ascontiguousarray(np.asarray(v_blocks, dtype=np.uint8))
    B, H, _, _ = kb.shape
    qb = _bits(q).reshape(B, -1, G)
    Hq = qb.shape[1]
    grp = Hq // H
    out = np.zeros((B, Hq, G))
    aw = np.zeros((B, Hq, G))
    for b in range(B):
        for h in range(H):
            K = decode(k_tables, kb[b, h, :seq_len], nthreads).astype(np.uint32) << 16
            V = decode(v_tables, vb[b, h, :seq_len], nthreads).astype(np.uint32) << 16
            Kf = K.view(np.float32).astype(np.float64)
            Vf = V.view(np.float32).astype(np.float64)
            for j in range(h * grp, (h + 1) * grp):
                qf = (qb[b, j].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                s = (Kf @ qf) * scale
                p = np.exp(s - s.max())
                p /= p.sum()
                out[b, j] = p @ Vf
                aw[b, j] = p @ np.abs(Vf)
    return out, aw
