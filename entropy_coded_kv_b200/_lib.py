"""ctypes declarations of libecco_b200.so (include/ecco.h).  No fallback: if the
library is missing or fails to load, importing the package raises."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libecco_b200.so")

ECCO_OK = 0
ECCO_ERR_ARG = -1
ECCO_ERR_ALIGN = -2
ECCO_ERR_TABLES = -3
ECCO_ERR_CUDA = -4
ECCO_ERR_DEVICE = -5
ECCO_ERR_UNSUPPORTED = -6
ECCO_ERR_WORKSPACE = -7
ECCO_ERR_TIMEOUT = -8
ATTENTION_STATIC_WS_BYTES = 4 << 20
SELECT_MINMAX = 0
SELECT_MSE = 1
TABLES_BYTES = 7952
MAX_SEGMENTS = 256

EXPORTED = [
    "ecco_tables_create", "ecco_tables_destroy", "ecco_select_encode", "ecco_decode", "ecco_decode_speculative",
    "ecco_decode_gemv", "ecco_decode_multi", "ecco_encode_multi", "ecco_strerror",
    "ecco_abi_version", "ecco_device_timeouts", "ecco_decode_attention",
    "ecco_decode_attention_workspace_bytes", "ecco_decode_attention_static", "ecco_select_encode_ex",
    "ecco_select_encode_act", "ecco_decode_act", "ecco_learn_tables", "ecco_huffman_lengths",
    "ecco_decode_attention_staged", "ecco_decode_attention_staged_workspace_bytes",
    "ecco_selftest_wait_timeout",
]


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "rows", "groups_per_row", "src_row_stride", "dst_row_stride", "src_offset", "dst_offset")]


class Segment(ctypes.Structure):
    _fields_ = [("tables", ctypes.c_void_p), ("src", ctypes.c_void_p), ("dst", ctypes.c_void_p),
                ("desc", Desc)]


STATS_FIELDS = ["n_groups", "n_zero", "n_clipped", "n_padded", "n_records", "n_nonfinite",
                "payload_bits", "reserved"]


class EccoError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} ({code})")
        self.code = code


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libecco_b200.so not built ({path}); run entropy_coded_kv_b200/build.py")
    L = ctypes.CDLL(path)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.ecco_tables_create.argtypes = [P, ctypes.c_size_t, ctypes.POINTER(P)]
    L.ecco_tables_destroy.argtypes = [P]
    L.ecco_select_encode.argtypes = [P, P, Desc, P, P, P]
    L.ecco_decode.argtypes = [P, P, Desc, P, P]
    L.ecco_decode_speculative.argtypes = [P, P, Desc, P, P]
    L.ecco_select_encode_ex.argtypes = [P, P, Desc, P, P, I, I, P]
    L.ecco_select_encode_act.argtypes = [P, P, Desc, P, P, P]
    L.ecco_learn_tables.argtypes = [P, I64, I, I, ctypes.c_uint64, P, ctypes.c_size_t, P]
    L.ecco_huffman_lengths.argtypes = [P, I, I, P]
    L.ecco_decode_act.argtypes = [P, P, Desc, P, P]
    L.ecco_decode_gemv.argtypes = [P, P, I64, I64, P, I, P, P]
    L.ecco_decode_multi.argtypes = [ctypes.POINTER(Segment), I, P]
    L.ecco_encode_multi.argtypes = [ctypes.POINTER(Segment), I, P, P]
    L.ecco_strerror.argtypes = [I]
    L.ecco_strerror.restype = ctypes.c_char_p
    L.ecco_abi_version.argtypes = []
    L.ecco_device_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    L.ecco_selftest_wait_timeout.argtypes = [P]
    L.ecco_decode_attention_workspace_bytes.argtypes = [I, I, I, I]
    L.ecco_decode_attention_static.argtypes = [P, P, P, P, I64, I, I, I, I, P, ctypes.c_float, P, P]
    L.ecco_decode_attention.argtypes = [P, P, P, P, I64, I, I, I, I, P, ctypes.c_float, P, P,
                                        ctypes.c_size_t, P]
    L.ecco_decode_attention_staged_workspace_bytes.argtypes = [I, I, I, I]
    L.ecco_decode_attention_staged.argtypes = L.ecco_decode_attention.argtypes
    sizes = ("ecco_decode_attention_workspace_bytes", "ecco_decode_attention_staged_workspace_bytes")
    for fn in EXPORTED:
        if fn != "ecco_strerror" and fn not in sizes:
            getattr(L, fn).restype = I
    for fn in sizes:
        getattr(L, fn).restype = ctypes.c_size_t
    _lib = L
    return L


def strerror(code: int) -> str:
    return load().ecco_strerror(int(code)).decode()


def check(code: int, what: str) -> None:
    if code != ECCO_OK:
        raise EccoError(code, what)
