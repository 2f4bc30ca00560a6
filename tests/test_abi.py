"""The C ABI library loads and exports every entry point include/ecco.h
declares; argument errors come back as codes before any CUDA call (CPU)."""
import ctypes
import os
import re

import pytest

import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200 import _lib
from entropy_coded_kv_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"^\s*(?:int|size_t|const char\s*\*)\s+(ecco_\w+)\s*\(", src, re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert {"ecco_tables_create", "ecco_select_encode", "ecco_decode", "ecco_decode_gemv"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert set(_lib.EXPORTED) == names


def test_header_constants_match_binding(lib):
    src = open(os.path.join(ROOT, "include", "ecco.h")).read()
    assert f"ECCO_TABLES_BYTES {_lib.TABLES_BYTES}u" in src
    consts = {m.group(1): m.group(2) for m in re.finditer(r"#define (ECCO_\w+) \(?(-?[0-9x]+)", src)}
    for name in ("OK", "ERR_ARG", "ERR_ALIGN", "ERR_TABLES", "ERR_CUDA", "ERR_DEVICE", "ERR_UNSUPPORTED",
                 "ERR_WORKSPACE", "ERR_TIMEOUT", "SELECT_MINMAX", "SELECT_MSE"):
        assert int(consts["ECCO_" + name], 0) == getattr(_lib, "ECCO_" + name if name.startswith(("OK", "ERR")) else name), name
    assert "ECCO_ATTENTION_STATIC_WS_BYTES (4u << 20)" in src and _lib.ATTENTION_STATIC_WS_BYTES == 4 << 20
    assert int(consts["ECCO_MAX_SEGMENTS"]) == _lib.MAX_SEGMENTS
    assert int(consts["ECCO_GROUP"]) == ecco.GROUP and int(consts["ECCO_GROUP_ACT"]) == ecco.GROUP_ACT
    assert lib.ecco_abi_version() == 1
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        assert _lib.strerror(code)


def test_argument_errors_need_no_gpu(lib):
    d = _lib.Desc(1, 1, 1, 1, 0, 0)
    assert lib.ecco_decode(None, None, d, None, None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_select_encode(None, None, d, None, None, None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_decode_gemv(None, None, 1, 128, None, 1, None, None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_decode_multi(None, -1, None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_decode_multi(None, 100000, None) == _lib.ECCO_ERR_ARG
    assert lib.ecco_tables_destroy(None) == _lib.ECCO_ERR_ARG
    h = ctypes.c_void_p()
    assert lib.ecco_tables_create(None, 7952, ctypes.byref(h)) == _lib.ECCO_ERR_ARG
    assert lib.ecco_tables_create(b"x" * 10, 10, ctypes.byref(h)) == _lib.ECCO_ERR_TABLES
    assert lib.ecco_decode_attention(None, None, None, None, 64, 1, 1, 1, 1, None, 1.0, None, None, 0,
                                     None) == _lib.ECCO_ERR_ARG
    # workspace: 130 floats (128 partial sums, max, sum) per query head and 512-token split
    assert lib.ecco_decode_attention_workspace_bytes(2, 8, 4, 4096) == 4 * 130 * 2 * 8 * 4 * 8
    assert lib.ecco_decode_attention_workspace_bytes(1, 1, 1, 513) == 4 * 130 * 2
    assert lib.ecco_decode_attention_workspace_bytes(1, 1, 9, 10) == 0
    assert lib.ecco_decode_attention_workspace_bytes(1, 1, 1, 0) == 0
    # staged: partials of 256-token splits rounded up to 256 B, 256 B of slack,
    # then K and V rows of one chunk (a multiple of 512 tokens within 1 GiB, at
    # most the sequence rounded up to 512)
    assert lib.ecco_decode_attention_staged_workspace_bytes(8, 8, 4, 4096) == (
        4 * 130 * 8 * 8 * 4 * 16 + 256 + 2 * 64 * 4096 * 256)
    assert lib.ecco_decode_attention_staged_workspace_bytes(1, 8, 4, 131072) == (
        4 * 130 * 8 * 4 * 512 + 256 + 2 * 8 * 131072 * 256)
    assert lib.ecco_decode_attention_staged_workspace_bytes(64, 32, 1, 8192) == (
        4 * 130 * 64 * 32 * 32 + 256 + 2 * 64 * 32 * 1024 * 256)
    assert lib.ecco_decode_attention_staged_workspace_bytes(1, 1, 1, 513) == 1792 + 256 + 2 * 1024 * 256
    assert lib.ecco_decode_attention_staged_workspace_bytes(1, 1, 9, 10) == 0
    assert lib.ecco_decode_attention_staged(None, None, None, None, 64, 1, 1, 1, 1, None, 1.0, None, None, 0,
                                            None) == _lib.ECCO_ERR_ARG
    bad = bytearray(7952)
    assert lib.ecco_tables_create(bytes(bad), 7952, ctypes.byref(h)) == _lib.ECCO_ERR_TABLES


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "entropy_coded_kv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", src, re.M), f
                assert "ecco_oracle" not in src, f
