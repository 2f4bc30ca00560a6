"""Ecco 512-bit block codec for LLM tensors on B200 (sm_100a).

Thin PyTorch binding over libecco_b200.so (include/ecco.h): it only turns
tensors into device pointers and the current CUDA stream into a handle.  Every
step of encode, decode and decode+GEMV runs in the library's kernels; there is
no CPU or eager-PyTorch fallback.

Method: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression" (arXiv 2505.06901), review page sections
"What carries the argument" and "Core claim".
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import EccoError, Desc, Segment, STATS_FIELDS

GROUP = 128
GROUP_ACT = 64  # activation format: 64 values per 64-byte block
BLOCK_BYTES = 64

__all__ = ["Tables", "encode", "decode", "decode_gemv", "decode_multi", "encode_multi",
           "Prepared", "prepare_encode", "prepare_decode",
           "decode_attention", "attention_workspace_bytes", "decode_attention_static",
           "decode_attention_staged", "attention_staged_workspace_bytes",
           "encode_act", "decode_act", "GROUP_ACT", "learn_tables", "huffman_lengths",
           "new_stats", "read_stats", "flat_desc", "kv_append_desc", "EccoError", "Desc"]


class Tables:
    """Device-resident tables of one tensor, built from a table blob (bytes)."""

    def __init__(self, blob: bytes, device=None):
        lib = _lib.load()
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        if dev.type != "cuda":
            raise ValueError("tables live on a CUDA device")
        self.device = dev
        buf = ctypes.create_string_buffer(bytes(blob), len(blob))
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _lib.check(lib.ecco_tables_create(buf, len(blob), ctypes.byref(h)), "ecco_tables_create")
        self._h = h
        self.blob = bytes(blob)

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise ValueError("tables destroyed")
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None:
            with torch.cuda.device(self.device):
                _lib.load().ecco_tables_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _stream(dev) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def flat_desc(n_groups: int) -> Desc:
    return Desc(1, int(n_groups), int(n_groups), int(n_groups), 0, 0)


def kv_append_desc(rows: int, new_tokens: int, total_tokens: int, start: int) -> Desc:
    """Encode [rows, new_tokens] groups from a contiguous tensor into token
    positions start..start+new_tokens of a [rows, total_tokens] block cache."""
    return Desc(int(rows), int(new_tokens), int(new_tokens), int(total_tokens), 0, int(start))


def _check_tensor(t: torch.Tensor, dtype, name: str, device):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise TypeError(f"{name} must be a {dtype} tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, tables on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def new_stats(device) -> torch.Tensor:
    """A zeroed device buffer for ecco_stats (8 x u64)."""
    return torch.zeros(len(STATS_FIELDS), dtype=torch.int64, device=device)


def read_stats(stats: torch.Tensor) -> dict:
    v = stats.cpu().tolist()
    return {k: int(x) for k, x in zip(STATS_FIELDS, v)}


def encode(x: torch.Tensor, tables: Tables, out: torch.Tensor | None = None,
           stats: torch.Tensor | None = None, desc: Desc | None = None, select: int = _lib.SELECT_MINMAX,
           n_patterns: int = 64) -> torch.Tensor:
    """bf16 groups of 128 -> uint8 blocks [n_groups, 64].  With `desc`, `x` and
    `out` are the full source / destination buffers the descriptor indexes.
    `select` / `n_patterns` choose the pattern-selection variant
    (ecco_select_encode_ex); the defaults are the method's own."""
    _check_tensor(x, torch.bfloat16, "x", tables.device)
    if desc is None:
        if x.numel() % GROUP:
            raise ValueError("x.numel() must be a multiple of 128")
        desc = flat_desc(x.numel() // GROUP)
    if out is None:
        if desc.rows * desc.groups_per_row != x.numel() // GROUP or desc.dst_offset:
            raise ValueError("pass `out` when the descriptor does not map x one-to-one")
        out = torch.empty((x.numel() // GROUP, BLOCK_BYTES), dtype=torch.uint8, device=x.device)
    _check_tensor(out, torch.uint8, "out", tables.device)
    _bounds(desc, x.numel() // GROUP, out.numel() // BLOCK_BYTES)
    sp = ctypes.c_void_p(stats.data_ptr()) if stats is not None else None
    if select == _lib.SELECT_MINMAX and n_patterns == 64:
        rc = _lib.load().ecco_select_encode(tables.handle, ctypes.c_void_p(x.data_ptr()), desc,
                                            ctypes.c_void_p(out.data_ptr()), sp, _stream(x.device))
        _lib.check(rc, "ecco_select_encode")
    else:
        rc = _lib.load().ecco_select_encode_ex(tables.handle, ctypes.c_void_p(x.data_ptr()), desc,
                                               ctypes.c_void_p(out.data_ptr()), sp, int(select), int(n_patterns),
                                               _stream(x.device))
        _lib.check(rc, "ecco_select_encode_ex")
    return out


def decode(blocks: torch.Tensor, tables: Tables, out: torch.Tensor | None = None,
           desc: Desc | None = None, speculative: bool = False) -> torch.Tensor:
    """uint8 blocks [n, 64] -> bf16 [n, 128].  speculative=True runs the
    warp-parallel decoder (ecco_decode_speculative): same output."""
    _check_tensor(blocks, torch.uint8, "blocks", tables.device)
    n_blocks = blocks.numel() // BLOCK_BYTES
    if desc is None:
        desc = flat_desc(n_blocks)
    if out is None:
        out = torch.empty((desc.rows * desc.groups_per_row, GROUP), dtype=torch.bfloat16, device=blocks.device)
    _check_tensor(out, torch.bfloat16, "out", tables.device)
    _bounds(desc, n_blocks, out.numel() // GROUP)
    fn = "ecco_decode_speculative" if speculative else "ecco_decode"
    rc = getattr(_lib.load(), fn)(tables.handle, ctypes.c_void_p(blocks.data_ptr()), desc,
                                  ctypes.c_void_p(out.data_ptr()), _stream(blocks.device))
    _lib.check(rc, fn)
    return out


def decode_gemv(blocks: torch.Tensor, tables: Tables, rows: int, cols: int, x: torch.Tensor,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """y[b, r] = sum_k W~[r, k] x[b, k] (fp32), W~ the decoded rows x cols matrix."""
    _check_tensor(blocks, torch.uint8, "blocks", tables.device)
    _check_tensor(x, torch.bfloat16, "x", tables.device)
    if x.dim() == 1:
        x = x.view(1, -1)
    batch = x.shape[0]
    if x.shape[1] != cols or blocks.numel() != rows * (cols // GROUP) * BLOCK_BYTES:
        raise ValueError("shape mismatch")
    if out is None:
        out = torch.empty((batch, rows), dtype=torch.float32, device=x.device)
    _check_tensor(out, torch.float32, "out", tables.device)
    rc = _lib.load().ecco_decode_gemv(tables.handle, ctypes.c_void_p(blocks.data_ptr()), rows, cols,
                                      ctypes.c_void_p(x.data_ptr()), batch,
                                      ctypes.c_void_p(out.data_ptr()), _stream(x.device))
    _lib.check(rc, "ecco_decode_gemv")
    return out


def attention_workspace_bytes(batch: int, kv_heads: int, group: int, seq_len: int) -> int:
    return int(_lib.load().ecco_decode_attention_workspace_bytes(batch, kv_heads, group, seq_len))


def attention_staged_workspace_bytes(batch: int, kv_heads: int, group: int, seq_len: int) -> int:
    return int(_lib.load().ecco_decode_attention_staged_workspace_bytes(batch, kv_heads, group, seq_len))


def decode_attention(k_blocks: torch.Tensor, v_blocks: torch.Tensor, k_tables: Tables, v_tables: Tables,
                     q: torch.Tensor, seq_len: int, scale: float, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Decode-phase attention over a compressed KV cache.

    k_blocks / v_blocks: uint8 [B, Hkv, S_cap, 64]; q: bf16 [B, Hkv * G, 128].
    Returns fp32 [B, Hkv * G, 128]: softmax over the first seq_len tokens of
    scale * q . K~, applied to V~ (K~, V~ decoded inside the kernel)."""
    return _attention("ecco_decode_attention", attention_workspace_bytes, k_blocks, v_blocks, k_tables,
                      v_tables, q, seq_len, scale, out, workspace)


def decode_attention_staged(k_blocks: torch.Tensor, v_blocks: torch.Tensor, k_tables: Tables, v_tables: Tables,
                            q: torch.Tensor, seq_len: int, scale: float, out: torch.Tensor | None = None,
                            workspace: torch.Tensor | None = None) -> torch.Tensor:
    """decode_attention computed in stages: each chunk of tokens is decoded by
    the block decoder into a scratch in the workspace, then attended.  Same
    arguments and result.  The workspace holds a chunk's decoded K and V rows
    (up to 1 GiB, attention_staged_workspace_bytes); pass one to reuse it
    across calls."""
    return _attention("ecco_decode_attention_staged", attention_staged_workspace_bytes, k_blocks, v_blocks,
                      k_tables, v_tables, q, seq_len, scale, out, workspace)


def _attention(fn, ws_bytes, k_blocks, v_blocks, k_tables, v_tables, q, seq_len, scale, out, workspace):
    _check_tensor(k_blocks, torch.uint8, "k_blocks", k_tables.device)
    _check_tensor(v_blocks, torch.uint8, "v_blocks", v_tables.device)
    _check_tensor(q, torch.bfloat16, "q", k_tables.device)
    if k_blocks.dim() != 4 or k_blocks.shape[-1] != BLOCK_BYTES or v_blocks.shape != k_blocks.shape:
        raise ValueError("k_blocks / v_blocks must be [B, Hkv, S_cap, 64] of the same shape")
    B, H, s_cap, _ = k_blocks.shape
    if q.dim() != 3 or q.shape[0] != B or q.shape[2] != GROUP or q.shape[1] % H:
        raise ValueError("q must be [B, Hkv * G, 128]")
    G = q.shape[1] // H
    if out is None:
        out = torch.empty((B, H * G, GROUP), dtype=torch.float32, device=q.device)
    _check_tensor(out, torch.float32, "out", k_tables.device)
    need = ws_bytes(B, H, G, seq_len)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check_tensor(workspace, torch.uint8, "workspace", k_tables.device)
    rc = getattr(_lib.load(), fn)(
        k_tables.handle, v_tables.handle, ctypes.c_void_p(k_blocks.data_ptr()),
        ctypes.c_void_p(v_blocks.data_ptr()), s_cap, B, H, G, int(seq_len), ctypes.c_void_p(q.data_ptr()),
        float(scale), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel(), _stream(q.device))
    _lib.check(rc, fn)
    return out


def decode_attention_static(k_blocks: torch.Tensor, v_blocks: torch.Tensor, k_tables: Tables, v_tables: Tables,
                            q: torch.Tensor, seq_len: int, scale: float,
                            out: torch.Tensor | None = None) -> torch.Tensor:
    """decode_attention with the library's static device workspace (no
    workspace argument, nothing allocated by the call when `out` is given).
    Calls that can overlap on one device race on that workspace."""
    _check_tensor(k_blocks, torch.uint8, "k_blocks", k_tables.device)
    _check_tensor(v_blocks, torch.uint8, "v_blocks", v_tables.device)
    _check_tensor(q, torch.bfloat16, "q", k_tables.device)
    if k_blocks.dim() != 4 or k_blocks.shape[-1] != BLOCK_BYTES or v_blocks.shape != k_blocks.shape:
        raise ValueError("k_blocks / v_blocks must be [B, Hkv, S_cap, 64] of the same shape")
    B, H, s_cap, _ = k_blocks.shape
    if q.dim() != 3 or q.shape[0] != B or q.shape[2] != GROUP or q.shape[1] % H:
        raise ValueError("q must be [B, Hkv * G, 128]")
    G = q.shape[1] // H
    if out is None:
        out = torch.empty((B, H * G, GROUP), dtype=torch.float32, device=q.device)
    _check_tensor(out, torch.float32, "out", k_tables.device)
    rc = _lib.load().ecco_decode_attention_static(
        k_tables.handle, v_tables.handle, ctypes.c_void_p(k_blocks.data_ptr()),
        ctypes.c_void_p(v_blocks.data_ptr()), s_cap, B, H, G, int(seq_len), ctypes.c_void_p(q.data_ptr()),
        float(scale), ctypes.c_void_p(out.data_ptr()), _stream(q.device))
    _lib.check(rc, "ecco_decode_attention_static")
    return out


def encode_act(x: torch.Tensor, tables: Tables, out: torch.Tensor | None = None,
               stats: torch.Tensor | None = None, desc: Desc | None = None) -> torch.Tensor:
    """Activation format: bf16 groups of 64 -> uint8 blocks [n_groups, 64]."""
    _check_tensor(x, torch.bfloat16, "x", tables.device)
    if desc is None:
        if x.numel() % GROUP_ACT:
            raise ValueError("x.numel() must be a multiple of 64")
        desc = flat_desc(x.numel() // GROUP_ACT)
    if out is None:
        if desc.rows * desc.groups_per_row != x.numel() // GROUP_ACT or desc.dst_offset:
            raise ValueError("pass `out` when the descriptor does not map x one-to-one")
        out = torch.empty((x.numel() // GROUP_ACT, BLOCK_BYTES), dtype=torch.uint8, device=x.device)
    _check_tensor(out, torch.uint8, "out", tables.device)
    _bounds(desc, x.numel() // GROUP_ACT, out.numel() // BLOCK_BYTES)
    sp = ctypes.c_void_p(stats.data_ptr()) if stats is not None else None
    rc = _lib.load().ecco_select_encode_act(tables.handle, ctypes.c_void_p(x.data_ptr()), desc,
                                            ctypes.c_void_p(out.data_ptr()), sp, _stream(x.device))
    _lib.check(rc, "ecco_select_encode_act")
    return out


def decode_act(blocks: torch.Tensor, tables: Tables, out: torch.Tensor | None = None,
               desc: Desc | None = None) -> torch.Tensor:
    """Activation format: uint8 blocks [n, 64] -> bf16 [n, 64]."""
    _check_tensor(blocks, torch.uint8, "blocks", tables.device)
    n_blocks = blocks.numel() // BLOCK_BYTES
    if desc is None:
        desc = flat_desc(n_blocks)
    if out is None:
        out = torch.empty((desc.rows * desc.groups_per_row, GROUP_ACT), dtype=torch.bfloat16, device=blocks.device)
    _check_tensor(out, torch.bfloat16, "out", tables.device)
    _bounds(desc, n_blocks, out.numel() // GROUP_ACT)
    rc = _lib.load().ecco_decode_act(tables.handle, ctypes.c_void_p(blocks.data_ptr()), desc,
                                     ctypes.c_void_p(out.data_ptr()), _stream(blocks.device))
    _lib.check(rc, "ecco_decode_act")
    return out


def learn_tables(sample: torch.Tensor, seed: int = 0, n_patterns: int = 64, group: int = GROUP) -> bytes:
    """Table blob learned on the GPU (ecco_learn_tables) from a bf16 device
    tensor whose numel is a multiple of `group` (128, or 64 for activations)."""
    if not isinstance(sample, torch.Tensor) or sample.dtype != torch.bfloat16 or sample.device.type != "cuda":
        raise TypeError("sample must be a bf16 CUDA tensor")
    x = sample.contiguous()
    if x.numel() % group:
        raise ValueError(f"sample.numel() must be a multiple of {group}")
    blob = ctypes.create_string_buffer(_lib.TABLES_BYTES)
    with torch.cuda.device(x.device):
        rc = _lib.load().ecco_learn_tables(ctypes.c_void_p(x.data_ptr()), x.numel() // group, group, n_patterns,
                                           int(seed) & (2 ** 64 - 1), blob, _lib.TABLES_BYTES, _stream(x.device))
    _lib.check(rc, "ecco_learn_tables")
    return blob.raw


def huffman_lengths(weights, max_len: int = 8):
    """Optimal length-limited prefix-code lengths (package-merge, host)."""
    import numpy as np
    w = np.ascontiguousarray(np.asarray(weights, dtype=np.float64))
    out = np.zeros(w.size, dtype=np.uint8)
    rc = _lib.load().ecco_huffman_lengths(ctypes.c_void_p(w.ctypes.data), w.size, max_len,
                                          ctypes.c_void_p(out.ctypes.data))
    _lib.check(rc, "ecco_huffman_lengths")
    return out


@dataclass
class Seg:
    tables: Tables
    src: torch.Tensor
    dst: torch.Tensor
    desc: Desc | None = None


def _segments(segs, src_dtype, dst_dtype, src_unit, dst_unit):
    arr = (Segment * max(1, len(segs)))()
    for i, s in enumerate(segs):
        _check_tensor(s.src, src_dtype, "src", s.tables.device)
        _check_tensor(s.dst, dst_dtype, "dst", s.tables.device)
        d = s.desc or flat_desc(s.src.numel() // src_unit)
        _bounds(d, s.src.numel() // src_unit, s.dst.numel() // dst_unit)
        arr[i] = Segment(s.tables.handle, s.src.data_ptr(), s.dst.data_ptr(), d)
    return arr


class Prepared:
    """Segments checked and marshalled once, for a multi-segment call repeated
    on the same buffers (a per-token KV append over every layer): the call then
    only passes the prepared array and the current stream.  It keeps the
    tensors and tables alive; their contents may change between calls, their
    storage may not."""

    def __init__(self, segs: list[Seg], kind: str):
        if kind not in ("encode", "decode"):
            raise ValueError("kind is 'encode' or 'decode'")
        self.kind, self.segs = kind, list(segs)
        if kind == "encode":
            self.arr = _segments(self.segs, torch.bfloat16, torch.uint8, GROUP, BLOCK_BYTES)
        else:
            self.arr = _segments(self.segs, torch.uint8, torch.bfloat16, BLOCK_BYTES, GROUP)
        self.device = self.segs[0].tables.device if self.segs else None

    def __len__(self):
        return len(self.segs)


def prepare_encode(segs: list[Seg]) -> Prepared:
    return Prepared(segs, "encode")


def prepare_decode(segs: list[Seg]) -> Prepared:
    return Prepared(segs, "decode")


def _marshalled(segs, kind, src_dtype, dst_dtype, src_unit, dst_unit):
    if isinstance(segs, Prepared):
        if segs.kind != kind:
            raise ValueError(f"segments prepared for {segs.kind}, not {kind}")
        return segs.arr, len(segs), segs.device
    return _segments(segs, src_dtype, dst_dtype, src_unit, dst_unit), len(segs), segs[0].tables.device


def decode_multi(segs: list[Seg] | Prepared) -> None:
    if not len(segs):
        return
    arr, n, dev = _marshalled(segs, "decode", torch.uint8, torch.bfloat16, BLOCK_BYTES, GROUP)
    rc = _lib.load().ecco_decode_multi(arr, n, _stream(dev))
    _lib.check(rc, "ecco_decode_multi")


def encode_multi(segs: list[Seg] | Prepared, stats: torch.Tensor | None = None) -> None:
    if not len(segs):
        return
    arr, n, dev = _marshalled(segs, "encode", torch.bfloat16, torch.uint8, GROUP, BLOCK_BYTES)
    sp = ctypes.c_void_p(stats.data_ptr()) if stats is not None else None
    rc = _lib.load().ecco_encode_multi(arr, n, sp, _stream(dev))
    _lib.check(rc, "ecco_encode_multi")


def _bounds(d: Desc, n_src: int, n_dst: int) -> None:
    """Host-side check that the descriptor stays inside both buffers."""
    if d.rows == 0 or d.groups_per_row == 0:
        return
    last_src = d.src_offset + (d.rows - 1) * d.src_row_stride + d.groups_per_row
    last_dst = d.dst_offset + (d.rows - 1) * d.dst_row_stride + d.groups_per_row
    if min(d.rows, d.groups_per_row, d.src_row_stride, d.dst_row_stride, d.src_offset, d.dst_offset) < 0:
        raise ValueError("negative descriptor field")
    if last_src > n_src or last_dst > n_dst:
        raise ValueError(f"descriptor exceeds buffers (src {last_src}>{n_src} or dst {last_dst}>{n_dst})")
