"""Seeded synthetic inputs shared by the tests, the smoke check and bench.py.

This module holds no arithmetic of the codec.  It makes random tensors with the
shapes and value distributions of the five workloads, packs table blobs (a file
format), and draws random *valid* table sets (sorted centroids, complete prefix
codes) for adversarial parity cases.

Workloads (shapes from the Llama-3-8B family; the review page's own data --
LLaMA/Mistral weights, a Pile calibration set -- is not available here and these
synthetic inputs stand in for it):

  c1  one 256 x 1024 matrix, N(0, 0.02^2), exactly round(0.001 N) entries set to
      +-0.4 (+-20 sigma, random sign), seed 0.
  c2  one layer's KV cache, K and V each [8, 8, 4096, 128] (batch, KV heads,
      tokens, head_dim): N(0, 1) times a per-(tensor, head, channel)
      LogNormal(0, 0.5) scale, with 4 of 128 channels per (tensor, head) times 15,
      seed 1.  Calibration sample: same distribution, seed 2.
  c3  one MLP weight 14336 x 4096, Student-t(5) * 0.02, seed 3; activation x and
      a batch-16 X drawn N(0, 1).
  c4  32 layers x {q, k, v, o, gate, up, down} with Llama-3-8B shapes,
      Student-t(5) * 0.02, seed 4.
  c5  32 layers x {K, V} x [1, 8, 131072, 128] with the c2 distribution, seed 5;
      per-layer calibration samples [1, 8, 4096, 128], seed 105.
"""
from __future__ import annotations

import struct

import numpy as np
import torch

G = 128
NPAT = 64
NCENT = 15
NBOOK = 4
NSYM = 16
LMAX = 8
TABLES_MAGIC = 0x31434345  # "ECC1"
TABLES_VERSION = 1
TABLES_BYTES = 16 + NPAT * NCENT * 4 + NPAT * NBOOK * NSYM

C4_SHAPES = [
    ("q", 4096, 4096),
    ("k", 1024, 4096),
    ("v", 1024, 4096),
    ("o", 4096, 4096),
    ("gate", 14336, 4096),
    ("up", 14336, 4096),
    ("down", 4096, 14336),
]
C4_LAYERS = 32


# ------------------------------------------------------------------ tables blob
def pack_tables(S_t: float, C: np.ndarray, lens: np.ndarray) -> bytes:
    """Serialises a table set: header, fp32 centroids [64][15], u8 lengths [64][4][16]."""
    C = np.ascontiguousarray(np.asarray(C, dtype=np.float32).reshape(NPAT, NCENT))
    lens = np.ascontiguousarray(np.asarray(lens, dtype=np.uint8).reshape(NPAT, NBOOK, NSYM))
    hdr = struct.pack("<IIfI", TABLES_MAGIC, TABLES_VERSION, float(np.float32(S_t)), 0)
    out = hdr + C.tobytes() + lens.tobytes()
    assert len(out) == TABLES_BYTES
    return out


def unpack_tables(blob: bytes):
    magic, ver, st, _ = struct.unpack_from("<IIfI", blob, 0)
    C = np.frombuffer(blob, dtype=np.float32, count=NPAT * NCENT, offset=16).reshape(NPAT, NCENT)
    lens = np.frombuffer(blob, dtype=np.uint8, count=NPAT * NBOOK * NSYM,
                         offset=16 + NPAT * NCENT * 4).reshape(NPAT, NBOOK, NSYM)
    return magic, ver, np.float32(st), C.copy(), lens.copy()


def random_complete_lengths(rng: np.random.Generator, nsym: int = NSYM, lmax: int = LMAX) -> np.ndarray:
    """Random code-length vector of a complete binary prefix code (Kraft sum 1)
    with every length in 1..lmax: grow a random full binary tree with nsym
    leaves by splitting random leaves that are shallower than lmax."""
    depths = [0]
    while len(depths) < nsym:
        cand = [i for i, d in enumerate(depths) if d < lmax]
        i = cand[int(rng.integers(len(cand)))]
        d = depths.pop(i)
        depths += [d + 1, d + 1]
    depths = np.array(depths, dtype=np.uint8)
    rng.shuffle(depths)
    return depths


def random_tables(seed: int, S_t: float | None = None, spread: float = 1.0) -> bytes:
    """A random valid table set: strictly increasing centroids in about
    (-spread, spread), random complete codes with lengths 1..8."""
    rng = np.random.default_rng(seed)
    C = np.zeros((NPAT, NCENT), dtype=np.float32)
    for p in range(NPAT):
        while True:
            c = np.sort(rng.uniform(-spread, spread, NCENT)).astype(np.float32)
            if np.all(np.diff(c) > 0):
                break
        C[p] = c
    lens = np.zeros((NPAT, NBOOK, NSYM), dtype=np.uint8)
    for p in range(NPAT):
        for h in range(NBOOK):
            lens[p, h] = random_complete_lengths(rng)
    if S_t is None:
        S_t = float(rng.uniform(1e-4, 1e-2))
    return pack_tables(S_t, C, lens)


# ------------------------------------------------------------------ samplers
def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def student_t(shape, df: int, g: torch.Generator, device) -> torch.Tensor:
    """Student-t with integer df: z0 / sqrt(sum_{i=1..df} z_i^2 / df), fp32."""
    z0 = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(df):
        z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        chi.addcmul_(z, z)
    return z0 / torch.sqrt(chi / df)


def c1_matrix(device="cpu", seed: int = 0, rows: int = 256, cols: int = 1024) -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn(rows * cols, generator=g, device=device, dtype=torch.float32) * 0.02
    n_out = int(round(0.001 * rows * cols))
    idx = torch.randperm(rows * cols, generator=g, device=device)[:n_out]
    sign = torch.randint(0, 2, (n_out,), generator=g, device=device).float() * 2 - 1
    x[idx] = 0.4 * sign
    return x.reshape(rows, cols).to(torch.bfloat16)


def kv_cache(shape, seed: int, device="cpu", n_outlier_ch: int = 4, outlier_mult: float = 15.0,
             sigma: float = 0.5) -> tuple[torch.Tensor, torch.Tensor]:
    """(K, V), each `shape` = [B, H, S, D]: N(0,1) times a per-(tensor, head,
    channel) LogNormal(0, sigma) scale; n_outlier_ch channels per (tensor, head)
    are multiplied by outlier_mult."""
    B, H, S, D = shape
    g = _gen(seed, device)
    out = []
    for _t in range(2):
        scale = torch.exp(torch.randn(H, D, generator=g, device=device) * sigma)
        for h in range(H):
            ch = torch.randperm(D, generator=g, device=device)[:n_outlier_ch]
            scale[h, ch] *= outlier_mult
        z = torch.randn(B, H, S, D, generator=g, device=device, dtype=torch.float32)
        out.append((z * scale.view(1, H, 1, D)).to(torch.bfloat16))
    return out[0], out[1]


def c2_kv(device="cpu", seed: int = 1, shape=(8, 8, 4096, 128)):
    return kv_cache(shape, seed, device)


def c2_calibration(device="cpu", seed: int = 2, shape=(8, 8, 4096, 128)):
    return kv_cache(shape, seed, device)


def c3_weight(device="cpu", seed: int = 3, rows: int = 14336, cols: int = 4096) -> torch.Tensor:
    g = _gen(seed, device)
    return (student_t((rows, cols), 5, g, device) * 0.02).to(torch.bfloat16)


def activations(n: int, batch: int = 1, device="cpu", seed: int = 33) -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(batch, n, generator=g, device=device).to(torch.bfloat16)


def c4_tensor(layer: int, name: str, device="cpu", seed: int = 4) -> torch.Tensor:
    idx = [n for n, _, _ in C4_SHAPES].index(name)
    _, rows, cols = C4_SHAPES[idx]
    g = _gen(seed * 1000 + layer * len(C4_SHAPES) + idx, device)
    return (student_t((rows, cols), 5, g, device) * 0.02).to(torch.bfloat16)


def c5_layer(layer: int, device="cpu", seed: int = 5, seq: int = 131072):
    return kv_cache((1, 8, seq, 128), seed * 1000 + layer, device)


def c5_calibration(layer: int, device="cpu", seed: int = 105):
    return kv_cache((1, 8, 4096, 128), seed * 1000 + layer, device)


def hidden_states(tokens: int, hidden: int = 4096, seed: int = 6, device="cpu", n_outlier_ch: int = 8,
                  outlier_mult: float = 20.0, sigma: float = 0.5) -> torch.Tensor:
    """Activations [tokens, hidden] bf16 for the 64-value-group format: N(0,1)
    times a per-channel LogNormal(0, sigma) scale, n_outlier_ch channels
    multiplied by outlier_mult (the channel-outlier shape of LLM activations)."""
    g = _gen(seed, device)
    scale = torch.exp(torch.randn(hidden, generator=g, device=device) * sigma)
    ch = torch.randperm(hidden, generator=g, device=device)[:n_outlier_ch]
    scale[ch] *= outlier_mult
    z = torch.randn(tokens, hidden, generator=g, device=device, dtype=torch.float32)
    return (z * scale.view(1, hidden)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
