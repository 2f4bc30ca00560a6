"""Offline calibration: learns one tensor's table blob from a sample.

The review page ("Ecco: Improving Memory Bandwidth and Capacity for LLMs via
Entropy-aware Cache Compression") says the patterns and codebooks are learned
once, offline, on a calibration set ("What carries the argument"; free
parameters S = 64, H = 4, 15 centroids; referee comment 1: code lengths limited
to 8 bits, with no construction given).  This module is that offline step:
host-side numpy, not on the timed path.  Its construction is this library's own:

  1. S_t = absmax(sample) / 448 (the per-tensor FP16-to-FP8 factor, Fig. 4).
  2. Every sample group is scaled by its FP8 group scale; the element of largest
     magnitude is set aside (it becomes symbol 15).
  3. Each group's 127 remaining values are summarised by 15 equal-count
     quantile means; k-means (k-means++ seeding) over these 15-vectors gives
     64 initial patterns.
  4. Lloyd refinement in the encoder's own terms: groups are assigned to
     patterns by the online min/max rule, values to centroids by thresholds,
     and each centroid moves to the mean of its values.
  5. Per pattern, the symbol histograms of its groups are split into 4
     clusters; each cluster gets an optimal length-limited prefix code
     (package-merge, Larmore & Hirschberg 1990, lengths <= 8, every symbol
     codable), and groups move to the codebook that codes them shortest.
"""
from __future__ import annotations

import numpy as np
import torch

G = 128
NPAT = 64
NCENT = 15
NBOOK = 4
NSYM = 16
LMAX = 8
TABLES_MAGIC = 0x31434345


def package_merge(weights, lmax: int = LMAX) -> np.ndarray:
    """Optimal prefix-code lengths with every length <= lmax (package-merge)."""
    w = [float(v) for v in weights]
    n = len(w)
    if n == 1:
        return np.array([1], dtype=np.uint8)
    if n > (1 << lmax):
        raise ValueError("alphabet too large for the length limit")
    leaves = sorted(((w[i], (i,)) for i in range(n)), key=lambda t: (t[0], t[1]))
    cur = list(leaves)
    for _ in range(lmax - 1):
        pk = [(cur[2 * k][0] + cur[2 * k + 1][0], cur[2 * k][1] + cur[2 * k + 1][1])
              for k in range(len(cur) // 2)]
        merged, a, b = [], 0, 0
        while a < len(leaves) or b < len(pk):
            if b >= len(pk) or (a < len(leaves) and leaves[a][0] <= pk[b][0]):
                merged.append(leaves[a]); a += 1
            else:
                merged.append(pk[b]); b += 1
        cur = merged
    lens = np.zeros(n, dtype=np.int64)
    for _, syms in cur[: 2 * n - 2]:
        for s in syms:
            lens[s] += 1
    return lens.astype(np.uint8)


def _e4m3_round(r: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.clip(r, -448.0, 448.0).astype(np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float32).numpy()


def normalise_groups(X: np.ndarray, S_t: np.float32):
    """Scaled groups: returns (u [n, group] fp32, m [n], keep mask)."""
    mag = np.abs(X)
    m = np.argmax(mag, axis=1)
    xm = X[np.arange(len(X)), m]
    s = (np.float32(S_t) * _e4m3_round(xm / np.float32(S_t))).astype(np.float32)
    keep = s != 0
    u = np.zeros_like(X)
    inv = np.where(keep, np.float32(1.0) / np.where(keep, s, 1), 0).astype(np.float32)
    u[keep] = X[keep] * inv[keep, None]
    return u, m, keep


def _kmeanspp(F: np.ndarray, k: int, rng) -> np.ndarray:
    n = len(F)
    centers = [F[int(rng.integers(n))]]
    d2 = ((F - centers[0]) ** 2).sum(1)
    for _ in range(1, k):
        tot = d2.sum()
        i = int(rng.integers(n)) if tot <= 0 else int(rng.choice(n, p=d2 / tot))
        centers.append(F[i])
        d2 = np.minimum(d2, ((F - F[i]) ** 2).sum(1))
    return np.array(centers, dtype=np.float64)


def _kmeans(F: np.ndarray, k: int, rng, iters: int = 20) -> np.ndarray:
    F64 = F.astype(np.float64)
    C = _kmeanspp(F64, k, rng)
    for _ in range(iters):
        d = (F64 ** 2).sum(1)[:, None] - 2 * F64 @ C.T + (C ** 2).sum(1)[None, :]
        a = np.argmin(d, axis=1)
        for j in range(k):
            sel = a == j
            if sel.any():
                C[j] = F64[sel].mean(0)
            else:
                C[j] = F64[int(rng.integers(len(F64)))]
    return C


def _strictly_increasing(c: np.ndarray) -> np.ndarray:
    c = np.sort(np.clip(c, -4.0, 4.0).astype(np.float32))
    for j in range(1, len(c)):
        if not c[j] > c[j - 1]:
            c[j] = np.nextafter(c[j - 1], np.float32(np.inf))
    return c


def _thresholds(C: np.ndarray) -> np.ndarray:
    return ((C[:, :-1] + C[:, 1:]).astype(np.float32) * np.float32(0.5)).astype(np.float32)


def _assign_minmax(umin, umax, C):
    e = (umin[:, None] - C[None, :, 0]) ** 2 + (umax[:, None] - C[None, :, -1]) ** 2
    return np.argmin(e, axis=1)


def _quantise(u_rows, T_rows):
    # symbol = number of thresholds strictly below the value
    return (u_rows[:, :, None] > T_rows[:, None, :]).sum(-1)


def learn_tables(sample: torch.Tensor, seed: int = 0, max_groups: int = 16384,
                 refine_iters: int = 4, codebook_iters: int = 6, npat: int = NPAT, group: int = G) -> bytes:
    """Learns a table blob from a bf16 (or float) sample whose numel % 128 == 0.
    npat < 64 learns that many patterns (the compressor's 16-pattern variant,
    free parameters: "reduced from 64"); rows npat..63 repeat row 0 and are
    never chosen by an encoder that searches npat patterns.  group = 64 learns
    tables for the activation format (64-value groups, same blob layout)."""
    if group not in (G, 64):
        raise ValueError("group must be 128 or 64")
    if not 1 <= npat <= NPAT:
        raise ValueError("npat must be in 1..64")
    X = sample.detach().float().reshape(-1, group).cpu().numpy().astype(np.float32)
    X = np.where(np.isfinite(X), X, 0).astype(np.float32)
    absmax = float(np.abs(X).max()) if X.size else 0.0
    S_t = np.float32(absmax / 448.0) if absmax > 0 else np.float32(1.0)
    S_t = np.float32(min(max(S_t, np.float32(2.0 ** -60)), np.float32(2.0 ** 60)))
    rng = np.random.default_rng(seed)
    if len(X) > max_groups:
        X = X[np.sort(rng.choice(len(X), max_groups, replace=False))]
    u, m, keep = normalise_groups(X, S_t)
    u, m = u[keep], m[keep]
    n = len(u)
    if n < NPAT:
        u = (np.concatenate([u, np.zeros((NPAT - n + 1, group), np.float32)]) if n
             else np.zeros((NPAT + 1, group), np.float32))
        m = np.concatenate([m, np.zeros(len(u) - n, np.int64)]) if n else np.zeros(len(u), np.int64)
        n = len(u)
    mask = np.ones_like(u, dtype=bool)
    mask[np.arange(n), m] = False
    rest = u[mask].reshape(n, group - 1)

    srt = np.sort(rest, axis=1)
    edges = np.linspace(0, group - 1, NCENT + 1).round().astype(int)
    F = np.stack([srt[:, edges[j]:edges[j + 1]].mean(1) for j in range(NCENT)], axis=1)
    C = _kmeans(F, npat, rng)
    C = np.stack([_strictly_increasing(c) for c in C])

    umin, umax = rest.min(1), rest.max(1)
    for _ in range(refine_iters):
        p = _assign_minmax(umin, umax, C)
        T = _thresholds(C)
        sym = _quantise(rest, T[p])
        for q in range(npat):
            sel = p == q
            if not sel.any():
                continue
            vals, syms = rest[sel].ravel(), sym[sel].ravel()
            sums = np.bincount(syms, weights=vals, minlength=NCENT)
            cnts = np.bincount(syms, minlength=NCENT)
            newc = C[q].astype(np.float64).copy()
            nz = cnts > 0
            newc[nz] = sums[nz] / cnts[nz]
            C[q] = _strictly_increasing(newc)

    p = _assign_minmax(umin, umax, C)
    T = _thresholds(C)
    sym_rest = _quantise(rest, T[p])
    hist = np.zeros((n, NSYM), dtype=np.int64)
    for s in range(NCENT):
        hist[:, s] = (sym_rest == s).sum(1)
    hist[:, 15] = 1
    lens = np.zeros((NPAT, NBOOK, NSYM), dtype=np.uint8)
    glob_len = package_merge(hist.sum(0) + 1)
    for q in range(npat):
        Hq = hist[p == q]
        if len(Hq) == 0:
            lens[q, :] = glob_len
            continue
        base = Hq.sum(0) + 1
        if len(Hq) < NBOOK:
            lens[q, :] = package_merge(base)
            continue
        P = Hq / Hq.sum(1, keepdims=True)
        centers = _kmeans(P, NBOOK, rng, iters=10)
        a = np.argmin(((P[:, None, :] - centers[None]) ** 2).sum(-1), axis=1)
        books = np.zeros((NBOOK, NSYM), dtype=np.uint8)
        for _ in range(codebook_iters):
            for h in range(NBOOK):
                sel = a == h
                books[h] = package_merge(Hq[sel].sum(0) + 1 if sel.any() else base)
            a = np.argmin(Hq @ books.T.astype(np.int64), axis=1)
        lens[q] = books
    if npat < NPAT:
        C = np.concatenate([C, np.repeat(C[:1], NPAT - npat, axis=0)])
        lens[npat:] = lens[0]
    from struct import pack
    Cb = np.ascontiguousarray(C.astype(np.float32))
    blob = pack("<IIfI", TABLES_MAGIC, 1, float(S_t), 0) + Cb.tobytes() + np.ascontiguousarray(lens).tobytes()
    assert len(blob) == 16 + NPAT * NCENT * 4 + NPAT * NBOOK * NSYM
    return blob
