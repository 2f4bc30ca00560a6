"""Optimal length-limited prefix codes by exhaustive dynamic programming --
TEST INFRASTRUCTURE (only tests/ may import it).

The minimal total length sum_i w_i l_i over prefix codes with 1 <= l_i <= L
(Kraft: sum_i 2^-l_i <= 1).  With weights sorted heaviest first an optimal
code has non-decreasing lengths, so the search runs over (symbol, last length,
Kraft budget used in units of 2^-L).  Used to check that a library code is
optimal under the 8-bit limit the review page's referee comment 1 quotes
("Ecco: Improving Memory Bandwidth and Capacity for LLMs via Entropy-aware
Cache Compression", Sec. 4.2: code lengths limited to 2-8 bits).
"""
from __future__ import annotations

from functools import lru_cache


def optimal_cost(weights, max_len: int) -> float:
    ws = sorted((float(w) for w in weights), reverse=True)
    n = len(ws)
    units = 1 << max_len

    @lru_cache(maxsize=None)
    def best(i: int, lmin: int, used: int) -> float:
        if i == n:
            return 0.0
        out = float("inf")
        for l in range(lmin, max_len + 1):
            u = used + (units >> l)
            if u <= units:
                out = min(out, ws[i] * l + best(i + 1, l, u))
        return out

    return best(0, 1, 0)
