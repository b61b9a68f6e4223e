"""Launch-shape choices for the LSA library (host-side heuristics, no computation)."""
from __future__ import annotations

import math

B200_SMS = 148


def split_for(T: int, H: int, cap: int = 2564, sms: int = B200_SMS) -> int:
    """Split-KV chunk count for sparse attention.

    The tensor-core kernel (128 heads) runs one CTA per SM, two CTAs (V halves) per
    (token, split), 32 rows per tile, and pays about two tiles' worth of set-up per CTA
    (loading the 147 KB query block).  Pick the split count minimising
    waves x (tiles per split + 2).  Other head counts use the warp-MMA kernel with
    T * H / 32 CTAs at two per SM.
    """
    if H != 128:
        base = max(1, T * max(1, H // 32))
        return int(max(1, min(16, -(-sms * 2 // base))))
    best, best_cost = 1, float("inf")
    for n in range(1, 33):
        if n > 1 and cap / n < 64:
            break
        ctas = 2 * T * n
        cost = math.ceil(ctas / sms) * (math.ceil(cap / n / 32) + 2)
        if cost < best_cost - 1e-9:
            best, best_cost = n, cost
    return best
