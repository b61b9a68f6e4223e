"""Launch-shape choices for the LSA library (host-side heuristics, no computation)."""
from __future__ import annotations

import math

B200_SMS = 148


def split_for(T: int, H: int, cap: int = 2564, sms: int = B200_SMS, layers: int = 1) -> int:
    """Split-KV chunk count for sparse attention.

    The tensor-core kernel (128 heads) runs one CTA per SM, two CTAs (V halves) per
    (token, split), 32 rows per tile, and pays about two tiles' worth of set-up per CTA
    (loading the 147 KB query block).  Pick the split count minimising
    waves x (tiles per split + 2) + (12 when split: the partial outputs and the merge).  A fused
    step runs the layers that share an index on two streams, so up to two layers' CTAs are
    resident together (``layers``).  Measured on the 128K decode (32 tokens, 2 layers):
    0.193 / 0.215 / 0.230 ms per step for 1 / 2 / 3 splits.  Other head counts use the
    warp-MMA kernel with T * H / 32 CTAs at two per SM.
    """
    if H != 128:
        base = max(1, T * max(1, H // 32))
        return int(max(1, min(16, -(-sms * 2 // base))))
    best, best_cost = 1, float("inf")
    for n in range(1, 33):
        if n > 1 and cap / n < 64:
            break
        ctas = 2 * T * n * max(1, min(2, layers))
        cost = math.ceil(ctas / sms) * (math.ceil(cap / n / 32) + 2) + (12 if n > 1 else 0)
        if cost < best_cost - 1e-9:
            best, best_cost = n, cost
    return best
