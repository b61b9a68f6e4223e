"""Launch-shape choices for the LSA library (host-side heuristics, no computation)."""
from __future__ import annotations

B200_SMS = 148


def split_for(T: int, H: int, sms: int = B200_SMS, ctas_per_sm: int = 2) -> int:
    """Split-KV chunk count so that T x (H / 32) x n_split attention CTAs fill the GPU."""
    base = max(1, T * max(1, H // 32))
    n = -(-sms * ctas_per_sm // base)
    return int(max(1, min(16, n)))
