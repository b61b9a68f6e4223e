"""The LSA hot path by its plain definitions, float64 (oracle; test infrastructure only).

Per query token t at absolute position ``pos`` (keys 0..pos visible):

1. indexer score of every visible key          -- ``indexer_scores``
2. (HI) block keys, block scores, coarse recall -- ``block_keys``, ``hi_candidates``
3. top-k by (score desc, position asc)          -- ``topk``
4. union with the sink tokens and the SI window -- ``union_fixed``
5. softmax attention over the selected rows     -- ``attention``
6. (split-KV) log-sum-exp merge of partials     -- ``merge_partials``

Cross-layer index reuse (CLI) is step 5 run again with another layer's query and KV
cache on the index list of steps 1-4, unchanged; it needs no function of its own.
Sources are named in the package docstring ([explainer], [release], [notes]).
"""
from __future__ import annotations

import numpy as np


def indexer_scores(q: np.ndarray, w: np.ndarray, K: np.ndarray) -> np.ndarray:
    """I(s) = sum_h w_h * ReLU(q_h . k_s) for every key row k_s of K.

    q: [H_I, d_I] float64, w: [H_I], K: [n, d_I]  ->  [n].
    [release] "LongCat 稀疏注意力": LSA evolves from DSA's lightning indexer, whose
    scoring cost is the bottleneck; [explainer] "DSA 的瓶颈" likewise.  The pages print
    no formula: this is the DSA indexer form (per-head dot product, ReLU, weighted head
    sum), with no extra scale and w used as given.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    logits = K @ q.T                                   # [n, H_I]
    return np.maximum(logits, 0.0) @ np.asarray(w, dtype=np.float64)


def fp8_queries(q: np.ndarray) -> np.ndarray:
    """The indexer queries of the FP8-query mode: each row q_h (one head of one token) scaled by
    the power of two 2**s that brings its largest magnitude m into [128, 256)
    (s = 7 - floor(log2 m), clamped to [-126, 126]; s = 0 for an all-zero row), rounded to
    e4m3 (``formats.e4m3_round``) and scaled back by 2**-s.

    The DSA-style indexer usually runs its queries in FP8 ([release] "LongCat 稀疏注意力":
    LSA grows out of DSA's lightning indexer, whose scoring cost is the bottleneck).  The pages
    fix no quantisation; the per-row power-of-two scale is this library's reading (exact to
    undo, so the score differs from the BF16-query score only by the e4m3 rounding of q).
    q: [H_I, d_I] -> [H_I, d_I] float64.
    """
    from .formats import e4m3_round
    q = np.asarray(q, dtype=np.float64)
    m = np.max(np.abs(q), axis=-1)
    _, E = np.frexp(np.where(m > 0, m, 1.0))
    s = np.where(m > 0, np.clip(7 - (E - 1), -126, 126), 0)
    sc = np.ldexp(1.0, s)[..., None]
    return e4m3_round(q * sc) / sc


def indexer_scores_fp8q(q: np.ndarray, w: np.ndarray, K: np.ndarray) -> np.ndarray:
    """``indexer_scores`` with the queries of the FP8-query mode (``fp8_queries``)."""
    return indexer_scores(fp8_queries(q), w, K)


def topk(scores: np.ndarray, positions: np.ndarray, k: int) -> np.ndarray:
    """The min(k, n) positions ranked first by (score descending, position ascending).

    [explainer] "① LSA": each query picks its top-k keys through the indexer.  The order
    on equal scores (lower position first) makes the selection unique; -0 equals +0.
    Returned in ranking order (not sorted by position).
    """
    scores = np.asarray(scores, dtype=np.float64)
    positions = np.asarray(positions, dtype=np.int64)
    if np.isnan(scores).any():
        raise ValueError("NaN indexer score")
    order = np.lexsort((positions, -scores))          # primary: -score, secondary: position
    return positions[order[:max(0, min(k, scores.size))]]


def window_start(pos: int, window: int, align: int = 0) -> int:
    """First position of the SI window: pos-window+1 clipped at 0, or -- with ``align`` > 0 -- that
    position rounded down to a multiple of ``align`` (the block-aligned window).

    [release] SI bullet: the contiguous part of the selection is read with hardware-aligned
    accesses.  The plain reading keeps the window's extent exactly ``window`` positions; the
    aligned reading starts it at the row block that holds pos-window+1, so the window covers
    whole blocks up to the query (``window`` to ``window + align - 1`` positions).
    """
    b = max(0, pos - window + 1)
    return (b // align) * align if align > 0 else b


def union_fixed(selected: np.ndarray, pos: int, n_sink: int, window: int, align: int = 0) -> np.ndarray:
    """Ascending, de-duplicated union of the top-k picks, the sinks and the SI window.

    Sinks: positions 0..n_sink-1 ([explainer] "① LSA": a few fixed sink tokens keep the
    sparse softmax stable).  Window: the last ``window`` visible positions
    pos-window+1..pos, the contiguous, sequentially read part of the selection budget
    that streaming-aware indexing adds to the dynamic picks ([release] SI bullet); with
    ``align``, from ``window_start(pos, window, align)``.  Both are clipped to the visible
    range 0..pos.
    """
    sinks = np.arange(0, min(n_sink, pos + 1), dtype=np.int64)
    win = np.arange(window_start(pos, window, align), pos + 1, dtype=np.int64) if window > 0 else \
        np.zeros(0, dtype=np.int64)
    return np.union1d(np.union1d(np.asarray(selected, dtype=np.int64), sinks), win)


def union_fixed_budget(scores: np.ndarray, positions: np.ndarray, k: int, pos: int, n_sink: int,
                       window: int, align: int = 0) -> np.ndarray:
    """Fixed-budget SI selection: the sinks and the window as in ``union_fixed``, plus the top-k
    (``topk`` order) of the visible positions OUTSIDE both, so the three sets are disjoint and
    the list holds min(k, outside) + |sinks| + |window| positions, ascending.

    [release] SI bullet: the selection budget is split between a contiguous, hardware-aligned
    part and the dynamic picks.  Read as a budget, the dynamic part should not spend picks on
    positions the fixed part already holds; ``union_fixed`` is the other reading (top-k over all
    visible positions, then the union).  scores / positions: the visible keys (any order).
    """
    scores = np.asarray(scores, dtype=np.float64)
    positions = np.asarray(positions, dtype=np.int64)
    a = min(n_sink, pos + 1)
    b = max(a, window_start(pos, window, align)) if window > 0 else pos + 1
    outside = (positions >= a) & (positions < b)
    picks = topk(scores[outside], positions[outside], k)
    return union_fixed(picks, pos, n_sink, window, align)


def block_keys(K: np.ndarray, length: int, block_size: int) -> np.ndarray:
    """Block key = arithmetic mean of the (dequantised) keys of the block's existing tokens.

    K: [>= length, d_I] rows of one sequence.  Returns [ceil(length / block_size), d_I];
    the last block may be partial and is averaged over the tokens it has.
    [release] HI bullet: a coarse block-level approximate score first; the pages do not
    say how a block is summarised -- the mean of its keys is taken.
    """
    K = np.asarray(K[:length], dtype=np.float64)
    nblk = (length + block_size - 1) // block_size
    out = np.empty((nblk, K.shape[1]), dtype=np.float64)
    for b in range(nblk):
        out[b] = K[b * block_size:(b + 1) * block_size].mean(axis=0)
    return out


def hi_candidates(q: np.ndarray, w: np.ndarray, kbar: np.ndarray, pos: int, block_size: int,
                  n_recall: int) -> np.ndarray:
    """Coarse recall of HI: the positions of the ``n_recall`` best visible blocks.

    Block score J(b) = sum_h w_h * ReLU(q_h . kbar_b) (the indexer formula on block keys);
    a block is visible when its first token is visible (b * block_size <= pos); recall
    = top-n_recall blocks by (J desc, b asc); candidates = the visible tokens of the
    recalled blocks, ascending.  [release] HI bullet: block-level approximate scoring,
    coarse recall, then fine token selection among the recalled candidates.
    """
    n_vis = pos // block_size + 1
    J = indexer_scores(q, w, kbar[:n_vis])
    blocks = np.sort(topk(J, np.arange(n_vis), n_recall))
    cand = (blocks[:, None] * block_size + np.arange(block_size)[None, :]).reshape(-1)
    return cand[cand <= pos]


def select(q: np.ndarray, w: np.ndarray, K: np.ndarray, pos: int, k: int, n_sink: int, window: int,
           hi: bool = False, length: int | None = None, block_size: int = 64, n_recall: int = 0,
           kbar: np.ndarray | None = None):
    """Index list of one query token (steps 1-4).  Returns (idx ascending, scores of 0..pos or None).

    K holds the sequence's indexer keys as float64 rows 0.. (at least 0..pos; for HI the
    whole sequence, ``length`` rows, unless ``kbar`` is given).
    """
    if not hi:
        s = indexer_scores(q, w, K[:pos + 1])
        picks = topk(s, np.arange(pos + 1), k)
        return union_fixed(picks, pos, n_sink, window), s
    if kbar is None:
        kbar = block_keys(K, length, block_size)
    cand = hi_candidates(q, w, kbar, pos, block_size, n_recall)
    s = indexer_scores(q, w, K[cand])
    picks = topk(s, cand, k)
    return union_fixed(picks, pos, n_sink, window), None


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, sm_scale: float):
    """Softmax attention of all heads of one query over the given rows.

    q: [H, D], K: [n, D], V: [n, Dv]  ->  (o [H, Dv], lse [H]) with
    z = sm_scale * q K^T, p = softmax(z) per head (max subtracted), o = p V,
    lse = log sum_j exp(z_j) (natural log).  An empty row set gives o = 0, lse = -inf.
    [explainer] "① LSA": attention reads only the selected keys plus the sinks.  In the
    MLA-absorbed layout V is the first Dv dims of the shared latent row.
    """
    q = np.asarray(q, dtype=np.float64)
    H = q.shape[0]
    if K.shape[0] == 0:
        return np.zeros((H, V.shape[1])), np.full(H, -np.inf)
    z = sm_scale * (q @ np.asarray(K, dtype=np.float64).T)      # [H, n]
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    s = e.sum(axis=1, keepdims=True)
    o = (e @ np.asarray(V, dtype=np.float64)) / s
    return o, m[:, 0] + np.log(s[:, 0])


def merge_partials(os: list, lses: list):
    """Combine partial attentions over disjoint row subsets: lse = log sum_s e^{lse_s},
    o = sum_s e^{lse_s - lse} o_s.  [explainer] "③ KVP 解码切分示意": each shard computes a
    partial attention, the partial results are then merged.  Empty partials (lse = -inf)
    contribute nothing.
    """
    lses = np.stack([np.asarray(l, dtype=np.float64) for l in lses])      # [S, H]
    os = np.stack([np.asarray(o, dtype=np.float64) for o in os])          # [S, H, Dv]
    m = lses.max(axis=0)
    finite = np.isfinite(m)
    msafe = np.where(finite, m, 0.0)
    wts = np.where(np.isfinite(lses), np.exp(lses - msafe[None, :]), 0.0)
    tot = wts.sum(axis=0)
    lse = np.where(finite, msafe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    o = np.einsum("sh,shd->hd", wts, os) / np.where(tot > 0, tot, 1.0)[:, None]
    return o, lse
