"""The whole LSA path for single query tokens of a synthetic workload (oracle; test infrastructure).

Inputs are regenerated on the host from ``lsa_synth`` (never read back from a GPU) and
decoded exactly; the arithmetic is ``oracle.lsa``.  Only the rows a query needs are
built, so sampled queries of the full-size workloads stay affordable.
"""
from __future__ import annotations

import numpy as np

from lsa_synth import workloads as W

from . import formats, lsa

_CHUNK = 1 << 16


def query_context(w: W.Workload, p: W.Pass, token: int):
    """(sequence b, position pos, length L_b, q_I float64 [H_I, d_I], w float64 [H_I]) of a token."""
    q_seq, q_pos = W.query_rows(w, p)
    b, pos = int(q_seq[token]), int(q_pos[token])
    L = int(W.lengths(w)[b])
    qi = formats.bf16_to_f64(W.idx_q_bits(w, p, [token])[0])
    wi = W.idx_w(w, p, [token])[0].astype(np.float64)
    return b, pos, L, qi, wi


def index_keys(w: W.Workload, p: W.Pass, b: int, rows, plan=None) -> np.ndarray:
    """Indexer key rows of sequence b, decoded to float64."""
    data, scale = W.idx_key_rows(w, p, b, rows, plan)
    return formats.decode_rows(data, scale)


def block_keys_of_sequence(w: W.Workload, p: W.Pass, b: int, length: int, plan=None) -> np.ndarray:
    """Block keys of a whole sequence, built chunk by chunk (chunks are whole blocks)."""
    out = []
    step = (_CHUNK // w.block_size) * w.block_size
    for r0 in range(0, length, step):
        r1 = min(length, r0 + step)
        K = index_keys(w, p, b, np.arange(r0, r1), plan)
        out.append(lsa.block_keys(K, r1 - r0, w.block_size))
    return np.concatenate(out, axis=0)


def index_list(w: W.Workload, p: W.Pass, token: int, plan=None):
    """(ascending index list, flat scores of 0..pos or None for HI) of one query token."""
    b, pos, L, qi, wi = query_context(w, p, token)
    if plan is None and p.name == "target" and (w.plant_frac > 0 or w.plant_blocks > 0):
        plan = W.plant_plan(w, p)
    if not w.hi:
        K = index_keys(w, p, b, np.arange(pos + 1), plan)
        return lsa.select(qi, wi, K, pos, w.k, w.n_sink, w.window)
    kbar = block_keys_of_sequence(w, p, b, L, plan)
    cand = lsa.hi_candidates(qi, wi, kbar, pos, w.block_size, w.n_recall)
    s = lsa.indexer_scores(qi, wi, index_keys(w, p, b, cand, plan))
    picks = lsa.topk(s, cand, w.k)
    return lsa.union_fixed(picks, pos, w.n_sink, w.window), None


def kv_decoded(w: W.Workload, layer: W.Layer, b: int, rows):
    """(K rows [n, D], V rows [n, Dv]) of a layer, float64."""
    data, scale = W.kv_rows(w, layer.tid_kv, b, rows, w.D)
    K = formats.decode_rows(data, scale)
    if layer.tid_v >= 0:
        vd, vs = W.kv_rows(w, layer.tid_v, b, rows, w.Dv)
        return K, formats.decode_rows(vd, vs)
    return K, K[:, :w.Dv]


def attend(w: W.Workload, p: W.Pass, layer: W.Layer, token: int, idx: np.ndarray):
    """(o [H, Dv], lse [H]) of one layer for one query token over the index list ``idx``."""
    q_seq, _ = W.query_rows(w, p)
    b = int(q_seq[token])
    q = formats.bf16_to_f64(W.attn_q_bits(w, layer, [token])[0])
    K, V = kv_decoded(w, layer, b, idx)
    return lsa.attention(q, K, V, w.sm_scale)


def run_query(w: W.Workload, p: W.Pass, token: int, plan=None):
    """Index list, flat scores and every layer's (o, lse) of one query token."""
    idx, scores = index_list(w, p, token, plan)
    outs = [attend(w, p, layer, token, idx) for layer in p.layers]
    return {"idx": idx, "scores": scores, "layers": outs}
