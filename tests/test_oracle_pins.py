"""Pins of the CPU oracle against things other than itself (CPU only).

Each test fixes a part of the oracle to an independent source: a hand-worked example,
brute force over tiny inputs written with plain Python loops, a library routine
(torch's FP8/BF16 conversions, float64 scaled_dot_product_attention), or an invariant
that the definitions imply.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import formats, lsa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_small.json")


def _g():
    with open(GOLDEN) as f:
        return json.load(f)


# ------------------------------------------------------------------ formats

def test_e4m3_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = formats.E4M3_TABLE
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert nan.sum() == 2                                   # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], mine[~nan])


def test_e4m3_spec_values():
    t = formats.E4M3_TABLE
    assert t[0x38] == 1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x08] == 2.0 ** -6                             # smallest normal
    assert t[0x01] == 2.0 ** -9                             # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9                         # largest subnormal
    assert t[0x80] == 0.0 and math.copysign(1, t[0x80]) < 0


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    mine = formats.bf16_to_f64(bits)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])


def test_scaled_rows_decode():
    codes = np.array([[0x38, 0xB8], [0x7E, 0x01]], dtype=np.uint8)
    v = formats.decode_rows(codes, np.array([0.5, 2.0], dtype=np.float32))
    assert np.array_equal(v, [[0.5, -0.5], [896.0, 2.0 ** -8]])


def test_e4m3_round_matches_torch_float8():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.normal(size=20000) * 40.0,                         # normals up to ~180
        rng.uniform(-2.0 ** -5, 2.0 ** -5, size=20000),        # around and below the smallest normal
        rng.uniform(-440.0, 440.0, size=5000),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(formats.e4m3_round(x.astype(np.float64)), ref)


def test_e4m3_round_grid_and_ties():
    t = formats.E4M3_TABLE
    pos = np.sort(np.unique(t[np.isfinite(t) & (t >= 0)]))
    assert np.array_equal(formats.e4m3_round(pos), pos)              # every value maps to itself
    assert np.array_equal(formats.e4m3_round(-pos), -pos)
    mids = (pos[:-1] + pos[1:]) / 2                                   # exact midpoints: ties to even code
    got = formats.e4m3_round(mids)
    code_of = {v: c for c, v in enumerate(t[:0x7F]) if np.isfinite(v)}
    for lo, hi, g in zip(pos[:-1], pos[1:], got):
        even = lo if code_of[lo] % 2 == 0 else hi
        assert g == even, (lo, hi, g)
    assert formats.e4m3_round(np.array([500.0, -1e6]))[0] == 448.0     # saturation
    assert formats.e4m3_round(np.array([-1e6]))[0] == -448.0
    assert formats.e4m3_round(np.array([2.0 ** -10]))[0] == 0.0         # half the smallest subnormal: tie to 0


def test_fp8_queries_scale_and_error_bound():
    rng = np.random.default_rng(4)
    # rows of very different magnitudes: the scale is per row (head), not per token
    q = rng.normal(size=(6, 128)) * np.array([1e3, 1.0, 1e-3, 3.0, 1e-6, 0.0])[:, None]
    q8 = lsa.fp8_queries(q)
    for h in range(6):
        m = np.abs(q[h]).max()
        if m == 0:
            assert np.all(q8[h] == 0)
            continue
        s = 7 - math.floor(math.log2(m))
        assert 128 <= m * 2.0 ** s < 256
        big = np.abs(q[h]) * 2.0 ** s >= 2.0 ** -6                   # normal after scaling
        err = np.abs(q8[h] - q[h])
        assert np.all(err[big] <= 2.0 ** -4 * np.abs(q[h][big]))      # 3 mantissa bits, round to nearest
        assert np.all(err[~big] <= 2.0 ** -10 * 2.0 ** -s)            # half a subnormal step
    assert np.abs(q8[0] - q[0]).max() > 0                             # it does round


def test_fp8_query_scores_on_representable_queries():
    rng = np.random.default_rng(5)
    # entries k / 4 with |k| <= 15: exactly representable after any power-of-two scale that
    # keeps the row maximum in [128, 256) (4 significant bits), so the rounding is the identity
    q = rng.integers(-15, 16, size=(8, 128)) / 4.0 * np.array([2.0 ** j for j in range(-3, 5)])[:, None]
    q[:, 0] = 3.75 * np.array([2.0 ** j for j in range(-3, 5)])           # a known maximum per row
    K = rng.normal(size=(50, 128))
    w = rng.normal(size=8)
    assert np.array_equal(lsa.fp8_queries(q), q)
    assert np.array_equal(lsa.indexer_scores_fp8q(q, w, K), lsa.indexer_scores(q, w, K))
    # and a query that is not representable scores differently
    q2 = q.copy()
    q2[:, 1] = 0.123456
    assert not np.array_equal(lsa.indexer_scores_fp8q(q2, w, K), lsa.indexer_scores(q2, w, K))


# ------------------------------------------------------------------ worked example

def test_worked_indexer():
    g = _g()["indexer"]
    s = lsa.indexer_scores(np.array(g["q"], float), np.array(g["w"], float), np.array(g["keys"], float))
    assert s.tolist() == g["scores"]


def test_worked_topk_and_union():
    g = _g()
    s = np.array(g["indexer"]["scores"], float)
    for case in g["topk"]["cases"]:
        assert lsa.topk(s, np.arange(6), case["k"]).tolist() == case["picks"]
    u = g["union"]
    picks = lsa.topk(s, np.arange(6), u["k"])
    assert lsa.union_fixed(picks, u["pos"], u["n_sink"], u["window"]).tolist() == u["index_list"]
    picks3 = lsa.topk(s[:4], np.arange(4), 1)
    assert lsa.union_fixed(picks3, 3, 2, 2).tolist() == u["pos_3_k_1_sink_2_window_2"]


def test_worked_si_variants():
    """The fixed-budget selection and the block-aligned window on the hand-worked example."""
    g = _g()
    s = np.array(g["indexer"]["scores"], float)
    v = g["si_variants"]
    pos = v["pos"]
    for c in v["cases"]:
        if c["fixed_budget"]:
            got = lsa.union_fixed_budget(s, np.arange(pos + 1), c["k"], pos, c["n_sink"], c["window"], c["align"])
        else:
            got = lsa.union_fixed(lsa.topk(s, np.arange(pos + 1), c["k"]), pos, c["n_sink"], c["window"], c["align"])
        assert got.tolist() == c["index_list"], c["why"]
        assert lsa.window_start(pos, c["window"], c["align"]) == c["window_start"]


def test_worked_hi():
    g = _g()
    q, w, K = (np.array(g["indexer"][n], float) for n in ("q", "w", "keys"))
    h = g["hi"]
    kbar = lsa.block_keys(K, 6, h["block_size"])
    assert kbar.tolist() == h["block_keys"]
    assert lsa.indexer_scores(q, w, kbar).tolist() == h["block_scores"]
    for r, key in ((2, "recall_2"), (1, "recall_1")):
        cand = lsa.hi_candidates(q, w, kbar, 5, h["block_size"], r)
        assert cand.tolist() == h[key]["candidates"]
        idx, _ = lsa.select(q, w, K, 5, 2, 1, 1, hi=True, length=6, block_size=2, n_recall=r)
        assert idx.tolist() == h[key]["index_list_k2_sink1_window1"]


def test_worked_attention_and_merge():
    g = _g()["attention"]
    o, lse = lsa.attention(np.array(g["q"], float), np.array(g["K_rows"], float),
                           np.array(g["V_rows"], float), math.log(2))
    assert abs(o[0, 0] - 9.0) < 1e-12 and abs(lse[0] - math.log(7)) < 1e-12
    o1, l1 = lsa.attention(np.array(g["q"], float), np.array(g["K_rows"][:1], float),
                           np.array(g["V_rows"][:1], float), math.log(2))
    o2, l2 = lsa.attention(np.array(g["q"], float), np.array(g["K_rows"][1:], float),
                           np.array(g["V_rows"][1:], float), math.log(2))
    assert abs(o1[0, 0] - 7) < 1e-12 and abs(l1[0]) < 1e-12
    assert abs(o2[0, 0] - 56 / 6) < 1e-12 and abs(l2[0] - math.log(6)) < 1e-12
    om, lm = lsa.merge_partials([o1, o2], [l1, l2])
    assert abs(om[0, 0] - 9) < 1e-12 and abs(lm[0] - math.log(7)) < 1e-12


# ------------------------------------------------------------------ brute force on tiny inputs

def _brute_scores(q, w, K):
    out = []
    for k in K:
        tot = 0.0
        for h in range(len(q)):
            dot = 0.0
            for d in range(len(k)):
                dot += q[h][d] * k[d]
            tot += w[h] * (dot if dot > 0 else 0.0)
        out.append(tot)
    return out


@pytest.mark.parametrize("seed", range(5))
def test_indexer_vs_loops(seed):
    rng = np.random.default_rng(seed)
    q, w, K = rng.normal(size=(3, 5)), rng.uniform(size=3), rng.normal(size=(11, 5))
    assert np.allclose(lsa.indexer_scores(q, w, K), _brute_scores(q.tolist(), w.tolist(), K.tolist()),
                       rtol=1e-13, atol=1e-13)


def test_indexer_invariants():
    rng = np.random.default_rng(7)
    q, w, K = rng.normal(size=(4, 6)), rng.uniform(size=4), rng.normal(size=(50, 6))
    s = lsa.indexer_scores(q, w, K)
    assert np.allclose(lsa.indexer_scores(q, 2 * w, K), 2 * s)              # linear in w
    perm = rng.permutation(4)
    assert np.allclose(lsa.indexer_scores(q[perm], w[perm], K), s)          # head order irrelevant
    assert np.allclose(lsa.indexer_scores(q, w, 3 * K), 3 * s)             # ReLU is positively homogeneous
    assert (s >= 0).all()
    assert np.all(lsa.indexer_scores(-np.abs(q), w, np.abs(K)) == 0)      # all heads negative -> 0


def _brute_topk_valid(scores, k, picks):
    """Every pick beats every non-pick under (score desc, position asc), and |picks| = min(k, n)."""
    n = len(scores)
    if len(picks) != min(k, n) or len(set(picks)) != len(picks):
        return False
    rest = [j for j in range(n) if j not in picks]
    return all(scores[a] > scores[b] or (scores[a] == scores[b] and a < b) for a in picks for b in rest)


def test_topk_brute_force_all_small_cases():
    rng = np.random.default_rng(3)
    for n in range(0, 8):
        for _ in range(20):
            s = rng.integers(-2, 3, size=n).astype(float)           # many ties
            for k in range(0, n + 2):
                picks = lsa.topk(s, np.arange(n), k).tolist()
                assert _brute_topk_valid(s.tolist(), k, picks)
                # ranking order: non-increasing score, positions ascending on ties
                for a, b in zip(picks, picks[1:]):
                    assert s[a] > s[b] or (s[a] == s[b] and a < b)


def test_topk_exhaustive_subset_search():
    """For tiny n the unique valid k-subset found by exhaustive search equals the oracle's picks."""
    rng = np.random.default_rng(5)
    for _ in range(30):
        n = int(rng.integers(1, 7))
        s = rng.integers(0, 3, size=n).astype(float)
        k = int(rng.integers(1, n + 1))
        valid = [set(c) for c in itertools.combinations(range(n), k)
                 if _brute_topk_valid(s.tolist(), k, list(c))]
        assert len(valid) == 1
        assert set(lsa.topk(s, np.arange(n), k).tolist()) == valid[0]


def test_topk_signed_zero_and_nan():
    s = np.array([0.0, -0.0, 0.0, -1.0])
    assert lsa.topk(s, np.arange(4), 2).tolist() == [0, 1]
    with pytest.raises(ValueError):
        lsa.topk(np.array([1.0, np.nan]), np.arange(2), 1)


def test_union_brute_force():
    rng = np.random.default_rng(11)
    for _ in range(200):
        pos = int(rng.integers(0, 40))
        sel = rng.choice(pos + 1, size=int(rng.integers(0, pos + 2)), replace=False)
        ns, W = int(rng.integers(0, 6)), int(rng.integers(0, 10))
        want = set(sel.tolist()) | {j for j in range(ns) if j <= pos} | {j for j in range(pos + 1) if j > pos - W}
        got = lsa.union_fixed(sel, pos, ns, W)
        assert got.tolist() == sorted(want)


# ------------------------------------------------------------------ attention

@pytest.mark.parametrize("seed", range(3))
def test_dense_equals_sdpa(seed):
    """Selecting every key (k >= context) gives dense attention; checked against torch SDPA in float64."""
    rng = np.random.default_rng(seed)
    H, n, D, Dv = 4, 37, 24, 16
    q, K = rng.normal(size=(H, D)), rng.normal(size=(n, D))
    V = K[:, :Dv]                                            # absorbed-MLA layout: V = first Dv dims
    scale = 1 / math.sqrt(D)
    s = lsa.indexer_scores(rng.normal(size=(2, D)), rng.uniform(size=2), K)
    idx = lsa.union_fixed(lsa.topk(s, np.arange(n), n + 5), n - 1, 4, 8)
    assert idx.tolist() == list(range(n))
    o, lse = lsa.attention(q, K[idx], V[idx], scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, H, n, D),
        torch.from_numpy(V)[None, None].expand(1, H, n, Dv), scale=scale)[0, :, 0, :].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    z = scale * q @ K.T
    assert np.allclose(lse, np.log(np.exp(z).sum(axis=1)), rtol=1e-13)


def test_attention_vs_loops_and_row_sums():
    rng = np.random.default_rng(4)
    H, n, D, Dv = 3, 9, 5, 4
    q, K, V = rng.normal(size=(H, D)), rng.normal(size=(n, D)), rng.normal(size=(n, Dv))
    o, lse = lsa.attention(q, K, V, 0.7)
    for h in range(H):
        z = [0.7 * sum(q[h][d] * K[j][d] for d in range(D)) for j in range(n)]
        m = max(z)
        e = [math.exp(x - m) for x in z]
        tot = sum(e)
        p = [x / tot for x in e]
        assert abs(sum(p) - 1) < 1e-12
        for c in range(Dv):
            assert abs(o[h][c] - sum(p[j] * V[j][c] for j in range(n))) < 1e-12
        assert abs(lse[h] - (m + math.log(tot))) < 1e-12
    # softmax weights are a probability vector: o of an all-ones V is exactly 1
    o1, _ = lsa.attention(q, K, np.ones((n, 2)), 0.7)
    assert np.allclose(o1, 1.0, atol=1e-14)


def test_attention_large_logits_stable():
    q = np.array([[1000.0, 0.0]])
    K = np.array([[1.0, 0.0], [0.999, 0.0]])
    o, lse = lsa.attention(q, K, np.array([[1.0], [0.0]]), 1.0)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    assert abs(o[0, 0] - 1 / (1 + math.exp(-1.0))) < 1e-12


def test_empty_selection():
    o, lse = lsa.attention(np.ones((2, 3)), np.zeros((0, 3)), np.zeros((0, 3)), 1.0)
    assert (o == 0).all() and np.isneginf(lse).all()


@pytest.mark.parametrize("n_split", [1, 2, 3, 7])
def test_merge_of_splits_equals_full(n_split):
    rng = np.random.default_rng(n_split)
    H, n, D = 4, 29, 8
    q, K, V = rng.normal(size=(H, D)), rng.normal(size=(n, D)), rng.normal(size=(n, D))
    o, lse = lsa.attention(q, K, V, 0.4)
    parts = np.array_split(np.arange(n), n_split)
    res = [lsa.attention(q, K[p], V[p], 0.4) for p in parts]
    res.append(lsa.attention(q, K[:0], V[:0], 0.4))          # an empty split contributes nothing
    om, lm = lsa.merge_partials([r[0] for r in res], [r[1] for r in res])
    assert np.allclose(om, o, rtol=1e-12, atol=1e-12) and np.allclose(lm, lse, rtol=1e-13)


# ------------------------------------------------------------------ HI / CLI invariants

@pytest.mark.parametrize("seed", range(4))
def test_hi_all_blocks_recalled_equals_flat(seed):
    rng = np.random.default_rng(seed)
    L, bs, d = 203, 16, 8                                    # ragged last block
    q, w, K = rng.normal(size=(4, d)), rng.uniform(size=4), rng.normal(size=(L, d))
    pos = L - 1 - seed
    flat, _ = lsa.select(q, w, K, pos, 20, 4, 8)
    hi, _ = lsa.select(q, w, K, pos, 20, 4, 8, hi=True, length=L, block_size=bs, n_recall=1000)
    assert flat.tolist() == hi.tolist()


def test_hi_candidates_are_whole_recalled_blocks():
    rng = np.random.default_rng(9)
    L, bs, d = 300, 32, 8
    q, w, K = rng.normal(size=(2, d)), rng.uniform(size=2), rng.normal(size=(L, d))
    kbar = lsa.block_keys(K, L, bs)
    assert np.allclose(kbar[-1], K[288:300].mean(axis=0))   # partial block: mean over its 12 tokens
    cand = lsa.hi_candidates(q, w, kbar, 250, bs, 3)
    blocks = sorted(set((cand // bs).tolist()))
    assert len(blocks) == 3 and (cand <= 250).all()
    J = lsa.indexer_scores(q, w, kbar[:250 // bs + 1])
    best = sorted(np.argsort(-J, kind="stable")[:3].tolist())
    assert blocks == best


# ------------------------------------------------------------------ fixed-budget SI selection

def test_fixed_budget_union_brute_force():
    rng = np.random.default_rng(11)
    for trial in range(300):
        n = int(rng.integers(1, 40))
        pos = int(rng.integers(0, n))
        k = int(rng.integers(0, 12))
        n_sink = int(rng.integers(0, 5))
        window = int(rng.integers(0, 8))
        sc = rng.integers(0, 4, size=pos + 1).astype(np.float64)       # many ties
        got = lsa.union_fixed_budget(sc, np.arange(pos + 1), k, pos, n_sink, window)
        sinks = set(range(min(n_sink, pos + 1)))
        win = set(range(max(0, pos - window + 1), pos + 1)) if window > 0 else set()
        rest = [j for j in range(pos + 1) if j not in sinks and j not in win]
        # brute force: rank the rest by (score desc, position asc), take k
        best = sorted(rest, key=lambda j: (-sc[j], j))[:k]
        want = sorted(sinks | win | set(best))
        assert got.tolist() == want
        assert len(got) == len(sinks | win) + min(k, len(rest))          # exact budget, disjoint parts


def test_fixed_budget_equals_plain_union_when_picks_avoid_the_fixed_sets():
    pos, k, n_sink, window = 999, 50, 4, 100
    sc = np.zeros(pos + 1)
    sc[300:350] = 10.0 + np.arange(50)                 # the top-50 lie outside sinks and window
    cols = np.arange(pos + 1)
    plain = lsa.union_fixed(lsa.topk(sc, cols, k), pos, n_sink, window)
    assert np.array_equal(lsa.union_fixed_budget(sc, cols, k, pos, n_sink, window), plain)
    sc[995] = 100.0                                    # a top score inside the window
    plain = lsa.union_fixed(lsa.topk(sc, cols, k), pos, n_sink, window)
    budget = lsa.union_fixed_budget(sc, cols, k, pos, n_sink, window)
    assert len(budget) == len(plain) + 1               # the budget spends that pick elsewhere


# ------------------------------------------------------------------ block-aligned SI window

def test_aligned_window_brute_force():
    """The aligned window covers every position from the 64-row block holding pos-W+1 up to pos:
    brute force over small cases, its extent between W and W + 63, and the plain window when
    pos-W+1 is itself on a block boundary."""
    rng = np.random.default_rng(13)
    for _ in range(300):
        pos = int(rng.integers(0, 400))
        W = int(rng.integers(0, 200))
        ns = int(rng.integers(0, 6))
        sel = rng.choice(pos + 1, size=int(rng.integers(0, min(pos + 2, 30))), replace=False)
        first = max(0, pos - W + 1)
        blk = first - first % 64
        win = set(range(blk, pos + 1)) if W > 0 else set()
        want = set(sel.tolist()) | {j for j in range(ns) if j <= pos} | win
        assert lsa.union_fixed(sel, pos, ns, W, align=64).tolist() == sorted(want)
        if W > 0:
            assert W <= len(win) <= W + 63 or len(win) == pos + 1
        if W > 0 and first % 64 == 0:
            assert lsa.union_fixed(sel, pos, ns, W, align=64).tolist() == lsa.union_fixed(sel, pos, ns, W).tolist()
    assert lsa.window_start(1000, 512, 64) == 448 and lsa.window_start(1000, 512) == 489
    assert lsa.window_start(100, 512, 64) == 0 and lsa.window_start(575, 512, 64) == 64


def test_aligned_window_fixed_budget_brute_force():
    rng = np.random.default_rng(17)
    for _ in range(300):
        pos = int(rng.integers(0, 300))
        k = int(rng.integers(0, 12))
        n_sink = int(rng.integers(0, 5))
        window = int(rng.integers(0, 100))
        sc = rng.integers(0, 4, size=pos + 1).astype(np.float64)
        got = lsa.union_fixed_budget(sc, np.arange(pos + 1), k, pos, n_sink, window, align=64)
        sinks = set(range(min(n_sink, pos + 1)))
        first = max(0, pos - window + 1)
        win = set(range(first - first % 64, pos + 1)) if window > 0 else set()
        rest = [j for j in range(pos + 1) if j not in sinks and j not in win]
        best = sorted(rest, key=lambda j: (-sc[j], j))[:k]
        assert got.tolist() == sorted(sinks | win | set(best))
