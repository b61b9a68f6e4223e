"""GPU parity: the CUDA library against the float64 CPU oracle on the same seeded inputs.

Tolerances (from the definitions of the path and its precision):
* indexer / block scores: relative 1e-3, with a floor at 1% of the row's RMS score for
  entries near zero (ReLU sums of cancelling dot products);
* top-k: exact index lists when the selection runs on identical scores; >= 99.9% overlap
  against the oracle's own float64 scores;
* attention (BF16 output): max-abs 1e-2 and relative L2 5e-3;
* determinism: bitwise identical outputs across runs at a fixed n_split.
"""
import math

import numpy as np
import pytest
import torch

from lsa_synth import device as D
from lsa_synth import gen
from lsa_synth import workloads as W
from oracle import formats, lsa as olsa, run

from long_context_sparse_indexer_b200 import lsa

from . import gpu_helpers as H

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_decode": W.WORKLOADS["tiny_decode"],
    "cli_small": W.scaled("decode_cli_128k", B=3, len_lo=2500, len_hi=5200),
    "mtp_small": W.scaled("mtp_256k", B=2, len_lo=3001, len_hi=3001),
    "prefill_small": W.scaled("prefill_32k", len_lo=3000, len_hi=3000, passes=(W._target_pass(64, 1),)),
    "hi_small": W.scaled("decode_hi_1m", B=2, len_lo=20000, len_hi=20000),
    # FP8 scales whose per-sequence stride is not 16-byte aligned (the tensor-core indexer
    # reads them directly instead of by TMA), and a 64-dim FP8 indexer (warp-MMA kernel).
    "cli_unaligned": W.scaled("decode_cli_128k", B=3, len_lo=2500, len_hi=5200, seed=12),
    "cli_d64": W.scaled("decode_cli_128k", B=2, len_lo=3000, len_hi=4100, d_I=64, seed=13),
    # BF16 indexer keys at d_I = 128 (the tensor-core row scorer), query groups of 1 and of 4
    "cli_bf16": W.scaled("decode_cli_128k", B=3, len_lo=2500, len_hi=5200, idx_fp8=False, seed=14),
    "mtp_bf16": W.scaled("mtp_256k", B=2, len_lo=3001, len_hi=3001, idx_fp8=False, seed=15),
}
FLAT = ["tiny_decode", "cli_small", "mtp_small", "prefill_small", "cli_unaligned", "cli_d64", "cli_bf16", "mtp_bf16"]
L_ALLOC = {"cli_unaligned": 5203}

_cache = {}


def wt_of(name):
    if name not in _cache:
        _cache[name] = D.build_workload(SMALL[name], "cuda", L_alloc=L_ALLOC.get(name))
    return _cache[name]


def tokens_to_check(w, p, limit=6):
    T = w.T(p)
    if T <= limit:
        return list(range(T))
    return sorted({0, 1, T // 2, T - 2, T - 1})


# ------------------------------------------------------------------ inputs

@pytest.mark.parametrize("name", list(SMALL))
def test_device_inputs_match_host_generator(cuda, name):
    w = SMALL[name]
    wt = wt_of(name)
    plan = None
    for pi, p in enumerate(w.passes):
        pt = wt.passes[pi]
        T = w.T(p)
        assert np.array_equal(pt.q_idx.view(torch.int16).cpu().numpy().view(np.uint16), W.idx_q_bits(w, p))
        assert np.array_equal(pt.w.cpu().numpy(), W.idx_w(w, p))
        if p.name == "target" and (w.plant_frac or w.plant_blocks):
            plan = W.plant_plan(w, p)
        for b in range(w.B):
            L = int(W.lengths(w)[b])
            rows = np.unique(np.concatenate([np.arange(0, 70), np.arange(L - 70, L),
                                             plan[0][b][:50] if plan is not None and p.name == "target"
                                             else np.zeros(0, np.int64)]))
            data, scale = W.idx_key_rows(w, p, b, rows, plan if p.name == "target" else None)
            got = pt.k_idx[b, torch.from_numpy(rows).cuda()].cpu()
            if scale is None:
                assert np.array_equal(got.view(torch.int16).numpy().view(np.uint16), data)
            else:
                assert np.array_equal(got.numpy(), data)
                assert np.array_equal(pt.k_scale[b, torch.from_numpy(rows).cuda()].cpu().numpy(), scale)
            for li, layer in enumerate(p.layers):
                kd, ks = W.kv_rows(w, layer.tid_kv, b, rows[:20], w.D)
                g = pt.layers[li]["kv"][b, torch.from_numpy(rows[:20]).cuda()].cpu()
                if ks is None:
                    assert np.array_equal(g.view(torch.int16).numpy().view(np.uint16), kd)
                else:
                    assert np.array_equal(g.numpy(), kd)
        toks = [0, T - 1]
        for li, layer in enumerate(p.layers):
            got = pt.layers[li]["q"][toks].view(torch.int16).cpu().numpy().view(np.uint16)
            assert np.array_equal(got, W.attn_q_bits(w, layer, toks))


# ------------------------------------------------------------------ indexer scores

@pytest.mark.parametrize("name", FLAT)
def test_flat_index_scores(cuda, name):
    w = SMALL[name]
    wt = wt_of(name)
    for pi, p in enumerate(w.passes):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sc = H.flat_scores(wt, pi, st).cpu().numpy().astype(np.float64)
        assert lsa.read_device_status(st) == lsa.OK
        q_seq, q_pos = W.query_rows(w, p)
        plan = W.plant_plan(w, p) if p.name == "target" and (w.plant_frac or w.plant_blocks) else None
        for t in tokens_to_check(w, p):
            b, pos, L, qi, wi = run.query_context(w, p, t)
            K = run.index_keys(w, p, b, np.arange(pos + 1), plan)
            ref = olsa.indexer_scores(qi, wi, K)
            assert H.score_close(sc[t, :pos + 1], ref) < 1e-3
            assert np.all(np.isneginf(sc[t, pos + 1:wt.L_alloc]))


# The FP8-query mode needs the tensor-core indexer (FP8 keys, d_I = 128, H_I a multiple of 32).
Q8 = ["cli_small", "mtp_small", "prefill_small", "cli_unaligned"]


@pytest.mark.parametrize("name", Q8)
def test_fp8_query_index_scores(cuda, name):
    """FP8-query mode against the oracle's FP8-query scores (same query rounding; products of
    e4m3 values are exact, so only the FP32 accumulation differs), and visibly different from
    the exact BF16-query scores."""
    w = SMALL[name]
    wt = wt_of(name)
    for pi, p in enumerate(w.passes):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sc = H.flat_scores(wt, pi, st, q_fp8=True).cpu().numpy().astype(np.float64)
        assert lsa.read_device_status(st) == lsa.OK
        plan = W.plant_plan(w, p) if p.name == "target" and (w.plant_frac or w.plant_blocks) else None
        moved = 0.0
        for t in tokens_to_check(w, p):
            b, pos, L, qi, wi = run.query_context(w, p, t)
            K = run.index_keys(w, p, b, np.arange(pos + 1), plan)
            ref = olsa.indexer_scores_fp8q(qi, wi, K)
            assert H.score_close(sc[t, :pos + 1], ref) < 1e-4
            assert np.all(np.isneginf(sc[t, pos + 1:wt.L_alloc]))
            moved = max(moved, H.score_close(olsa.indexer_scores(qi, wi, K), ref))
        assert moved > 1e-3                      # the rounding of q is real: the mode changes the scores


def test_fp8_query_mode_unsupported_shapes(cuda):
    for name in ("tiny_decode", "cli_d64"):
        wt = wt_of(name)
        with pytest.raises(lsa.LsaError) as e:
            H.flat_scores(wt, 0, q_fp8=True)
        assert e.value.status == lsa.ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["cli_small", "mtp_small"])
def test_fp8_query_fused_selection(cuda, name):
    """The fused step in FP8-query mode selects what the oracle's top-k selects on the GPU's own
    FP8-query scores, and its attention matches the oracle on that index list."""
    w = SMALL[name]
    wt = wt_of(name)
    p = w.passes[0]
    sc = H.flat_scores(wt, 0, q_fp8=True).cpu().numpy().astype(np.float64)
    step, ws, idx, cnt, layers = H.decode_step(wt, 0, n_split=2, idx_q_fp8=True)
    step(ws)
    got = H.index_lists(idx, cnt)
    _, q_pos = W.query_rows(w, p)
    for t in range(w.T(p)):
        pos = int(q_pos[t])
        picks = olsa.topk(sc[t, :pos + 1], np.arange(pos + 1), w.k)
        assert got[t].tolist() == olsa.union_fixed(picks, pos, w.n_sink, w.window).tolist()


def test_hi_fine_scores_fp8_query(cuda):
    """HI fine stage in FP8-query mode: scores over recalled blocks equal the oracle's FP8-query
    scores at the blocks' positions."""
    w = SMALL["hi_small"]
    wt = wt_of("hi_small")
    p = w.passes[0]
    pt = wt.passes[0]
    T = pt.q_idx.shape[0]
    nblk = (wt.L_alloc + w.block_size - 1) // w.block_size
    n_cand = 6
    cand = torch.full((T, n_cand), -1, dtype=torch.int32)
    _, q_pos = W.query_rows(w, p)
    for t in range(T):
        vis = int(q_pos[t]) // w.block_size + 1
        picks = sorted({0, vis - 1, vis // 2, vis // 3, max(0, vis - 7)})
        cand[t, :len(picks)] = torch.tensor(picks, dtype=torch.int32)
    cand = cand.cuda()
    sc = torch.empty((T, n_cand * w.block_size), dtype=torch.float32, device="cuda")
    lsa.index_score(H.batch_of(wt), pt.q_idx, pt.w, H.idx_cache(wt), sc, cand_blocks=cand, block_size=w.block_size,
                    q_fp8=True)
    sc = sc.cpu().numpy().astype(np.float64)
    cand = cand.cpu().numpy()
    plan = W.plant_plan(w, p)
    assert nblk >= n_cand
    for t in tokens_to_check(w, p):
        b, pos, L, qi, wi = run.query_context(w, p, t)
        for j, blk in enumerate(cand[t]):
            cols = sc[t, j * w.block_size:(j + 1) * w.block_size]
            if blk < 0:
                assert np.all(np.isneginf(cols))
                continue
            rows = np.arange(blk * w.block_size, (blk + 1) * w.block_size)
            vis = rows <= pos
            K = run.index_keys(w, p, b, rows[vis], plan)
            ref = olsa.indexer_scores_fp8q(qi, wi, K)
            assert H.score_close(cols[vis], ref) < 1e-4
            assert np.all(np.isneginf(cols[~vis]))


@pytest.mark.parametrize("heads", [64, 16])
def test_block_keys_and_block_scores(cuda, heads):
    """Block keys against the oracle's means, block scores against the indexer formula on them;
    64 heads (32-column TMEM reads) and 16 heads (8-column reads, query rows padded to 32)."""
    if heads == 64:
        w, wt = SMALL["hi_small"], wt_of("hi_small")
    else:
        w = W.scaled("decode_hi_1m", B=2, len_lo=9000, len_hi=9000, H_I=16, seed=16)
        wt = D.build_workload(w, "cuda")
    p = w.passes[0]
    kbar_dev = H.block_keys(wt)
    kbar = H.block_key_values(kbar_dev)
    plan = W.plant_plan(w, p)
    nblk = kbar.shape[1]
    bsc = torch.empty((w.B, (nblk + 3) // 4 * 4), dtype=torch.float32, device="cuda")
    lsa.block_score(H.batch_of(wt), wt.passes[0].q_idx, wt.passes[0].w, kbar_dev, w.block_size, bsc, nblk)
    bsc = bsc.cpu().numpy().astype(np.float64)
    for t in range(w.T(p)):
        b, pos, L, qi, wi = run.query_context(w, p, t)
        ref_kbar = run.block_keys_of_sequence(w, p, b, L, plan)
        # the FP32 mean stored as hi + lo (16 significant bits): within 2^-16 of each key
        err = np.abs(kbar[b, :ref_kbar.shape[0]] - ref_kbar)
        assert np.all(err <= 2.0 ** -16 * np.abs(ref_kbar) + 1e-6 * np.abs(ref_kbar).max())
        nvis = pos // w.block_size + 1
        J = olsa.indexer_scores(qi, wi, ref_kbar[:nvis])
        assert H.score_close(bsc[t, :nvis], J) < 1e-3
        assert np.all(np.isneginf(bsc[t, nvis:nblk]))


# ------------------------------------------------------------------ top-k in isolation

def _host_score_rows(rng, T, n_cols, tie_levels):
    s = rng.integers(0, tie_levels, size=(T, n_cols)).astype(np.float32) * np.float32(0.25)
    s[:, ::7] = rng.normal(size=(T, (n_cols + 6) // 7)).astype(np.float32)
    s[:, 3::11] = -0.0
    s[:, 5::13] = -np.inf
    return s


@pytest.mark.parametrize("n_cols,k,n_sink,window,tie_levels", [
    (5000, 256, 4, 128, 3), (5000, 256, 4, 128, 1000), (3000, 2048, 4, 512, 5), (100, 300, 4, 16, 2),
    (70000, 2048, 4, 512, 50), (4097, 0, 4, 128, 3), (4097, 33, 0, 0, 4),
    # ~30000 keys share the threshold bin: more candidates than CTA 0's merged list holds, so
    # the cluster finishes with the full passes over its segments
    (70000, 2048, 4, 512, 2),
])
def test_topk_matches_oracle_exactly(cuda, n_cols, k, n_sink, window, tie_levels):
    rng = np.random.default_rng(n_cols + k)
    T = 5
    s = _host_score_rows(rng, T, n_cols, tie_levels)
    pos = np.array([n_cols - 1, n_cols // 2, 10, min(n_cols - 1, 3), n_cols - 2])
    s_masked = s.copy()
    for t in range(T):
        s_masked[t, pos[t] + 1:] = -np.inf
    batch = lsa.Batch(torch.tensor([n_cols], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"),
                      torch.from_numpy(pos.astype(np.int32)).cuda(), n_cols)
    cap = k + n_sink + window
    idx = torch.empty((T, max(cap, 1)), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s_masked).cuda(), n_cols, k, n_sink, window, idx, cnt, dev_status=st)
    assert lsa.read_device_status(st) == lsa.OK
    got = H.index_lists(idx, cnt)
    for t in range(T):
        valid = ~np.isneginf(s_masked[t])
        cols = np.nonzero(valid)[0]
        picks = olsa.topk(s_masked[t, cols].astype(np.float64), cols, k)
        want = olsa.union_fixed(picks, int(pos[t]), n_sink, window)
        assert got[t].tolist() == want.tolist()
        assert np.all(idx[t, cnt[t]:].cpu().numpy() == -1)


@pytest.mark.parametrize("T,n_cols,fixed_budget,tie_levels", [
    (63, 30000, False, 40),        # fewer than 64 rows: clusters of 8
    (64, 30000, False, 40),        # clusters of 2 (a row's half fits the shared-memory cache);
                                   # a wide threshold bin: the full passes over the segments
    (64, 30000, False, 100000),    # clusters of 2, few candidates: the compacted finish
    (64, 30000, True, 40),
    (64, 100000, False, 100000),   # clusters of 4 (a half does not fit, a quarter does)
    (64, 200000, False, 100000),   # clusters of 8 (a quarter does not fit either)
])
def test_topk_cluster_sizes(cuda, T, n_cols, fixed_budget, tie_levels):
    """The launch picks the cluster size per row from the row count and the row width; every
    choice must give the oracle's lists.  Positions differ per row (several rows see only part
    of the row), scores carry ties."""
    rng = np.random.default_rng(T * 1000 + n_cols + int(fixed_budget) + tie_levels)
    k, n_sink, window = 2048, 4, 512
    s = _host_score_rows(rng, T, n_cols, tie_levels)
    pos = rng.integers(n_cols // 3, n_cols, size=T)
    pos[:3] = [n_cols - 1, 700, 3000]
    for t in range(T):
        s[t, pos[t] + 1:] = -np.inf
    batch = lsa.Batch(torch.tensor([n_cols], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"),
                      torch.from_numpy(pos.astype(np.int32)).cuda(), n_cols)
    idx = torch.empty((T, k + n_sink + window), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s).cuda(), n_cols, k, n_sink, window, idx, cnt, dev_status=st,
             fixed_budget=fixed_budget)
    assert lsa.read_device_status(st) == lsa.OK
    got = H.index_lists(idx, cnt)
    for t in range(T):
        cols = np.nonzero(~np.isneginf(s[t]))[0]
        sc = s[t, cols].astype(np.float64)
        if fixed_budget:
            want = olsa.union_fixed_budget(sc, cols, k, int(pos[t]), n_sink, window)
        else:
            want = olsa.union_fixed(olsa.topk(sc, cols, k), int(pos[t]), n_sink, window)
        assert got[t].tolist() == want.tolist(), t


@pytest.mark.parametrize("n_cols", [3000, 70000])
def test_topk_all_equal_scores(cuda, n_cols):
    """Every visible score equal (as when every weighted ReLU sum is 0): the selection is the
    k lowest positions, then the union with the sinks and the window."""
    T, k, n_sink, window = 3, 2048, 4, 512
    pos = np.array([n_cols - 1, n_cols // 3, 100])
    s = np.zeros((T, n_cols), dtype=np.float32)
    for t in range(T):
        s[t, pos[t] + 1:] = -np.inf
    batch = lsa.Batch(torch.tensor([n_cols], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"),
                      torch.from_numpy(pos.astype(np.int32)).cuda(), n_cols)
    idx = torch.empty((T, k + n_sink + window), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s).cuda(), n_cols, k, n_sink, window, idx, cnt)
    got = H.index_lists(idx, cnt)
    for t in range(T):
        cols = np.arange(pos[t] + 1)
        picks = olsa.topk(s[t, cols].astype(np.float64), cols, k)
        assert picks.tolist() == list(range(min(k, pos[t] + 1)))      # ties: lowest positions
        want = olsa.union_fixed(picks, int(pos[t]), n_sink, window)
        assert got[t].tolist() == want.tolist()


@pytest.mark.parametrize("n_cols,k,n_sink,window,tie_levels", [
    (5000, 256, 4, 128, 3), (70000, 2048, 4, 512, 50), (70000, 2048, 4, 512, 2), (100, 300, 4, 16, 2),
])
def test_topk_fixed_budget(cuda, n_cols, k, n_sink, window, tie_levels):
    """Fixed-budget SI: the oracle's top-k over the positions outside the sinks and the window,
    then the (disjoint) union; the list holds exactly min(k, outside) + sinks + window."""
    rng = np.random.default_rng(n_cols + k + 7)
    T = 4
    s = _host_score_rows(rng, T, n_cols, tie_levels)
    pos = np.array([n_cols - 1, n_cols // 2, 10, n_cols - 2])
    for t in range(T):
        s[t, pos[t] + 1:] = -np.inf
    # the best scores of every row sit in its window and its sinks: the budget must skip them
    for t in range(T):
        s[t, max(0, pos[t] - 3):pos[t] + 1] = 1e6
        s[t, :2] = 1e6
    batch = lsa.Batch(torch.tensor([n_cols], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"),
                      torch.from_numpy(pos.astype(np.int32)).cuda(), n_cols)
    idx = torch.empty((T, k + n_sink + window), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s).cuda(), n_cols, k, n_sink, window, idx, cnt, fixed_budget=True)
    got = H.index_lists(idx, cnt)
    for t in range(T):
        cols = np.nonzero(~np.isneginf(s[t]))[0]
        want = olsa.union_fixed_budget(s[t, cols].astype(np.float64), cols, k, int(pos[t]), n_sink, window)
        assert got[t].tolist() == want.tolist()
        a = min(n_sink, pos[t] + 1)
        b = max(a, pos[t] - window + 1)
        outside = int(np.sum((cols >= a) & (cols < b)))
        assert len(got[t]) == min(k, outside) + a + (pos[t] + 1 - b)
        assert np.all(idx[t, cnt[t]:].cpu().numpy() == -1)


def test_topk_fixed_budget_candidate_blocks(cuda):
    rng = np.random.default_rng(2)
    T, bs, n_cand = 3, 64, 40
    blocks = np.stack([np.sort(rng.choice(500, size=n_cand, replace=False)) for _ in range(T)])
    blocks[:, 0] = 0                                          # the sinks' block is recalled
    blocks[2, -5:] = -1
    pos = np.array([500 * 64 - 1, 250 * 64 + 17, 30000])
    for t in range(T):                                        # and the window's last block
        last = int(pos[t]) // bs
        if last not in blocks[t]:
            blocks[t, 1] = last
        blocks[t] = np.sort(np.where(blocks[t] < 0, 10 ** 6, blocks[t]))
        blocks[t] = np.where(blocks[t] == 10 ** 6, -1, blocks[t])
    s = rng.integers(0, 20, size=(T, n_cand * bs)).astype(np.float32)
    for t in range(T):
        p_of_col = (blocks[t][:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
        bad = (np.repeat(blocks[t], bs) < 0) | (p_of_col > pos[t])
        s[t, bad] = -np.inf
        s[t, (p_of_col <= pos[t]) & (p_of_col > pos[t] - 50) & ~bad] = 1e6     # top scores in the window
    batch = lsa.Batch(torch.tensor([500 * 64], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"), torch.from_numpy(pos.astype(np.int32)).cuda(),
                      500 * 64)
    cb = torch.from_numpy(blocks.astype(np.int32)).cuda()
    k, ns, win = 300, 4, 100
    idx = torch.empty((T, k + ns + win), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s).cuda(), n_cand * bs, k, ns, win, idx, cnt, cand_blocks=cb, block_size=bs,
             fixed_budget=True)
    got = H.index_lists(idx, cnt)
    for t in range(T):
        p_of_col = (blocks[t][:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
        valid = ~np.isneginf(s[t])
        want = olsa.union_fixed_budget(s[t, valid].astype(np.float64), p_of_col[valid], k, int(pos[t]), ns, win)
        assert got[t].tolist() == want.tolist()


@pytest.mark.parametrize("fixed", [False, True])
@pytest.mark.parametrize("n_cols", [5000, 70000])
def test_topk_window_aligned(cuda, n_cols, fixed):
    """Block-aligned SI window: the window starts on the 64-row boundary at or below
    pos - window + 1; plain union and fixed budget, against the oracle's aligned reading."""
    rng = np.random.default_rng(n_cols + 3 * fixed)
    T, k, n_sink, window = 5, 300, 4, 100
    s = _host_score_rows(rng, T, n_cols, 50)
    pos = np.array([n_cols - 1, n_cols // 2 + 5, 130, 700, 63])
    for t in range(T):
        s[t, pos[t] + 1:] = -np.inf
    batch = lsa.Batch(torch.tensor([n_cols], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"),
                      torch.from_numpy(pos.astype(np.int32)).cuda(), n_cols)
    cap = k + n_sink + window + lsa.WINDOW_ALIGN - 1
    idx = torch.empty((T, cap), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s).cuda(), n_cols, k, n_sink, window, idx, cnt, dev_status=st,
             fixed_budget=fixed, window_aligned=True)
    assert lsa.read_device_status(st) == lsa.OK
    got = H.index_lists(idx, cnt)
    for t in range(T):
        cols = np.nonzero(~np.isneginf(s[t]))[0]
        sc = s[t, cols].astype(np.float64)
        if fixed:
            want = olsa.union_fixed_budget(sc, cols, k, int(pos[t]), n_sink, window, align=64)
        else:
            want = olsa.union_fixed(olsa.topk(sc, cols, k), int(pos[t]), n_sink, window, align=64)
        assert got[t].tolist() == want.tolist(), t
        assert np.all(idx[t, cnt[t]:].cpu().numpy() == -1)
    # ld_idx must leave room for the 63 extra window positions
    small = torch.empty((T, k + n_sink + window), dtype=torch.int32, device="cuda")
    with pytest.raises(lsa.LsaError):
        lsa.topk(batch, torch.from_numpy(s).cuda(), n_cols, k, n_sink, window, small, cnt, window_aligned=True)


def test_fused_step_window_aligned(cuda):
    w = SMALL["cli_small"]
    wt = wt_of("cli_small")
    p = w.passes[0]
    sc = H.flat_scores(wt).cpu().numpy().astype(np.float64)
    step, ws, idx, cnt, layers = H.decode_step(wt, 0, n_split=2, cap_extra=lsa.WINDOW_ALIGN - 1,
                                               si_window_aligned=True)
    assert step.index_capacity() == w.cap + lsa.WINDOW_ALIGN - 1
    step(ws)
    got = H.index_lists(idx, cnt)
    _, q_pos = W.query_rows(w, p)
    for t in range(w.T(p)):
        pos = int(q_pos[t])
        picks = olsa.topk(sc[t, :pos + 1], np.arange(pos + 1), w.k)
        assert got[t].tolist() == olsa.union_fixed(picks, pos, w.n_sink, w.window, align=64).tolist()
    t = w.T(p) - 1
    o_ref, _ = run.attend(w, p, p.layers[0], t, got[t])
    mx, rl2 = H.attn_errors(H.bf16_to_np(layers[0].o[t]), o_ref)
    assert mx < 1e-2 and rl2 < 5e-3


def test_topk_raw_and_candidate_blocks(cuda):
    rng = np.random.default_rng(1)
    T, bs, n_cand = 3, 64, 40
    blocks = np.stack([np.sort(rng.choice(500, size=n_cand, replace=False)) for _ in range(T)])
    blocks[2, -5:] = -1                                     # unused tail
    pos = np.array([500 * 64 - 1, 250 * 64 + 17, 30000])
    s = rng.integers(0, 20, size=(T, n_cand * bs)).astype(np.float32)
    for t in range(T):
        p_of_col = (blocks[t][:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
        bad = (np.repeat(blocks[t], bs) < 0) | (p_of_col > pos[t])
        s[t, bad] = -np.inf
    batch = lsa.Batch(torch.tensor([500 * 64], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"), torch.from_numpy(pos.astype(np.int32)).cuda(),
                      500 * 64)
    cb = torch.from_numpy(blocks.astype(np.int32)).cuda()
    k, ns, win = 300, 4, 100
    idx = torch.empty((T, k + ns + win), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    sd = torch.from_numpy(s).cuda()
    lsa.topk(batch, sd, n_cand * bs, k, ns, win, idx, cnt, cand_blocks=cb, block_size=bs)
    got = H.index_lists(idx, cnt)
    raw_idx = torch.empty((T, 50), dtype=torch.int32, device="cuda")
    lsa.topk(batch, sd, n_cand * bs, 50, 0, 0, raw_idx, cnt, raw=True)
    got_raw = H.index_lists(raw_idx, cnt)
    for t in range(T):
        p_of_col = (blocks[t][:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
        valid = ~np.isneginf(s[t])
        picks = olsa.topk(s[t, valid].astype(np.float64), p_of_col[valid], k)
        assert got[t].tolist() == olsa.union_fixed(picks, int(pos[t]), ns, win).tolist()
        cols = np.nonzero(valid)[0]
        assert got_raw[t].tolist() == sorted(olsa.topk(s[t, valid].astype(np.float64), cols, 50).tolist())


# ------------------------------------------------------------------ attention in isolation

@pytest.mark.parametrize("name", ["tiny_decode", "cli_small", "mtp_small"])
@pytest.mark.parametrize("n_split", [1, 3, 7])
def test_attention_on_oracle_index(cuda, name, n_split):
    w = SMALL[name]
    wt = wt_of(name)
    p = w.passes[0]
    toks = tokens_to_check(w, p, limit=4)
    T = w.T(p)
    plan = W.plant_plan(w, p) if (w.plant_frac or w.plant_blocks) else None
    lists = {t: run.index_list(w, p, t, plan)[0] for t in toks}
    cap = w.cap
    idx = torch.full((T, cap), -1, dtype=torch.int32)
    cnt = torch.zeros(T, dtype=torch.int32)
    for t, l in lists.items():
        idx[t, :len(l)] = torch.from_numpy(l.astype(np.int32))
        cnt[t] = len(l)
    idx, cnt = idx.cuda(), cnt.cuda()
    batch = H.batch_of(wt)
    for li, layer in enumerate(p.layers):
        kv, v = H.kv_cache(wt, 0, li)
        q = wt.passes[0].layers[li]["q"]
        o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
        ws = torch.empty(max(256, lsa.attn_workspace_size(T, w.H, w.Dv, n_split)), dtype=torch.uint8, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        lsa.sparse_attn(batch, q, kv, idx, cnt, w.sm_scale, o, lse, v=v, n_split=n_split, ws=ws, dev_status=st)
        assert lsa.read_device_status(st) == lsa.OK
        on, ln = H.bf16_to_np(o), lse.cpu().numpy()
        for t in toks:
            o_ref, lse_ref = run.attend(w, p, layer, t, lists[t])
            mx, rl2 = H.attn_errors(on[t], o_ref)
            assert mx < 1e-2 and rl2 < 5e-3, (t, mx, rl2)
            assert np.abs(ln[t] - lse_ref).max() < 1e-3 * max(1.0, np.abs(lse_ref).max())


@pytest.mark.parametrize("n_split", [1, 3, 7])
def test_attention_runs_of_consecutive_rows(cuda, n_split):
    """Tiles of 32 consecutive valid rows (one TMA box per atom) next to scattered tiles (row
    gathers): runs that start on and off a tile boundary, a run cut by the list's end, a run
    that ends at the query's position (the window), and a short run inside a scattered tile."""
    name = "cli_small"
    w = SMALL[name]
    wt = wt_of(name)
    p = w.passes[0]
    T = w.T(p)
    q_seq, q_pos = W.query_rows(w, p)
    rng = np.random.default_rng(7)
    lists = {}
    for t in range(T):
        pos = int(q_pos[t])
        scattered = np.sort(rng.choice(np.arange(200, 1500), size=45, replace=False))
        parts = [np.arange(0, 96),                       # three whole tiles from list offset 0
                 scattered[:5],                          # shifts the next run off the tile grid
                 np.arange(1600, 1670),                  # a run across two tile boundaries
                 scattered[5:],
                 np.arange(1700, 1708),                  # a run shorter than a tile
                 np.arange(pos - 99, pos + 1)]           # the window, ending at the query
        l = np.unique(np.concatenate(parts))
        l = l[l <= pos]
        lists[t] = l.astype(np.int64)
    cap = max(len(l) for l in lists.values())
    idx = torch.full((T, cap), -1, dtype=torch.int32)
    cnt = torch.zeros(T, dtype=torch.int32)
    for t, l in lists.items():
        idx[t, :len(l)] = torch.from_numpy(l.astype(np.int32))
        cnt[t] = len(l)
    idx, cnt = idx.cuda(), cnt.cuda()
    batch = H.batch_of(wt)
    layer = p.layers[0]
    kv, v = H.kv_cache(wt, 0, 0)
    q = wt.passes[0].layers[0]["q"]
    o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(256, lsa.attn_workspace_size(T, w.H, w.Dv, n_split)), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.sparse_attn(batch, q, kv, idx, cnt, w.sm_scale, o, lse, v=v, n_split=n_split, ws=ws, dev_status=st)
    assert lsa.read_device_status(st) == lsa.OK
    on, ln = H.bf16_to_np(o), lse.cpu().numpy()
    for t in range(T):
        o_ref, lse_ref = run.attend(w, p, layer, t, lists[t])
        mx, rl2 = H.attn_errors(on[t], o_ref)
        assert mx < 1e-2 and rl2 < 5e-3, (t, mx, rl2)
        assert np.abs(ln[t] - lse_ref).max() < 1e-3 * max(1.0, np.abs(lse_ref).max())


# ------------------------------------------------------------------ whole path

@pytest.mark.parametrize("name", list(SMALL))
def test_fused_path_end_to_end(cuda, name):
    w = SMALL[name]
    wt = wt_of(name)
    for pi, p in enumerate(w.passes):
        step, ws, idx, cnt, layers = H.decode_step(wt, pi, n_split=3)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        step(ws, st)
        assert lsa.read_device_status(st) == lsa.OK
        got = H.index_lists(idx, cnt)
        plan = W.plant_plan(w, p) if p.name == "target" and (w.plant_frac or w.plant_blocks) else None
        outs = [(H.bf16_to_np(L.o), L.lse.cpu().numpy()) for L in layers]
        for t in tokens_to_check(w, p, limit=4):
            ref = run.run_query(w, p, t, plan)
            a, b = set(got[t].tolist()), set(ref["idx"].tolist())
            assert len(a & b) >= 0.999 * len(b) and len(a) == len(b), (t, len(a), len(b), len(a & b))
            assert np.all(np.diff(got[t]) > 0)
            for li, layer in enumerate(p.layers):
                # where the lists differ (near-ties decided in FP32), the attention is checked on
                # the GPU's own list
                o_ref = ref["layers"][li][0] if a == b else run.attend(w, p, layer, t, got[t])[0]
                mx, rl2 = H.attn_errors(outs[li][0][t], o_ref)
                assert mx < 1e-2 and rl2 < 5e-3, (t, li, mx, rl2, a == b)


def test_fused_step_waits_for_the_prolog_event(cuda):
    """attn_q_ready: the attention layers wait for the caller's event (the MLA prolog writing their
    queries on another stream), the index selection does not need to.  The queries start as zeros
    and are written on a side stream after a delay; the outputs must equal those of a step whose
    queries were ready from the start, bit for bit, and so must the index lists."""
    wt = wt_of("cli_small")
    step, ws, idx_ref, cnt_ref, layers = H.decode_step(wt, 0, n_split=2)
    step(ws)
    torch.cuda.synchronize()
    ref = [L.o.clone() for L in layers]
    w = wt.w
    pt = wt.passes[0]
    q_late = [torch.zeros_like(L.q) for L in layers]
    lay = [lsa.Layer(q, L.kv, torch.full_like(L.o, float("nan")), torch.empty_like(L.lse), L.v)
           for q, L in zip(q_late, layers)]
    idx = torch.full_like(idx_ref, -7)
    cnt = torch.zeros_like(cnt_ref)
    ev = torch.cuda.Event()
    dec = lsa.DecodeStep(H.batch_of(wt), pt.q_idx, pt.w, H.idx_cache(wt), w.k, w.n_sink, w.window, lay, w.H, w.D,
                         w.Dv, w.sm_scale, n_split=2, idx_out=idx, count_out=cnt, attn_q_ready=ev)
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    side.wait_stream(main)
    with torch.cuda.stream(side):
        torch.cuda._sleep(20_000_000)                       # the "prolog" takes a while
        for q, L in zip(q_late, layers):
            q.copy_(L.q)
        ev.record(side)
    dec(ws, stream=main)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref) and torch.equal(cnt, cnt_ref)
    for a, b in zip(lay, ref):
        assert torch.equal(a.o.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["cli_small", "mtp_small"])
def test_pipeline_host_io_matches_device_path(cuda, name):
    """lsa_pipeline_*: queries copied in from pinned host memory into two slots of device
    buffers (which start zeroed), the fused decode, outputs copied back into host buffers
    (which start as garbage); after three steps every host output equals, bit for bit, the
    output of lsa_decode_fused called directly on the same queries."""
    w = SMALL[name]
    wt = wt_of(name)
    pi, pt = 0, wt.passes[0]
    step, ws, idx, cnt, layers = H.decode_step(wt, pi, n_split=3)
    step(ws)
    torch.cuda.synchronize()
    ref = [L.o.cpu() for L in layers]
    slots = []
    for s in range(2):
        q_idx, wv = torch.zeros_like(pt.q_idx), torch.zeros_like(pt.w)
        ins, lay = [q_idx, wv], []
        for L in layers:
            q = torch.zeros_like(L.q)
            ins.append(q)
            lay.append(lsa.Layer(q, L.kv, torch.zeros_like(L.o), torch.empty_like(L.lse), L.v))
        dec = lsa.DecodeStep(H.batch_of(wt, pi), q_idx, wv, H.idx_cache(wt, pi), w.k, w.n_sink, w.window, lay,
                             w.H, w.D, w.Dv, w.sm_scale, n_split=3, idx_out=idx, count_out=cnt)
        host_in = [t.cpu().contiguous().pin_memory() for t in [pt.q_idx, pt.w] + [L.q for L in layers]]
        host_out = [torch.full(L.o.shape, 7.0, dtype=L.o.dtype).pin_memory() for L in layers]
        slots.append((dec, list(zip(ins, host_in)), list(zip(host_out, [L.o for L in lay])), host_out))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pl = lsa.Pipeline(2)
    preps = [pl.prepare(s, [dec], [ws], h2d, d2h, st) for s, (dec, h2d, d2h, _) in enumerate(slots)]
    for i in range(3):
        pl.run(preps[i % 2])
    pl.join()
    torch.cuda.synchronize()
    assert lsa.read_device_status(st) == lsa.OK
    for _, _, _, host_out in slots:
        for li, h in enumerate(host_out):
            assert torch.equal(h, ref[li]), (li, (h.float() - ref[li].float()).abs().max())
    pl.close()


@pytest.mark.parametrize("name", FLAT)
def test_oracle_selection_on_gpu_scores_is_bit_exact(cuda, name):
    """The oracle's top-k + union, run on the GPU's own scores, gives the GPU's index list exactly."""
    w = SMALL[name]
    wt = wt_of(name)
    for pi, p in enumerate(w.passes):
        sc = H.flat_scores(wt, pi).cpu().numpy().astype(np.float64)
        step, ws, idx, cnt, _ = H.decode_step(wt, pi)
        step(ws)
        got = H.index_lists(idx, cnt)
        _, q_pos = W.query_rows(w, p)
        for t in range(w.T(p)):
            pos = int(q_pos[t])
            picks = olsa.topk(sc[t, :pos + 1], np.arange(pos + 1), w.k)
            assert got[t].tolist() == olsa.union_fixed(picks, pos, w.n_sink, w.window).tolist()


@pytest.mark.parametrize("name", ["cli_small", "hi_small", "mtp_small"])
def test_two_runs_bitwise_identical(cuda, name):
    wt = wt_of(name)
    res = []
    for _ in range(2):
        step, ws, idx, cnt, layers = H.decode_step(wt, 0, n_split=4)
        step(ws)
        torch.cuda.synchronize()
        res.append([idx.cpu(), cnt.cpu()] + [L.o.cpu() for L in layers] + [L.lse.cpu() for L in layers])
    for x, y in zip(*res):
        assert torch.equal(x.view(torch.uint8) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.uint8) if y.dtype == torch.bfloat16 else y)


def test_split_count_invariance(cuda):
    wt = wt_of("cli_small")
    outs = {}
    for ns in (1, 2, 5, 16):
        step, ws, idx, cnt, layers = H.decode_step(wt, 0, n_split=ns)
        step(ws)
        outs[ns] = [H.bf16_to_np(L.o) for L in layers]
    for ns in (2, 5, 16):
        for a, b in zip(outs[1], outs[ns]):
            mx, rl2 = H.attn_errors(a, b.astype(np.float64))
            assert mx < 1e-2 and rl2 < 5e-3


def test_hi_with_every_block_recalled_equals_flat(cuda):
    base = SMALL["hi_small"]
    w_all = W.scaled("decode_hi_1m", B=2, len_lo=20000, len_hi=20000, n_recall=400)
    w_flat = W.scaled("decode_hi_1m", B=2, len_lo=20000, len_hi=20000, hi=False)
    wt = wt_of("hi_small")
    res = []
    for w in (w_all, w_flat):
        wt2 = D.WorkloadTensors(w, wt.L_alloc, wt.seq_len, wt.passes)
        step, ws, idx, cnt, _ = H.decode_step(wt2, 0)
        step(ws)
        res.append(H.index_lists(idx, cnt))
    assert all(a.tolist() == b.tolist() for a, b in zip(*res))
    assert base.n_recall == 256


# ------------------------------------------------------------------ device-side data errors

def test_device_data_errors_are_reported(cuda):
    wt = wt_of("cli_small")
    pt = wt.passes[0]
    bad_pos = pt.q_pos.clone()
    bad_pos[1] = wt.L_alloc + 5
    batch = lsa.Batch(wt.seq_len, pt.q_seq, bad_pos, wt.L_alloc)
    sc = torch.empty((pt.q_idx.shape[0], wt.L_alloc), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.index_score(batch, pt.q_idx, pt.w, H.idx_cache(wt), sc, n_cols=wt.L_alloc, dev_status=st)
    assert lsa.read_device_status(st) == lsa.ERR_DEVICE_DATA
    assert torch.isneginf(sc[1]).all()                        # the bad token sees no key
    assert torch.isfinite(sc[0, :int(pt.q_pos[0]) + 1]).all()
    # the same bad position in the HI fine stage (every group scores all candidate columns)
    n_cand = 8
    cand = torch.arange(n_cand, dtype=torch.int32, device="cuda").repeat(pt.q_idx.shape[0], 1).contiguous()
    sc_hi = torch.empty((pt.q_idx.shape[0], n_cand * 64), dtype=torch.float32, device="cuda")
    st.zero_()
    lsa.index_score(batch, pt.q_idx, pt.w, H.idx_cache(wt), sc_hi, n_cols=n_cand * 64, cand_blocks=cand,
                    block_size=64, dev_status=st)
    assert lsa.read_device_status(st) == lsa.ERR_DEVICE_DATA
    assert torch.isneginf(sc_hi[1]).all()
    # NaN score
    good = H.batch_of(wt)
    sc = H.flat_scores(wt)
    sc[0, 3] = float("nan")
    idx = torch.empty((sc.shape[0], 2564), dtype=torch.int32, device="cuda")
    cnt = torch.empty(sc.shape[0], dtype=torch.int32, device="cuda")
    st.zero_()
    lsa.topk(good, sc, wt.L_alloc, 2048, 4, 512, idx, cnt, dev_status=st)
    assert lsa.read_device_status(st) == lsa.ERR_DEVICE_DATA
    # index outside the sequence
    st.zero_()
    sc = H.flat_scores(wt)
    lsa.topk(good, sc, wt.L_alloc, 2048, 4, 512, idx, cnt)
    idx[0, 5] = 10 ** 7
    kv, _ = H.kv_cache(wt, 0, 0)
    o = torch.empty((sc.shape[0], 128, 512), dtype=torch.bfloat16, device="cuda")
    lsa.sparse_attn(good, pt.layers[0]["q"], kv, idx, cnt, 0.04, o, dev_status=st)
    assert lsa.read_device_status(st) == lsa.ERR_DEVICE_DATA
    torch.cuda.synchronize()
