"""GPU parity on the code paths the benchmark itself runs.

The small parity cases give each CTA of the persistent tensor-core indexer at most a few key
tiles.  The decode benchmark runs one query token per sequence (query groups of one, 256-key
tiles) with many tiles per CTA, so its CTAs wrap the five-stage key ring and the four
accumulator slots and cross from one query group to the next.  These cases reproduce that
tiling at sizes the float64 oracle still checks column by column:

* every visible indexer score column of several tokens (first, middle, last) within the
  indexer tolerance (relative 1e-3, floor 1% of the row's RMS score);
* the oracle's top-k + union run on the GPU's own scores equals the GPU's index list exactly,
  for every token;
* top-k rows wider than the shared-memory cache (327,680 columns), which run the uncached
  kernel, equal the oracle's selection exactly, with and without a crowded threshold bin.
"""
import numpy as np
import pytest
import torch

from lsa_synth import device as D
from lsa_synth import workloads as W
from oracle import lsa as olsa, run

from long_context_sparse_indexer_b200 import lsa

from . import gpu_helpers as H

pytestmark = pytest.mark.gpu

N_SMS = 148
TILE = 256          # keys per tile of the tensor-core indexer for query groups of one (N = 64)

BENCH_TILING = {
    # 8 sequences of 60K-64K keys: about 13 tiles per CTA, a few CTAs cross a sequence boundary
    "decode_b8_64k": W.scaled("decode_cli_128k", B=8, len_lo=60000, len_hi=64000),
    # 48 sequences of 7K-9K keys: about 10 tiles per CTA, most CTAs cross one or two boundaries
    "decode_b48_8k": W.scaled("decode_cli_128k", B=48, len_lo=7000, len_hi=9000, seed=21),
}

_cache = {}


def wt_of(name):
    if name not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        _cache[name] = D.build_workload(BENCH_TILING[name], "cuda")
    return _cache[name]


def tiles_per_cta(w):
    return float(np.sum((W.lengths(w) + TILE - 1) // TILE)) / N_SMS


@pytest.mark.parametrize("name", list(BENCH_TILING))
def test_indexer_every_column_at_bench_tiling(cuda, name):
    w = BENCH_TILING[name]
    p = w.passes[0]
    assert p.q_per_seq == 1 and tiles_per_cta(w) >= 8          # the ring and the slots wrap
    wt = wt_of(name)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sc = H.flat_scores(wt, 0, st).cpu().numpy().astype(np.float64)
    assert lsa.read_device_status(st) == lsa.OK
    T = w.T(p)
    for t in sorted({0, T // 3, T // 2, T - 1}):
        b, pos, L, qi, wi = run.query_context(w, p, t)
        K = run.index_keys(w, p, b, np.arange(pos + 1))
        ref = olsa.indexer_scores(qi, wi, K)
        assert H.score_close(sc[t, :pos + 1], ref) < 1e-3, t
        assert np.all(np.isneginf(sc[t, pos + 1:wt.L_alloc])), t


@pytest.mark.parametrize("name", list(BENCH_TILING))
def test_oracle_selection_on_gpu_scores_bit_exact_at_bench_tiling(cuda, name):
    w = BENCH_TILING[name]
    p = w.passes[0]
    wt = wt_of(name)
    sc = H.flat_scores(wt, 0).cpu().numpy().astype(np.float64)
    step, ws, idx, cnt, layers = H.decode_step(wt, 0, n_split=1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    step(ws, st)
    assert lsa.read_device_status(st) == lsa.OK
    got = H.index_lists(idx, cnt)
    _, q_pos = W.query_rows(w, p)
    for t in range(w.T(p)):
        pos = int(q_pos[t])
        picks = olsa.topk(sc[t, :pos + 1], np.arange(pos + 1), w.k)
        assert got[t].tolist() == olsa.union_fixed(picks, pos, w.n_sink, w.window).tolist(), t
    # attention of one middle token on that list (the list is the GPU's own, so this checks the
    # attention kernel at the bench's split count whatever the selection)
    t = w.T(p) // 2
    outs = H.bf16_to_np(layers[0].o[t])
    o_ref, _ = run.attend(w, p, p.layers[0], t, got[t])
    mx, rl2 = H.attn_errors(outs, o_ref)
    assert mx < 1e-2 and rl2 < 5e-3, (mx, rl2)


@pytest.mark.parametrize("tie_levels", [50, 2])
def test_topk_rows_wider_than_the_cache(cuda, tie_levels):
    """n_cols = 400,000 > 8 CTAs x 40,960 cached columns: the kernel re-reads its segments from
    global memory.  tie_levels = 2 puts most keys in the threshold bin, so the cluster finishes
    with full passes instead of CTA 0's compacted list."""
    n_cols, k, n_sink, window, T = 400_000, 2048, 4, 512, 3
    rng = np.random.default_rng(tie_levels)
    s = rng.integers(0, tie_levels, size=(T, n_cols)).astype(np.float32) * np.float32(0.25)
    s[:, ::7] = rng.normal(size=(T, (n_cols + 6) // 7)).astype(np.float32)
    s[:, 3::11] = -0.0
    pos = np.array([n_cols - 1, n_cols // 2 + 3, 350_001])
    for t in range(T):
        s[t, pos[t] + 1:] = -np.inf
    batch = lsa.Batch(torch.tensor([n_cols], dtype=torch.int32, device="cuda"),
                      torch.zeros(T, dtype=torch.int32, device="cuda"),
                      torch.from_numpy(pos.astype(np.int32)).cuda(), n_cols)
    idx = torch.empty((T, k + n_sink + window), dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s).cuda(), n_cols, k, n_sink, window, idx, cnt, dev_status=st)
    assert lsa.read_device_status(st) == lsa.OK
    got = H.index_lists(idx, cnt)
    for t in range(T):
        cols = np.arange(pos[t] + 1)
        picks = olsa.topk(s[t, cols].astype(np.float64), cols, k)
        assert got[t].tolist() == olsa.union_fixed(picks, int(pos[t]), n_sink, window).tolist(), t
    # raw mode on the same rows: the selected columns themselves
    raw = torch.empty((T, k), dtype=torch.int32, device="cuda")
    lsa.topk(batch, torch.from_numpy(s).cuda(), n_cols, k, 0, 0, raw, cnt, raw=True)
    got_raw = H.index_lists(raw, cnt)
    for t in range(T):
        cols = np.arange(pos[t] + 1)
        assert got_raw[t].tolist() == sorted(olsa.topk(s[t, cols].astype(np.float64), cols, k).tolist()), t
