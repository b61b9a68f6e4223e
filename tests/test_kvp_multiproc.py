"""KVP across ranks on CPU: the KVP driver over two gloo processes, every step done by the oracle.

The driver (``long_context_sparse_indexer_b200.kvp.KVPDecode``) orders the per-shard steps and
runs the all-gathers between them; here its ``ops`` are float64 restatements of the steps from
the oracle's functions (the CUDA path is checked against them on the GPU).  Two ranks with two
shards each split every sequence's context into four contiguous ranges.  The result must be the
single-device definition:

* the index list equal, bit for bit, to the oracle's selection over the whole context -- the
  candidates exchanged are each shard's top-k, and every key of the global top-k is in its
  shard's top-k (ties are many: queries and keys are small integers, so scores are exact);
* the merged attention equal to the oracle's attention over the whole list within 1e-12
  (log-sum-exp merge of per-shard partials in shard order, float64).
"""
import datetime
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

from oracle import lsa as olsa

B, H_I, D_I, H, D, DV = 2, 4, 16, 8, 24, 16
K, N_SINK, WINDOW = 40, 3, 17
LENS = [301, 517]
SM_SCALE = 0.2
N_SHARDS = 4                      # 2 ranks x 2 shards


def problem():
    """Integer-valued queries and keys (exact float64 scores, many ties), random KV rows."""
    rng = np.random.default_rng(5)
    L = max(LENS)
    keys = rng.integers(-2, 3, size=(B, L, D_I)).astype(np.float64)
    qi = rng.integers(-2, 3, size=(B, H_I, D_I)).astype(np.float64)
    w = rng.integers(1, 4, size=(B, H_I)).astype(np.float64)
    kv = rng.normal(size=(B, L, D))
    q = rng.normal(size=(B, H, D))
    return keys, qi, w, kv, q


def shard_ranges(n_shards):
    """Per sequence: contiguous, disjoint ranges covering 0 .. len - 1, in position order."""
    out = []
    for s in range(n_shards):
        out.append([(LENS[b] * s // n_shards, LENS[b] * (s + 1) // n_shards) for b in range(B)])
    return out


class OracleOps:
    """The KVP steps in float64 from the oracle's functions, on CPU tensors."""

    def __init__(self, keys, kv, qi, w, q):
        self.keys, self.kv, self.qi, self.w, self.q = keys, kv, qi, w, q

    def shard_batch(self, batch, sh, tag):
        from long_context_sparse_indexer_b200 import lsa
        st, ln = sh.start.numpy(), sh.length.numpy()
        q_seq, q_pos = batch.q_seq.numpy(), batch.q_pos.numpy()
        lqp = np.array([min(max(q_pos[t] - st[b], 0), ln[b] - 1) for t, b in enumerate(q_seq)], dtype=np.int32)
        return lsa.Batch(torch.from_numpy(ln.astype(np.int32)), batch.q_seq, torch.from_numpy(lqp), sh.L_alloc)

    def scores(self, local, q_idx, w, sh, tag):
        T = local.q_seq.numel()
        out = np.full((T, sh.L_alloc), -np.inf)
        for t, b in enumerate(local.q_seq.numpy()):
            p = int(local.q_pos[t])
            out[t, :p + 1] = olsa.indexer_scores(q_idx[t].numpy(), w[t].numpy(), sh.k_idx.data[b, :p + 1].numpy())
        return torch.from_numpy(out)

    def candidates(self, local, q_pos_global, sh, scores, k, tag):
        T = scores.shape[0]
        pos = np.full((T, k), -1, dtype=np.int32)
        sco = np.full((T, k), -np.inf)
        for t, b in enumerate(local.q_seq.numpy()):
            st = int(sh.start[b])
            if int(q_pos_global[t]) < st:
                continue
            row = scores[t].numpy()
            cols = np.nonzero(np.isfinite(row))[0]
            picks = np.sort(olsa.topk(row[cols], cols, k))
            pos[t, :picks.size] = picks + st
            sco[t, :picks.size] = row[picks]
        return torch.from_numpy(pos), torch.from_numpy(sco)

    def select(self, batch, pos_all, score_all, k, n_sink, window):
        T = pos_all.shape[1]
        cap = k + n_sink + window
        idx = np.full((T, cap), -1, dtype=np.int32)
        cnt = np.zeros(T, dtype=np.int32)
        for t in range(T):
            p, s = pos_all[:, t].numpy().reshape(-1), score_all[:, t].numpy().reshape(-1)
            ok = p >= 0
            sel = olsa.union_fixed(olsa.topk(s[ok], p[ok], k), int(batch.q_pos[t]), n_sink, window)
            idx[t, :sel.size] = sel
            cnt[t] = sel.size
        return torch.from_numpy(idx), torch.from_numpy(cnt)

    def local_index(self, batch, sh, idx, cnt, tag):
        T, cap = idx.shape
        lidx = np.full((T, cap), -1, dtype=np.int32)
        lcnt = np.zeros(T, dtype=np.int32)
        for t, b in enumerate(batch.q_seq.numpy()):
            st, ln = int(sh.start[b]), int(sh.length[b])
            row = idx[t, :int(cnt[t])].numpy()
            mine = row[(row >= st) & (row < st + ln)] - st
            lidx[t, :mine.size] = mine
            lcnt[t] = mine.size
        return torch.from_numpy(lidx), torch.from_numpy(lcnt)

    def partial(self, local, q, kv, lidx, lcnt, sm_scale, n_split, Dv, tag):
        T, Hh = q.shape[0], q.shape[1]
        o = np.zeros((T, Hh, Dv))
        lse = np.full((T, Hh), -np.inf)
        for t, b in enumerate(local.q_seq.numpy()):
            rows = lidx[t, :int(lcnt[t])].numpy()
            Kr = kv.data[b, rows].numpy()
            o[t], lse[t] = olsa.attention(q[t].numpy(), Kr, Kr[:, :Dv], sm_scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, o_all, lse_all, tag):
        P, T = o_all.shape[0], o_all.shape[1]
        o = np.zeros(tuple(o_all.shape[1:]))
        lse = np.zeros(tuple(lse_all.shape[1:]))
        for t in range(T):
            o[t], lse[t] = olsa.merge_partials([o_all[p, t].numpy() for p in range(P)],
                                               [lse_all[p, t].numpy() for p in range(P)])
        return torch.from_numpy(o), torch.from_numpy(lse)


def run_kvp(rank, world, group):
    from long_context_sparse_indexer_b200 import kvp, lsa
    keys, qi, w, kv, q = problem()
    per = N_SHARDS // world
    shards = []
    for s in range(rank * per, (rank + 1) * per):
        rng_ = shard_ranges(N_SHARDS)[s]
        st = np.array([a for a, _ in rng_], dtype=np.int32)
        ln = np.array([e - a for a, e in rng_], dtype=np.int32)
        La = int(ln.max())
        kl = np.zeros((B, La, D_I))
        vl = np.zeros((B, La, D))
        for b in range(B):
            kl[b, :ln[b]] = keys[b, st[b]:st[b] + ln[b]]
            vl[b, :ln[b]] = kv[b, st[b]:st[b] + ln[b]]
        shards.append(kvp.Shard(torch.from_numpy(st), torch.from_numpy(ln), La, lsa.Cache(torch.from_numpy(kl)),
                                [lsa.Cache(torch.from_numpy(vl))]))
    batch = lsa.Batch(torch.tensor(LENS, dtype=torch.int32), torch.arange(B, dtype=torch.int32),
                      torch.tensor([l - 1 for l in LENS], dtype=torch.int32), max(LENS))
    step = kvp.KVPDecode(batch, torch.from_numpy(qi), torch.from_numpy(w), shards, K, N_SINK, WINDOW,
                         [torch.from_numpy(q)], DV, SM_SCALE, group=group, world=world,
                         ops=OracleOps(keys, kv, qi, w, q))
    return step()


def reference():
    keys, qi, w, kv, q = problem()
    out = []
    for b in range(B):
        pos = LENS[b] - 1
        idx, _ = olsa.select(qi[b], w[b], keys[b, :LENS[b]], pos, K, N_SINK, WINDOW)
        o, lse = olsa.attention(q[b], kv[b, idx], kv[b, idx, :DV], SM_SCALE)
        out.append((idx, o, lse))
    return out


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        idx, cnt, outs = run_kvp(rank, world, None)
        o, lse = outs[0]
        q.put((rank, idx.numpy(), cnt.numpy(), o.numpy(), lse.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _check(idx, cnt, o, lse):
    for b, (ridx, ro, rlse) in enumerate(reference()):
        assert idx[b, :cnt[b]].tolist() == ridx.tolist()
        assert np.all(idx[b, cnt[b]:] == -1)
        assert np.abs(o[b] - ro).max() < 1e-12 * max(1.0, np.abs(ro).max())
        assert np.abs(lse[b] - rlse).max() < 1e-12 * max(1.0, np.abs(rlse).max())


def test_kvp_two_ranks_match_single_device_definition():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted((q.get(timeout=240) for _ in procs), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for _, idx, cnt, o, lse in got:                 # every rank holds the same, single-device result
        _check(idx, cnt, o, lse)
    assert np.array_equal(got[0][1], got[1][1]) and np.array_equal(got[0][3], got[1][3])


def test_kvp_one_process_four_shards():
    idx, cnt, outs = run_kvp(0, 1, None)
    _check(idx.numpy(), cnt.numpy(), outs[0][0].numpy(), outs[0][1].numpy())


def test_shard_candidates_contain_the_global_top_k():
    """The property the exchange rests on, by brute force: on every shard split tried, the global
    top-k (score desc, position asc) is a subset of the union of the shards' own top-k."""
    rng = np.random.default_rng(11)
    for trial in range(30):
        n = int(rng.integers(20, 200))
        s = rng.integers(0, 4, size=n).astype(np.float64)
        k = int(rng.integers(1, 30))
        cuts = np.sort(rng.choice(np.arange(1, n), size=int(rng.integers(1, 5)), replace=False))
        bounds = [0, *cuts.tolist(), n]
        union = np.concatenate([np.arange(a, e)[np.isin(np.arange(a, e), olsa.topk(s[a:e], np.arange(a, e), k))]
                                for a, e in zip(bounds[:-1], bounds[1:])])
        glob = olsa.topk(s, np.arange(n), k)
        assert np.isin(glob, union).all()
        assert olsa.topk(s[union], union, k).tolist() == glob.tolist()
