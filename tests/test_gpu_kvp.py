"""KVP on the GPU: the sharded-context path of the C ABI against the single-device path and the oracle.

One process emulates several ranks' shards (the collectives are skipped with one rank; the data
crosses shards exactly as the all-gathers would lay it out).  Checks:

* the KVP index lists equal the fused single-device step's lists bit for bit (each shard's scores
  are the same kernel's scores of the same keys; the shard candidates contain the global top-k);
* every layer's merged attention within the attention tolerance of the oracle's attention on that
  list (max-abs 1e-2, relative L2 5e-3);
* lsa_sparse_attn_partial's FP32 result and lsa_merge_partials against the oracle, including empty
  partials (lse = -inf).
"""
import numpy as np
import pytest
import torch

from lsa_synth import device as D
from lsa_synth import workloads as W
from oracle import lsa as olsa, run

from long_context_sparse_indexer_b200 import kvp, lsa

from . import gpu_helpers as H

pytestmark = pytest.mark.gpu


def make_shards(wt, n_shards, pi=0):
    """Contiguous shards of every sequence, copied into per-shard caches (rows from 0)."""
    w = wt.w
    lens = W.lengths(w)
    pt = wt.passes[pi]
    shards = []
    for s in range(n_shards):
        st = np.array([int(lens[b]) * s // n_shards for b in range(w.B)], dtype=np.int32)
        en = np.array([int(lens[b]) * (s + 1) // n_shards for b in range(w.B)], dtype=np.int32)
        ln = en - st
        La = int(-(-int(ln.max()) // 64) * 64)
        k_loc = torch.zeros((w.B, La, w.d_I), dtype=pt.k_idx.dtype, device="cuda")
        s_loc = torch.ones((w.B, La), dtype=torch.float32, device="cuda") if pt.k_scale is not None else None
        kv_loc = []
        for L in pt.layers:
            kv_loc.append((torch.zeros((w.B, La, w.D), dtype=L["kv"].dtype, device="cuda"),
                           torch.ones((w.B, La), dtype=torch.float32, device="cuda") if L["kv_scale"] is not None
                           else None))
        for b in range(w.B):
            a, e = int(st[b]), int(en[b])
            k_loc[b, :e - a] = pt.k_idx[b, a:e]
            if s_loc is not None:
                s_loc[b, :e - a] = pt.k_scale[b, a:e]
            for (kv, ks), L in zip(kv_loc, pt.layers):
                kv[b, :e - a] = L["kv"][b, a:e]
                if ks is not None:
                    ks[b, :e - a] = L["kv_scale"][b, a:e]
        shards.append(kvp.Shard(torch.from_numpy(st).cuda(), torch.from_numpy(ln).cuda(), La,
                                lsa.Cache(k_loc, s_loc), [lsa.Cache(kv, ks) for kv, ks in kv_loc]))
    return shards


CASES = {
    "cli_3shards": (W.scaled("decode_cli_128k", B=3, len_lo=9000, len_hi=14000, seed=31), 3, 2),
    "mtp_2shards": (W.scaled("mtp_256k", B=2, len_lo=6001, len_hi=6001, seed=32), 2, 1),
}


@pytest.mark.parametrize("name", list(CASES))
def test_kvp_matches_single_device(cuda, name):
    w, n_shards, n_split = CASES[name]
    wt = D.build_workload(w, "cuda")
    p = w.passes[0]
    pt = wt.passes[0]
    step, ws, idx_ref, cnt_ref, layers = H.decode_step(wt, 0, n_split=1)
    step(ws)
    shards = make_shards(wt, n_shards)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dec = kvp.KVPDecode(H.batch_of(wt), pt.q_idx, pt.w, shards, w.k, w.n_sink, w.window,
                        [L["q"] for L in pt.layers], w.Dv, w.sm_scale, n_split=n_split, ops=kvp.LsaOps(dev_status=st))
    idx, cnt, outs = dec()
    torch.cuda.synchronize()
    assert lsa.read_device_status(st) == lsa.OK
    assert torch.equal(cnt, cnt_ref)
    assert torch.equal(idx, idx_ref)
    got = H.index_lists(idx, cnt)
    T = w.T(p)
    for li, layer in enumerate(p.layers):
        o = H.bf16_to_np(outs[li][0])
        for t in sorted({0, T // 2, T - 1}):
            o_ref, lse_ref = run.attend(w, p, layer, t, got[t])
            mx, rl2 = H.attn_errors(o[t], o_ref)
            assert mx < 1e-2 and rl2 < 5e-3, (li, t, mx, rl2)
            lse = outs[li][1][t].cpu().numpy()
            assert np.abs(lse - lse_ref).max() < 1e-3 * max(1.0, np.abs(lse_ref).max())


def test_partial_attention_and_merge_against_the_oracle(cuda):
    w = W.scaled("decode_cli_128k", B=2, len_lo=3000, len_hi=4000, seed=33)
    wt = D.build_workload(w, "cuda")
    p = w.passes[0]
    T = w.T(p)
    plan = None
    lists = {t: run.index_list(w, p, t, plan)[0] for t in range(T)}
    # two disjoint halves of each list (even / odd entries) and one empty part
    parts = [{t: l[0::2] for t, l in lists.items()}, {t: l[1::2] for t, l in lists.items()},
             {t: l[:0] for t, l in lists.items()}]
    kv, _ = H.kv_cache(wt, 0, 0)
    q = wt.passes[0].layers[0]["q"]
    o_parts = torch.empty((len(parts), T, w.H, w.Dv), dtype=torch.float32, device="cuda")
    l_parts = torch.empty((len(parts), T, w.H), dtype=torch.float32, device="cuda")
    for pi_, part in enumerate(parts):
        for n_split in (1, 3):
            idx = torch.full((T, w.cap), -1, dtype=torch.int32)
            cnt = torch.zeros(T, dtype=torch.int32)
            for t, l in part.items():
                idx[t, :len(l)] = torch.from_numpy(l.astype(np.int32))
                cnt[t] = len(l)
            ws = torch.empty(max(256, lsa.attn_workspace_size(T, w.H, w.Dv, n_split)), dtype=torch.uint8,
                             device="cuda")
            lsa.sparse_attn_partial(H.batch_of(wt), q, kv, idx.cuda(), cnt.cuda(), w.sm_scale, o_parts[pi_],
                                    l_parts[pi_], n_split=n_split, ws=ws)
            on, ln = o_parts[pi_].cpu().numpy().astype(np.float64), l_parts[pi_].cpu().numpy()
            for t, l in part.items():
                o_ref, lse_ref = run.attend(w, p, p.layers[0], t, l)
                if len(l) == 0:
                    assert np.all(on[t] == 0) and np.all(np.isneginf(ln[t]))
                    continue
                mx, rl2 = H.attn_errors(on[t], o_ref)
                assert mx < 1e-2 and rl2 < 5e-3, (pi_, n_split, t, mx, rl2)
                assert np.abs(ln[t] - lse_ref).max() < 1e-3 * max(1.0, np.abs(lse_ref).max())
    o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    lsa.merge_partials(o_parts, l_parts, o, lse)
    on = H.bf16_to_np(o)
    # the merge of the GPU's own partials by the oracle's rule, and the whole-list attention
    op_np, lp_np = o_parts.cpu().numpy().astype(np.float64), l_parts.cpu().numpy().astype(np.float64)
    for t in range(T):
        om, lm = olsa.merge_partials([op_np[i, t] for i in range(len(parts))], [lp_np[i, t] for i in range(len(parts))])
        assert np.abs(on[t] - om).max() <= 2.0 ** -8 * np.abs(om).max() + 1e-6
        assert np.abs(lse[t].cpu().numpy() - lm).max() < 1e-5 * max(1.0, np.abs(lm).max())
        o_ref, _ = run.attend(w, p, p.layers[0], t, lists[t])
        mx, rl2 = H.attn_errors(on[t], o_ref)
        assert mx < 1e-2 and rl2 < 5e-3, (t, mx, rl2)


@pytest.mark.parametrize("R,Dv", [(1, 512), (8, 512), (17, 512), (24, 512), (25, 512), (32, 512), (33, 512),
                                  (100, 512), (17, 200), (40, 136)])
def test_merge_partials_part_counts(cuda, R, Dv):
    """lsa_merge_partials against the oracle's merge for every kernel path: up to 24 partials held in
    registers, 25..32 with a second round trip, more than 32 through the block-per-head kernel; V
    widths that are not a multiple of 128; empty partials (lse = -inf), a head with every partial
    empty, and lse values far apart (one partial dominates)."""
    rng = np.random.default_rng(R * 1000 + Dv)
    T, H_ = 3, 24
    o_parts = rng.normal(size=(R, T, H_, Dv)).astype(np.float32)
    l_parts = (rng.normal(size=(R, T, H_)) * 3.0).astype(np.float32)
    l_parts[rng.random(size=(R, T, H_)) < 0.2] = -np.inf           # empty partials
    l_parts[:, 1, 5] = -np.inf                                     # a head with nothing at all
    l_parts[0, 2, 7] = 60.0                                        # one partial dominates
    o = torch.empty((T, H_, Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, H_), dtype=torch.float32, device="cuda")
    lsa.merge_partials(torch.from_numpy(o_parts).cuda(), torch.from_numpy(l_parts).cuda(), o, lse)
    on, ln = H.bf16_to_np(o), lse.cpu().numpy()
    for t in range(T):
        om, lm = olsa.merge_partials([o_parts[i, t].astype(np.float64) for i in range(R)],
                                     [l_parts[i, t].astype(np.float64) for i in range(R)])
        assert np.abs(on[t] - om).max() <= 2.0 ** -8 * np.abs(om).max() + 1e-6, t
        fin = np.isfinite(lm)
        assert np.array_equal(fin, np.isfinite(ln[t]))
        assert np.abs(ln[t][fin] - lm[fin]).max() < 1e-5 * max(1.0, np.abs(lm[fin]).max())
    assert np.all(on[1, 5] == 0) and np.isneginf(ln[1, 5])


def test_attention_with_many_splits(cuda):
    """lsa_sparse_attn with 40 splits (the wide merge) agrees with one split within the attention
    tolerance, on the oracle's own index lists."""
    wt = D.build_workload(W.scaled("decode_cli_128k", B=2, len_lo=6000, len_hi=8000, seed=5), "cuda")
    w = wt.w
    p = w.passes[0]
    T = w.T(p)
    lists = {t: run.index_list(w, p, t, None)[0] for t in range(T)}
    idx = torch.full((T, w.cap), -1, dtype=torch.int32)
    cnt = torch.zeros(T, dtype=torch.int32)
    for t, l in lists.items():
        idx[t, :len(l)] = torch.from_numpy(l.astype(np.int32))
        cnt[t] = len(l)
    idx, cnt = idx.cuda(), cnt.cuda()
    kv, _ = H.kv_cache(wt, 0, 0)
    q = wt.passes[0].layers[0]["q"]
    outs = {}
    for ns in (1, 40):
        o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
        ws = torch.empty(max(256, lsa.attn_workspace_size(T, w.H, w.Dv, ns)), dtype=torch.uint8, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        lsa.sparse_attn(H.batch_of(wt), q, kv, idx, cnt, w.sm_scale, o, lse, n_split=ns, ws=ws, dev_status=st)
        assert lsa.read_device_status(st) == lsa.OK
        outs[ns] = (H.bf16_to_np(o), lse.cpu().numpy())
    for t in range(T):
        o_ref, lse_ref = run.attend(w, p, p.layers[0], t, lists[t])
        for ns in (1, 40):
            mx, rl2 = H.attn_errors(outs[ns][0][t], o_ref)
            assert mx < 1e-2 and rl2 < 5e-3, (ns, t, mx, rl2)
            assert np.abs(outs[ns][1][t] - lse_ref).max() < 1e-3 * max(1.0, np.abs(lse_ref).max())
