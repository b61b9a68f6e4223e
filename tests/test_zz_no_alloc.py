"""lsa_sparse_attn_noalloc: sparse attention for callers that cannot allocate device memory.

Callers such as a serving runtime whose memory pool is closed to new allocations, or a
plugin host that owns every cudaMalloc, cannot hand lsa_sparse_attn a workspace for its
split-KV partials.  The no-allocation entry point keeps those partials in the library's
own static device array instead.  This test calls it through the C ABI twice in a row
and checks each result against lsa_sparse_attn with a caller-provided workspace, within
the attention tolerance the parity tests use (max-abs 1e-2, relative L2 5e-3).  It builds
its own inputs, so it runs alone in a fresh process as well as after the other tests;
it sits in a file collected last so that a run stopping at its first failure has already
run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from lsa_synth import device as D
from lsa_synth import workloads as W

from long_context_sparse_indexer_b200 import lsa

pytestmark = pytest.mark.gpu


def _errors(a: torch.Tensor, b: torch.Tensor):
    x = a.float().cpu().numpy().astype(np.float64)
    y = b.float().cpu().numpy().astype(np.float64)
    d = x - y
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(y), 1e-30))


def test_noalloc_attention_matches_workspace_entry_point(cuda):
    w = W.scaled("decode_cli_128k", B=4, len_lo=3000, len_hi=6000)
    p = w.passes[0]
    wt = D.build_workload(w, "cuda")
    pt = wt.passes[0]
    T = w.T(p)
    batch = lsa.Batch(wt.seq_len, pt.q_seq, pt.q_pos, wt.L_alloc, q_group=p.q_per_seq)
    # Index lists from the library's own indexer + top-k.
    ld = (wt.L_alloc + 3) // 4 * 4
    scores = torch.empty((T, ld), dtype=torch.float32, device="cuda")
    lsa.index_score(batch, pt.q_idx, pt.w, lsa.Cache(pt.k_idx, pt.k_scale), scores, n_cols=wt.L_alloc)
    idx = torch.empty((T, w.cap), dtype=torch.int32, device="cuda")
    cnt = torch.empty((T,), dtype=torch.int32, device="cuda")
    lsa.topk(batch, scores, wt.L_alloc, w.k, w.n_sink, w.window, idx, cnt)
    L = pt.layers[0]
    kv = lsa.Cache(L["kv"], L["kv_scale"])
    n_split = 4

    ref_o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    ws = torch.empty(lsa.attn_workspace_size(T, w.H, w.Dv, n_split), dtype=torch.uint8, device="cuda")
    lsa.sparse_attn(batch, L["q"], kv, idx, cnt, w.sm_scale, ref_o, ref_lse, n_split=n_split, ws=ws)
    torch.cuda.synchronize()

    lib = lsa.library()
    cb, ck = batch.c(), kv.c()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full((T, w.H, w.Dv), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((T, w.H), float("nan"), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = lib.lsa_sparse_attn_noalloc(ctypes.byref(cb), L["q"].data_ptr(), w.H, w.D, ctypes.byref(ck), None, w.Dv,
                                         idx.data_ptr(), idx.stride(0), cnt.data_ptr(), w.sm_scale, n_split,
                                         o.data_ptr(), lse.data_ptr(), st.data_ptr(), stream)
        assert rc == lsa.OK, (call, lsa.status_string(rc))
        assert lsa.read_device_status(st) == lsa.OK
        mx, rl2 = _errors(o, ref_o)
        assert mx < 1e-2 and rl2 < 5e-3, (call, mx, rl2)
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() < 1e-3

    # A request whose split partials exceed the static scratch is refused without launching.
    big = lsa.Batch(wt.seq_len, pt.q_seq.repeat(64), pt.q_pos.repeat(64), wt.L_alloc)
    rc = lib.lsa_sparse_attn_noalloc(ctypes.byref(big.c()), L["q"].data_ptr(), w.H, w.D, ctypes.byref(ck), None,
                                     w.Dv, idx.data_ptr(), idx.stride(0), cnt.data_ptr(), w.sm_scale, 64,
                                     ref_o.data_ptr(), None, None, stream)
    assert rc == lsa.ERR_WORKSPACE
