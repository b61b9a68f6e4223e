"""lsa_sparse_attn_noalloc: sparse attention for callers that cannot allocate device memory.

Callers such as a serving runtime whose memory pool is closed to new allocations, or a
plugin host that owns every cudaMalloc, cannot hand lsa_sparse_attn a workspace for its
split-KV partials.  The no-allocation entry point keeps those partials in the library's
own static device array instead.  It runs the same kernels at the same n_split, and the
library is deterministic, so its outputs must equal lsa_sparse_attn's bit for bit.  This
test calls it through the C ABI twice in a row (the array keeps the first call's contents)
and through the Python wrapper with one split (no scratch), and compares each result
with lsa_sparse_attn given a caller-provided workspace.  It builds its own inputs, so it
runs alone in a fresh process as well as after the other tests; it sits in a file
collected last so that a run stopping at its first failure has already run everything
else.
"""
import ctypes

import pytest
import torch

from lsa_synth import device as D
from lsa_synth import workloads as W

from long_context_sparse_indexer_b200 import lsa

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


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

    def reference(n_split):
        o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
        ws = torch.empty(max(256, lsa.attn_workspace_size(T, w.H, w.Dv, n_split)), dtype=torch.uint8, device="cuda")
        lsa.sparse_attn(batch, L["q"], kv, idx, cnt, w.sm_scale, o, lse, n_split=n_split, ws=ws)
        torch.cuda.synchronize()
        return o, lse

    n_split = 4
    ref_o, ref_lse = reference(n_split)
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
        assert torch.equal(_bits(o), _bits(ref_o)), (call, (o.float() - ref_o.float()).abs().max())
        assert torch.equal(_bits(lse), _bits(ref_lse)), call

    # One split needs no scratch (a null scratch pointer reaches the kernels): same bits as the
    # workspace entry point, through the Python wrapper.
    ref1_o, ref1_lse = reference(1)
    o1 = torch.full_like(ref1_o, float("nan"))
    lse1 = torch.full_like(ref1_lse, float("nan"))
    lsa.sparse_attn_noalloc(batch, L["q"], kv, idx, cnt, w.sm_scale, o1, lse1, n_split=1)
    torch.cuda.synchronize()
    assert torch.equal(_bits(o1), _bits(ref1_o)) and torch.equal(_bits(lse1), _bits(ref1_lse))

    # A request whose split partials exceed the static scratch is refused without launching.
    big = lsa.Batch(wt.seq_len, pt.q_seq.repeat(64), pt.q_pos.repeat(64), wt.L_alloc)
    rc = lib.lsa_sparse_attn_noalloc(ctypes.byref(big.c()), L["q"].data_ptr(), w.H, w.D, ctypes.byref(ck), None,
                                     w.Dv, idx.data_ptr(), idx.stride(0), cnt.data_ptr(), w.sm_scale, 64,
                                     ref_o.data_ptr(), None, None, stream)
    assert rc == lsa.ERR_WORKSPACE
    # An unsupported shape gets the status lsa_sparse_attn gives it, not the scratch-size one.
    rc = lib.lsa_sparse_attn_noalloc(ctypes.byref(big.c()), L["q"].data_ptr(), 48, w.D, ctypes.byref(ck), None,
                                     w.Dv, idx.data_ptr(), idx.stride(0), cnt.data_ptr(), w.sm_scale, 64,
                                     ref_o.data_ptr(), None, None, stream)
    assert rc == lsa.ERR_UNSUPPORTED
