"""Bounded waits: a wait limit shorter than the pipeline's own waits makes the kernels give up.

Every mbarrier wait of the tensor-core kernels is bounded.  lsa_set_wait_limit_ns shortens the
pipeline waits of the tensor-core indexer and block-score kernels (their drains keep the 2 s
bound), so a launch gives up on purpose: it must store LSA_ERR_TIMEOUT in the status word, drain
its copies and MMAs, free its tensor memory and return, leaving the context usable.  The next
launch with the default limit must then succeed and reproduce the earlier scores bit for bit.
"""
import pytest
import torch

from lsa_synth import device as D
from lsa_synth import workloads as W

from long_context_sparse_indexer_b200 import lsa

from . import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _timed_out_once(fn, tries=3):
    """Runs fn(status) with a 1 ns wait limit until the status word reports a timeout (a wait that
    happens to find its phase complete never gives up, so one try could in principle pass)."""
    prev = lsa.set_wait_limit_ns(1)
    try:
        for _ in range(tries):
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            fn(st)
            s = lsa.read_device_status(st)
            assert s in (lsa.OK, lsa.ERR_TIMEOUT), lsa.status_string(s)
            if s == lsa.ERR_TIMEOUT:
                return True
        return False
    finally:
        lsa.set_wait_limit_ns(prev)


def test_indexer_gives_up_and_the_context_stays_usable(cuda):
    w = W.scaled("decode_cli_128k", B=8, len_lo=20000, len_hi=30000, seed=41)
    wt = D.build_workload(w, "cuda")
    ref = H.flat_scores(wt).clone()
    torch.cuda.synchronize()
    assert _timed_out_once(lambda st: H.flat_scores(wt, 0, st))
    assert lsa.set_wait_limit_ns(0) == 0                # the default is back
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    again = H.flat_scores(wt, 0, st)
    assert lsa.read_device_status(st) == lsa.OK
    assert torch.equal(again, ref)


def test_block_scores_give_up_and_the_context_stays_usable(cuda):
    w = W.scaled("decode_hi_1m", B=2, len_lo=200000, len_hi=200000, seed=42)
    wt = D.build_workload(w, "cuda")
    kbar = H.block_keys(wt)
    T = w.T(w.passes[0])
    nblk = kbar.shape[1]
    pt = wt.passes[0]

    def run(st=None):
        sc = torch.full((T, (nblk + 3) // 4 * 4), float("nan"), dtype=torch.float32, device="cuda")
        lsa.block_score(H.batch_of(wt), pt.q_idx, pt.w, kbar, w.block_size, sc, nblk, dev_status=st)
        return sc

    ref = run()
    torch.cuda.synchronize()
    assert _timed_out_once(run)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    again = run(st)
    assert lsa.read_device_status(st) == lsa.OK
    assert torch.equal(again[:, :nblk], ref[:, :nblk])
