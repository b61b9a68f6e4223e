"""Oracle on the synthetic workloads: properties the definitions and the input recipe fix (CPU only)."""
import numpy as np

from lsa_synth import workloads as W
from oracle import lsa, run


def test_tiny_decode_planted_positions_selected():
    w = W.WORKLOADS["tiny_decode"]
    p = w.passes[0]
    r = run.run_query(w, p, 0)
    rows, _ = W.plant_plan(w, p)
    assert np.isin(rows[0], r["idx"]).all()
    idx = r["idx"]
    assert np.all(np.diff(idx) > 0) and idx[0] == 0 and idx[-1] == 4095
    assert 256 + 0 <= idx.size <= w.cap
    assert set(range(4)) <= set(idx.tolist()) and set(range(4096 - 128, 4096)) <= set(idx.tolist())
    o, lse = r["layers"][0]
    assert o.shape == (16, 128) and np.isfinite(o).all() and np.isfinite(lse).all()


def test_hi_planted_blocks_recalled():
    w = W.scaled("decode_hi_1m", len_lo=16384, len_hi=16384, B=2)
    p = w.passes[0]
    rows, _ = W.plant_plan(w, p)
    for t in range(2):
        idx, _ = run.index_list(w, p, t)
        assert np.isin(rows[t], idx).all()


def test_hi_full_recall_equals_flat_on_workload():
    w = W.scaled("decode_hi_1m", len_lo=3000, len_hi=3000, B=1, n_recall=10 ** 6, window=100, k=300)
    flat = W.scaled("decode_hi_1m", len_lo=3000, len_hi=3000, B=1, hi=False, window=100, k=300)
    a, _ = run.index_list(w, w.passes[0], 0)
    b, _ = run.index_list(flat, flat.passes[0], 0)
    assert a.tolist() == b.tolist()


def test_cli_layers_share_index_and_differ_in_output():
    w = W.scaled("decode_cli_128k", B=2, len_lo=2000, len_hi=3000)
    p = w.passes[0]
    r = run.run_query(w, p, 1)
    assert len(r["layers"]) == 2
    (o0, _), (o1, _) = r["layers"]
    assert not np.allclose(o0, o1)
    # the second layer's output is attention over the very same index list
    o1b, _ = run.attend(w, p, p.layers[1], 1, r["idx"])
    assert np.array_equal(o1, o1b)


def test_mtp_draft_steps_reuse_step1_index():
    w = W.scaled("mtp_256k", B=2, len_lo=3000, len_hi=3000)
    d = w.passes[1]
    assert d.q_per_seq == 1 and len(d.layers) == 3
    assert len({l.tid_kv for l in d.layers}) == 1 and len({l.tid_q for l in d.layers}) == 3
    r = run.run_query(w, d, 0)
    assert len(r["layers"]) == 3


def test_softmax_normalisation_on_workload():
    """o of an all-ones V equals 1: the selected rows' weights sum to one."""
    w = W.scaled("prefill_32k", len_lo=4096, len_hi=4096)
    p = w.passes[0]
    idx, _ = run.index_list(w, p, 5)
    from oracle import formats
    q = formats.bf16_to_f64(W.attn_q_bits(w, p.layers[0], [5])[0])
    K, _ = run.kv_decoded(w, p.layers[0], 0, idx)
    o, _ = lsa.attention(q, K, np.ones((len(idx), 3)), w.sm_scale)
    assert np.allclose(o, 1.0, atol=1e-13)
