"""Helpers for the GPU parity tests: run the library on device-built synthetic inputs."""
from __future__ import annotations

import numpy as np
import torch

from lsa_synth import device as D
from lsa_synth import workloads as W

from long_context_sparse_indexer_b200 import lsa


def batch_of(wt: D.WorkloadTensors, pi: int = 0) -> lsa.Batch:
    p = wt.w.passes[pi]
    return lsa.Batch(wt.seq_len, wt.passes[pi].q_seq, wt.passes[pi].q_pos, wt.L_alloc, q_group=p.q_per_seq)


def idx_cache(wt: D.WorkloadTensors, pi: int = 0) -> lsa.Cache:
    pt = wt.passes[pi]
    return lsa.Cache(pt.k_idx, pt.k_scale)


def kv_cache(wt: D.WorkloadTensors, pi: int, li: int):
    L = wt.passes[pi].layers[li]
    return lsa.Cache(L["kv"], L["kv_scale"]), (lsa.Cache(L["v"]) if L["v"] is not None else None)


def flat_scores(wt: D.WorkloadTensors, pi: int = 0, status=None, q_fp8: bool = False) -> torch.Tensor:
    pt = wt.passes[pi]
    T = pt.q_idx.shape[0]
    ld = (wt.L_alloc + 3) // 4 * 4
    sc = torch.full((T, ld), float("nan"), dtype=torch.float32, device=pt.q_idx.device)
    lsa.index_score(batch_of(wt, pi), pt.q_idx, pt.w, idx_cache(wt, pi), sc, n_cols=wt.L_alloc, dev_status=status,
                    q_fp8=q_fp8)
    return sc


def block_keys(wt: D.WorkloadTensors, pi: int = 0, status=None) -> torch.Tensor:
    w = wt.w
    kbar = lsa.block_keys_buffer(w.B, wt.L_alloc, w.block_size, w.d_I, wt.seq_len.device)
    kbar.zero_()
    lsa.block_keys(batch_of(wt, pi), idx_cache(wt, pi), w.block_size, kbar, dev_status=status)
    return kbar


def block_key_values(kbar: torch.Tensor) -> np.ndarray:
    """The block keys a block-key buffer holds, hi + lo, in float64: [B, nblk, d_I]."""
    x = kbar.float().cpu().numpy().astype(np.float64)
    d = x.shape[-1] // 2
    return x[..., :d] + x[..., d:]


def decode_step(wt: D.WorkloadTensors, pi: int = 0, n_split: int = 1, kbar=None, cap_extra: int = 0,
                idx_q_fp8: bool = False, si_window_aligned: bool = False):
    """Builds lsa.DecodeStep for a pass plus its output tensors."""
    w = wt.w
    pt = wt.passes[pi]
    T = pt.q_idx.shape[0]
    dev = pt.q_idx.device
    layers = []
    for li, L in enumerate(pt.layers):
        kv, v = kv_cache(wt, pi, li)
        o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((T, w.H), dtype=torch.float32, device=dev)
        layers.append(lsa.Layer(L["q"], kv, o, lse, v))
    cap = w.cap + cap_extra
    idx = torch.empty((T, cap), dtype=torch.int32, device=dev)
    cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    if w.hi and kbar is None:
        kbar = block_keys(wt, pi)
    step = lsa.DecodeStep(batch_of(wt, pi), pt.q_idx, pt.w, idx_cache(wt, pi), w.k, w.n_sink, w.window, layers,
                          w.H, w.D, w.Dv, w.sm_scale, n_split=n_split, hi=w.hi, block_size=w.block_size,
                          n_recall=w.n_recall, kbar=kbar, idx_out=idx, count_out=cnt, idx_q_fp8=idx_q_fp8,
                          si_window_aligned=si_window_aligned)
    ws = torch.empty(max(256, step.workspace_size()), dtype=torch.uint8, device=dev)
    return step, ws, idx, cnt, layers


def index_lists(idx: torch.Tensor, cnt: torch.Tensor):
    ih, ch = idx.cpu().numpy(), cnt.cpu().numpy()
    return [ih[t, :ch[t]].astype(np.int64) for t in range(len(ch))]


def score_close(gpu: np.ndarray, ref: np.ndarray, rtol: float = 1e-3):
    """Relative error of indexer scores, with a floor at 1% of the row's RMS score for near-zero entries."""
    floor = 1e-2 * np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    err = np.abs(gpu - ref) / np.maximum(np.abs(ref), floor)
    return float(err.max()) if err.size else 0.0


def attn_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    """(max-abs error, relative L2 error) of an attention output."""
    d = o_gpu.astype(np.float64) - o_ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(o_ref), 1e-30))


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)
