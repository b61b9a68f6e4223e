"""Benchmark of the LSA hot path on B200: LSA decode queries/s and achieved HBM bandwidth.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl lsa|reference]

A step is one pass of the whole path over one batch of synthetic input already resident
in HBM: indexer (flat, or HI block scores -> recall -> fine scores), top-k with sinks and
SI window, then sparse attention for every layer / draft step sharing the index, with
split-KV merge.  Default workload: batched decode at 64K-128K context with cross-layer
index reuse (32 sequences, 2 layers).  Multi-GPU (torchrun): every rank runs its own
batch (weak scaling, no collective on the data path); value = all ranks' queries / the
slowest rank's time.  ``--impl reference`` times the float64 CPU oracle on a bounded
sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lsa_synth import workloads as W  # noqa: E402

METRIC = "LSA decode queries/s at 128K & 1M ctx; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0


def bf16_peak():
    """Dense BF16 tensor throughput for a kernel timed alone (the burst figure)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def indexer_flops(w, p):
    """Algorithmic flops of one flat indexer pass: 2 * H_I * d_I per (query, visible key)."""
    _, q_pos = W.query_rows(w, p)
    return float(2 * w.H_I * w.d_I) * float(np.sum(q_pos.astype(np.int64) + 1))


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ the GPU arm

def build_step(w, wt, pi, n_split, q8=False):
    from long_context_sparse_indexer_b200 import lsa
    pt = wt.passes[pi]
    p = w.passes[pi]
    T = pt.q_idx.shape[0]
    dev = pt.q_idx.device
    batch = lsa.Batch(wt.seq_len, pt.q_seq, pt.q_pos, wt.L_alloc, q_group=p.q_per_seq)
    layers = []
    for L in pt.layers:
        o = torch.empty((T, w.H, w.Dv), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((T, w.H), dtype=torch.float32, device=dev)
        layers.append(lsa.Layer(L["q"], lsa.Cache(L["kv"], L["kv_scale"]), o, lse,
                                lsa.Cache(L["v"]) if L["v"] is not None else None))
    kbar = None
    if w.hi:
        kbar = lsa.block_keys_buffer(w.B, wt.L_alloc, w.block_size, w.d_I, dev)
        lsa.block_keys(batch, lsa.Cache(pt.k_idx, pt.k_scale), w.block_size, kbar)
    idx = torch.empty((T, w.cap), dtype=torch.int32, device=dev)
    cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    step = lsa.DecodeStep(batch, pt.q_idx, pt.w, lsa.Cache(pt.k_idx, pt.k_scale), w.k, w.n_sink, w.window, layers,
                          w.H, w.D, w.Dv, w.sm_scale, n_split=n_split, hi=w.hi, block_size=w.block_size,
                          n_recall=w.n_recall, kbar=kbar, idx_out=idx, count_out=cnt, idx_q_fp8=q8)
    ws = torch.empty(max(256, step.workspace_size()), dtype=torch.uint8, device=dev)
    return dict(step=step, ws=ws, idx=idx, cnt=cnt, layers=layers, batch=batch, kbar=kbar, T=T, n_split=n_split, q8=q8)


def slot_copy(w, wt, pi, sd):
    """A second set of device buffers for one pass of the step (queries in, outputs out), with
    its own DecodeStep sharing the caches, batch, workspace and index outputs of `sd`.
    Returns (step, device inputs, device outputs)."""
    from long_context_sparse_indexer_b200 import lsa
    pt = wt.passes[pi]
    q_idx, wv = pt.q_idx.clone(), pt.w.clone()
    layers, qs = [], []
    for L, Ls in zip(pt.layers, sd["layers"]):
        q = L["q"].clone()
        qs.append(q)
        layers.append(lsa.Layer(q, Ls.kv, torch.empty_like(Ls.o), torch.empty_like(Ls.lse), Ls.v))
    step = lsa.DecodeStep(sd["batch"], q_idx, wv, lsa.Cache(pt.k_idx, pt.k_scale), w.k, w.n_sink, w.window, layers,
                          w.H, w.D, w.Dv, w.sm_scale, n_split=sd["n_split"], hi=w.hi, block_size=w.block_size,
                          n_recall=w.n_recall, kbar=sd["kbar"], idx_out=sd["idx"], count_out=sd["cnt"],
                          idx_q_fp8=sd["q8"])
    return step, [q_idx, wv] + qs, [L.o for L in layers]


def launches_per_step(w, splits):
    per = 0
    for p, n_split in zip(w.passes, splits):
        per += 4 if w.hi else 2
        per += len(p.layers) * (2 if n_split > 1 else 1)
    return per


def algorithmic_bytes(w, wt, steps_data):
    """Bytes the method must move per step (see the design notes): indexer keys once per pass, HI
    block keys + recalled keys, selected KV rows once per layer (union over a sequence's tokens),
    q / w / o / lse.  Returns (total, indexer_bytes_of_first_pass)."""
    lens = W.lengths(w)
    kb = w.d_I * (1 if w.idx_fp8 else 2) + (4 if w.idx_fp8 else 0)
    rowb = w.D * (1 if w.kv_fp8 else 2) + (4 if w.kv_fp8 else 0)
    total = 0
    idx_first = 0
    for pi, p in enumerate(w.passes):
        sd = steps_data[pi]
        T = sd["T"]
        _, q_pos = W.query_rows(w, p)
        qw = T * (w.H_I * w.d_I * 2 + w.H_I * 4)
        if w.hi:
            vis_blocks = sum(int(q_pos[t]) // w.block_size + 1 for t in range(T))
            ib = vis_blocks * w.d_I * 4 + T * w.n_recall * w.block_size * kb + qw
        else:
            seq_max = {}
            for t in range(T):
                b = int(t // p.q_per_seq)
                seq_max[b] = max(seq_max.get(b, 0), int(q_pos[t]) + 1)
            ib = sum(seq_max.values()) * kb + qw
        if pi == 0:
            idx_first = ib
        total += ib
        idx = sd["idx"].cpu().numpy()
        cnt = sd["cnt"].cpu().numpy()
        rows = 0
        for b in range(w.B):
            toks = range(b * p.q_per_seq, (b + 1) * p.q_per_seq)
            u = np.unique(np.concatenate([idx[t, :cnt[t]] for t in toks]))
            rows += u.size
        kvb = rows * rowb
        distinct_kv = len({L.tid_kv for L in p.layers})
        per_layer_io = T * (w.H * w.D * 2 + w.H * w.Dv * 2 + w.H * 4)
        total += kvb * distinct_kv + per_layer_io * len(p.layers)
        if distinct_kv < len(p.layers):   # draft steps: same rows, read again by each step's query
            total += kvb * (len(p.layers) - distinct_kv)
    return total, idx_first


def rank_workload(w, rank: int, world: int):
    """The workload rank `rank` runs: same shapes on every rank (weak scaling), its own seed."""
    return W.scaled(w.name, B=w.B, seed=w.seed + 1000 * rank) if world > 1 else w


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's value (all ranks take part; a plain return at world == 1)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_region(fn, steps, stream):
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def attention_flops(w, steps_data):
    """Algorithmic flops of the attention of one step: 2 * H * (Dqk + Dv) per (query, selected row,
    layer) -- the QK^T and PV contractions."""
    tot = 0.0
    for p, sd in zip(w.passes, steps_data):
        rows = float(sd["cnt"].sum().item())
        tot += 2.0 * w.H * (w.D + w.Dv) * rows * len(p.layers)
    return tot


def graph_of(fn):
    """fn captured once into a CUDA graph (on a side stream), or None if capture fails."""
    try:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                fn(s)
        torch.cuda.synchronize()
        return g
    except Exception as e:  # capture unsupported: eager launches
        print(f"[bench] graph capture failed, timing eager launches: {e}", file=sys.stderr)
        return None


def time_alone(fn, stream, n):
    """Average CUDA-event duration of fn() on `stream` over n back-to-back launches (after 3 warm)."""
    for _ in range(3):
        fn()
    return time_region(fn, n, stream)


def measure(name, args, rank, world, local_rank, headline):
    """One workload: its step (all passes, all layers) captured in a CUDA graph, W warm-up steps,
    a sustained untimed load (so the clock samples describe the steady state), then exactly K
    steps between CUDA events; the dominant kernels timed alone for the rooflines; with
    `headline`, also the end-to-end rate through the host-buffer pipeline."""
    from lsa_synth import device as D
    from long_context_sparse_indexer_b200 import launch, lsa

    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS[name]
    if args.batch and headline:
        w = W.scaled(name, B=args.batch)
    w = rank_workload(w, rank, world)
    wt = D.build_workload(w, dev)
    stream = torch.cuda.current_stream()
    forced = [int(x) for x in args.n_split.split(",")] if (args.n_split and headline) else []
    sds = [build_step(w, wt, pi, forced[min(pi, len(forced) - 1)] if forced
                      else launch.split_for(w.T(p), w.H, w.cap, layers=len(p.layers)), q8=args.idx_q8)
           for pi, p in enumerate(w.passes)]

    def step(s=None):
        for sd in sds:
            sd["step"](sd["ws"], stream=s if s is not None else stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    graph = None if args.no_graph else graph_of(step)
    fn = (lambda: graph.replay()) if graph is not None else step
    for _ in range(3):
        fn()

    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        time.sleep(0.05)                     # let the sampler start
        # The K timed steps, then a sustained window of about args.load_ms timed on its own: its
        # rate is the steady state under the power cap, and the clock samples cover both.
        ms = time_region(fn, args.steps, stream)
        n_sus = max(args.steps, int(args.load_ms / max(ms, 1e-3)))
        ms_sus = time_region(fn, n_sus, stream) if args.load_ms > 0 else None
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ms, world, dev)
    if ms_sus is not None:
        ms_sus = max_over_ranks(ms_sus, world, dev)

    q_per_step = w.queries_per_step()
    value = q_per_step * world / (ms / 1e3)
    total_bytes, idx_bytes = algorithmic_bytes(w, wt, sds)
    hbm, src = peaks()
    bf16, bsrc = bf16_peak()
    res = {"workload": w.name, "value": value, "unit": "queries/s", "ms_per_step": ms,
           "algorithmic_gb_per_step": total_bytes / 1e9, "step_hbm_gbs": total_bytes / (ms / 1e3) / 1e9,
           "step_hbm_frac": total_bytes / (ms / 1e3) / 1e9 / hbm,
           "n_split": [sd["n_split"] for sd in sds], "launch": "cuda_graph" if graph is not None else "eager",
           "clocks": clk.summary()}
    if ms_sus is not None:
        res["sustained"] = {"steps": n_sus, "ms_per_step": ms_sus, "value": q_per_step * world / (ms_sus / 1e3),
                            "step_hbm_frac": total_bytes / (ms_sus / 1e3) / 1e9 / hbm}

    # Dominant kernels timed alone on the same inputs, against their rooflines.
    sd0, pt0 = sds[0], wt.passes[0]
    k_cache = lsa.Cache(pt0.k_idx, pt0.k_scale)
    n_alone = max(10, args.steps)
    if not w.hi:
        ld = (wt.L_alloc + 3) // 4 * 4
        sc = torch.empty((sd0["T"], ld), dtype=torch.float32, device=dev)
        idx_fn = lambda: lsa.index_score(sd0["batch"], pt0.q_idx, pt0.w, k_cache, sc, n_cols=wt.L_alloc,  # noqa
                                         stream=stream, q_fp8=args.idx_q8)
        kern = "index_score (flat indexer, FP8 queries)" if args.idx_q8 else "index_score (flat indexer)"
    else:
        nblk = (wt.L_alloc + w.block_size - 1) // w.block_size
        sc = torch.empty((sd0["T"], (nblk + 3) // 4 * 4), dtype=torch.float32, device=dev)
        idx_fn = lambda: lsa.block_score(sd0["batch"], pt0.q_idx, pt0.w, sd0["kbar"], w.block_size, sc, nblk,  # noqa
                                         stream=stream)
        kern = "block_score (HI coarse scores, tensor cores)"
        lens = W.lengths(w)
        idx_bytes = sum((int(l) - 1) // w.block_size + 1 for l in lens) * w.d_I * 4
    kms = time_alone(idx_fn, stream, n_alone)
    achieved = idx_bytes / (kms / 1e3) / 1e9
    roof = {"bound": "hbm", "kernel": kern, "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": indexer_traffic(kern, idx_bytes), "peak_source": f"{src} hbm_gbs",
            "launch_ms": kms, "algorithmic_bytes_per_launch": idx_bytes}
    if not w.hi:
        # The flat indexer issues FP8 MMAs (e4m3 x e4m3, two query terms): peak = measured BF16
        # burst x 2 (the nominal FP8 / BF16 ratio).  Tensor-bound when its flops at that peak take
        # longer than its bytes at the HBM peak (prefill; not decode).
        flops = indexer_flops(w, w.passes[0])
        fp8 = 2.0 * bf16
        if flops / (fp8 * 1e12) > idx_bytes / (hbm * 1e9):
            tf = flops / (kms / 1e3) / 1e12
            roof.update({"bound": "tensor", "achieved": tf, "peak": fp8, "unit": "TFLOP/s", "frac": tf / fp8,
                         "peak_source": f"{bsrc} bf16_tflops x 2 (FP8 MMA)", "algorithmic_flops_per_launch": flops,
                         "algorithmic_bytes_per_launch": idx_bytes})
    res["roofline"] = roof

    # Attention of the first pass alone, its layers on two streams as in the step (layer l on
    # branch l mod 2), against the tensor roofline when its flops dominate (prefill), else HBM.
    # Bytes: the rows of the union of a sequence's lists once per layer (as in the step's
    # algorithmic bytes), plus q / o / lse; flops: every (query, selected row) pair.
    att_layers = sd0["layers"]
    one = lsa.attn_workspace_size(sd0["T"], w.H, w.Dv, sd0["n_split"])
    ws_att = [torch.empty(max(256, one), dtype=torch.uint8, device=dev) for _ in range(2)]
    side = torch.cuda.Stream(device=dev)
    ev_fork, ev_join = torch.cuda.Event(), torch.cuda.Event()

    def att_fn():
        ev_fork.record(stream)
        side.wait_event(ev_fork)
        for li, L in enumerate(att_layers):
            lsa.sparse_attn(sd0["batch"], L.q, L.kv, sd0["idx"], sd0["cnt"], w.sm_scale, L.o, L.lse, v=L.v,
                            n_split=sd0["n_split"], ws=ws_att[li & 1], stream=stream if li % 2 == 0 else side)
        ev_join.record(side)
        stream.wait_event(ev_join)
    ams = time_alone(att_fn, stream, n_alone)
    p0 = w.passes[0]
    idx_h, cnt_h = sd0["idx"].cpu().numpy(), sd0["cnt"].cpu().numpy()
    rows = float(cnt_h.sum())
    urows = sum(np.unique(np.concatenate([idx_h[t, :cnt_h[t]] for t in range(b * p0.q_per_seq,
                                                                             (b + 1) * p0.q_per_seq)])).size
                for b in range(w.B))
    rowb = w.D * (1 if w.kv_fp8 else 2) + (4 if w.kv_fp8 else 0)
    att_bytes = len(att_layers) * (urows * rowb + sd0["T"] * (w.H * w.D * 2 + w.H * w.Dv * 2 + w.H * 4))
    att_flops = 2.0 * w.H * (w.D + w.Dv) * rows * len(att_layers)
    a_roof = {"kernel": "sparse_attn (+ split merge)", "launch_ms": ams, "algorithmic_bytes_per_launch": att_bytes,
              "algorithmic_flops_per_launch": att_flops}
    if att_flops / (bf16 * 1e12) > att_bytes / (hbm * 1e9):
        tf = att_flops / (ams / 1e3) / 1e12
        a_roof.update({"bound": "tensor", "achieved": tf, "peak": bf16, "unit": "TFLOP/s", "frac": tf / bf16,
                       "peak_source": f"{bsrc} bf16_tflops (BF16 MMA)"})
    else:
        gb = att_bytes / (ams / 1e3) / 1e9
        a_roof.update({"bound": "hbm", "achieved": gb, "peak": hbm, "unit": "GB/s", "frac": gb / hbm,
                       "peak_source": f"{src} hbm_gbs"})
    res["attention_roofline"] = a_roof

    if headline:
        res["e2e"] = e2e_rate(w, wt, sds, args, world, dev, stream, q_per_step)
        res["gpu_launches"] = launches_per_step(w, [sd["n_split"] for sd in sds]) * args.steps
        res["config"] = {"workload": w.name, "description": w.description, "batch": w.B,
                         "queries_per_step_per_gpu": q_per_step,
                         "ctx": [int(W.lengths(w).min()), int(W.lengths(w).max())],
                         "k": w.k, "n_sink": w.n_sink, "window": w.window, "hi": w.hi,
                         "layers_per_index": [len(p.layers) for p in w.passes],
                         "indexer_queries": "fp8 (per-head power-of-two scale)" if args.idx_q8 else "bf16 (exact)",
                         "n_split": res["n_split"], "parallelism": f"replicas x{world} (batch per GPU)",
                         "launch": res["launch"],
                         "l2": "inputs larger than L2 (indexer keys + selected KV rows per step >> 126 MB)"}
    del sds, wt, graph
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res, w


def e2e_rate(w, wt, sds, args, world, dev, stream, q_per_step):
    """End to end through the public API with host buffers: the pipelined driver of the C ABI
    (lsa_pipeline_*).  Every step copies its queries (indexer q and w, every layer's q) from
    pinned host memory into one of two slots of device buffers, runs the fused calls on that
    slot and copies every layer's output back to pinned host memory; the copies of one step
    overlap the decode of its neighbours.  The timed region ends after the last step's copy-out."""
    from long_context_sparse_indexer_b200 import lsa
    n_slots = max(2, args.slots)
    pl = lsa.Pipeline(n_slots, stream)
    preps, h2d_bytes, d2h_bytes = [], 0, 0
    for slot in range(n_slots):
        decs, h2d, d2h = [], [], []
        for pi, pt in enumerate(wt.passes):
            sd = sds[pi]
            if slot == 0:
                dec, ins, outs = sd["step"], [pt.q_idx, pt.w] + [L["q"] for L in pt.layers], [L.o for L in sd["layers"]]
            else:
                dec, ins, outs = slot_copy(w, wt, pi, sd)
            decs.append(dec)
            for d in ins:
                h = torch.empty(d.shape, dtype=d.dtype, pin_memory=True)
                h.copy_(d)
                h2d.append((d, h))
            for d in outs:
                d2h.append((torch.empty(d.shape, dtype=d.dtype, pin_memory=True), d))
        preps.append(pl.prepare(slot, decs, [sd["ws"] for sd in sds], h2d, d2h))
        h2d_bytes = sum(h.numel() * h.element_size() for _, h in h2d)
        d2h_bytes = sum(h.numel() * h.element_size() for h, _ in d2h)

    def e2e_run(n):
        for i in range(n):
            pl.run(preps[i % n_slots])
        pl.join()

    e2e_run(4)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    pl.close()
    return {"value": q_per_step * world / (e2e_ms / 1e3), "unit": "queries/s", "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes, "ms_per_step": e2e_ms}


def code_digest(src: bytes) -> str:
    """SHA-256 of a C++/CUDA source's code: comments removed, whitespace runs collapsed, so that an
    edit of the comments keeps the digest and any edit of the code changes it."""
    import hashlib
    import re
    text = src.decode("utf-8")
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode("utf-8")).hexdigest()


def indexer_traffic(kern: str, idx_bytes: float):
    """DRAM bytes per launch of the dominant kernel, from the committed ncu figures.

    profiles/indexer_traffic.json (flat tensor-core indexer) and profiles/block_score_traffic.json
    (HI block scores) record the ratio of measured DRAM traffic to algorithmic bytes of a capture
    of that kernel and the digest of the kernel source's code it was taken on (code_digest); the
    ratio is applied only while the source still has that digest (otherwise the counters describe
    another kernel and the field is null)."""
    if kern.startswith("index_score"):
        rec, src_file = "indexer_traffic.json", "index_score_tc.cu"
    elif kern.startswith("block_score"):
        rec, src_file = "block_score_traffic.json", "row_score_tc.cu"
    else:
        return None
    try:
        with open(os.path.join(ROOT, "profiles", rec)) as f:
            d = json.load(f)
        src = open(os.path.join(ROOT, "long_context_sparse_indexer_b200", "csrc", src_file), "rb").read()
    except (OSError, ValueError):
        return None
    if code_digest(src) != d.get("code_sha256"):
        return None
    return float(d["dram_bytes_over_algorithmic"]) * idx_bytes


# ------------------------------------------------------------------ the CPU oracle (baseline / reference arm)

def oracle_sample(w, n_tokens=1, min_seconds=0.0):
    """Times the float64 oracle's compute (selection + attention) on pre-decoded inputs of sampled tokens.

    The compute over the sampled tokens repeats until at least `min_seconds` have been spent;
    returns (tokens processed, seconds)."""
    from oracle import formats, lsa as olsa, run
    p = w.passes[0]
    T = w.T(p)
    toks = sorted(set(np.linspace(0, T - 1, n_tokens).astype(int).tolist()))
    plan = W.plant_plan(w, p) if (w.plant_frac or w.plant_blocks) else None
    prepared = []
    for t in toks:
        b, pos, L, qi, wi = run.query_context(w, p, t)
        K = run.index_keys(w, p, b, np.arange(L if w.hi else pos + 1), plan)
        prepared.append((t, b, pos, L, qi, wi, K))
    done, dt = 0, 0.0
    while done == 0 or dt < min_seconds:
        t0 = time.perf_counter()
        for (t, b, pos, L, qi, wi, K) in prepared:
            idx, _ = olsa.select(qi, wi, K, pos, w.k, w.n_sink, w.window, hi=w.hi, length=L,
                                 block_size=w.block_size, n_recall=w.n_recall)
            for layer in p.layers:
                q = formats.bf16_to_f64(W.attn_q_bits(w, layer, [t])[0])
                Kr, Vr = run.kv_decoded(w, layer, b, idx)
                olsa.attention(q, Kr, Vr, w.sm_scale)
        dt += time.perf_counter() - t0
        done += len(prepared)
    return done, dt


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def run_reference(args, rank, world):
    w = W.WORKLOADS[args.workload]
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_sample(w, 1)
    n_q, tot = 0, 0.0
    for _ in range(args.steps):
        n, dt = oracle_sample(w, 1)
        n_q += n
        tot += dt
    v = n_q / tot
    cores = cpu_cores()
    sample = (f"{args.steps} step(s) of 1 query token of {w.name} (all of its layers), inputs decoded "
              f"beforehand; float64 numpy/BLAS")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded counter-based generator)",
            "config": {"workload": w.name, "description": w.description},
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": v, "unit": "queries/s"},
            "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_stages(args, local_rank):
    """Each kernel of the workload's first pass timed alone: a CUDA graph of 20 back-to-back
    launches, replayed 5 times after one replay of warm-up (CUDA events on the launching stream).
    Prints one JSON line {"stages_us": {...}} -- a breakdown of the step, not the bench line."""
    from lsa_synth import device as D
    from long_context_sparse_indexer_b200 import launch, lsa
    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS[args.workload]
    if args.batch:
        w = W.scaled(args.workload, B=args.batch)
    wt = D.build_workload(w, dev)
    p, pt = w.passes[0], wt.passes[0]
    T = w.T(p)
    ns = int(args.n_split.split(",")[0]) if args.n_split else launch.split_for(T, w.H, w.cap, layers=len(p.layers))
    sd = build_step(w, wt, 0, ns, q8=args.idx_q8)
    batch, kc = sd["batch"], lsa.Cache(pt.k_idx, pt.k_scale)
    idx, cnt = sd["idx"], sd["cnt"]
    stages = {}
    if w.hi:
        kbar = sd["kbar"]
        nblk = kbar.shape[1]
        bsc = torch.empty((T, (nblk + 3) // 4 * 4), dtype=torch.float32, device=dev)
        cand = torch.empty((T, w.n_recall), dtype=torch.int32, device=dev)
        ccnt = torch.empty((T,), dtype=torch.int32, device=dev)
        ncols = w.n_recall * w.block_size
        fsc = torch.empty((T, ncols), dtype=torch.float32, device=dev)
        stages["block_score"] = lambda: lsa.block_score(batch, pt.q_idx, pt.w, kbar, w.block_size, bsc, nblk)
        stages["recall_topk"] = lambda: lsa.topk(batch, bsc, nblk, w.n_recall, 0, 0, cand, ccnt, raw=True)
        stages["fine_index_score"] = lambda: lsa.index_score(batch, pt.q_idx, pt.w, kc, fsc, cand_blocks=cand,
                                                             block_size=w.block_size, q_fp8=args.idx_q8)
        stages["fine_topk"] = lambda: lsa.topk(batch, fsc, ncols, w.k, w.n_sink, w.window, idx, cnt,
                                               cand_blocks=cand, block_size=w.block_size)
    else:
        ld = (wt.L_alloc + 3) // 4 * 4
        sc = torch.empty((T, ld), dtype=torch.float32, device=dev)
        stages["index_score"] = lambda: lsa.index_score(batch, pt.q_idx, pt.w, kc, sc, n_cols=wt.L_alloc,
                                                        q_fp8=args.idx_q8)
        stages["topk"] = lambda: lsa.topk(batch, sc, wt.L_alloc, w.k, w.n_sink, w.window, idx, cnt)
    L0 = sd["layers"][0]
    ws = torch.empty(max(256, lsa.attn_workspace_size(T, w.H, w.Dv, ns)), dtype=torch.uint8, device=dev)
    stages[f"attention_one_layer_n_split_{ns}"] = lambda: lsa.sparse_attn(batch, L0.q, L0.kv, idx, cnt, w.sm_scale,
                                                                          L0.o, L0.lse, v=L0.v, n_split=ns, ws=ws)
    stages["fused_step"] = lambda: sd["step"](sd["ws"])
    sd["step"](sd["ws"])                          # index lists for the stages that read them
    torch.cuda.synchronize()
    out = {}
    for name, f in stages.items():
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s_ = torch.cuda.Stream(device=dev)
        s_.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s_):
            with torch.cuda.graph(g, stream=s_):
                for _ in range(20):
                    f()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(5):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / 100 * 1e3
    print(json.dumps({"workload": w.name, "n_split": ns, "stages_us": out}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_cli_128k", choices=list(W.WORKLOADS))
    ap.add_argument("--impl", default="lsa", choices=["lsa", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the sequence count (small profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="measure only --workload (by default a single-GPU run of the 128K decode also measures the "
                         "1M-context HI decode and the 32K prefill chunk)")
    ap.add_argument("--load-ms", type=float, default=250.0,
                    help="sustained window after each timed region, timed on its own (steady state under the "
                         "power cap; the clock samples cover it); 0 = none")
    ap.add_argument("--slots", type=int, default=2, help="device buffer slots of the host-buffer pipeline")
    ap.add_argument("--idx-q8", action="store_true", help="indexer in FP8-query mode (lsa_index_score_q8)")
    ap.add_argument("--n-split", default="", help="override the split-KV chunk count: one value, or one per pass")
    ap.add_argument("--stages", action="store_true",
                    help="print the time of each kernel of the step alone (CUDA graphs) instead of the bench line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    torch.cuda.set_device(local_rank)
    if args.stages:
        run_stages(args, local_rank)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    head, w = measure(args.workload, args, rank, world, local_rank, headline=True)
    res = {
        "metric": METRIC, "value": head["value"], "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16+fp8", "data": "synthetic (seeded counter-based generator)",
        "config": head["config"],
        "algorithmic_gb_per_step": head["algorithmic_gb_per_step"], "step_hbm_gbs": head["step_hbm_gbs"],
        "step_hbm_frac": head["step_hbm_frac"],
        "roofline": head["roofline"], "attention_roofline": head["attention_roofline"],
        "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
    }
    if "sustained" in head:
        res["sustained"] = head["sustained"]
    if world == 1 and not args.no_extras and args.workload == "decode_cli_128k" and not args.batch:
        # The metric names two context lengths (128K and 1M); the prefill chunk carries the tensor
        # roofline.  Each is measured the same way (graph, warm-up, sustained load, K timed steps).
        res["workloads"] = {}
        for nm in ("decode_hi_1m", "prefill_32k"):
            r, _ = measure(nm, args, rank, world, local_rank, headline=False)
            res["workloads"][nm] = r
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            n, dt = oracle_sample(W.WORKLOADS[args.workload], 2, min_seconds=10.0)
            res["cpu_baseline"] = {"value": n / dt, "unit": "queries/s", "cores": cpu_cores(), "kind": "oracle",
                                   "sample": f"2 query tokens of {w.name} (all layers), computed {n // 2} times "
                                             f"({n} tokens), float64 numpy/BLAS, inputs decoded beforehand; "
                                             f"{dt:.1f} s"}
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
