"""KVP decode: one context sharded over ranks (one process per GPU), exchanges over NCCL.

Explainer page ("如何在 5 万张国产芯片训练出 1.6T 万亿参数模型？"), section "③ KVP 解码切分示意",
and the release post's section "推理" (decode nodes): the KV cache of a long sequence is split
over devices, each computes partial results over its shard, and the partial results are merged.

Each rank holds ``shards``: contiguous row ranges of every sequence (its indexer keys and its KV
rows, stored from row 0 of the rank's own caches); shard g = rank * len(shards) + s covers
positions before those of shard g + 1.  One step:

1. per local shard: local batch, indexer scores, the shard's top-k as (position, score) pairs;
2. all-gather of the pairs over the ranks (shard order);
3. the global selection (top-k by (score desc, position asc), sinks, window) -- every rank
   computes the same list, the single-device one;
4. per layer and local shard: the selected rows the shard holds, partial attention over them
   (FP32 result and log-sum-exp);
5. all-gather of the partial results (shard order), log-sum-exp merge in shard order.

Every computation is a call of the C ABI (``lsa.kvp_*``, ``lsa.index_score``,
``lsa.sparse_attn_partial``, ``lsa.merge_partials``) through :class:`LsaOps`; this module only
orders them and runs the collectives (``torch.distributed.all_gather``, NCCL between GPUs).
The exchanged bytes per step and token are shards x k x 8 (candidates) and, per layer,
shards x H x (Dv + 1) x 4 (partial results).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

from . import lsa


@dataclass
class Shard:
    """Rows start[b] .. start[b] + length[b] - 1 of every sequence b, held from row 0 of the local
    caches (L_alloc rows each)."""
    start: torch.Tensor            # int32 [B]
    length: torch.Tensor           # int32 [B]
    L_alloc: int
    k_idx: lsa.Cache               # local indexer keys
    kv: List[lsa.Cache] = field(default_factory=list)   # local KV cache of each attention layer


class LsaOps:
    """The KVP steps as calls of the CUDA library on one device, with output buffers kept between
    calls (keyed by role and shard), all on one stream."""

    def __init__(self, stream=None, dev_status: Optional[torch.Tensor] = None):
        self.stream = stream
        self.dev_status = dev_status
        self._bufs = {}

    def _buf(self, key, shape, dtype, device):
        b = self._bufs.get(key)
        if b is None or tuple(b.shape) != tuple(shape) or b.dtype != dtype or b.device != device:
            b = torch.empty(shape, dtype=dtype, device=device)
            self._bufs[key] = b
        return b

    def shard_batch(self, batch: lsa.Batch, sh: Shard, tag) -> lsa.Batch:
        dev = batch.q_pos.device
        lsl = self._buf(("lsl", tag), (batch.seq_len.numel(),), torch.int32, dev)
        lqp = self._buf(("lqp", tag), (batch.q_pos.numel(),), torch.int32, dev)
        return lsa.kvp_shard_batch(batch, sh.L_alloc, sh.start, sh.length, lsl, lqp, self.dev_status, self.stream)

    def scores(self, local: lsa.Batch, q_idx: torch.Tensor, w: torch.Tensor, sh: Shard, tag) -> torch.Tensor:
        T = q_idx.shape[0]
        sc = self._buf(("sc", tag), (T, (sh.L_alloc + 3) // 4 * 4), torch.float32, q_idx.device)
        lsa.index_score(local, q_idx, w, sh.k_idx, sc, n_cols=sh.L_alloc, dev_status=self.dev_status,
                        stream=self.stream)
        return sc

    def candidates(self, local: lsa.Batch, q_pos_global: torch.Tensor, sh: Shard, scores: torch.Tensor, k: int, tag):
        T, dev = scores.shape[0], scores.device
        pos = self._buf(("cp", tag), (T, k), torch.int32, dev)
        sco = self._buf(("cs", tag), (T, k), torch.float32, dev)
        cnt = self._buf(("cc", tag), (T,), torch.int32, dev)
        lsa.kvp_candidates(local, q_pos_global, sh.start, scores, sh.L_alloc, k, pos, sco, cnt, self.dev_status,
                           self.stream)
        return pos, sco

    def select(self, batch: lsa.Batch, pos_all: torch.Tensor, score_all: torch.Tensor, k: int, n_sink: int,
               window: int):
        P, T, kp = pos_all.shape
        dev = pos_all.device
        cap = k + n_sink + window
        idx = self._buf(("idx",), (T, cap), torch.int32, dev)
        cnt = self._buf(("cnt",), (T,), torch.int32, dev)
        ws = self._buf(("selws",), (max(256, lsa.kvp_select_workspace_size(T, P, kp)),), torch.uint8, dev)
        lsa.kvp_select(batch, pos_all, score_all, k, n_sink, window, idx, cnt, ws, self.dev_status, self.stream)
        return idx, cnt

    def local_index(self, batch: lsa.Batch, sh: Shard, idx: torch.Tensor, cnt: torch.Tensor, tag):
        lidx = self._buf(("lidx", tag), tuple(idx.shape), torch.int32, idx.device)
        lcnt = self._buf(("lcnt", tag), tuple(cnt.shape), torch.int32, idx.device)
        lsa.kvp_local_index(batch, sh.start, sh.length, idx, cnt, lidx, lcnt, self.dev_status, self.stream)
        return lidx, lcnt

    def partial(self, local: lsa.Batch, q: torch.Tensor, kv: lsa.Cache, lidx: torch.Tensor, lcnt: torch.Tensor,
                sm_scale: float, n_split: int, Dv: int, tag):
        T, H = q.shape[0], q.shape[1]
        o = self._buf(("op", tag), (T, H, Dv), torch.float32, q.device)
        l = self._buf(("lp", tag), (T, H), torch.float32, q.device)
        ws = self._buf(("aws", tag), (max(256, lsa.attn_workspace_size(T, H, Dv, n_split)),), torch.uint8, q.device)
        lsa.sparse_attn_partial(local, q, kv, lidx, lcnt, sm_scale, o, l, Dv=Dv, n_split=n_split, ws=ws,
                                dev_status=self.dev_status, stream=self.stream)
        return o, l

    def merge(self, o_all: torch.Tensor, lse_all: torch.Tensor, tag):
        _, T, H, Dv = o_all.shape
        o = self._buf(("o", tag), (T, H, Dv), torch.bfloat16, o_all.device)
        lse = self._buf(("lse", tag), (T, H), torch.float32, o_all.device)
        lsa.merge_partials(o_all.contiguous(), lse_all.contiguous(), o, lse, stream=self.stream)
        return o, lse


class KVPDecode:
    """One LSA decode step with the context sharded over ``world`` ranks of ``group`` (and over the
    ``shards`` of this rank).  With world == 1 the collectives are skipped (the shards of one
    process are then the whole context: the same path on one GPU)."""

    def __init__(self, batch: lsa.Batch, q_idx: torch.Tensor, w: torch.Tensor, shards: Sequence[Shard], k: int,
                 n_sink: int, window: int, layer_q: Sequence[torch.Tensor], Dv: int, sm_scale: float,
                 n_split: int = 1, group=None, world: int = 1, ops=None):
        self.batch, self.q_idx, self.w = batch, q_idx, w
        self.shards = list(shards)
        self.k, self.n_sink, self.window = int(k), int(n_sink), int(window)
        self.layer_q = list(layer_q)
        self.Dv, self.sm_scale, self.n_split = int(Dv), float(sm_scale), int(n_split)
        self.group, self.world = group, int(world)
        self.ops = ops if ops is not None else LsaOps()

    def _gather(self, x: torch.Tensor) -> torch.Tensor:
        """Concatenation over the ranks (rank order) of x [n_local, ...] -> [world * n_local, ...]."""
        if self.world <= 1:
            return x
        import torch.distributed as dist
        parts = [torch.empty_like(x) for _ in range(self.world)]
        dist.all_gather(parts, x.contiguous(), group=self.group)
        return torch.cat(parts, dim=0)

    def __call__(self):
        """Returns (idx [T, cap], count [T], [(o [T, H, Dv] bf16, lse [T, H]) per layer])."""
        ops = self.ops
        locals_, pos, sco = [], [], []
        for s, sh in enumerate(self.shards):
            lb = ops.shard_batch(self.batch, sh, s)
            sc = ops.scores(lb, self.q_idx, self.w, sh, s)
            p, v = ops.candidates(lb, self.batch.q_pos, sh, sc, self.k, s)
            locals_.append(lb)
            pos.append(p)
            sco.append(v)
        pos_all = self._gather(torch.stack(pos))
        sco_all = self._gather(torch.stack(sco))
        idx, cnt = ops.select(self.batch, pos_all, sco_all, self.k, self.n_sink, self.window)
        lists = [ops.local_index(self.batch, sh, idx, cnt, s) for s, sh in enumerate(self.shards)]
        outs = []
        for li, q in enumerate(self.layer_q):
            po, pl = [], []
            for s, (sh, lb, (lidx, lcnt)) in enumerate(zip(self.shards, locals_, lists)):
                o, l = ops.partial(lb, q, sh.kv[li], lidx, lcnt, self.sm_scale, self.n_split, self.Dv, (li, s))
                po.append(o)
                pl.append(l)
            o_all = self._gather(torch.stack(po))
            l_all = self._gather(torch.stack(pl))
            outs.append(ops.merge(o_all, l_all, li))
        return idx, cnt, outs
