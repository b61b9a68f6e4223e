"""Synthetic LSA workloads: shapes, seeds and the host-side generation of every input.

The five named workloads follow the five benchmark settings of the LSA hot path
(tiny decode, 32K prefill chunk, 128K batched decode with cross-layer index reuse,
1M decode with hierarchical indexing, speculative MTP verify + draft).  ``scaled``
derives small variants with the same structure for parity tests the CPU oracle
finishes in seconds.

A workload has one or more *passes*.  A pass is one indexer run (one index per query
token) whose index list is consumed by several attention *layers* (cross-layer index
reuse).  The speculative workload has a target pass (4 verify tokens per sequence,
two layers sharing the index) and a draft pass (one index per sequence, consumed by
the three draft steps over the draft KV cache).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field

import numpy as np

from . import gen


@dataclass(frozen=True)
class Layer:
    tid_kv: int                 # latent KV cache (MLA layout) or K cache (separate layout)
    tid_q: int                  # attention query of this layer / draft step
    tid_v: int = -1             # separate V cache, -1 for the MLA layout (V = first Dv dims of KV)


@dataclass(frozen=True)
class Pass:
    name: str
    q_per_seq: int              # indexed query tokens per sequence, at positions L-q_per_seq .. L-1
    tid_idx_keys: int
    tid_idx_q: int
    tid_idx_w: int
    layers: tuple               # Layer entries consuming this pass's index lists
    queries_per_seq: int        # query tokens this pass completes per sequence (for queries/s)


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    len_lo: int                 # sequence lengths ~ U[len_lo, len_hi] (integers); equal => fixed
    len_hi: int
    H_I: int
    d_I: int
    idx_fp8: bool               # FP8 e4m3 indexer keys with a per-token scale, else BF16
    k: int
    n_sink: int
    window: int
    H: int
    D: int                      # attention QK dim (576 latent for MLA, 128 for the separate layout)
    Dv: int
    kv_fp8: bool
    sm_scale: float
    passes: tuple
    hi: bool = False
    block_size: int = 64
    n_recall: int = 0
    plant_frac: float = 0.0     # fraction of positions planted along the query direction
    plant_blocks: int = 0       # number of planted blocks per sequence
    description: str = ""
    extra: dict = field(default_factory=dict)

    # ------------------------------------------------------------ derived sizes
    @property
    def separate_v(self) -> bool:
        return self.passes[0].layers[0].tid_v >= 0

    @property
    def cap(self) -> int:
        """Maximum index-list length per query: top-k plus sinks plus window."""
        return self.k + self.n_sink + self.window

    def T(self, p: Pass) -> int:
        return self.B * p.q_per_seq

    def queries_per_step(self) -> int:
        return sum(self.B * p.queries_per_seq for p in self.passes)


def _target_pass(q_per_seq: int, n_layers: int, separate_v: bool = False) -> Pass:
    layers = tuple(Layer(gen.TID_KV + l, gen.TID_Q + l, gen.TID_V + l if separate_v else -1)
                   for l in range(n_layers))
    return Pass("target", q_per_seq, gen.TID_IDX_KEYS, gen.TID_IDX_Q, gen.TID_IDX_W, layers, q_per_seq)


def _draft_pass(n_steps: int) -> Pass:
    layers = tuple(Layer(gen.TID_KV + 8, gen.TID_Q + 8 + s) for s in range(n_steps))
    return Pass("draft", 1, gen.TID_DRAFT_IDX_KEYS, gen.TID_DRAFT_IDX_Q, gen.TID_DRAFT_IDX_W, layers, n_steps)


WORKLOADS = {
    "tiny_decode": Workload(
        name="tiny_decode", seed=0, B=1, len_lo=4096, len_hi=4096, H_I=8, d_I=64, idx_fp8=False,
        k=256, n_sink=4, window=128, H=16, D=128, Dv=128, kv_fp8=False, sm_scale=1.0 / math.sqrt(128),
        passes=(_target_pass(1, 1, separate_v=True),), plant_frac=0.01,
        description="decode, batch 1, context 4096, 8x64 BF16 indexer, 16 heads over one KV head (d=128)"),
    "prefill_32k": Workload(
        name="prefill_32k", seed=1, B=1, len_lo=32768, len_hi=32768, H_I=64, d_I=128, idx_fp8=True,
        k=2048, n_sink=4, window=512, H=128, D=576, Dv=512, kv_fp8=False, sm_scale=1.0 / math.sqrt(576),
        passes=(_target_pass(2048, 1),),
        description="prefill chunk: 2048 causal queries (positions 30720-32767) over a 32K context"),
    "decode_cli_128k": Workload(
        name="decode_cli_128k", seed=2, B=32, len_lo=65536, len_hi=131072, H_I=64, d_I=128, idx_fp8=True,
        k=2048, n_sink=4, window=512, H=128, D=576, Dv=512, kv_fp8=False, sm_scale=1.0 / math.sqrt(576),
        passes=(_target_pass(1, 2),),
        description="batched decode, batch 32, context U[64K,128K], one FP8 indexer pass serving 2 layers"),
    "decode_hi_1m": Workload(
        name="decode_hi_1m", seed=3, B=4, len_lo=1 << 20, len_hi=1 << 20, H_I=64, d_I=128, idx_fp8=True,
        k=2048, n_sink=4, window=1024, H=128, D=576, Dv=512, kv_fp8=False, sm_scale=1.0 / math.sqrt(576),
        passes=(_target_pass(1, 1),), hi=True, block_size=64, n_recall=256, plant_blocks=16,
        description="1M-context decode, batch 4, hierarchical indexing (64-token blocks, recall 256)"),
    "mtp_256k": Workload(
        name="mtp_256k", seed=4, B=64, len_lo=262144, len_hi=262144, H_I=64, d_I=128, idx_fp8=True,
        k=2048, n_sink=4, window=512, H=128, D=576, Dv=512, kv_fp8=True, sm_scale=1.0 / math.sqrt(576),
        passes=(_target_pass(4, 2), _draft_pass(3)),
        description="speculative decode, batch 64, context 256K: 4 verify tokens (index shared by 2 "
                    "layers) + 3 draft steps reusing one index; FP8 KV"),
}

ORDER = ("tiny_decode", "prefill_32k", "decode_cli_128k", "decode_hi_1m", "mtp_256k")


def scaled(name: str, **changes) -> Workload:
    """A variant of a named workload with some fields replaced (same seed unless given)."""
    return dataclasses.replace(WORKLOADS[name], **changes)


# ---------------------------------------------------------------- host generation

def lengths(w: Workload) -> np.ndarray:
    if w.len_lo == w.len_hi:
        return np.full(w.B, w.len_lo, dtype=np.int64)
    key = gen.tensor_key(w.seed, gen.TID_LENGTHS)
    h = gen.words(key, np.arange(w.B, dtype=np.uint64))
    span = np.uint64(w.len_hi - w.len_lo + 1)
    return (w.len_lo + (h % span).astype(np.int64)).astype(np.int64)


def query_rows(w: Workload, p: Pass):
    """(q_seq, q_pos) of the pass's query tokens: token j of sequence b sits at L_b - q_per_seq + j."""
    L = lengths(w)
    q_seq = np.repeat(np.arange(w.B, dtype=np.int64), p.q_per_seq)
    q_pos = np.concatenate([np.arange(L[b] - p.q_per_seq, L[b], dtype=np.int64) for b in range(w.B)])
    return q_seq, q_pos


def idx_q_bits(w: Workload, p: Pass, tokens=None) -> np.ndarray:
    """Indexer queries as BF16 bits, [n_tokens, H_I, d_I]."""
    T = w.T(p)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    ctr = (tokens.astype(np.uint64)[:, None] * np.uint64(w.H_I * w.d_I)
           + np.arange(w.H_I * w.d_I, dtype=np.uint64)[None, :])
    x = gen.normal_f32(gen.tensor_key(w.seed, p.tid_idx_q), ctr)
    return gen.f32_to_bf16_bits(x).reshape(len(tokens), w.H_I, w.d_I)


def idx_w(w: Workload, p: Pass, tokens=None) -> np.ndarray:
    """Indexer head weights ~ U(0,1), float32 [n_tokens, H_I]."""
    T = w.T(p)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    ctr = tokens.astype(np.uint64)[:, None] * np.uint64(w.H_I) + np.arange(w.H_I, dtype=np.uint64)[None, :]
    return gen.uniform_f32(gen.tensor_key(w.seed, p.tid_idx_w), ctr)


def attn_q_bits(w: Workload, layer: Layer, tokens) -> np.ndarray:
    """Attention queries as BF16 bits, [n_tokens, H, D]."""
    tokens = np.asarray(tokens)
    ctr = (tokens.astype(np.uint64)[:, None] * np.uint64(w.H * w.D)
           + np.arange(w.H * w.D, dtype=np.uint64)[None, :])
    x = gen.normal_f32(gen.tensor_key(w.seed, layer.tid_q), ctr)
    return gen.f32_to_bf16_bits(x).reshape(len(tokens), w.H, w.D)


def plant_plan(w: Workload, p: Pass):
    """Planted rows per sequence and the planting direction per sequence.

    Returns (rows, directions): rows[b] is a sorted int64 array of cache rows of sequence b
    (empty when nothing is planted), directions is float32 [B, d_I].  Planting uses the
    first indexed query token of each sequence.
    """
    L = lengths(w)
    rows, dirs = [], np.zeros((w.B, w.d_I), dtype=np.float32)
    for b in range(w.B):
        if w.plant_frac > 0:
            n = int(round(w.plant_frac * L[b]))
            r = gen.choose_without_replacement(w.seed, gen.TID_PLANT, b, int(L[b]), n)
        elif w.plant_blocks > 0:
            nblk = (int(L[b]) + w.block_size - 1) // w.block_size
            blk = gen.choose_without_replacement(w.seed, gen.TID_PLANT, b, nblk, w.plant_blocks)
            r = (blk[:, None] * w.block_size + np.arange(w.block_size)[None, :]).reshape(-1)
            r = r[r < L[b]]
        else:
            r = np.zeros(0, dtype=np.int64)
        rows.append(np.asarray(r, dtype=np.int64))
        if r.size:
            qb = gen.bf16_bits_to_f32(idx_q_bits(w, p, [b * p.q_per_seq])[0])
            dirs[b] = gen.query_direction(qb)
    return rows, dirs


def _cache_rows_f32(key: int, b: int, rows: np.ndarray, dim: int) -> np.ndarray:
    return gen.normal_f32(key, gen.cache_ctr(b, rows, dim))


def idx_key_rows(w: Workload, p: Pass, b: int, rows, plan=None):
    """Indexer key cache rows of sequence b.

    FP8 caches return (codes uint8 [n, d_I], scale float32 [n]); BF16 caches return
    (bits uint16 [n, d_I], None).
    """
    rows = np.asarray(rows, dtype=np.int64)
    x = _cache_rows_f32(gen.tensor_key(w.seed, p.tid_idx_keys), b, rows, w.d_I)
    if p.name == "target" and (w.plant_frac > 0 or w.plant_blocks > 0):
        prow, pdir = plan if plan is not None else plant_plan(w, p)
        hit = np.isin(rows, prow[b])
        if hit.any():
            x[hit] = gen.planted_rows(x[hit], pdir[b])
    if w.idx_fp8:
        return gen.quantize_rows_e4m3(x)
    return gen.f32_to_bf16_bits(x), None


def kv_rows(w: Workload, tid: int, b: int, rows, dim: int):
    """KV cache rows (BF16 bits, or FP8 codes + scale) of sequence b for cache tensor ``tid``."""
    rows = np.asarray(rows, dtype=np.int64)
    x = _cache_rows_f32(gen.tensor_key(w.seed, tid), b, rows, dim)
    if w.kv_fp8:
        return gen.quantize_rows_e4m3(x)
    return gen.f32_to_bf16_bits(x), None
