"""Python binding of the LSA C ABI (include/lsa.h): argument marshalling only.

Every computation runs in the CUDA library ``_lsa.so``; this module turns torch tensors
into the pointers, strides and structs the C functions take, and raises ``LsaError`` on
a non-OK status.  There is no fallback: importing this module on a machine without the
built library fails.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"LSA CUDA library not built: {LIB_PATH} (run python -m long_context_sparse_indexer_b200.build)")
_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_DATA, ERR_TIMEOUT = range(7)
BF16, FP8_E4M3, FP32 = 0, 1, 2
TOPK_RAW = 1
TOPK_EXCLUDES_FIXED = 2
TOPK_WINDOW_ALIGNED = 4
WINDOW_ALIGN = 64

c_i32, c_i64, c_u32, c_f32, c_vp, c_size = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float,
                                             ctypes.c_void_p, ctypes.c_size_t)


class LsaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = _lib.lsa_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})" if what else f"{msg} (status {status})")


class CCache(ctypes.Structure):
    _fields_ = [("data", c_vp), ("scale", c_vp), ("dtype", c_i32), ("dim", c_i32),
                ("seq_stride", c_i64), ("tok_stride", c_i64), ("scale_seq_stride", c_i64)]


class CBatch(ctypes.Structure):
    _fields_ = [("B", c_i32), ("T", c_i32), ("q_group", c_i32), ("L_alloc", c_i32),
                ("seq_len", c_vp), ("q_seq", c_vp), ("q_pos", c_vp)]


class CLayer(ctypes.Structure):
    _fields_ = [("q", c_vp), ("kv", CCache), ("v", CCache), ("o", c_vp), ("lse", c_vp)]


class CDecodeParams(ctypes.Structure):
    _fields_ = [("batch", CBatch), ("q_idx", c_vp), ("w", c_vp), ("H_I", c_i32), ("k_idx", CCache),
                ("k", c_i32), ("n_sink", c_i32), ("window", c_i32),
                ("hi", c_i32), ("block_size", c_i32), ("n_recall", c_i32), ("kbar", c_vp),
                ("kbar_seq_stride", c_i64),
                ("H", c_i32), ("Dqk", c_i32), ("Dv", c_i32), ("sm_scale", c_f32), ("n_split", c_i32),
                ("n_layers", c_i32), ("layers", ctypes.POINTER(CLayer)),
                ("idx_out", c_vp), ("idx_ld", c_i64), ("count_out", c_vp), ("idx_q_fp8", c_i32),
                ("si_fixed_budget", c_i32), ("si_window_aligned", c_i32), ("attn_q_ready", c_vp)]


_P = ctypes.POINTER
_lib.lsa_index_score.argtypes = [_P(CBatch), c_vp, c_vp, c_i32, _P(CCache), c_vp, c_i32, c_i32, c_vp, c_i64,
                                 c_i32, c_vp, c_vp]
_lib.lsa_index_score_q8.argtypes = _lib.lsa_index_score.argtypes
_lib.lsa_block_keys.argtypes = [_P(CBatch), _P(CCache), c_i32, c_vp, c_i64, c_vp, c_vp]
_lib.lsa_block_score.argtypes = [_P(CBatch), c_vp, c_vp, c_i32, c_i32, c_vp, c_i64, c_i32, c_vp, c_i64, c_i32,
                                 c_vp, c_vp]
_lib.lsa_topk.argtypes = [_P(CBatch), c_vp, c_i64, c_i32, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_u32, c_vp,
                          c_i64, c_vp, c_vp, c_vp]
_lib.lsa_sparse_attn.argtypes = [_P(CBatch), c_vp, c_i32, c_i32, _P(CCache), _P(CCache), c_i32, c_vp, c_i64, c_vp,
                                 c_f32, c_i32, c_vp, c_vp, c_vp, c_size, c_vp, c_vp]
_lib.lsa_sparse_attn_noalloc.argtypes = [_P(CBatch), c_vp, c_i32, c_i32, _P(CCache), _P(CCache), c_i32, c_vp, c_i64,
                                         c_vp, c_f32, c_i32, c_vp, c_vp, c_vp, c_vp]
_lib.lsa_attn_workspace_size.argtypes = [c_i32, c_i32, c_i32, c_i32]
_lib.lsa_attn_workspace_size.restype = c_size
_lib.lsa_decode_fused.argtypes = [_P(CDecodeParams), c_vp, c_size, c_vp, c_vp]
_lib.lsa_decode_workspace_size.argtypes = [_P(CDecodeParams)]
_lib.lsa_decode_workspace_size.restype = c_size
_lib.lsa_decode_index_capacity.argtypes = [_P(CDecodeParams)]
_lib.lsa_decode_index_capacity.restype = c_i32
_lib.lsa_read_device_status.argtypes = [c_vp, c_vp]
_lib.lsa_sparse_attn_partial.argtypes = [_P(CBatch), c_vp, c_i32, c_i32, _P(CCache), _P(CCache), c_i32, c_vp, c_i64,
                                         c_vp, c_f32, c_i32, c_vp, c_vp, c_vp, c_size, c_vp, c_vp]
_lib.lsa_merge_partials.argtypes = [c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp]
_lib.lsa_kvp_shard_batch.argtypes = [_P(CBatch), c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]
_lib.lsa_kvp_candidates.argtypes = [_P(CBatch), c_vp, c_vp, c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]
_lib.lsa_kvp_select_workspace_size.argtypes = [c_i32, c_i32, c_i32]
_lib.lsa_kvp_select_workspace_size.restype = c_size
_lib.lsa_kvp_select.argtypes = [_P(CBatch), c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_i64, c_vp, c_vp,
                                c_size, c_vp, c_vp]
_lib.lsa_kvp_local_index.argtypes = [_P(CBatch), c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp]


class CCopy(ctypes.Structure):
    _fields_ = [("dst", c_vp), ("src", c_vp), ("bytes", c_size)]


_lib.lsa_pipeline_create.argtypes = [ctypes.POINTER(c_vp), c_i32, c_vp]
_lib.lsa_pipeline_step.argtypes = [c_vp, c_i32, ctypes.POINTER(_P(CDecodeParams)), c_i32, ctypes.POINTER(c_vp),
                                   ctypes.POINTER(c_size), _P(CCopy), c_i32, _P(CCopy), c_i32, c_vp]
_lib.lsa_pipeline_join.argtypes = [c_vp]
_lib.lsa_pipeline_destroy.argtypes = [c_vp]
_lib.lsa_status_string.argtypes = [c_i32]
_lib.lsa_status_string.restype = ctypes.c_char_p
_lib.lsa_version.restype = c_i32
_lib.lsa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.lsa_set_wait_limit_ns.restype = ctypes.c_uint64
for _f in ("lsa_index_score", "lsa_index_score_q8", "lsa_block_keys", "lsa_block_score", "lsa_topk", "lsa_sparse_attn",
           "lsa_sparse_attn_noalloc", "lsa_decode_fused", "lsa_read_device_status", "lsa_sparse_attn_partial",
           "lsa_merge_partials", "lsa_kvp_shard_batch", "lsa_kvp_candidates", "lsa_kvp_select", "lsa_kvp_local_index"):
    getattr(_lib, _f).restype = c_i32

EXPORTS = ("lsa_index_score", "lsa_index_score_q8", "lsa_block_keys", "lsa_block_score", "lsa_topk", "lsa_sparse_attn",
           "lsa_sparse_attn_noalloc", "lsa_attn_workspace_size", "lsa_decode_fused", "lsa_decode_workspace_size", "lsa_read_device_status",
           "lsa_status_string", "lsa_version", "lsa_pipeline_create", "lsa_pipeline_step", "lsa_pipeline_join",
           "lsa_pipeline_destroy", "lsa_sparse_attn_partial", "lsa_merge_partials", "lsa_kvp_shard_batch",
           "lsa_kvp_candidates", "lsa_kvp_select_workspace_size", "lsa_kvp_select", "lsa_kvp_local_index",
           "lsa_set_wait_limit_ns", "lsa_decode_index_capacity")


def library() -> ctypes.CDLL:
    return _lib


def _check(status: int, what: str) -> None:
    if status != OK:
        raise LsaError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ------------------------------------------------------------------ descriptors

@dataclass
class Batch:
    """Query tokens: q_seq / q_pos / seq_len are int32 device tensors."""
    seq_len: torch.Tensor
    q_seq: torch.Tensor
    q_pos: torch.Tensor
    L_alloc: int
    q_group: int = 1

    def c(self) -> CBatch:
        return CBatch(int(self.seq_len.numel()), int(self.q_seq.numel()), int(self.q_group), int(self.L_alloc),
                      _ptr(self.seq_len), _ptr(self.q_seq), _ptr(self.q_pos))


@dataclass
class Cache:
    """A per-sequence cache [B, L_alloc, dim]: uint8 FP8 codes (+ float scale [B, L_alloc]) or bf16."""
    data: torch.Tensor
    scale: Optional[torch.Tensor] = None

    @property
    def dtype(self) -> int:
        if self.data.dtype == torch.uint8 or self.data.dtype == torch.float8_e4m3fn:
            return FP8_E4M3
        if self.data.dtype == torch.bfloat16:
            return BF16
        raise ValueError(f"unsupported cache dtype {self.data.dtype}")

    def c(self) -> CCache:
        d = self.data
        assert d.dim() == 3 and d.stride(2) == 1
        sc = self.scale
        sss = int(sc.stride(0)) if sc is not None else 0
        return CCache(_ptr(d), _ptr(sc), self.dtype, int(d.shape[2]), int(d.stride(0)), int(d.stride(1)), sss)


_EMPTY_CACHE = CCache(None, None, 0, 0, 0, 0, 0)


# ------------------------------------------------------------------ entry points

def index_score(batch: Batch, q_idx: torch.Tensor, w: torch.Tensor, k_idx: Cache, scores: torch.Tensor,
                n_cols: int = 0, cand_blocks: Optional[torch.Tensor] = None, block_size: int = 0,
                dev_status: Optional[torch.Tensor] = None, stream=None, q_fp8: bool = False) -> None:
    """lsa_index_score (lsa_index_score_q8 with q_fp8): flat scores (cand_blocks None) or HI fine
    scores over recalled blocks."""
    cb, ck = batch.c(), k_idx.c()
    n_cand = int(cand_blocks.shape[1]) if cand_blocks is not None else 0
    fn, name = (_lib.lsa_index_score_q8, "lsa_index_score_q8") if q_fp8 else (_lib.lsa_index_score, "lsa_index_score")
    _check(fn(ctypes.byref(cb), _ptr(q_idx), _ptr(w), int(q_idx.shape[1]), ctypes.byref(ck),
              _ptr(cand_blocks), n_cand, int(block_size), _ptr(scores), int(scores.stride(0)),
              int(n_cols), _ptr(dev_status), _stream(stream)), name)


def block_keys_buffer(B: int, L_alloc: int, block_size: int, d_I: int, device) -> torch.Tensor:
    """An (uninitialised) block-key buffer in the layout lsa_block_keys writes:
    [B, ceil(L_alloc / block_size), 2 * d_I] BF16, each row the (hi, lo) halves of one block key."""
    nblk = (L_alloc + block_size - 1) // block_size
    return torch.empty((B, nblk, 2 * d_I), dtype=torch.bfloat16, device=device)


def block_keys(batch: Batch, k_idx: Cache, block_size: int, kbar: torch.Tensor,
               dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """lsa_block_keys into `kbar` (see block_keys_buffer for its layout)."""
    cb, ck = batch.c(), k_idx.c()
    _check(_lib.lsa_block_keys(ctypes.byref(cb), ctypes.byref(ck), int(block_size), _ptr(kbar), int(kbar.stride(0)),
                               _ptr(dev_status), _stream(stream)), "lsa_block_keys")


def block_score(batch: Batch, q_idx: torch.Tensor, w: torch.Tensor, kbar: torch.Tensor, block_size: int,
                scores: torch.Tensor, n_cols: int, dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    cb = batch.c()
    _check(_lib.lsa_block_score(ctypes.byref(cb), _ptr(q_idx), _ptr(w), int(q_idx.shape[1]), int(q_idx.shape[2]),
                                _ptr(kbar), int(kbar.stride(0)), int(block_size), _ptr(scores), int(scores.stride(0)),
                                int(n_cols), _ptr(dev_status), _stream(stream)), "lsa_block_score")


def topk(batch: Batch, scores: torch.Tensor, n_cols: int, k: int, n_sink: int, window: int, idx: torch.Tensor,
         count: torch.Tensor, cand_blocks: Optional[torch.Tensor] = None, block_size: int = 0, raw: bool = False,
         dev_status: Optional[torch.Tensor] = None, stream=None, fixed_budget: bool = False,
         window_aligned: bool = False) -> None:
    cb = batch.c()
    n_cand = int(cand_blocks.shape[1]) if cand_blocks is not None else 0
    _check(_lib.lsa_topk(ctypes.byref(cb), _ptr(scores), int(scores.stride(0)), int(n_cols), _ptr(cand_blocks),
                         n_cand, int(block_size), int(k), int(n_sink), int(window),
                         (TOPK_RAW if raw else 0) | (TOPK_EXCLUDES_FIXED if fixed_budget else 0)
                         | (TOPK_WINDOW_ALIGNED if window_aligned else 0),
                         _ptr(idx), int(idx.stride(0)), _ptr(count), _ptr(dev_status), _stream(stream)), "lsa_topk")


def attn_workspace_size(T: int, H: int, Dv: int, n_split: int) -> int:
    return int(_lib.lsa_attn_workspace_size(T, H, Dv, n_split))


def sparse_attn(batch: Batch, q: torch.Tensor, kv: Cache, idx: torch.Tensor, count: torch.Tensor, sm_scale: float,
                o: torch.Tensor, lse: Optional[torch.Tensor] = None, v: Optional[Cache] = None, Dv: int = 0,
                n_split: int = 1, ws: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                stream=None) -> None:
    cb, ck = batch.c(), kv.c()
    cv = v.c() if v is not None else None
    H, Dqk = int(q.shape[1]), int(q.shape[2])
    Dv = int(Dv or o.shape[2])
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.lsa_sparse_attn(ctypes.byref(cb), _ptr(q), H, Dqk, ctypes.byref(ck),
                                ctypes.byref(cv) if cv is not None else None, Dv, _ptr(idx), int(idx.stride(0)),
                                _ptr(count), float(sm_scale), int(n_split), _ptr(o), _ptr(lse), _ptr(ws), wsb,
                                _ptr(dev_status), _stream(stream)), "lsa_sparse_attn")


NOALLOC_SCRATCH_BYTES = 32 << 20


def sparse_attn_noalloc(batch: Batch, q: torch.Tensor, kv: Cache, idx: torch.Tensor, count: torch.Tensor,
                        sm_scale: float, o: torch.Tensor, lse: Optional[torch.Tensor] = None,
                        v: Optional[Cache] = None, Dv: int = 0, n_split: int = 1,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """lsa_sparse_attn_noalloc: sparse_attn for callers that cannot allocate device memory.

    The split partials live in the library's static device scratch array (32 MiB per GPU,
    shared by every call, so calls must not overlap on the GPU); nothing is allocated.
    """
    cb, ck = batch.c(), kv.c()
    cv = v.c() if v is not None else None
    H, Dqk = int(q.shape[1]), int(q.shape[2])
    Dv = int(Dv or o.shape[2])
    _check(_lib.lsa_sparse_attn_noalloc(ctypes.byref(cb), _ptr(q), H, Dqk, ctypes.byref(ck),
                                        ctypes.byref(cv) if cv is not None else None, Dv, _ptr(idx),
                                        int(idx.stride(0)), _ptr(count), float(sm_scale), int(n_split), _ptr(o),
                                        _ptr(lse), _ptr(dev_status), _stream(stream)), "lsa_sparse_attn_noalloc")


def sparse_attn_partial(batch: Batch, q: torch.Tensor, kv: Cache, idx: torch.Tensor, count: torch.Tensor,
                        sm_scale: float, o_part: torch.Tensor, lse_part: torch.Tensor, v: Optional[Cache] = None,
                        Dv: int = 0, n_split: int = 1, ws: Optional[torch.Tensor] = None,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """lsa_sparse_attn_partial: sparse_attn with an FP32 result (o_part [T, H, Dv] float, lse_part [T, H])."""
    cb, ck = batch.c(), kv.c()
    cv = v.c() if v is not None else None
    H, Dqk = int(q.shape[1]), int(q.shape[2])
    Dv = int(Dv or o_part.shape[2])
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.lsa_sparse_attn_partial(ctypes.byref(cb), _ptr(q), H, Dqk, ctypes.byref(ck),
                                        ctypes.byref(cv) if cv is not None else None, Dv, _ptr(idx),
                                        int(idx.stride(0)), _ptr(count), float(sm_scale), int(n_split), _ptr(o_part),
                                        _ptr(lse_part), _ptr(ws), wsb, _ptr(dev_status), _stream(stream)),
           "lsa_sparse_attn_partial")


def merge_partials(o_parts: torch.Tensor, lse_parts: torch.Tensor, o: torch.Tensor, lse: Optional[torch.Tensor] = None,
                   stream=None) -> None:
    """lsa_merge_partials: o_parts [R, T, H, Dv] float, lse_parts [R, T, H] -> o [T, H, Dv] bf16 (+ lse)."""
    R, T, H, Dv = (int(x) for x in o_parts.shape)
    assert o_parts.is_contiguous() and lse_parts.is_contiguous() and o.is_contiguous()
    _check(_lib.lsa_merge_partials(_ptr(o_parts), _ptr(lse_parts), R, T, H, Dv, _ptr(o), _ptr(lse), _stream(stream)),
           "lsa_merge_partials")


def kvp_shard_batch(batch: Batch, L_alloc_local: int, shard_start: torch.Tensor, shard_len: torch.Tensor,
                    local_seq_len: torch.Tensor, local_q_pos: torch.Tensor, dev_status: Optional[torch.Tensor] = None,
                    stream=None) -> Batch:
    """lsa_kvp_shard_batch: the shard's local batch (same q_seq, local lengths and positions)."""
    cb = batch.c()
    _check(_lib.lsa_kvp_shard_batch(ctypes.byref(cb), int(L_alloc_local), _ptr(shard_start), _ptr(shard_len),
                                    _ptr(local_seq_len), _ptr(local_q_pos), _ptr(dev_status), _stream(stream)),
           "lsa_kvp_shard_batch")
    return Batch(local_seq_len, batch.q_seq, local_q_pos, int(L_alloc_local), batch.q_group)


def kvp_candidates(local: Batch, q_pos_global: torch.Tensor, shard_start: torch.Tensor, scores: torch.Tensor,
                   n_cols: int, k: int, cand_pos: torch.Tensor, cand_score: torch.Tensor, cand_count: torch.Tensor,
                   dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    cb = local.c()
    _check(_lib.lsa_kvp_candidates(ctypes.byref(cb), _ptr(q_pos_global), _ptr(shard_start), _ptr(scores),
                                   int(scores.stride(0)), int(n_cols), int(k), _ptr(cand_pos), _ptr(cand_score),
                                   _ptr(cand_count), _ptr(dev_status), _stream(stream)), "lsa_kvp_candidates")


def kvp_select_workspace_size(T: int, n_parts: int, k_part: int) -> int:
    return int(_lib.lsa_kvp_select_workspace_size(T, n_parts, k_part))


def kvp_select(batch: Batch, cand_pos: torch.Tensor, cand_score: torch.Tensor, k: int, n_sink: int, window: int,
               idx: torch.Tensor, count: torch.Tensor, ws: torch.Tensor, dev_status: Optional[torch.Tensor] = None,
               stream=None) -> None:
    """lsa_kvp_select: cand_pos / cand_score [n_parts, T, k_part] (shard order) -> idx [T, cap], count [T]."""
    n_parts, _, k_part = (int(x) for x in cand_pos.shape)
    cb = batch.c()
    _check(_lib.lsa_kvp_select(ctypes.byref(cb), _ptr(cand_pos), _ptr(cand_score), n_parts, k_part, int(k),
                               int(n_sink), int(window), _ptr(idx), int(idx.stride(0)), _ptr(count), _ptr(ws),
                               ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)), "lsa_kvp_select")


def kvp_local_index(batch: Batch, shard_start: torch.Tensor, shard_len: torch.Tensor, idx: torch.Tensor,
                    count: torch.Tensor, local_idx: torch.Tensor, local_count: torch.Tensor,
                    dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    cb = batch.c()
    _check(_lib.lsa_kvp_local_index(ctypes.byref(cb), _ptr(shard_start), _ptr(shard_len), _ptr(idx),
                                    int(idx.stride(0)), _ptr(count), _ptr(local_idx), int(local_idx.stride(0)),
                                    _ptr(local_count), _ptr(dev_status), _stream(stream)), "lsa_kvp_local_index")


@dataclass
class Layer:
    q: torch.Tensor
    kv: Cache
    o: torch.Tensor
    lse: Optional[torch.Tensor] = None
    v: Optional[Cache] = None


class DecodeStep:
    """Marshalled parameters of lsa_decode_fused (built once, launched many times)."""

    def __init__(self, batch: Batch, q_idx: torch.Tensor, w: torch.Tensor, k_idx: Cache, k: int, n_sink: int,
                 window: int, layers: Sequence[Layer], H: int, Dqk: int, Dv: int, sm_scale: float, n_split: int = 1,
                 hi: bool = False, block_size: int = 64, n_recall: int = 0, kbar: Optional[torch.Tensor] = None,
                 idx_out: Optional[torch.Tensor] = None, count_out: Optional[torch.Tensor] = None,
                 idx_q_fp8: bool = False, si_fixed_budget: bool = False, si_window_aligned: bool = False,
                 attn_q_ready=None):
        """attn_q_ready: a torch.cuda.Event recorded once the layers' attention queries are written
        (the attention waits for it, the indexer and top-k do not), or None."""
        self._keep = (batch, q_idx, w, k_idx, list(layers), kbar, idx_out, count_out, attn_q_ready)
        arr = (CLayer * max(1, len(layers)))()
        for i, L in enumerate(layers):
            arr[i] = CLayer(_ptr(L.q), L.kv.c(), L.v.c() if L.v is not None else _EMPTY_CACHE, _ptr(L.o), _ptr(L.lse))
        self._layers = arr
        self.p = CDecodeParams(batch.c(), _ptr(q_idx), _ptr(w), int(q_idx.shape[1]), k_idx.c(), int(k), int(n_sink),
                               int(window), int(bool(hi)), int(block_size), int(n_recall), _ptr(kbar),
                               int(kbar.stride(0)) if kbar is not None else 0, int(H), int(Dqk), int(Dv),
                               float(sm_scale), int(n_split), len(layers), arr, _ptr(idx_out),
                               int(idx_out.stride(0)) if idx_out is not None else 0, _ptr(count_out),
                               int(bool(idx_q_fp8)), int(bool(si_fixed_budget)), int(bool(si_window_aligned)),
                               None)
        self._attn_q_ready = attn_q_ready

    def workspace_size(self) -> int:
        return int(_lib.lsa_decode_workspace_size(ctypes.byref(self.p)))

    def index_capacity(self) -> int:
        return int(_lib.lsa_decode_index_capacity(ctypes.byref(self.p)))

    def __call__(self, ws: torch.Tensor, dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
        if self._attn_q_ready is not None:
            # torch creates an event's CUDA handle at its first record: read it at each call
            self.p.attn_q_ready = self._attn_q_ready.cuda_event or None
        _check(_lib.lsa_decode_fused(ctypes.byref(self.p), _ptr(ws), ws.numel() * ws.element_size(),
                                     _ptr(dev_status), _stream(stream)), "lsa_decode_fused")


class Pipeline:
    """lsa_pipeline_*: pipelined host-buffer decode (copy-in, fused decode, copy-out on three
    streams, ordered per device-buffer slot).  `prepare` marshals one slot's step once; `run`
    issues it (no synchronisation); `join` orders the decode stream after every copy issued."""

    class Prepared:
        def __init__(self, slot, steps, wss, h2d, d2h, dev_status):
            self.slot = int(slot)
            self._keep = (steps, wss, h2d, d2h, dev_status)
            n = len(steps)
            self.params = (_P(CDecodeParams) * max(1, n))(*[ctypes.pointer(st.p) for st in steps])
            self.ws = (c_vp * max(1, n))(*[_ptr(w) for w in wss])
            self.ws_bytes = (c_size * max(1, n))(*[w.numel() * w.element_size() for w in wss])
            self.n = n
            self.h2d = (CCopy * max(1, len(h2d)))(*[CCopy(_ptr(d), _ptr(h), h.numel() * h.element_size())
                                                    for d, h in h2d])
            self.n_h2d = len(h2d)
            self.d2h = (CCopy * max(1, len(d2h)))(*[CCopy(_ptr(h), _ptr(d), d.numel() * d.element_size())
                                                    for h, d in d2h])
            self.n_d2h = len(d2h)
            self.dev_status = _ptr(dev_status)

    def __init__(self, n_slots: int = 2, stream=None):
        h = c_vp()
        _check(_lib.lsa_pipeline_create(ctypes.byref(h), int(n_slots), _stream(stream)), "lsa_pipeline_create")
        self._h = h

    def prepare(self, slot: int, steps: Sequence["DecodeStep"], wss: Sequence[torch.Tensor],
                h2d: Sequence[tuple], d2h: Sequence[tuple], dev_status: Optional[torch.Tensor] = None) -> "Pipeline.Prepared":
        """h2d: (device tensor, pinned host tensor) pairs; d2h: (pinned host tensor, device tensor) pairs."""
        for d, h in list(h2d) + [(d, h) for h, d in d2h]:
            assert d.is_cuda and not h.is_cuda and d.is_contiguous() and h.is_contiguous()
            assert d.numel() * d.element_size() == h.numel() * h.element_size()
        return Pipeline.Prepared(slot, list(steps), list(wss), list(h2d), list(d2h), dev_status)

    def run(self, pr: "Pipeline.Prepared") -> None:
        _check(_lib.lsa_pipeline_step(self._h, pr.slot, pr.params, pr.n, pr.ws, pr.ws_bytes, pr.h2d, pr.n_h2d,
                                      pr.d2h, pr.n_d2h, pr.dev_status), "lsa_pipeline_step")

    def join(self) -> None:
        _check(_lib.lsa_pipeline_join(self._h), "lsa_pipeline_join")

    def close(self) -> None:
        if self._h:
            _check(_lib.lsa_pipeline_destroy(self._h), "lsa_pipeline_destroy")
            self._h = c_vp()

    def __del__(self):
        try:
            if self._h:
                _lib.lsa_pipeline_destroy(self._h)
        except Exception:
            pass


def read_device_status(dev_status: torch.Tensor, stream=None) -> int:
    return int(_lib.lsa_read_device_status(_ptr(dev_status), _stream(stream)))


def status_string(status: int) -> str:
    return _lib.lsa_status_string(status).decode()


def version() -> int:
    return int(_lib.lsa_version())


def set_wait_limit_ns(ns: int) -> int:
    """lsa_set_wait_limit_ns (diagnostic): returns the previous limit (0 = the 2 s default)."""
    return int(_lib.lsa_set_wait_limit_ns(int(ns)))
