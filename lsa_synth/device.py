"""GPU-side construction of the synthetic workloads (same bytes as the host generator).

Builds every tensor a workload needs directly in device memory with the filler in
``csrc/synth_fill.cu`` (compiled in-tree to ``_synth.so``), so caches of tens of GB never
pass through the host.  Only small index tensors (lengths, positions, planted rows,
planting directions) are computed on the host and copied.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np
import torch

from . import gen
from . import workloads as W

_HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(_HERE, "_synth.so")
SRC = os.path.join(_HERE, "csrc", "synth_fill.cu")


def build(force: bool = False) -> str:
    if force or not os.path.exists(SO) or os.path.getmtime(SO) < os.path.getmtime(SRC):
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
        cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
               "-shared", SRC, "-o", SO]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("synth_fill build failed:\n" + res.stdout + res.stderr)
    return SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise ImportError(f"{SO} not built (python -c 'import lsa_synth.device as d; d.build()')")
        lib = ctypes.CDLL(SO)
        lib.synth_fill_rows.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p]
        lib.synth_fill_uniform.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p]
        _lib = lib
    return _lib


def _stream():
    return torch.cuda.current_stream().cuda_stream


def fill_rows(out: torch.Tensor, scale: torch.Tensor | None, key: int, cache_mode: bool, L_alloc: int,
              rows: torch.Tensor | None = None, dirs: torch.Tensor | None = None) -> None:
    fmt = {torch.bfloat16: 0, torch.uint8: 1, torch.float32: 2}[out.dtype]
    dim = out.shape[-1]
    n_rows = rows.numel() if rows is not None else out.numel() // dim
    err = _load().synth_fill_rows(out.data_ptr(), scale.data_ptr() if scale is not None else None, fmt, n_rows, dim,
                                  int(cache_mode), int(L_alloc), key,
                                  rows.data_ptr() if rows is not None else None,
                                  dirs.data_ptr() if dirs is not None else None, _stream())
    if err:
        raise RuntimeError(f"synth_fill_rows failed: cuda error {err}")


def fill_uniform(out: torch.Tensor, key: int) -> None:
    err = _load().synth_fill_uniform(out.data_ptr(), out.numel(), key, _stream())
    if err:
        raise RuntimeError(f"synth_fill_uniform failed: cuda error {err}")


@dataclass
class PassTensors:
    q_seq: torch.Tensor
    q_pos: torch.Tensor
    q_idx: torch.Tensor            # bf16 [T, H_I, d_I]
    w: torch.Tensor                # f32 [T, H_I]
    k_idx: torch.Tensor            # uint8 or bf16 [B, L_alloc, d_I]
    k_scale: torch.Tensor | None   # f32 [B, L_alloc]
    layers: list = field(default_factory=list)   # per layer: dict(q, kv, kv_scale, v)


@dataclass
class WorkloadTensors:
    w: W.Workload
    L_alloc: int
    seq_len: torch.Tensor
    passes: list


def _cache(B: int, L: int, dim: int, fp8: bool, dev):
    if fp8:
        return (torch.empty((B, L, dim), dtype=torch.uint8, device=dev),
                torch.empty((B, L), dtype=torch.float32, device=dev))
    return torch.empty((B, L, dim), dtype=torch.bfloat16, device=dev), None


def build_workload(w: W.Workload, device="cuda", L_alloc: int | None = None) -> WorkloadTensors:
    """All input tensors of a workload, generated on the GPU."""
    build()
    dev = torch.device(device)
    lens = W.lengths(w)
    L_alloc = int(L_alloc or -(-int(lens.max()) // 64) * 64)     # rows per sequence, a multiple of 64
    seq_len = torch.from_numpy(lens.astype(np.int32)).to(dev)
    passes = []
    kv_done = {}
    for p in w.passes:
        q_seq, q_pos = W.query_rows(w, p)
        T = w.T(p)
        q_idx = torch.empty((T, w.H_I, w.d_I), dtype=torch.bfloat16, device=dev)
        fill_rows(q_idx, None, gen.tensor_key(w.seed, p.tid_idx_q), False, 1)
        wt = torch.empty((T, w.H_I), dtype=torch.float32, device=dev)
        fill_uniform(wt, gen.tensor_key(w.seed, p.tid_idx_w))
        k_idx, k_scale = _cache(w.B, L_alloc, w.d_I, w.idx_fp8, dev)
        key = gen.tensor_key(w.seed, p.tid_idx_keys)
        fill_rows(k_idx, k_scale, key, True, L_alloc)
        if p.name == "target" and (w.plant_frac > 0 or w.plant_blocks > 0):
            rows, dirs = W.plant_plan(w, p)
            flat = np.concatenate([b * L_alloc + r for b, r in enumerate(rows)]).astype(np.int64)
            if flat.size:
                fill_rows(k_idx, k_scale, key, True, L_alloc, rows=torch.from_numpy(flat).to(dev),
                          dirs=torch.from_numpy(dirs).to(dev))
        layers = []
        for layer in p.layers:
            q = torch.empty((T, w.H, w.D), dtype=torch.bfloat16, device=dev)
            fill_rows(q, None, gen.tensor_key(w.seed, layer.tid_q), False, 1)
            if layer.tid_kv not in kv_done:
                kv, kv_scale = _cache(w.B, L_alloc, w.D, w.kv_fp8, dev)
                fill_rows(kv, kv_scale, gen.tensor_key(w.seed, layer.tid_kv), True, L_alloc)
                v = None
                if layer.tid_v >= 0:
                    v, _ = _cache(w.B, L_alloc, w.Dv, False, dev)
                    fill_rows(v, None, gen.tensor_key(w.seed, layer.tid_v), True, L_alloc)
                kv_done[layer.tid_kv] = (kv, kv_scale, v)
            kv, kv_scale, v = kv_done[layer.tid_kv]
            layers.append(dict(q=q, kv=kv, kv_scale=kv_scale, v=v))
        passes.append(PassTensors(torch.from_numpy(q_seq.astype(np.int32)).to(dev),
                                  torch.from_numpy(q_pos.astype(np.int32)).to(dev), q_idx, wt, k_idx, k_scale,
                                  layers))
    return WorkloadTensors(w, L_alloc, seq_len, passes)
