"""The C ABI without a GPU: every symbol of include/lsa.h is exported, host validation rejects bad calls."""
import ctypes
import os
import re

import pytest
import torch

from long_context_sparse_indexer_b200 import lsa

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lsa.h")


def declared():
    txt = open(HDR).read()
    return sorted(set(re.findall(r"^\s*(?:lsa_status|size_t|const char\*|int|uint64_t)\s+(lsa_\w+)\s*\(", txt, re.M)))


def test_every_declared_symbol_is_exported():
    names = declared()
    assert len(names) >= 11
    lib = lsa.library()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(lsa.EXPORTS)


def test_status_strings_and_version():
    assert lsa.version() == 1
    for s in range(7):
        assert lsa.status_string(s)
    assert "unknown" in lsa.status_string(99)


def _batch(T=1, B=1, q_group=1, L=100):
    return lsa.CBatch(B, T, q_group, L, 16, 16, 16)        # fake device pointers: never dereferenced


def _cache(dtype=lsa.FP8_E4M3, dim=128, scale=16, data=4096):
    return lsa.CCache(data, scale, dtype, dim, 100 * dim, dim, 100)


def test_index_score_rejects_bad_arguments():
    lib = lsa.library()
    b, c = _batch(), _cache()
    call = lambda bb, cc, H_I=64, ld=100, n=100, q=16, w=16, sc=16: lib.lsa_index_score(  # noqa: E731
        ctypes.byref(bb), q, w, H_I, ctypes.byref(cc), None, 0, 0, sc, ld, n, None, None)
    assert call(b, c, H_I=48) == lsa.ERR_UNSUPPORTED
    assert call(b, _cache(dim=96)) == lsa.ERR_UNSUPPORTED
    assert call(b, _cache(scale=None)) == lsa.ERR_INVALID_ARG              # FP8 without scale
    assert call(b, _cache(data=4097)) == lsa.ERR_INVALID_ARG               # misaligned rows
    assert call(b, c, n=101) == lsa.ERR_INVALID_ARG                        # n_cols > ld
    assert call(_batch(T=3, q_group=2), c) == lsa.ERR_INVALID_ARG          # T not a multiple of q_group
    assert call(b, c, q=None) == lsa.ERR_INVALID_ARG
    assert call(b, _cache(dtype=7)) == lsa.ERR_UNSUPPORTED
    assert lib.lsa_index_score(None, 16, 16, 64, ctypes.byref(c), None, 0, 0, 16, 100, 100, None, None) \
        == lsa.ERR_INVALID_ARG


def test_block_calls_reject_bad_arguments():
    """lsa_block_keys / lsa_block_score: layout of the block-key buffer, supported shapes, and an
    empty batch as a no-op (L_alloc = 100, block size 64: 2 blocks of 2 * 128 BF16 each)."""
    lib = lsa.library()
    b, c = _batch(), _cache()
    keys = lambda bb=b, cc=c, bs=64, kbar=4096, stride=512: lib.lsa_block_keys(  # noqa: E731
        ctypes.byref(bb) if bb is not None else None, ctypes.byref(cc), bs, kbar, stride, None, None)
    assert keys(bb=None) == lsa.ERR_INVALID_ARG
    assert keys(kbar=None) == lsa.ERR_INVALID_ARG
    assert keys(bs=0) == lsa.ERR_INVALID_ARG and keys(bs=1025) == lsa.ERR_INVALID_ARG
    assert keys(stride=504) == lsa.ERR_INVALID_ARG                          # below 2 blocks x 2 d_I
    assert keys(stride=516) == lsa.ERR_INVALID_ARG                          # not 16-byte rows
    assert keys(kbar=4104) == lsa.ERR_INVALID_ARG                           # kbar not 16-byte aligned
    assert keys(cc=_cache(dtype=7)) == lsa.ERR_UNSUPPORTED
    assert keys(cc=_cache(scale=None)) == lsa.ERR_INVALID_ARG
    assert keys(bb=lsa.CBatch(1, 0, 1, 100, None, None, None)) == lsa.ERR_INVALID_ARG   # no lengths

    score = lambda bb=b, H_I=64, d_I=128, kbar=4096, stride=512, bs=64, ld=2, n=2, q=16, w=16, sc=16:         lib.lsa_block_score(ctypes.byref(bb), q, w, H_I, d_I, kbar, stride, bs, sc, ld, n, None, None)  # noqa: E731
    assert score(H_I=48) == lsa.ERR_UNSUPPORTED
    assert score(d_I=96) == lsa.ERR_UNSUPPORTED
    assert score(bs=0) == lsa.ERR_INVALID_ARG
    assert score(n=3, ld=3) == lsa.ERR_INVALID_ARG                          # more columns than blocks
    assert score(n=2, ld=1) == lsa.ERR_INVALID_ARG                          # n_cols > ld
    assert score(stride=504) == lsa.ERR_INVALID_ARG
    assert score(q=None) == lsa.ERR_INVALID_ARG and score(sc=None) == lsa.ERR_INVALID_ARG
    assert score(q=24) == lsa.ERR_INVALID_ARG and score(kbar=4104) == lsa.ERR_INVALID_ARG
    assert score(bb=lsa.CBatch(1, 0, 1, 100, 16, None, None)) == lsa.OK     # no query: nothing to do


def test_topk_rejects_bad_arguments():
    lib = lsa.library()
    b = _batch()
    call = lambda k=10, ns=4, win=8, ld_idx=22, flags=0, cand=None: lib.lsa_topk(  # noqa: E731
        ctypes.byref(b), 16, 100, 100, cand, 1 if cand else 0, 64 if cand else 0, k, ns, win, flags, 16, ld_idx, 16,
        None, None)
    assert call(ld_idx=21) == lsa.ERR_INVALID_ARG                          # capacity below k + sinks + window
    assert call(k=-1) == lsa.ERR_INVALID_ARG
    assert call(flags=lsa.TOPK_RAW) == lsa.ERR_INVALID_ARG                 # raw mode takes no sinks/window
    assert call(flags=8) == lsa.ERR_UNSUPPORTED
    assert call(flags=lsa.TOPK_RAW | lsa.TOPK_EXCLUDES_FIXED, ns=0, win=0) == lsa.ERR_INVALID_ARG   # raw has no fixed part


def test_attention_rejects_bad_arguments():
    lib = lsa.library()
    b = _batch()
    kv = _cache(dtype=lsa.BF16, dim=576, scale=None)
    call = lambda H=128, Dqk=576, Dv=512, ns=1, ws=None, wsb=0, scale=0.04, kvc=kv: lib.lsa_sparse_attn(  # noqa
        ctypes.byref(b), 4096, H, Dqk, ctypes.byref(kvc), None, Dv, 16, 100, 16, scale, ns, 4096, 16, ws, wsb, None,
        None)
    assert call(H=100) == lsa.ERR_UNSUPPORTED
    assert call(Dv=256) == lsa.ERR_UNSUPPORTED
    assert call(ns=0) == lsa.ERR_INVALID_ARG
    assert call(ns=65) == lsa.ERR_INVALID_ARG
    assert call(scale=float("nan")) == lsa.ERR_INVALID_ARG
    assert call(ns=4) == lsa.ERR_WORKSPACE                                 # split partials need a workspace
    need = lsa.attn_workspace_size(1, 128, 512, 4)
    assert need >= 4 * 128 * 512 * 4
    assert call(ns=4, ws=4096, wsb=need - 1) == lsa.ERR_WORKSPACE
    assert lsa.attn_workspace_size(5, 128, 512, 1) == 0


def test_noalloc_attention_checks_shapes_before_its_scratch_size():
    """The no-allocation entry point returns what lsa_sparse_attn returns for the same bad
    arguments, and LSA_ERR_WORKSPACE only for a valid request its static scratch cannot hold
    (no GPU: every one of these returns before the first CUDA call)."""
    lib = lsa.library()
    kv = _cache(dtype=lsa.BF16, dim=576, scale=None)
    big = _batch(T=200)
    call = lambda b, H=128, ns=64: lib.lsa_sparse_attn_noalloc(  # noqa
        ctypes.byref(b), 4096, H, 576, ctypes.byref(kv), None, 512, 16, 100, 16, 0.04, ns, 4096, 16, None, None)
    assert call(big, H=100) == lsa.ERR_UNSUPPORTED          # shape first, although 200 x 64 x 100 rows > scratch
    assert call(big, ns=0) == lsa.ERR_INVALID_ARG
    assert call(big) == lsa.ERR_WORKSPACE                   # 200 x 64 x 128 partial rows of 2 KB > 32 MiB
    assert lsa.attn_workspace_size(200, 128, 512, 64) > lsa.NOALLOC_SCRATCH_BYTES


def test_noalloc_scratch_size_matches_the_header():
    m = re.search(r"#define\s+LSA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", open(HDR).read())
    assert m, "LSA_NOALLOC_SCRATCH_BYTES not found in the header"
    assert int(m.group(1)) << int(m.group(2)) == lsa.NOALLOC_SCRATCH_BYTES


def test_batches_beyond_the_grid_limit_are_refused():
    """More than 65,535 query tokens in one call: LSA_ERR_UNSUPPORTED before any launch."""
    lib = lsa.library()
    b = _batch(T=65536)
    kv = _cache(dtype=lsa.BF16, dim=576, scale=None)
    assert lib.lsa_sparse_attn(ctypes.byref(b), 4096, 128, 576, ctypes.byref(kv), None, 512, 16, 100, 16, 0.04, 1,
                               4096, 16, None, 0, None, None) == lsa.ERR_UNSUPPORTED
    assert lib.lsa_topk(ctypes.byref(b), 16, 100, 100, None, 0, 0, 10, 0, 0, 0, 16, 10, 16, None,
                        None) == lsa.ERR_UNSUPPORTED


def test_fused_rejects_bad_arguments():
    lib = lsa.library()
    p = lsa.CDecodeParams()
    p.batch = _batch()
    p.k, p.n_sink, p.window = 10, 4, 8
    p.H_I = 64
    p.k_idx = _cache()
    p.n_layers = 1
    p.layers = None
    assert lib.lsa_decode_fused(ctypes.byref(p), 4096, 1 << 30, None, None) == lsa.ERR_INVALID_ARG
    p.n_layers = 0
    p.hi, p.block_size, p.n_recall = 1, 64, 0
    assert lib.lsa_decode_fused(ctypes.byref(p), 4096, 1 << 30, None, None) == lsa.ERR_INVALID_ARG
    p.hi = 0
    need = lib.lsa_decode_workspace_size(ctypes.byref(p))
    assert need > 0
    assert lib.lsa_decode_fused(ctypes.byref(p), 4096, need - 1, None, None) == lsa.ERR_WORKSPACE
    assert lib.lsa_decode_fused(ctypes.byref(p), 4097, need, None, None) == lsa.ERR_WORKSPACE


def test_binding_refuses_to_run_without_cuda_library_on_missing_build(tmp_path, monkeypatch):
    import importlib
    import long_context_sparse_indexer_b200.lsa as mod
    monkeypatch.setattr(os.path, "exists", lambda p: False if p.endswith("_lsa.so") else os.path.isfile(p))
    with pytest.raises(ImportError):
        importlib.reload(mod)
    monkeypatch.undo()
    importlib.reload(mod)


def test_pipeline_rejects_bad_arguments():
    """lsa_pipeline_*: argument checks happen before any CUDA call (no device needed)."""
    lib = lsa.library()
    out = ctypes.c_void_p()
    assert lib.lsa_pipeline_create(None, 2, None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_pipeline_create(ctypes.byref(out), 0, None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_pipeline_create(ctypes.byref(out), 9, None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_pipeline_step(None, 0, None, 0, None, None, None, 0, None, 0, None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_pipeline_join(None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_pipeline_destroy(None) == lsa.ERR_INVALID_ARG


def test_struct_layouts_match_the_header(tmp_path):
    """Every ctypes mirror of a header struct has the header's size and field offsets (checked
    by compiling a C program against include/lsa.h)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    mirrors = {"lsa_cache": lsa.CCache, "lsa_batch": lsa.CBatch, "lsa_layer": lsa.CLayer,
               "lsa_decode_params": lsa.CDecodeParams, "lsa_copy": lsa.CCopy}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "lsa.h"', "int main(void) {"]
    for cname, cls in mirrors.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run([gcc, "-std=c11", "-I", inc, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {}
    for line in out:
        if line:
            parts = line.split()
            got[tuple(parts[:-1])] = int(parts[-1])
    for cname, cls in mirrors.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert got[(cname, fname)] == getattr(cls, fname).offset, (cname, fname)


def test_kvp_and_partial_calls_reject_bad_arguments():
    """The KVP calls, the FP32 partial attention and the merge validate on the host (no GPU: each of
    these returns before any CUDA call)."""
    lib = lsa.library()
    b = _batch(T=2, B=1)
    # lsa_merge_partials: sizes, alignment, the token limit
    assert lib.lsa_merge_partials(16, 16, 0, 2, 128, 512, 16, None, None) == lsa.ERR_INVALID_ARG     # no parts
    assert lib.lsa_merge_partials(16, 16, 2, 2, 128, 500, 16, None, None) == lsa.ERR_INVALID_ARG     # Dv % 8
    assert lib.lsa_merge_partials(None, 16, 2, 2, 128, 512, 16, None, None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_merge_partials(24, 16, 2, 2, 128, 512, 16, None, None) == lsa.ERR_INVALID_ARG     # unaligned
    assert lib.lsa_merge_partials(16, 16, 2, 70000, 128, 512, 16, None, None) == lsa.ERR_UNSUPPORTED
    assert lib.lsa_merge_partials(16, 16, 2, 0, 128, 512, 16, None, None) == lsa.OK                  # nothing to do
    # lsa_kvp_select: part counts, workspace
    need = lsa.kvp_select_workspace_size(2, 4, 100)
    assert need >= 2 * 4 * 100 * 8
    sel = lambda n_parts=4, k_part=100, ws=4096, wsb=need: lib.lsa_kvp_select(  # noqa
        ctypes.byref(b), 16, 16, n_parts, k_part, 100, 4, 16, 16, 200, 16, ws, wsb, None, None)
    assert sel(n_parts=0) == lsa.ERR_INVALID_ARG
    assert sel(k_part=0) == lsa.ERR_INVALID_ARG
    assert sel(ws=None) == lsa.ERR_WORKSPACE
    assert sel(wsb=need - 1) == lsa.ERR_WORKSPACE
    assert sel(ws=4100) == lsa.ERR_WORKSPACE                                               # not 256-byte aligned
    # lsa_kvp_local_index: the local list must be at least as wide as the global one
    assert lib.lsa_kvp_local_index(ctypes.byref(b), 16, 16, 16, 200, 16, 16, 199, 16, None, None) == lsa.ERR_INVALID_ARG
    # lsa_kvp_candidates: k >= 1, pointers
    assert lib.lsa_kvp_candidates(ctypes.byref(b), 16, 16, 16, 100, 100, 0, 16, 16, 16, None, None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_kvp_candidates(ctypes.byref(b), None, 16, 16, 100, 100, 8, 16, 16, 16, None, None) == lsa.ERR_INVALID_ARG
    # lsa_kvp_shard_batch
    assert lib.lsa_kvp_shard_batch(ctypes.byref(b), 0, 16, 16, 16, 16, None, None) == lsa.ERR_INVALID_ARG
    assert lib.lsa_kvp_shard_batch(ctypes.byref(b), 64, None, 16, 16, 16, None, None) == lsa.ERR_INVALID_ARG
    # lsa_sparse_attn_partial: both FP32 outputs are required; otherwise lsa_sparse_attn's checks
    kv = _cache(dtype=lsa.BF16, dim=576, scale=None)
    part = lambda o=4096, l=4096, H=128: lib.lsa_sparse_attn_partial(  # noqa
        ctypes.byref(b), 4096, H, 576, ctypes.byref(kv), None, 512, 16, 100, 16, 0.04, 1, o, l, None, 0, None, None)
    assert part(o=None) == lsa.ERR_INVALID_ARG
    assert part(l=None) == lsa.ERR_INVALID_ARG
    assert part(H=100) == lsa.ERR_UNSUPPORTED


def test_wait_limit_setter_and_index_capacity():
    assert lsa.set_wait_limit_ns(5) == 0                  # the default is 0 (2 s)
    assert lsa.set_wait_limit_ns(0) == 5
    p = lsa.CDecodeParams()
    p.k, p.n_sink, p.window = 2048, 4, 512
    lib = lsa.library()
    assert lib.lsa_decode_index_capacity(ctypes.byref(p)) == 2564
    p.si_window_aligned = 1
    assert lib.lsa_decode_index_capacity(ctypes.byref(p)) == 2564 + lsa.WINDOW_ALIGN - 1
    p.window = 0
    assert lib.lsa_decode_index_capacity(ctypes.byref(p)) == 2052
