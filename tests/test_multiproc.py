"""Multi-rank host logic of the benchmark, on CPU: two processes over gloo.

On N GPUs every rank runs its own batch of the workload (weak scaling, no collective on
the data path), timing is the maximum over ranks, and the reference arm runs on rank 0
only.  These checks need no GPU: the ranks exchange host values over gloo.
"""
import datetime
import os
import socket
from types import SimpleNamespace

import torch
import torch.multiprocessing as mp

import bench
from lsa_synth import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        w = bench.rank_workload(W.WORKLOADS["decode_cli_128k"], rank, world)
        ref = bench.run_reference(SimpleNamespace(workload="tiny_decode", steps=1, warmup=0), rank, world)
        dist.barrier()
        q.put((rank, slowest, w.seed, w.B, w.name, None if ref is None else ref["impl"]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=240) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    (r0, m0, s0, b0, n0, ref0), (r1, m1, s1, b1, n1, ref1) = got
    assert (r0, r1) == (0, 1)
    assert m0 == m1 == 2.5                          # every rank reports the slowest rank's time
    assert n0 == n1 == "decode_cli_128k" and b0 == b1 == W.WORKLOADS["decode_cli_128k"].B
    assert s0 != s1                                 # own batch per rank (weak scaling)
    assert ref0 == "reference" and ref1 is None     # the reference arm runs on rank 0 only


def test_single_rank_is_identity():
    w = W.WORKLOADS["decode_cli_128k"]
    assert bench.rank_workload(w, 0, 1) is w
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25


def test_traffic_records_follow_the_code_not_the_comments():
    """The committed DRAM-traffic ratios apply while the kernel's code is the one they were
    captured on: a comment edit keeps the digest, a code edit (one token) changes it."""
    src = b"// header\nint f(int x) {  /* block\n comment */ return x + 1; // tail\n}\n"
    assert bench.code_digest(src) == bench.code_digest(b"int f(int x) { return x + 1;\n}")
    assert bench.code_digest(src) == bench.code_digest(src.replace(b"// tail", b"// another note"))
    assert bench.code_digest(src) != bench.code_digest(src.replace(b"x + 1", b"x + 2"))
    assert bench.indexer_traffic("attention", 1.0) is None      # no record for that kernel
