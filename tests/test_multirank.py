"""The N > 1 path of bench.py, on CPU with the gloo backend (world size 2).

Under torchrun the indexer problem is split by query rows (each rank a
contiguous, pair-balanced range; the split itself is checked against the
oracle in test_shard.py), the job time is the max over ranks and rank 0
reports the problem's rows over that time.  The sparse attention workloads
run one independent problem per rank.  These tests run two real processes to
check the reduction, the per-rank row ranges and the reference arm's rank
handling.
"""
from __future__ import annotations

import argparse
import datetime
import os
import socket

import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    own_ms = [3.0, 7.5][rank]
    mx = bench.allreduce_max(own_ms, device="cpu")
    bench.barrier()
    from sparse_attention_top_n1_b200 import shard
    p, inp = bench.make_workload("dsa_prefill")
    pieces = shard.shard(p, world, inp.get("act_q"), inp.get("act_k"))[rank]
    q.put((rank, mx, p.rows, [(pc.r0, pc.r1) for pc in pieces]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_split_one_problem():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    (r0, mx0, rows0, s0), (r1, mx1, rows1, s1) = out
    assert mx0 == mx1 == 7.5                 # the slowest rank's time
    assert rows0 == rows1 == 8192            # one problem, seen by both
    # the two ranks' ranges tile the rows; the causal triangle puts more rows on rank 0
    spans = sorted(s0 + s1)
    assert spans[0][0] == 0 and spans[-1][1] == 8192
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    assert s0[-1][1] > 4096
    # whole-job value: the problem's rows over the slowest rank's time
    assert abs(bench.job_value(rows0, 10, 7.5) - rows0 * 10 / 7.5e-3) < 1e-6


def test_reference_arm_other_ranks_exit_without_work(capsys):
    args = argparse.Namespace(workload="tiny", steps=1, warmup=3)
    assert bench.run_reference(args, 2, 1) == 0
    assert capsys.readouterr().out == ""


def test_single_process_reduction_is_identity():
    assert bench.allreduce_max(4.25, device="cpu") == 4.25
    assert not torch.distributed.is_initialized()


def test_sfa_reference_arm_other_ranks_exit_without_work(capsys):
    args = argparse.Namespace(workload="sfa_decode", steps=1, warmup=3)
    assert bench.sfa_reference(args, 1) == 0
    assert capsys.readouterr().out == ""


def test_sfa_ranks_draw_independent_problems():
    p0, x0 = bench.sfa_workload("sfa_decode", 0)
    p1, x1 = bench.sfa_workload("sfa_decode", 1)
    assert p0.N1 == p1.N1 and p0.sparse_count == p1.sparse_count and p0.rows == p1.rows
    assert not torch.equal(x0["query"], x1["query"])
