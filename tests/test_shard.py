"""Row sharding of one problem over ranks (sparse_attention_top_n1_b200.shard).

Each rank computes a contiguous range of output rows with rewritten actual
lengths that keep every row's causal diagonal; the key is replicated and no
data crosses ranks.  The check is against the fp64 oracle: the oracle run on
every rank's pieces, concatenated in row order, must equal the oracle run on
the whole problem bit for bit (indices and values), across BSND, TND and
paged keys, both sparse modes, compressed keys and sink/window rows.  One
test does this with two real gloo processes, the others in one process for
1 to 7 ranks.
"""
from __future__ import annotations

import dataclasses
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth
from sparse_attention_top_n1_b200 import shard

CASES = {
    "bsnd_mode3": dict(layout_q="BSND", layout_k="BSND", B=3, S1=37, S2=90, sparse_mode=3),
    "bsnd_mode0": dict(layout_q="BSND", layout_k="BSND", B=3, S1=37, S2=90, sparse_mode=0),
    "bsnd_q_longer": dict(layout_q="BSND", layout_k="BSND", B=2, S1=60, S2=30, sparse_mode=3,
                          ragged=False),
    "tnd_mode3": dict(layout_q="TND", layout_k="TND", B=4, S1=40, S2=70, sparse_mode=3),
    "tnd_mode0": dict(layout_q="TND", layout_k="TND", B=4, S1=40, S2=70, sparse_mode=0),
    "pa_mode3": dict(layout_q="BSND", layout_k="PA_BSND", B=5, S1=7, S2=300, sparse_mode=3,
                     block_size=32),
    "pa_decode": dict(layout_q="BSND", layout_k="PA_BSND", B=9, S1=1, S2=400, sparse_mode=3,
                      block_size=16),
    "tnd_pa_mode3": dict(layout_q="TND", layout_k="PA_BSND", B=3, S1=30, S2=200, sparse_mode=3,
                         block_size=64),
    "bsnd_cmp4": dict(layout_q="BSND", layout_k="BSND", B=2, S1=50, S2=40, sparse_mode=3,
                      cmp_ratio=4),
    "tnd_cmp8": dict(layout_q="TND", layout_k="TND", B=3, S1=60, S2=20, sparse_mode=3, cmp_ratio=8),
    "bsnd_window": dict(layout_q="BSND", layout_k="BSND", B=2, S1=45, S2=80, sparse_mode=3,
                        init_num=3, local_num=5),
    "tnd_quant": dict(layout_q="TND", layout_k="TND", B=3, S1=40, S2=60, sparse_mode=3, quant=True),
}


def make_case(name, seed=0):
    kw = dict(CASES[name])
    kw.setdefault("N1", 4)
    kw.setdefault("D", 16)
    kw.setdefault("sparse_count", 12)
    return synth.make_random(seed, **kw)


def run_pieces(p, inp, pieces):
    """The oracle on every piece (its own problem and views of the inputs)."""
    outs = []
    for pc in pieces:
        sub_p = dataclasses.replace(p, **pc.fields)
        sub = shard.piece_inputs(pc, p, inp)
        r = oracle.run(sub_p, sub, nthreads=1)
        assert r["idx"].shape[0] == pc.r1 - pc.r0
        outs.append((pc.r0, r["idx"], r["val"]))
    return outs


def assemble(p, parts):
    idx = np.full((p.rows, p.sparse_count), 12345, dtype=np.int32)
    val = np.full((p.rows, p.sparse_count), 7.0, dtype=np.float32)
    seen = np.zeros(p.rows, dtype=np.int64)
    for r0, i, v in parts:
        idx[r0:r0 + i.shape[0]] = i
        val[r0:r0 + v.shape[0]] = v
        seen[r0:r0 + i.shape[0]] += 1
    return idx, val, seen


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("world", [1, 2, 3, 7])
def test_shards_reassemble_the_whole_problem(name, world):
    p, inp = make_case(name, seed=world)
    full = oracle.run(p, inp, nthreads=1)
    per_rank = shard.shard(p, world, inp.get("act_q"), inp.get("act_k"), inp.get("cmp_residual_k"))
    assert len(per_rank) == world
    parts = [x for pieces in per_rank for x in run_pieces(p, inp, pieces)]
    idx, val, seen = assemble(p, parts)
    assert np.all(seen == 1), "every row is computed exactly once"
    np.testing.assert_array_equal(idx, full["idx"])
    np.testing.assert_array_equal(val.view(np.uint32), full["val"].view(np.uint32))


@pytest.mark.parametrize("name", ["bsnd_mode3", "tnd_mode3", "pa_decode"])
def test_every_row_range_reassembles(name):
    """Any cut, not only the balanced ones: every contiguous range [r0, r1)."""
    p, inp = make_case(name, seed=11)
    full = oracle.run(p, inp, nthreads=1)
    aq, ak, cr = inp.get("act_q"), inp.get("act_k"), inp.get("cmp_residual_k")
    R = p.rows
    step = max(1, R // 9)
    for r0 in range(0, R, step):
        for r1 in range(r0 + 1, R + 1, step):
            pieces = shard.pieces_for_range(p, r0, r1, aq, ak, cr)
            assert len(pieces) <= 3
            parts = run_pieces(p, inp, pieces)
            covered = sorted((a, a + i.shape[0]) for a, i, _ in parts)
            assert covered[0][0] == r0 and covered[-1][1] == r1
            for a, i, v in parts:
                np.testing.assert_array_equal(i, full["idx"][a:a + i.shape[0]])
                np.testing.assert_array_equal(v.view(np.uint32), full["val"][a:a + v.shape[0]].view(np.uint32))


def test_ranges_are_balanced_by_visible_pairs():
    p, inp = synth.make_dsa_prefill(S=2048)
    cost = shard.row_costs(p)
    # right-down causal with Sq = Sk: row i sees i + 1 keys
    np.testing.assert_array_equal(cost, np.arange(1, 2049))
    ranges = shard.split_rows(cost, 4)
    sums = [int(cost[a:b].sum()) + 64 * (b - a) for a, b in ranges]
    assert ranges[0][0] == 0 and ranges[-1][1] == 2048
    assert max(sums) - min(sums) <= 2 * (2048 + 64)
    # later rows see more keys, so the later ranges are shorter
    lens = [b - a for a, b in ranges]
    assert lens == sorted(lens, reverse=True)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, names, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        for name in names:
            p, inp = make_case(name, seed=5)
            pieces = shard.shard(p, world, inp.get("act_q"), inp.get("act_k"),
                                 inp.get("cmp_residual_k"))[rank]
            parts = run_pieces(p, inp, pieces)
            # every rank sends its rows to rank 0 (a test-side gather: the
            # indexer itself exchanges nothing)
            gathered = [None] * world
            dist.all_gather_object(gathered, parts)
            if rank == 0:
                full = oracle.run(p, inp, nthreads=1)
                idx, val, seen = assemble(p, [x for g in gathered for x in g])
                ok = (bool(np.all(seen == 1)) and np.array_equal(idx, full["idx"])
                      and np.array_equal(val.view(np.uint32), full["val"].view(np.uint32)))
                q.put((name, ok, [len(g) for g in gathered]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_one_problem():
    names = ["bsnd_mode3", "bsnd_mode0", "tnd_mode3", "pa_mode3", "pa_decode", "tnd_cmp8"]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, names, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = [q.get(timeout=180) for _ in names]
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    for name, ok, npieces in res:
        assert ok, name
        assert all(n >= 1 for n in npieces), name
