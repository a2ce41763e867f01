"""Host-side checks of the benchmark's algorithmic work counts (no GPU).

The roofline fractions divide these counts by measured times, so they are
checked against independent counts: the oracle's per-row visible-key counts
for the indexer, a direct count of the valid index entries for the sparse
attention consumer, and the FLOP formulas (2*N1*D per visible pair for the
scores; 2*N1*(D + Dv) per selected key for the attention).
"""
from __future__ import annotations

import numpy as np
import torch

import bench
import oracle
import synth
from synth import sfa as ssfa


def test_indexer_pairs_match_the_oracle_visible_counts():
    for seed, kw in [(60, dict(layout_q="BSND", layout_k="BSND", sparse_mode=3)),
                     (61, dict(layout_q="TND", layout_k="TND", sparse_mode=3)),
                     (62, dict(layout_q="BSND", layout_k="PA_BSND", sparse_mode=0))]:
        p, x = synth.make_random(seed, B=3, S1=21, S2=150, N1=16, sparse_count=32, **kw)
        c = bench.work_counts(p, x)
        orc = oracle.run(p, x)
        assert c["pairs"] == int(orc["nvis"].sum())
        assert c["flops"] == 2.0 * p.N1 * p.D * c["pairs"]


def test_named_workload_pairs():
    p, x = bench.make_workload("cfg2")
    c = bench.work_counts(p, x)
    assert c["pairs"] == 2 * 512 * 4096                     # mode 0: every key
    assert c["flops"] == 2.0 * 32 * 64 * c["pairs"]
    p, x = synth.make_dsa_prefill(S=256)                    # the DSA recipe at a small S
    c = bench.work_counts(p, x)
    assert c["pairs"] == 256 * 257 // 2                     # right-down causal triangle


def test_sparse_attention_counts():
    p, x = ssfa.make_sfa(63, B=2, S1=10, S2=90, q_lens=[10, 6], N1=32, K=48, holes=0.3)
    pairs, flops, gathered, io = bench.sfa_counts(p, x)
    idx = x["sparse_indices"].reshape(p.rows, p.sparse_count)
    assert pairs == int((idx >= 0).sum())
    assert flops == 2.0 * p.N1 * (p.D + p.Dv) * pairs
    assert gathered == pairs * (p.D + p.Dv) * 2
    assert io == p.rows * p.N1 * (p.D + p.Dv) * 2 + idx.numel() * 4 + p.rows * p.N1 * 4


def test_job_value_is_whole_job_rows_over_slowest_time():
    assert bench.job_value(1024, 20, 1, 2.0) == 1024 * 20 / 2e-3
    assert bench.job_value(1024, 20, 4, 2.0) == 4 * 1024 * 20 / 2e-3
