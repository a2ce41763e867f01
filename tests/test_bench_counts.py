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
    pairs, flops, gathered, compulsory = bench.sfa_counts(p, x)
    idx = x["sparse_indices"].reshape(p.rows, p.sparse_count)
    assert pairs == int((idx >= 0).sum())
    assert flops == 2.0 * p.N1 * (p.D + p.Dv) * pairs
    assert gathered == pairs * (p.D + p.Dv) * 2
    # distinct selected keys per batch, counted directly
    distinct = 0
    for b, (lo, hi) in enumerate([(0, 10), (10, 20)]):
        keys = set()
        for r in range(lo, hi):
            keys |= {int(j) for j in idx[r] if j >= 0}
        distinct += len(keys)
    io = p.rows * p.N1 * (p.D + p.Dv) * 2 + idx.numel() * 4 + p.rows * p.N1 * 4
    assert compulsory == io + distinct * (p.D + p.Dv) * 2


def test_job_value_is_the_problems_rows_over_the_slowest_time():
    assert bench.job_value(1024, 20, 2.0) == 1024 * 20 / 2e-3


def test_roofline_takes_the_slower_bound():
    # paged decode shape: 64 FLOP per byte is below the ridge point, so HBM bounds it
    r = bench.roofline(0.2, 3.65e10, 5.72e8, 1673.8, "t", 6446.3, "h")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - (5.72e8 / 6446.3e9) / 0.2e-3) < 1e-12
    assert abs(r["achieved"] - 5.72e8 / 0.2e-3 / 1e9) < 1e-9
    # DSA prefill shape: tensor-bound
    r = bench.roofline(0.7, 5.5e11, 2.7e8, 1673.8, "t", 6446.3, "h")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - (5.5e11 / 1673.8e12) / 0.7e-3) < 1e-12


def test_8bit_peak_falls_back_only_when_the_measurement_is_missing_or_low():
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0}
    v, src = bench.tensor_peak("e4m3", peaks, "m", {"fp8_tflops": 3100.0, "how": "x"})
    assert v == 3100.0 and "measured in this run" in src
    v, src = bench.tensor_peak("int8", peaks, "m", {"int8_tops": 200.0, "how": "x"})
    assert v == 3200.0 and src.startswith("assumed")
    v, src = bench.tensor_peak("bf16", peaks, "m", None)
    assert v == 1600.0


def test_default_workload_is_the_largest_configuration():
    sizes = {}
    for name in bench.CONFIGS:
        p, x = bench.make_workload(name)
        sizes[name] = bench.work_counts(p, x)["flops"]
    assert max(sizes, key=sizes.get) == bench.DEFAULT_WORKLOAD == "quant_varlen"


def test_end_to_end_pieces_tile_the_rows():
    """The overlapped end-to-end leg splits a problem into contiguous row
    pieces (the multi-GPU row split); they must cover every row once."""
    import numpy as np

    from sparse_attention_top_n1_b200 import shard
    for name, want in (("cfg2", 1), ("dsa_prefill", 2), ("quant_varlen", 7), ("paged_decode", 1)):
        p, inp = bench.make_workload(name)
        n = bench.e2e_pieces(p)
        assert n == want, name
        aq, ak, cr = inp.get("act_q"), inp.get("act_k"), inp.get("cmp_residual_k")
        cost = shard.row_costs(p, aq, ak, cr)
        seen = np.zeros(p.rows, dtype=np.int64)
        for r0, r1 in shard.split_rows(cost, n):
            for pc in shard.pieces_for_range(p, r0, r1, aq, ak, cr):
                seen[pc.r0:pc.r1] += 1
        assert np.all(seen == 1), name
