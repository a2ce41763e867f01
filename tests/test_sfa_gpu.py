"""GPU parity of the sparse attention consumer against the fp64 oracle.

Every case runs li_sparse_attention through the C ABI on seeded inputs and
compares each output element with oracle/sfa.py.  The bound follows from the
arithmetic: the logits accumulate exact 16-bit products in fp32; the softmax
weights enter the P.V product rounded to the input type (relative error
u = 2^-9 for bf16, 2^-12 for fp16, and the normaliser sums the same rounded
weights, so the result stays a convex combination whose weights are off by at
most 2u relative); the output is rounded once more (u relative).  Hence per
element |gpu - oracle| <= 2u * max|v| + 2u * |oracle| (+1e-6), and the
log-sum-exp is off by at most 2u plus the fp32 logit error.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.sfa as osfa
import sparse_attention_top_n1_b200 as li
from synth import sfa as ssfa

pytestmark = pytest.mark.gpu

U = {"bf16": 2.0 ** -9, "fp16": 2.0 ** -12}


def run_gpu(p, x, status=True):
    dev = torch.device("cuda", 0)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    pr = li.make_sfa_params(p)
    st = torch.zeros(1, dtype=torch.int32, device=dev) if status else None
    out, lse = li.sparse_attention(pr, d["query"], d["key"], d["value"], d["sparse_indices"],
                                   act_seq_q=d.get("act_q"), act_seq_k=d.get("act_k"),
                                   block_table=d.get("block_table"), status=st)
    assert li.li_last_launch_count() == (1 if p.rows else 0)
    torch.cuda.synchronize()
    return (out.float().cpu().numpy(), lse.cpu().numpy(),
            int(st.item()) if status else 0)


def check(p, x, rows=None, expect_flags=0, chunk=None):
    """GPU against oracle on `rows` (all when None), the oracle taken `chunk`
    rows at a time when given (bounded host memory at full size)."""
    out, lse, flags = run_gpu(p, x)
    assert flags == expect_flags, "device status 0x%x" % flags
    rows = list(range(p.rows)) if rows is None else list(rows)
    step = chunk or max(1, len(rows))
    for c0 in range(0, len(rows), step):
        part = rows[c0:c0 + step]
        compare(p, x, out[part], lse[part], osfa.run(p, x, rows=part))


def compare(p, x, out, lse, ref):
    u = U[p.dtype]
    vmax = float(x["value"].float().abs().max())
    err = np.abs(out - ref["out"])
    tol = 2 * u * vmax + 2 * u * np.abs(ref["out"]) + 1e-6
    bad = err > tol
    assert not bad.any(), "out: %d elements off, worst %.3g at %s (tol %.3g)" % (
        bad.sum(), err.max(), np.unravel_index(np.argmax(err - tol), err.shape), tol.flat[np.argmax(err - tol)])
    fin = np.isfinite(ref["lse"])
    assert np.array_equal(np.isfinite(lse), fin), "lse: -inf pattern differs"
    assert np.all(np.isneginf(lse[~fin]))
    lerr = np.abs(lse[fin] - ref["lse"][fin])
    assert lerr.size == 0 or lerr.max() <= 2 * u + 1e-4, "lse off by %.3g" % lerr.max()
    # empty rows are exact zeros
    assert np.all(out[~fin.any(axis=1)] == 0)


CASES = {
    # name: make_sfa kwargs
    "bsnd_bf16_n64_ragged": dict(seed=30, B=2, S1=40, S2=300, q_lens=[40, 25], k_lens=[300, 170], N1=64, K=128),
    "bsnd_bf16_n16_tail": dict(seed=31, B=1, S1=33, S2=250, N1=16, K=100, holes=0.3),
    "tnd_fp16_n32": dict(seed=32, layout_q="TND", layout_kv="TND", dtype="fp16", B=3, q_lens=[17, 0, 29],
                         k_lens=[90, 40, 260], N1=32, K=96),
    "pa_bf16_n128": dict(seed=33, layout_kv="PA_BSND", B=3, S1=8, q_lens=[8, 8, 5], k_lens=[500, 64, 333],
                         N1=128, K=200, block_size=64),
    "pa_fp16_n64_tnd_q": dict(seed=34, layout_q="TND", layout_kv="PA_BSND", dtype="fp16", B=2, q_lens=[3, 6],
                              k_lens=[1000, 129], N1=64, K=256, block_size=128),
    "k1": dict(seed=35, B=1, S1=20, S2=50, N1=64, K=1),
    "k64_noncausal_scale": dict(seed=36, B=2, S1=12, S2=80, N1=32, K=64, causal=False, softmax_scale=0.3),
    "big_scale": dict(seed=37, B=1, S1=16, S2=128, N1=16, K=64, causal=False, softmax_scale=4.0),
    # few rows: each row's keys are split over a cluster of 2, 4 or 8 CTAs
    "split2_bsnd": dict(seed=41, B=2, S1=3, S2=1500, N1=32, K=600, causal=False),
    "split4_pa_n128": dict(seed=42, layout_kv="PA_BSND", B=3, S1=2, k_lens=[1500, 2000, 900], N1=128,
                           K=1100, block_size=64),
    "split8_pa_decode": dict(seed=43, layout_kv="PA_BSND", B=4, S1=1, k_lens=[3000, 5000, 2500, 4100], N1=64,
                             K=2048, block_size=128, holes=0.1),
    "split8_n16_bsnd": dict(seed=44, B=2, S1=1, S2=3000, N1=16, K=2048, causal=False),
    "split4_tnd_pa_fp16": dict(seed=45, layout_q="TND", layout_kv="PA_BSND", dtype="fp16", B=3, q_lens=[1, 2, 1],
                               k_lens=[3000, 1500, 2200], N1=32, K=1200, block_size=32),
    "pa_block_not_pow2": dict(seed=46, layout_kv="PA_BSND", B=2, S1=3, k_lens=[700, 450], N1=64, K=300,
                              block_size=48),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_sfa_parity(name):
    kw = dict(CASES[name])
    p, x = ssfa.make_sfa(**kw)
    check(p, x)


def test_sfa_out_of_range_entries_are_skipped_and_flagged():
    p, x = ssfa.make_sfa(38, B=2, S1=24, S2=100, N1=64, K=64, junk=0.5)
    check(p, x, expect_flags=li.DEV_BAD_INDEX)


def test_sfa_bad_block_is_skipped_and_flagged():
    p, x = ssfa.make_sfa(39, layout_kv="PA_BSND", B=2, S1=4, k_lens=[200, 300], N1=16, K=64, block_size=64)
    bt = x["block_table"].clone()
    bt[1, 2] = 99                                          # beyond the pool
    x2 = dict(x)
    x2["block_table"] = bt
    out, lse, flags = run_gpu(p, x2)
    assert flags & li.DEV_BAD_BLOCK
    # batch 0 does not touch the bad block: its rows match the oracle on the good table
    ref = osfa.run(p, x, rows=list(range(4)))
    u = U[p.dtype]
    vmax = float(x["value"].float().abs().max())
    assert np.all(np.abs(out[:4] - ref["out"]) <= 2 * u * vmax + 2 * u * np.abs(ref["out"]) + 1e-6)


def test_sfa_all_empty_rows():
    p, x = ssfa.make_sfa(40, B=1, S1=8, S2=64, N1=64, K=128)
    x["sparse_indices"] = torch.full_like(x["sparse_indices"], -1)
    out, lse, flags = run_gpu(p, x)
    assert flags == 0
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_sfa_prefill_workload_all_rows():
    """The DSA prefill consumer at full size (8192 rows, K = 2048, 64 heads),
    every row against the oracle (512 rows at a time)."""
    p, x = ssfa.make_sfa_prefill()
    check(p, x, chunk=512)


def test_sfa_decode_workload_full():
    """The paged decode consumer at full size: 64 rows over a paged pool, K = 2048."""
    p, x = ssfa.make_sfa_decode()
    check(p, x)


def test_sfa_consumes_indexer_output():
    """The two-stage pipeline: the indexer's Top-k (GPU) feeds the attention
    (GPU); compared with the attention oracle on the oracle's own indices
    (the two index sets agree up to the Top-k tolerance band, so this test
    uses the oracle's indices for both sides)."""
    import oracle
    import synth
    p, x = synth.make_random(41, layout_q="BSND", layout_k="BSND", B=1, S1=48, S2=512, N1=64, D=128,
                             sparse_count=128, sparse_mode=3, ragged=False)
    orc = oracle.run(p, x)
    g = torch.Generator().manual_seed(41)
    value = torch.randn(1, 512, 1, 128, generator=g).to(torch.bfloat16)
    sp = ssfa.SfaProblem(layout_q="BSND", layout_kv="BSND", dtype="bf16", B=1, S1=48, S2=512, N1=64,
                         sparse_count=128)
    sx = dict(query=x["query"], key=x["key"], value=value,
              sparse_indices=torch.from_numpy(orc["idx"]).reshape(48, 1, 128).contiguous())
    check(sp, sx)
