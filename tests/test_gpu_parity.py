"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases span several 128-key tiles with ragged tails and cover every
layout pair, both sparse modes, bf16/fp16/fp8, head counts that need padding,
paged block sizes 16..1024 (also non-contiguous pools), padding rows and rows
with no visible key.  Exact-integer cases must match the oracle bit for bit
(indices, including lower-index tie-breaks, and values).  The named workloads
run at full size: completely where the oracle is fast enough, else on a
seeded row sample.
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_top_n1_b200 as li
import synth
from parity import check_against_oracle, check_all_rows, sample_rows, to_device

pytestmark = pytest.mark.gpu


def run_gpu(p, inputs):
    d = to_device(inputs)
    pr = li.make_params(p)
    ws = li.alloc_workspace(pr)
    idx, val = li.indexer(pr, d["query"], d["key"], d["weights"], act_seq_q=d.get("act_q"),
                          act_seq_k=d.get("act_k"), block_table=d.get("block_table"),
                          q_scale=d.get("q_scale"), k_scale=d.get("k_scale"),
                          cmp_residual_k=d.get("cmp_residual_k"), workspace=ws)
    assert li.li_last_launch_count() == 3
    flags = li.li_read_device_status(ws)
    torch.cuda.synchronize()
    gi = idx.cpu().numpy().reshape(p.rows, p.sparse_count)
    gv = val.cpu().numpy().reshape(p.rows, p.sparse_count) if p.return_value else None
    return gi, gv, flags


def small(seed, **kw):
    base = dict(B=2, S1=40, S2=300, N1=8, D=128, sparse_count=64, return_value=1)
    base.update(kw)
    return synth.make_random(seed, **base)


CASES = {
    "bsnd_mode0": dict(sparse_mode=0),
    "bsnd_mode3": dict(sparse_mode=3),
    "bsnd_mode3_full": dict(sparse_mode=3, ragged=False, S1=300),
    "bsnd_fp16_d64_n32": dict(dtype_qk="fp16", dtype_w="fp32", D=64, N1=32, sparse_mode=0),
    "bsnd_n64": dict(N1=64, S1=20, sparse_mode=3),
    "bsnd_n3_padded_heads": dict(N1=3, sparse_mode=3),
    "bsnd_n17_padded_heads": dict(N1=17, sparse_mode=0, dtype_w="fp16"),
    "bsnd_n1": dict(N1=1, sparse_mode=3, S1=70),
    "bsnd_k1": dict(sparse_count=1, sparse_mode=3),
    "bsnd_k_over_visible": dict(sparse_count=400, sparse_mode=3),
    "bsnd_empty_rows": dict(empty_rows=True, B=4, sparse_mode=3),
    "bsnd_q_longer_than_k": dict(S1=300, S2=100, ragged=False, sparse_mode=3),
    "tnd_mode3": dict(layout_q="TND", layout_k="TND", sparse_mode=3, B=3),
    "tnd_mode0": dict(layout_q="TND", layout_k="TND", sparse_mode=0, B=3),
    "pa16": dict(layout_k="PA_BSND", block_size=16, sparse_mode=3),
    "pa48": dict(layout_k="PA_BSND", block_size=48, sparse_mode=3),
    "pa64_strided": dict(layout_k="PA_BSND", block_size=64, key_block_pad=8, sparse_mode=3),
    "pa128": dict(layout_k="PA_BSND", block_size=128, sparse_mode=0, S2=700),
    "pa256": dict(layout_k="PA_BSND", block_size=256, sparse_mode=3, S2=700),
    "pa1024": dict(layout_k="PA_BSND", block_size=1024, sparse_mode=3, S2=1500),
    "tnd_q_pa_k": dict(layout_q="TND", layout_k="PA_BSND", block_size=32, sparse_mode=0),
    "decode_pa": dict(layout_k="PA_BSND", block_size=128, S1=1, ragged=False, sparse_mode=3,
                      N1=64, S2=1000, B=5),
    "quant_tnd": dict(layout_q="TND", layout_k="TND", quant=True, dtype_w="fp32", N1=64,
                      S1=60, S2=300, sparse_mode=3),
    "quant_pa": dict(layout_k="PA_BSND", quant=True, dtype_w="fp32", block_size=64, N1=64,
                     sparse_mode=3),
    "quant_bsnd_n8": dict(quant=True, dtype_w="fp32", sparse_mode=0),
    "int8_tnd_fp16": dict(layout_q="TND", layout_k="TND", quant=True, quant_dtype="int8",
                          dtype_scale="fp16", dtype_w="fp16", N1=64, S1=60, S2=300, sparse_mode=3),
    "int8_pa_fp32": dict(layout_k="PA_BSND", quant=True, quant_dtype="int8", dtype_w="fp32",
                         block_size=32, N1=64, sparse_mode=3),
    "int8_bsnd_n5": dict(quant=True, quant_dtype="int8", dtype_scale="fp16", dtype_w="bf16",
                         N1=5, sparse_mode=0),
    "sink_local_bsnd": dict(sparse_mode=3, init_num=4, local_num=8),
    "sink_only_tnd": dict(layout_q="TND", layout_k="TND", sparse_mode=3, init_num=16),
    "local_only_pa": dict(layout_k="PA_BSND", block_size=64, sparse_mode=0, local_num=32),
    "sink_local_fill_k": dict(sparse_mode=3, sparse_count=16, init_num=6, local_num=10),
    "sink_local_long_rows": dict(sparse_mode=0, S1=3, S2=20000, ragged=False, sparse_count=256,
                                 init_num=5, local_num=7),
    "cmp4_bsnd": dict(sparse_mode=3, cmp_ratio=4),
    "cmp2_tnd_q_pa_k": dict(layout_q="TND", layout_k="PA_BSND", block_size=32, sparse_mode=3,
                            cmp_ratio=2),
    "cmp128_bsnd_n64": dict(sparse_mode=3, cmp_ratio=128, N1=64, S1=40, S2=300),
    "cmp8_mode0": dict(sparse_mode=0, cmp_ratio=8),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_small_case_parity(name):
    p, inp = small(zlib.crc32(name.encode()) % 1000, **CASES[name])
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


@pytest.mark.parametrize("name", ["bsnd_mode3", "bsnd_fp16_d64_n32", "tnd_mode3", "pa48",
                                  "bsnd_n3_padded_heads", "quant_tnd", "quant_pa", "decode_pa",
                                  "int8_tnd_fp16", "int8_pa_fp32", "sink_local_bsnd", "cmp4_bsnd"])
def test_exact_integer_parity(name):
    """Small-integer inputs: every product and sum is exact in fp32, so the GPU
    must reproduce the oracle exactly, ties broken toward the lower index."""
    p, inp = small(500 + len(name), **CASES[name])
    g = torch.Generator().manual_seed(7)
    inp = dict(inp)
    for key in ("query", "key", "weights"):
        t = inp[key]
        inp[key] = torch.randint(-3, 4, t.shape, generator=g).to(torch.float32).to(t.dtype)
    if p.quant:
        for key in ("q_scale", "k_scale"):
            e = torch.randint(-2, 3, inp[key].shape, generator=g).to(torch.float32)
            inp[key] = torch.pow(2.0, e).to(inp[key].dtype)
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    o = oracle.run(p, inp)
    np.testing.assert_array_equal(gi, o["idx"])
    np.testing.assert_array_equal(gv, o["val"])


def test_v2_compressed_example_full():
    """The CANN V2 guide's call example: 130 original key tokens compressed
    4:1 into 32 keys with 2 residual tokens, right-down causal over them."""
    p, inp = synth.make_v2_compressed()
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


def test_dsa_prefill_window_workload_all_rows():
    p, inp = synth.make_dsa_prefill_window()
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_all_rows(p, inp, gi, gv)


def test_quant_int8_readme_example_full():
    """The VllmQuantLightningIndexer README's A3 call: int8 q/k over the full
    int8 range (|q.k| up to 2^21), fp16 scales and weights, PA keys."""
    p, inp = synth.make_quant_int8_pa()
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


def test_quant_int8_varlen_all_rows():
    p, inp = synth.make_quant_varlen_int8(return_value=1)
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_all_rows(p, inp, gi, gv)


def test_tiny_workload():
    p, inp = synth.make_tiny()
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


def test_cfg2_workload_full():
    p, inp = synth.make_cfg2()
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


def test_dsa_prefill_workload_all_rows():
    p, inp = synth.make_dsa_prefill()
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_all_rows(p, inp, gi, gv)


def test_paged_decode_workload_full():
    p, inp = synth.make_paged_decode(return_value=1)
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


def test_quant_varlen_workload_all_rows():
    p, inp = synth.make_quant_varlen(return_value=1)
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_all_rows(p, inp, gi, gv)


# ------------------------------------------------------------------ Top-k stage alone

def _topk_reference(rows_np, lens, k):
    R = rows_np.shape[0]
    idx = np.full((R, k), -1, dtype=np.int32)
    val = np.full((R, k), -np.inf, dtype=np.float32)
    for r in range(R):
        n = lens[r]
        v = rows_np[r, :n]
        order = np.lexsort((np.arange(n), -v.astype(np.float64)))[:k]
        idx[r, :len(order)] = order
        val[r, :len(order)] = v[order]
    return idx, val


@pytest.mark.parametrize("ld,k,kind", [(4096, 1024, "normal"), (300, 64, "quarters"),
                                       (8192, 2048, "quarters"), (40000, 2048, "normal"),
                                       (40000, 512, "quarters"), (64, 100, "normal"),
                                       (4096, 1024, "levels"), (16384, 2048, "levels"),
                                       (2048, 2048, "levels"), (5000, 700, "constant"),
                                       (65536, 2048, "levels"), (70000, 1, "normal"),
                                       (140000, 2048, "normal"), (20000, 2048, "constant"),
                                       (16384, 8192, "normal"), (12000, 4096, "levels"),
                                       (9000, 8192, "quarters"), (65536, 8192, "normal"),
                                       (40000, 4096, "levels"), (140000, 8192, "normal"),
                                       (30000, 8192, "constant")])
def test_topk_stage_exact(ld, k, kind):
    """Exact against a lexsort reference.  'quarters' (values on a 0.25 grid,
    every 7th -0.0) and 'constant' rows force the radix fallback; 'levels'
    (~7 keys per distinct value) keeps the bucket path with ties inside and
    at the threshold bucket.  Rows longer than 16384 keys run on a cluster of
    CTAs (bucket path, radix fallback, and beyond 131072 keys the streamed
    radix path)."""
    g = torch.Generator().manual_seed(ld + k)
    R = 12
    x = torch.randn(R, ld, generator=g)
    if kind == "quarters":                           # many exact ties, +0 and -0
        x = torch.round(x * 4) / 4
        x[:, ::7] = -0.0
    elif kind == "levels":
        x = torch.randint(0, max(ld // 7, 1), (R, ld), generator=g).to(torch.float32) / 7.0 - 3.0
    elif kind == "constant":
        x = torch.full((R, ld), 1.5)
    lens = torch.randint(1, ld + 1, (R,), generator=g).to(torch.int32)
    lens[0] = ld
    lens[1] = min(k, ld)
    d = x.cuda()
    idx = torch.empty(R, k, dtype=torch.int32, device="cuda")
    val = torch.empty(R, k, dtype=torch.float32, device="cuda")
    li.li_topk(d, ld, lens.cuda(), R, k, idx, val)
    torch.cuda.synchronize()
    ri, rv = _topk_reference(x.numpy(), lens.numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ri)
    np.testing.assert_array_equal(val.cpu().numpy(), rv)


# ------------------------------------------------------------------ device status word

def test_device_flag_bad_cmp_residual():
    """A residual outside [0, cmp_ratio) is clamped and flagged, not trusted."""
    p, inp = small(9, sparse_mode=3, cmp_ratio=4)
    inp = dict(inp)
    inp["cmp_residual_k"] = torch.tensor([5, 1], dtype=torch.int32)
    _, _, flags = run_gpu(p, inp)
    assert flags & li.DEV_BAD_KLEN


def test_device_flags_bad_lengths_and_blocks():
    p, inp = small(3, layout_k="PA_BSND", block_size=64, sparse_mode=3)
    inp = dict(inp)
    bt = inp["block_table"].clone()
    bt[0, 0] = p.num_blocks + 5                      # outside the pool: skipped, flagged
    inp["block_table"] = bt
    _, _, flags = run_gpu(p, inp)
    assert flags & li.DEV_BAD_BLOCK
    p2, inp2 = small(4, sparse_mode=3)
    inp2 = dict(inp2)
    ak = inp2["act_k"].clone()
    ak[1] = p2.S2 + 10                               # longer than the key tensor: clamped
    inp2["act_k"] = ak
    _, _, flags = run_gpu(p2, inp2)
    assert flags & li.DEV_BAD_KLEN


def test_device_flags_negative_scale():
    p, inp = small(5, layout_q="TND", layout_k="TND", quant=True, dtype_w="fp32",
                   sparse_mode=3)
    inp = dict(inp)
    ks = inp["k_scale"].clone()
    ks[3] = -1.0
    inp["k_scale"] = ks
    _, _, flags = run_gpu(p, inp)
    assert flags & li.DEV_NEG_SCALE


def test_bounded_wait_expires_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    li.li_selftest_bounded_wait(status, 5_000_000)    # 5 ms, nothing ever arrives
    torch.cuda.synchronize()
    assert int(status.item()) & li.DEV_TIMEOUT
    # the context is still usable afterwards
    p, inp = synth.make_tiny()
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


def test_repeat_calls_are_deterministic():
    p, inp = small(9, sparse_mode=3, N1=64, S1=64, S2=700)
    a = run_gpu(p, inp)
    b = run_gpu(p, inp)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# ------------------------------------------------------------------ sparse_count above 2048

@pytest.mark.parametrize("k", [4096, 8192])
def test_large_sparse_count_decode_rows(k):
    """sparse_count up to 8192 (CANN guide, "约束说明"): decode-length paged
    rows of 16 k to 65 k keys, every row against the oracle."""
    p, inp = synth.make_paged_decode(seed=40 + k, B=6, lo=16384, hi=65536, return_value=1)
    p.sparse_count = k
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv)


@pytest.mark.parametrize("k", [4096, 8192])
def test_large_sparse_count_causal_prefill(k):
    """Right-down causal prefill with k of 4096 and 8192: rows shorter than k
    are sorted whole, longer ones selected; sampled rows of both kinds."""
    p, inp = synth.make_dsa_prefill(seed=41 + k, S=12288, return_value=1)
    p.sparse_count = k
    gi, gv, flags = run_gpu(p, inp)
    assert flags == 0
    check_against_oracle(p, inp, gi, gv, rows=sample_rows(p, n_random=48, edge=8, seed=k))
