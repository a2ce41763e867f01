"""Pins of the sparse attention oracle against what the mathematics fixes.

Each pin checks the fp64 oracle (oracle/sfa.py) against a fact that does not
come from the oracle itself: a closed form (one selected key returns its value
row; a zero query averages the values; huge logit gaps pick the argmax), a
library routine on a special case (torch's scaled_dot_product_attention when
every key is selected), or an invariance the definition implies (index order,
-1 and out-of-range entries, the key layout, folding a power-of-two scale into
the query).  The planted-mistake test shows that every mutation the oracle
can plant fails at least one pin.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle.sfa as osfa
from synth import sfa as ssfa

MUTATIONS = (1, 2, 3, 4, 5, 6)


def _set_row(inputs, r, entries):
    idx = inputs["sparse_indices"].clone()
    K = idx.shape[-1]
    row = torch.full((K,), -1, dtype=torch.int32)
    row[:len(entries)] = torch.tensor(entries, dtype=torch.int32)
    idx[r, 0] = row
    out = dict(inputs)
    out["sparse_indices"] = idx
    return out


def _dec(t):
    return t.to(torch.float64).numpy()


def pin_single_key(mut):
    p, x = ssfa.make_sfa(11, B=1, S1=8, S2=40, N1=16, K=8, causal=False)
    x = _set_row(x, 3, [17])
    r = osfa.run(p, x, rows=[3], mutation=mut)
    v = _dec(x["value"]).reshape(-1, p.Dv)[17]
    q = _dec(x["query"]).reshape(p.rows, p.N1, p.D)[3]
    k = _dec(x["key"]).reshape(-1, p.D)[17]
    ok = np.array_equal(r["out"][0], np.broadcast_to(v, (p.N1, p.Dv)))
    ok &= np.allclose(r["lse"][0], p.scale * (q @ k), rtol=1e-12, atol=1e-12)
    return bool(ok)


def pin_zero_query_mean(mut):
    p, x = ssfa.make_sfa(12, B=1, S1=4, S2=64, N1=16, K=16, causal=False)
    x["query"] = torch.zeros_like(x["query"])
    sel = [3, 9, 10, 33, 50, 61]
    x = _set_row(x, 2, sel)
    r = osfa.run(p, x, rows=[2], mutation=mut)
    v = _dec(x["value"]).reshape(-1, p.Dv)[sel].mean(axis=0)
    ok = np.allclose(r["out"][0], np.broadcast_to(v, (p.N1, p.Dv)), rtol=0, atol=1e-14)
    ok &= np.allclose(r["lse"][0], math.log(len(sel)), rtol=0, atol=1e-14)
    return bool(ok)


def pin_order_invariance(mut):
    p, x = ssfa.make_sfa(13, B=1, S1=4, S2=64, N1=16, K=16, causal=False)
    sel = [5, 1, 44, 23, 8, 60, 31]
    a = osfa.run(p, _set_row(x, 1, sel), rows=[1], mutation=mut)
    b = osfa.run(p, _set_row(x, 1, sel[::-1] + [-1, -1]), rows=[1], mutation=mut)
    return bool(np.allclose(a["out"], b["out"], rtol=1e-13, atol=1e-13)
                and np.allclose(a["lse"], b["lse"], rtol=1e-13, atol=1e-13))


def pin_library_sdpa(mut):
    """Every key selected: plain attention, as torch's library routine computes it."""
    S2 = 48
    p, x = ssfa.make_sfa(14, B=1, S1=6, S2=S2, N1=16, K=S2, causal=False)
    x["sparse_indices"] = torch.arange(S2, dtype=torch.int32).repeat(p.rows, 1, 1).contiguous()
    r = osfa.run(p, x, mutation=mut)
    q = x["query"].to(torch.float64).reshape(p.rows, p.N1, p.D).transpose(0, 1)   # [N1, S1, D]
    k = x["key"].to(torch.float64).reshape(1, S2, p.D).expand(p.N1, S2, p.D)
    v = x["value"].to(torch.float64).reshape(1, S2, p.Dv).expand(p.N1, S2, p.Dv)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=p.scale)
    ref = ref.transpose(0, 1).numpy()
    lref = torch.logsumexp(p.scale * q @ k.transpose(1, 2), dim=-1).transpose(0, 1).numpy()
    return bool(np.allclose(r["out"], ref, rtol=1e-10, atol=1e-12)
                and np.allclose(r["lse"], lref, rtol=1e-12, atol=1e-12))


def pin_huge_gap_argmax(mut):
    """Logit gaps of thousands: the softmax is one-hot on the best key (and must
    not overflow)."""
    p, x = ssfa.make_sfa(15, B=1, S1=2, S2=32, N1=16, K=8, causal=False, softmax_scale=2048.0)
    sel = [2, 7, 19, 30]
    x = _set_row(x, 0, sel)
    r = osfa.run(p, x, rows=[0], mutation=mut)
    q = _dec(x["query"]).reshape(p.rows, p.N1, p.D)[0]
    k = _dec(x["key"]).reshape(-1, p.D)[sel]
    v = _dec(x["value"]).reshape(-1, p.Dv)[sel]
    lg = 2048.0 * q @ k.T
    best = lg.argmax(axis=1)
    gap = np.sort(lg, axis=1)[:, -1] - np.sort(lg, axis=1)[:, -2]
    assert gap.min() > 750, "fixture: gaps must underflow exp"
    ok = np.all(np.isfinite(r["out"])) and np.allclose(r["out"][0], v[best], rtol=0, atol=1e-20)
    ok &= np.allclose(r["lse"][0], lg.max(axis=1), rtol=1e-12, atol=1e-9)
    return bool(ok)


def pin_skips_invalid(mut):
    p, x = ssfa.make_sfa(16, B=1, S1=4, S2=40, N1=16, K=12, causal=False)
    clean = osfa.run(p, _set_row(x, 2, [4, 11, 27]), rows=[2], mutation=mut)
    dirty = osfa.run(p, _set_row(x, 2, [-1, 4, 40, 11, -1, 43, 27, -1]), rows=[2], mutation=mut)
    return bool(np.allclose(clean["out"], dirty["out"], rtol=0, atol=0)
                and np.allclose(clean["lse"], dirty["lse"], rtol=0, atol=0))


def pin_layout_invariance(mut):
    """The same logical batches laid out as BSND, TND and a paged pool agree."""
    p, x = ssfa.make_sfa(17, B=2, S1=5, S2=24, N1=16, K=8)
    outs = [osfa.run(p, x, mutation=mut)]
    # TND: concatenate the batches
    pt = ssfa.SfaProblem(**{**p.__dict__, "layout_q": "TND", "layout_kv": "TND", "T1": 10, "T2": 48,
                            "S1": 0, "S2": 0})
    xt = dict(x)
    xt["query"] = x["query"].reshape(10, p.N1, p.D)
    xt["key"] = x["key"].reshape(48, 1, p.D)
    xt["value"] = x["value"].reshape(48, 1, p.Dv)
    xt["act_q"] = torch.tensor([5, 10], dtype=torch.int32)
    xt["act_k"] = torch.tensor([24, 48], dtype=torch.int32)
    outs.append(osfa.run(pt, xt, mutation=mut))
    # paged: blocks of 8 keys, batch b's block j at pool slot perm
    pp = ssfa.SfaProblem(**{**p.__dict__, "layout_kv": "PA_BSND", "block_size": 8, "num_blocks": 6,
                            "max_blocks_per_seq": 3})
    xp = dict(x)
    order = [4, 0, 5, 2, 3, 1]                         # pool slot of logical block (b*3 + j)
    kb = x["key"].reshape(6, 8, 1, p.D)
    vb = x["value"].reshape(6, 8, 1, p.Dv)
    pool_k = torch.empty_like(kb)
    pool_v = torch.empty_like(vb)
    for lb, slot in enumerate(order):
        pool_k[slot] = kb[lb]
        pool_v[slot] = vb[lb]
    xp["key"], xp["value"] = pool_k, pool_v
    xp["block_table"] = torch.tensor([order[:3], order[3:]], dtype=torch.int32)
    xp["act_k"] = torch.tensor([24, 24], dtype=torch.int32)
    outs.append(osfa.run(pp, xp, mutation=mut))
    return all(np.array_equal(outs[0]["out"], o["out"]) and np.array_equal(outs[0]["lse"], o["lse"])
               for o in outs[1:])


def pin_scale_fold(mut):
    """scale 1/4 applied by the op equals the query multiplied by 1/4 (exact in
    bf16) with scale 1."""
    p, x = ssfa.make_sfa(18, B=1, S1=4, S2=32, N1=16, K=8, causal=False, softmax_scale=0.25)
    a = osfa.run(p, x, mutation=mut)
    p1 = ssfa.SfaProblem(**{**p.__dict__, "softmax_scale": 1.0})
    x1 = dict(x)
    x1["query"] = (x["query"].to(torch.float32) * 0.25).to(x["query"].dtype)
    assert torch.equal(x1["query"].to(torch.float32), x["query"].to(torch.float32) * 0.25)
    b = osfa.run(p1, x1, mutation=mut)
    return bool(np.allclose(a["out"], b["out"], rtol=1e-13, atol=1e-13))


def pin_empty_rows(mut):
    p, x = ssfa.make_sfa(19, B=2, S1=6, S2=16, q_lens=[6, 3], N1=16, K=4, causal=False)
    x = _set_row(x, 1, [])
    r = osfa.run(p, x, mutation=mut)
    ok = np.all(r["out"][1] == 0) and np.all(np.isneginf(r["lse"][1]))
    ok &= np.all(r["out"][6 + 3:] == 0) and np.all(np.isneginf(r["lse"][6 + 3:]))   # padding rows
    return bool(ok)


def pin_split_merge(mut):
    """Attention over a key set equals the merge of attention over any split of
    it: with (out_s, lse_s) per part, LSE = logsumexp_s lse_s and
    out = sum_s exp(lse_s - LSE) * out_s (the rule split rows are merged by)."""
    p, x = ssfa.make_sfa(21, B=1, S1=3, S2=200, N1=16, K=96, causal=False)
    full = osfa.run(p, x, rows=[1], mutation=mut)
    row = x["sparse_indices"][1, 0].tolist()
    parts = [row[:17], row[17:60], row[60:]]
    outs, lses = [], []
    for part in parts:
        r = osfa.run(p, _set_row(x, 1, part), rows=[1], mutation=mut)
        outs.append(r["out"][0])
        lses.append(r["lse"][0])
    L = np.logaddexp.reduce(np.stack(lses), axis=0)                  # [N1]
    merged = sum(np.exp(l - L)[:, None] * o for l, o in zip(lses, outs))
    return bool(np.allclose(merged, full["out"][0], rtol=1e-12, atol=1e-12)
                and np.allclose(L, full["lse"][0], rtol=1e-12, atol=1e-12))


PINS = [pin_single_key, pin_zero_query_mean, pin_order_invariance, pin_library_sdpa,
        pin_huge_gap_argmax, pin_skips_invalid, pin_layout_invariance, pin_scale_fold,
        pin_empty_rows, pin_split_merge]


@pytest.mark.parametrize("pin", PINS, ids=[f.__name__ for f in PINS])
def test_sfa_oracle_pin(pin):
    assert pin(0)


@pytest.mark.parametrize("mut", MUTATIONS)
def test_sfa_planted_mistake_is_caught(mut):
    import warnings
    failed = []
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        with np.errstate(all="ignore"):
            for pin in PINS:
                try:
                    ok = pin(mut)
                except Exception:
                    ok = False
                if not ok:
                    failed.append(pin.__name__)
    assert failed, "mutation %d passes every pin" % mut


def test_sfa_synth_index_rows_are_valid():
    """The generator's rows: distinct entries, inside the causal range, -1 pad."""
    p, x = ssfa.make_sfa(20, B=2, S1=40, S2=100, q_lens=[40, 33], k_lens=[100, 70], N1=16, K=32)
    idx = x["sparse_indices"].reshape(p.rows, p.sparse_count)
    for b, (Sq, Sk) in enumerate([(40, 100), (33, 70)]):
        for i in range(40):
            row = idx[b * 40 + i]
            v = row[row >= 0]
            if i >= Sq:
                assert v.numel() == 0
                continue
            nvis = min(Sk, i + 1 + Sk - Sq)
            assert v.numel() == min(32, nvis)
            assert len(set(v.tolist())) == v.numel()
            assert int(v.max()) < nvis
