"""Pins for the fp64 oracle: it is checked against things other than itself.

* exhaustive decoder checks against torch's own dtype conversions;
* an independent numpy brute force (the TileLang guide's golden recipe:
  einsum -> ReLU -> x weights -> sum over heads -> sorted Top-k) on
  small-integer inputs, where every sum is exact in fp64, so indices
  (including the lower-index tie-break) and values must agree exactly;
* a textbook reduction: one head, unit weight, positive inputs -> the score
  is a plain dot product and the result is torch.topk of an fp64 matmul;
* closed forms worked out by hand;
* invariants (monotone output, causal visibility, all-zero-ReLU rows, key
  permutation, padding, PA == BSND, TND == per-sequence BSND, quant with
  unit scales == plain path, power-of-two scale equivariance);
* planted mistakes: every mutation the oracle can be built with is caught
  by at least one of the checks above.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from brute import brute


# ---------------------------------------------------------------- helpers

def integerize(p, inputs, seed, lo=-3, hi=3, scale_pow2=False):
    """Replace q/k/w (and scales) by small integers (exact in every dtype)."""
    g = torch.Generator().manual_seed(seed)
    out = dict(inputs)
    for name in ("query", "key", "weights"):
        t = inputs[name]
        vals = torch.randint(lo, hi + 1, t.shape, generator=g).to(torch.float32)
        out[name] = vals.to(t.dtype)
    if p.quant:
        for name in ("q_scale", "k_scale"):
            t = inputs[name]
            if scale_pow2:
                e = torch.randint(-2, 3, t.shape, generator=g).to(torch.float32)
                out[name] = torch.pow(2.0, e).to(t.dtype)
            else:
                out[name] = torch.ones_like(t)
    return out


def assert_same(p, inputs, mutation=0):
    o = oracle.run(p, inputs, mutation=mutation)
    bi, bv = brute(p, inputs)
    np.testing.assert_array_equal(o["idx"], bi.astype(np.int32))
    np.testing.assert_array_equal(o["v64"], bv)


CASES = [
    dict(layout_q="BSND", layout_k="BSND", sparse_mode=0),
    dict(layout_q="BSND", layout_k="BSND", sparse_mode=3),
    dict(layout_q="BSND", layout_k="BSND", sparse_mode=3, ragged=False),
    dict(layout_q="TND", layout_k="TND", sparse_mode=3),
    dict(layout_q="TND", layout_k="TND", sparse_mode=0),
    dict(layout_q="BSND", layout_k="PA_BSND", sparse_mode=3, block_size=16),
    dict(layout_q="TND", layout_k="PA_BSND", sparse_mode=0, block_size=32),
    dict(layout_q="BSND", layout_k="PA_BSND", sparse_mode=3, block_size=16, key_block_pad=3),
    dict(layout_q="BSND", layout_k="BSND", sparse_mode=3, dtype_qk="fp16", dtype_w="fp32"),
    dict(layout_q="TND", layout_k="TND", sparse_mode=3, quant=True, dtype_w="fp32"),
    dict(layout_q="BSND", layout_k="PA_BSND", sparse_mode=3, quant=True, dtype_w="fp32",
         block_size=16),
    dict(layout_q="BSND", layout_k="BSND", sparse_mode=3, empty_rows=True),
    dict(layout_q="TND", layout_k="TND", sparse_mode=3, quant=True, quant_dtype="int8",
         dtype_scale="fp16", dtype_w="fp16"),
    dict(layout_q="BSND", layout_k="PA_BSND", sparse_mode=0, quant=True, quant_dtype="int8",
         dtype_w="fp32", block_size=16),
    dict(layout_q="BSND", layout_k="BSND", sparse_mode=3, init_num=2, local_num=3),
    dict(layout_q="TND", layout_k="PA_BSND", sparse_mode=0, block_size=16, init_num=4, local_num=1),
    dict(layout_q="BSND", layout_k="BSND", sparse_mode=3, cmp_ratio=4),
    dict(layout_q="TND", layout_k="PA_BSND", sparse_mode=3, block_size=16, cmp_ratio=2),
]


def small(seed, **kw):
    base = dict(B=2, S1=9, S2=40, N1=3, D=8, sparse_count=12, return_value=1)
    base.update(kw)
    return synth.make_random(seed, **base)


# ---------------------------------------------------------------- decoders

def _codes16():
    return torch.arange(65536, dtype=torch.int32).to(torch.int16)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_decoder_16bit_exhaustive(dt):
    t = _codes16().view(dt)
    got = oracle.decode(t)
    ref = t.to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    np.testing.assert_array_equal(got[m], ref[m])


def test_decoder_e4m3_exhaustive():
    t = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    got = oracle.decode(t)
    ref = t.to(torch.float32).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    np.testing.assert_array_equal(got[m], ref[m])
    assert np.nanmax(got) == 448.0 and np.isnan(got[0x7F]) and np.isnan(got[0xFF])


def test_decoder_int8_exhaustive():
    t = torch.arange(-128, 128, dtype=torch.int32).to(torch.int8)
    np.testing.assert_array_equal(oracle.decode(t), np.arange(-128, 128, dtype=np.float64))


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("ci", range(len(CASES)))
@pytest.mark.parametrize("seed", [11, 12])
def test_brute_force_exact_integers(ci, seed):
    p, inp = small(seed, **CASES[ci])
    inp = integerize(p, inp, seed, scale_pow2=True)
    assert_same(p, inp)


@pytest.mark.parametrize("ci", [0, 1, 3, 5, 8, 9])
def test_brute_force_random_floats(ci):
    p, inp = small(100 + ci, **CASES[ci])
    o = oracle.run(p, inp)
    bi, bv = brute(p, inp)
    np.testing.assert_array_equal(o["idx"], bi.astype(np.int32))
    fin = np.isfinite(bv)
    np.testing.assert_array_equal(np.isfinite(o["v64"]), fin)
    np.testing.assert_allclose(o["v64"][fin], bv[fin], rtol=1e-12, atol=1e-12)


def test_tiny_workload_brute_force():
    p, inp = synth.make_tiny()
    o = oracle.run(p, inp)
    bi, bv = brute(p, inp)
    np.testing.assert_array_equal(o["idx"], bi.astype(np.int32))
    np.testing.assert_allclose(o["v64"], bv, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- textbook

def test_textbook_single_head_is_dot_product_topk():
    """N1=1, W=1, positive q/k: s(t) = q.k_t, so Top-k is torch.topk of a matmul."""
    g = torch.Generator().manual_seed(5)
    S1, S2, D, kk = 7, 300, 32, 50
    q = torch.rand(1, S1, 1, D, generator=g).to(torch.bfloat16)
    k = torch.rand(1, S2, 1, D, generator=g).to(torch.bfloat16)
    w = torch.ones(1, S1, 1, dtype=torch.bfloat16)
    p = synth.Problem(B=1, S1=S1, S2=S2, N1=1, D=D, sparse_count=kk, sparse_mode=0,
                      return_value=1)
    o = oracle.run(p, dict(query=q, key=k, weights=w))
    s = q[0, :, 0].double() @ k[0, :, 0].double().T          # [S1, S2]
    ref = torch.topk(s, kk, dim=1, largest=True, sorted=True)
    np.testing.assert_array_equal(o["idx"], ref.indices.numpy().astype(np.int32))
    np.testing.assert_allclose(o["v64"], ref.values.numpy(), rtol=1e-13)


# ---------------------------------------------------------------- closed forms

def test_hand_worked_example():
    """Two heads on orthogonal axes; every score is worked out by hand.

    q_0 = e_0, q_1 = e_1, W = (2, -1); key t = (a_t, b_t, 0, 0) so
    s(t) = 2 relu(a_t) - relu(b_t):
      t : a, b   -> s
      0 : 1, 0   ->  2
      1 : 3, 1   ->  5
      2 :-2, 0   ->  0
      3 : 2, 4   ->  0
      4 : 1,-5   ->  2
      5 : 0, 3   -> -3
    Sorted (score desc, index asc): 1(5), 0(2), 4(2), 2(0), 3(0), 5(-3).
    With mode 3 and Sq = 2, Sk = 6 the first query (i=0) sees t <= 4 and the
    second (i=1) sees every key.
    """
    q = torch.zeros(1, 2, 2, 4)
    q[0, :, 0, 0] = 1
    q[0, :, 1, 1] = 1
    ab = [(1, 0), (3, 1), (-2, 0), (2, 4), (1, -5), (0, 3)]
    k = torch.zeros(1, 6, 1, 4)
    for t, (a, b) in enumerate(ab):
        k[0, t, 0, 0] = a
        k[0, t, 0, 1] = b
    w = torch.tensor([[[2.0, -1.0], [2.0, -1.0]]])
    inp = dict(query=q.to(torch.bfloat16), key=k.to(torch.bfloat16), weights=w.to(torch.bfloat16))
    p = synth.Problem(B=1, S1=2, S2=6, N1=2, D=4, sparse_count=7, sparse_mode=3, return_value=1)
    o = oracle.run(p, inp)
    ninf = -np.inf
    np.testing.assert_array_equal(o["idx"][0], [1, 0, 4, 2, 3, -1, -1])
    np.testing.assert_array_equal(o["v64"][0], [5, 2, 2, 0, 0, ninf, ninf])
    np.testing.assert_array_equal(o["idx"][1], [1, 0, 4, 2, 3, 5, -1])
    np.testing.assert_array_equal(o["v64"][1], [5, 2, 2, 0, 0, -3, ninf])
    assert list(o["nvis"]) == [5, 6]
    # mode 0: both rows see all six keys
    p.sparse_mode = 0
    o = oracle.run(p, inp)
    np.testing.assert_array_equal(o["idx"][0], [1, 0, 4, 2, 3, 5, -1])


def test_quant_hand_worked_example():
    """Dequant before ReLU: s = W * relu(sq * sk * (q.k)); with sq*sk < 0 the
    raw dot product's sign flips before the ReLU (README formula order)."""
    q = torch.tensor([[[[1.0, 2.0]]]])          # [B=1,S1=1,N1=1,D=2]
    k = torch.tensor([[[[1.0, 1.0]]], [[[-1.0, 0.5]]], [[[2.0, -2.0]]]]).reshape(1, 3, 1, 2)
    w = torch.tensor([[[0.5]]])
    qs = torch.tensor([[[2.0]]])
    ks = torch.tensor([[[4.0], [1.0], [-1.0]]]).reshape(1, 3, 1)
    # dots: 3, 0, -2 ; scaled: 3*8 = 24, 0, -2*2*-1 = 4 ; s = 0.5*relu: 12, 0, 2
    p = synth.Problem(B=1, S1=1, S2=3, N1=1, D=2, sparse_count=3, sparse_mode=0,
                      return_value=1, quant=True, dtype_qk="e4m3", dtype_w="fp32",
                      dtype_scale="fp32")
    inp = dict(query=q.to(torch.float8_e4m3fn), key=k.to(torch.float8_e4m3fn), weights=w,
               q_scale=qs.reshape(1, 1, 1), k_scale=ks)
    o = oracle.run(p, inp)
    np.testing.assert_array_equal(o["idx"][0], [0, 2, 1])
    np.testing.assert_array_equal(o["v64"][0], [12.0, 2.0, 0.0])


# ---------------------------------------------------------------- invariants

def test_monotone_and_visible_and_padding():
    p, inp = small(7, layout_q="BSND", layout_k="BSND", sparse_mode=3, S1=20, S2=30,
                   sparse_count=25)
    o = oracle.run(p, inp)
    aq, ak = inp["act_q"], inp["act_k"]
    for r in range(p.rows):
        b, i = divmod(r, p.S1)
        Sq, Sk = int(aq[b]), int(ak[b])
        nv = 0 if i >= Sq else max(0, min(Sk, i + 1 + Sk - Sq))
        assert o["nvis"][r] == nv
        n = min(nv, p.sparse_count)
        v = o["v64"][r]
        assert np.all(np.diff(v[:n]) <= 0)
        assert np.all(o["idx"][r, n:] == -1) and np.all(np.isneginf(v[n:]))
        assert np.all(o["idx"][r, :n] >= 0) and np.all(o["idx"][r, :n] < nv)
        assert len(set(o["idx"][r, :n].tolist())) == n


def test_all_zero_relu_row_gives_first_k_indices():
    """Every q.k <= 0 (q >= 0, k <= 0): all scores are 0 and ties go to the
    lowest indices, so the output is 0..k-1 with value 0."""
    g = torch.Generator().manual_seed(3)
    q = torch.rand(1, 4, 4, 16, generator=g).to(torch.bfloat16)
    k = (-torch.rand(1, 50, 1, 16, generator=g)).to(torch.bfloat16)
    w = torch.randn(1, 4, 4, generator=g).to(torch.bfloat16)
    p = synth.Problem(B=1, S1=4, S2=50, N1=4, D=16, sparse_count=20, sparse_mode=0,
                      return_value=1)
    o = oracle.run(p, dict(query=q, key=k, weights=w))
    for r in range(4):
        np.testing.assert_array_equal(o["idx"][r], np.arange(20))
        np.testing.assert_array_equal(o["v64"][r], np.zeros(20))


def test_key_permutation_permutes_indices():
    p, inp = small(21, layout_q="BSND", layout_k="BSND", sparse_mode=0, ragged=False,
                   B=1, S2=64, sparse_count=20)
    o = oracle.run(p, inp)
    perm = torch.randperm(64, generator=torch.Generator().manual_seed(1))
    inv = torch.argsort(perm)
    inp2 = dict(inp)
    inp2["key"] = inp["key"][:, perm]
    o2 = oracle.run(p, inp2)
    # key j of the permuted problem is key perm[j] of the original; tied
    # scores may reorder (ties go to the lower index), so compare the values
    # everywhere and the indices where the value is unique in its row
    mapped = perm.numpy()[o2["idx"]]
    np.testing.assert_array_equal(o2["v64"], o["v64"])
    for r in range(p.rows):
        v = o["v64"][r]
        uniq = np.array([np.sum(v == x) == 1 for x in v])
        assert uniq.sum() > p.sparse_count // 2
        np.testing.assert_array_equal(mapped[r][uniq], o["idx"][r][uniq])
    del inv


def test_pa_equals_bsnd_on_same_logical_keys():
    p, inp = small(31, layout_q="BSND", layout_k="PA_BSND", sparse_mode=3, block_size=16)
    o = oracle.run(p, inp)
    # gather the logical key sequence of every batch into a BSND tensor
    ak = inp["act_k"]
    S2 = int(ak.max())
    kb = torch.zeros(p.B, S2, 1, p.D, dtype=inp["key"].dtype)
    for b in range(p.B):
        for t in range(int(ak[b])):
            kb[b, t] = inp["key"][int(inp["block_table"][b, t // 16]), t % 16]
    p2 = synth.Problem(**{**p.__dict__, "layout_k": "BSND", "S2": S2})
    inp2 = dict(query=inp["query"], key=kb, weights=inp["weights"], act_q=inp["act_q"],
                act_k=ak)
    o2 = oracle.run(p2, inp2)
    np.testing.assert_array_equal(o["idx"], o2["idx"])
    np.testing.assert_array_equal(o["v64"], o2["v64"])


def test_tnd_equals_per_sequence_bsnd():
    p, inp = small(41, layout_q="TND", layout_k="TND", sparse_mode=3)
    o = oracle.run(p, inp)
    cq, ck = inp["act_q"].tolist(), inp["act_k"].tolist()
    for b in range(p.B):
        q0 = cq[b - 1] if b else 0
        k0 = ck[b - 1] if b else 0
        Sq, Sk = cq[b] - q0, ck[b] - k0
        if Sq == 0:
            continue
        pb = synth.Problem(B=1, S1=Sq, S2=Sk, N1=p.N1, D=p.D, sparse_count=p.sparse_count,
                           sparse_mode=3, return_value=1, dtype_qk=p.dtype_qk, dtype_w=p.dtype_w)
        ib = dict(query=inp["query"][q0:q0 + Sq].unsqueeze(0), key=inp["key"][k0:k0 + Sk].unsqueeze(0),
                  weights=inp["weights"][q0:q0 + Sq].unsqueeze(0))
        ob = oracle.run(pb, ib)
        np.testing.assert_array_equal(o["idx"][q0:q0 + Sq], ob["idx"])
        np.testing.assert_array_equal(o["v64"][q0:q0 + Sq], ob["v64"])


def test_quant_unit_scales_equal_plain_path():
    p, inp = small(51, layout_q="TND", layout_k="TND", sparse_mode=3, quant=True, dtype_w="fp32")
    inp = dict(inp)
    inp["q_scale"] = torch.ones_like(inp["q_scale"])
    inp["k_scale"] = torch.ones_like(inp["k_scale"])
    o = oracle.run(p, inp)
    # every e4m3 value is exact in bf16 (3 < 7 fraction bits, |x| <= 448)
    p2 = synth.Problem(**{**p.__dict__, "quant": False, "dtype_qk": "bf16"})
    inp2 = dict(inp)
    inp2["query"] = inp["query"].to(torch.float32).to(torch.bfloat16)
    inp2["key"] = inp["key"].to(torch.float32).to(torch.bfloat16)
    o2 = oracle.run(p2, inp2)
    np.testing.assert_array_equal(o["idx"], o2["idx"])
    np.testing.assert_array_equal(o["v64"], o2["v64"])


def test_quant_int8_unit_scales_equal_plain_path():
    p, inp = small(52, layout_q="BSND", layout_k="PA_BSND", sparse_mode=3, quant=True,
                   quant_dtype="int8", dtype_scale="fp16", dtype_w="fp16", block_size=16)
    inp = dict(inp)
    inp["q_scale"] = torch.ones_like(inp["q_scale"])
    inp["k_scale"] = torch.ones_like(inp["k_scale"])
    o = oracle.run(p, inp)
    # every int8 value is an integer of magnitude <= 128, exact in bf16
    p2 = synth.Problem(**{**p.__dict__, "quant": False, "dtype_qk": "bf16"})
    inp2 = dict(inp)
    inp2["query"] = inp["query"].to(torch.float32).to(torch.bfloat16)
    inp2["key"] = inp["key"].to(torch.float32).to(torch.bfloat16)
    o2 = oracle.run(p2, inp2)
    np.testing.assert_array_equal(o["idx"], o2["idx"])
    np.testing.assert_array_equal(o["v64"], o2["v64"])


def test_int8_quantizer_round_trip():
    """The int8 input recipe: codes are round-half-even(x / (absmax/127)),
    so code * scale is within half a step of x and the row's absmax maps to
    +-127."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(50, 4, 16, generator=g)
    codes, scale = synth.quantize_int8_per_row(x)
    assert codes.dtype == torch.int8
    back = codes.to(torch.float32) * scale.unsqueeze(-1)
    assert torch.all((back - x).abs() <= 0.5 * scale.unsqueeze(-1) * (1 + 1e-6))
    assert torch.all(codes.abs().to(torch.int32).amax(-1) == 127)


def test_v2_compressed_example_visible_counts():
    """The CANN V2 guide's example: S2 = 130 original tokens, cmp_ratio = 4,
    so 32 compressed keys and 2 residual tokens; with S1 = 64 right-down
    causal queries, query i sees the compressed keys whose 4 tokens all lie at
    or before original position i + 130 - 64, i.e. floor((i + 67) / 4) of
    them (16 for the first query, all 32 for the last)."""
    p, inp = synth.make_v2_compressed()
    o = oracle.run(p, inp)
    expect = np.array([min(32, (i + 67) // 4) for i in range(64)] * 2)
    np.testing.assert_array_equal(o["nvis"], expect)
    assert expect[0] == 16 and expect[63] == 32
    # every row keeps min(32, visible) keys, all of them visible
    for r in range(p.rows):
        got = o["idx"][r]
        assert np.all(got[:min(32, expect[r])] < expect[r]) and np.all(got[expect[r]:] == -1)


def test_cmp_ratio_one_is_the_plain_mask():
    p, inp = small(91, layout_q="BSND", layout_k="BSND", sparse_mode=3)
    o = oracle.run(p, inp)
    p2 = synth.Problem(**{**p.__dict__, "cmp_ratio": 1})
    o2 = oracle.run(p2, dict(inp, cmp_residual_k=torch.zeros(p.B, dtype=torch.int32)))
    np.testing.assert_array_equal(o["idx"], o2["idx"])


def test_sink_and_local_hand_worked_example():
    """One head, unit weight, D=1: s(t) = relu(q*k_t).  Keys 0..7 score
    0,5,1,7,2,6,3,4 (q=1); with k=4, init_num=1, local_num=1 the sink key 0
    (score 0) and the local key 7 (score 4) are kept whatever their score, and
    the two best others (keys 3 and 5) fill the rest; order by score desc."""
    q = torch.ones(1, 1, 1, 1)
    k = torch.tensor([0.0, 5, 1, 7, 2, 6, 3, 4]).reshape(1, 8, 1, 1)
    w = torch.ones(1, 1, 1)
    p = synth.Problem(B=1, S1=1, S2=8, N1=1, D=1, sparse_count=4, sparse_mode=0,
                      return_value=1, dtype_qk="bf16", dtype_w="bf16", init_num=1, local_num=1)
    inp = dict(query=q.to(torch.bfloat16), key=k.to(torch.bfloat16), weights=w.to(torch.bfloat16))
    o = oracle.run(p, inp)
    np.testing.assert_array_equal(o["idx"][0], [3, 5, 7, 0])
    np.testing.assert_array_equal(o["v64"][0], [7.0, 6.0, 4.0, 0.0])
    p.local_num = 3                                  # keys 0, 5, 6, 7 forced: they fill k = 4
    o = oracle.run(p, inp)
    np.testing.assert_array_equal(o["idx"][0], [5, 7, 6, 0])


def test_sink_and_local_keys_always_kept():
    """Every row keeps its first init_num and last local_num visible keys,
    the output stays ordered, and the other kept keys beat every dropped one."""
    p, inp = small(81, layout_q="BSND", layout_k="BSND", sparse_mode=3, S1=30, S2=60,
                   sparse_count=10, init_num=3, local_num=4)
    o = oracle.run(p, inp, want_scores=True)
    for r in range(p.rows):
        nv = int(o["nvis"][r])
        got = [int(t) for t in o["idx"][r] if t >= 0]
        assert len(got) == min(nv, p.sparse_count)
        forced = set(range(min(3, nv))) | set(range(max(0, nv - 4), nv))
        assert forced <= set(got)
        v = o["v64"][r][:len(got)]
        assert np.all(np.diff(v) <= 0)
        others = [t for t in got if t not in forced]
        dropped = [t for t in range(nv) if t not in set(got)]
        if others and dropped:
            sc = o["scores"][r]
            assert min(sc[t] for t in others) >= max(sc[t] for t in dropped)


def test_quant_power_of_two_scale_equivariance():
    """Uniform positive scales c_q, c_k scale every score by c_q*c_k exactly."""
    p, inp = small(61, layout_q="TND", layout_k="TND", sparse_mode=0, quant=True, dtype_w="fp32")
    inp = dict(inp)
    inp["q_scale"] = torch.ones_like(inp["q_scale"])
    inp["k_scale"] = torch.ones_like(inp["k_scale"])
    o = oracle.run(p, inp)
    inp["q_scale"] = torch.full_like(inp["q_scale"], 4.0)
    inp["k_scale"] = torch.full_like(inp["k_scale"], 0.125)
    o2 = oracle.run(p, inp)
    np.testing.assert_array_equal(o["idx"], o2["idx"])
    np.testing.assert_array_equal(o2["v64"], o["v64"] * 0.5)


def test_decode_causal_equals_full():
    """A single-token query under right-down causal sees all of its keys."""
    p, inp = small(71, layout_q="BSND", layout_k="PA_BSND", sparse_mode=3, S1=1, ragged=False,
                   block_size=16)
    o3 = oracle.run(p, inp)
    p.sparse_mode = 0
    o0 = oracle.run(p, inp)
    np.testing.assert_array_equal(o3["idx"], o0["idx"])


def test_row_subset_matches_full_run():
    p, inp = small(81, layout_q="TND", layout_k="TND", sparse_mode=3)
    full = oracle.run(p, inp, want_scores=True)
    rows = [p.rows - 1, 0, 3]
    sub = oracle.run(p, inp, rows=rows, want_scores=True)
    np.testing.assert_array_equal(sub["idx"], full["idx"][rows])
    np.testing.assert_array_equal(sub["v64"], full["v64"][rows])
    # the returned score row agrees with the selected values
    for j, r in enumerate(rows):
        n = int(sub["nvis"][j])
        sel = sub["idx"][j][: min(n, p.sparse_count)]
        np.testing.assert_array_equal(sub["scores"][j][sel], sub["v64"][j][: len(sel)])


# ---------------------------------------------------------------- planted mistakes

def _pin_suite(mutation):
    """Run a cross-section of the pins against a (possibly mutated) oracle."""
    failures = 0
    for ci in (1, 3, 5, 9, 14, 16):
        p, inp = small(200 + ci, **CASES[ci])
        inp = integerize(p, inp, 200 + ci, scale_pow2=True)
        try:
            assert_same(p, inp, mutation=mutation)
        except AssertionError:
            failures += 1
    return failures


def test_unmutated_oracle_passes_pin_suite():
    assert _pin_suite(0) == 0


@pytest.mark.parametrize("mutation", [1, 2, 3, 4, 5, 6, 7])
def test_each_planted_mistake_is_caught(mutation):
    assert _pin_suite(mutation) > 0
