"""Seeded synthetic inputs for the LightningIndexer workloads.

This module only draws and lays out input tensors; it holds none of the
indexer's arithmetic (no dot products, no ReLU, no weighting, no Top-k).
Both the fp64 oracle and the CUDA path consume what it returns, so it is the
one piece of code they share.

Every tensor is drawn on the CPU with ``torch.Generator().manual_seed(seed)``
in fp32 and then cast to its storage dtype.  The shapes follow the workloads
named by the pages:

* ``tiny``         -- a small bf16 BSND case (8 heads, 256 keys, k=64, mask 0).
* ``cfg2``         -- the TileLang test shape (CANN TileLang LightningIndexer
                      guide, section "调用示例与精度验证"): B=2, S1=512,
                      S2=4096, G=32, D=64, k=1024, fp16 q/k, fp32 weights.
* ``dsa_prefill``  -- DeepSeek-style prefill: S1=S2=8192, N1=64, D=128,
                      k=2048, right-down causal, values returned.
* ``paged_decode`` -- 64 single-token queries over PA_BSND keys (block 128)
                      with ragged lengths in [4096, 65536] and a block table
                      that is a random permutation of the physical pool.
* ``quant_varlen`` -- TND fp8-e4m3 q/k with per-token-head absmax scales
                      (VllmQuantLightningIndexer README, "功能说明"), 4
                      sequences of 2048/4096/8192/16384 tokens.
* ``quant_varlen_int8`` -- the same sequences with int8 q/k and fp16 scales
                      and weights (the README's A2/A3 dtypes, "参数说明").
* ``quant_int8_pa`` -- the README's A3 call example ("Atlas A3 推理系列产品调用
                      说明"): B=24, S1=4, S2=512, PA_BSND block 128, int8 q/k
                      uniform over the int8 range, fp16 scales U[0, 10], fp16
                      weights U[0, 0.01], k=512, mask 0.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

DTYPES = {
    "bf16": torch.bfloat16,
    "fp16": torch.float16,
    "fp32": torch.float32,
    "e4m3": torch.float8_e4m3fn,
    "int8": torch.int8,
}
E4M3_MAX = 448.0
INT8_MAX = 127.0
INT64_MAX = (1 << 63) - 1


@dataclasses.dataclass
class Problem:
    """Static description of one indexer call (the op attributes + dims)."""

    layout_q: str = "BSND"          # BSND | TND
    layout_k: str = "BSND"          # BSND | TND | PA_BSND
    dtype_qk: str = "bf16"          # bf16 | fp16 | e4m3 | int8
    dtype_w: str = "bf16"           # bf16 | fp16 | fp32
    dtype_scale: str = "fp32"       # fp32 | fp16 (quant only)
    quant: bool = False
    B: int = 1
    S1: int = 0                     # BSND query length (max)
    S2: int = 0                     # BSND key length (max)
    T1: int = 0                     # TND total query tokens
    T2: int = 0                     # TND total key tokens
    N1: int = 1
    N2: int = 1
    D: int = 128
    num_blocks: int = 0             # PA pool blocks
    block_size: int = 0             # PA block size
    max_blocks_per_seq: int = 0     # PA block_table second dim
    key_block_stride: int = 0       # PA elements between consecutive blocks (0 = dense)
    sparse_count: int = 2048
    sparse_mode: int = 3
    return_value: int = 0
    pre_tokens: int = INT64_MAX
    next_tokens: int = INT64_MAX
    max_seqlen_k: int = 0           # host-side bound on any key length (0 = derive)
    init_num: int = 0               # sink tokens always selected (first visible keys)
    local_num: int = 0              # local window always selected (last visible keys)
    cmp_ratio: int = 1              # original tokens per (compressed) key

    @property
    def rows(self) -> int:
        """Number of query rows (one output row of k slots per row)."""
        return self.B * self.S1 if self.layout_q == "BSND" else self.T1


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def _normal(g, shape, dtype: str) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(DTYPES[dtype])


def quantize_e4m3_per_row(x: torch.Tensor):
    """Per-(token, head) absmax quantisation to fp8 e4m3 (input recipe).

    scale = absmax(x[..., :]) / 448 (1 where the absmax is 0); the stored code
    is torch's round-to-nearest-even cast of x / scale.  Returns (codes, scale).
    """
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (x / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes, scale.to(torch.float32)


# --------------------------------------------------------------------------
# The named workloads
# --------------------------------------------------------------------------

def quantize_int8_per_row(x: torch.Tensor):
    """Per-(token, head) absmax quantisation to int8 (input recipe).

    scale = absmax(x[..., :]) / 127 (1 where the absmax is 0); the stored code
    is round-half-to-even of x / scale, clamped to [-127, 127].  Returns
    (codes, scale) with fp32 scales.
    """
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / INT8_MAX, torch.ones_like(amax))
    codes = torch.round(x / scale.unsqueeze(-1)).clamp(-INT8_MAX, INT8_MAX).to(torch.int8)
    return codes, scale.to(torch.float32)


QUANTIZERS = {"e4m3": quantize_e4m3_per_row, "int8": quantize_int8_per_row}


def make_tiny(seed: int = 0):
    p = Problem(layout_q="BSND", layout_k="BSND", dtype_qk="bf16", dtype_w="bf16",
                B=1, S1=32, S2=256, N1=8, N2=1, D=128, sparse_count=64,
                sparse_mode=0, return_value=1)
    g = _gen(seed)
    q = _normal(g, (1, 32, 8, 128), "bf16")
    k = _normal(g, (1, 256, 1, 128), "bf16")
    w = _normal(g, (1, 32, 8), "bf16")
    return p, dict(query=q, key=k, weights=w)


def make_cfg2(seed: int = 1, return_value: int = 1):
    """TileLang test shape: q [B,S1,N2*G,D] fp16, weights [B,S1,N2,G] fp32."""
    B, S1, S2, G, D = 2, 512, 4096, 32, 64
    p = Problem(layout_q="BSND", layout_k="BSND", dtype_qk="fp16", dtype_w="fp32",
                B=B, S1=S1, S2=S2, N1=G, N2=1, D=D, sparse_count=1024,
                sparse_mode=0, return_value=return_value)
    g = _gen(seed)
    q = _normal(g, (B, S1, G, D), "fp16")
    k = _normal(g, (B, S2, 1, D), "fp16")
    w = _normal(g, (B, S1, 1, G), "fp32").reshape(B, S1, G)
    return p, dict(query=q, key=k, weights=w)


def make_dsa_prefill(seed: int = 2, S: int = 8192, return_value: int = 1):
    N1, D = 64, 128
    p = Problem(layout_q="BSND", layout_k="BSND", dtype_qk="bf16", dtype_w="bf16",
                B=1, S1=S, S2=S, N1=N1, N2=1, D=D, sparse_count=2048,
                sparse_mode=3, return_value=return_value)
    g = _gen(seed)
    q = _normal(g, (1, S, N1, D), "bf16")
    k = _normal(g, (1, S, 1, D), "bf16")
    w = _normal(g, (1, S, N1), "bf16")
    return p, dict(query=q, key=k, weights=w)


def make_paged_decode(seed: int = 3, B: int = 64, lo: int = 4096, hi: int = 65536,
                      block_size: int = 128, max_blocks_per_seq: int = 512,
                      return_value: int = 0, sparse_count: int = 2048):
    """PA_BSND decode: key pool holds exactly the blocks the lengths need.

    Draw order: q, w, lengths, key pool, block permutation.  Unused table
    entries are -1 so that a stray read of them is visible.
    """
    N1, D = 64, 128
    g = _gen(seed)
    q = _normal(g, (B, 1, N1, D), "bf16")
    w = _normal(g, (B, 1, N1), "bf16")
    lens = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64)
    nblk = (lens + block_size - 1) // block_size
    assert int(nblk.max()) <= max_blocks_per_seq
    pool = int(nblk.sum())
    key = _normal(g, (pool, block_size, 1, D), "bf16")
    perm = torch.randperm(pool, generator=g)
    table = torch.full((B, max_blocks_per_seq), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        n = int(nblk[b])
        table[b, :n] = perm[off:off + n].to(torch.int32)
        off += n
    p = Problem(layout_q="BSND", layout_k="PA_BSND", dtype_qk="bf16", dtype_w="bf16",
                B=B, S1=1, S2=0, N1=N1, N2=1, D=D, num_blocks=pool,
                block_size=block_size, max_blocks_per_seq=max_blocks_per_seq,
                sparse_count=sparse_count, sparse_mode=3, return_value=return_value,
                max_seqlen_k=int(lens.max()))
    return p, dict(query=q, key=key, weights=w, act_k=lens.to(torch.int32), block_table=table)


def make_quant_varlen(seed: int = 4, lens=(2048, 4096, 8192, 16384), return_value: int = 0,
                      sparse_count: int = 2048, qdtype: str = "e4m3", dtype_scale: str = "fp32",
                      dtype_w: str = "fp32"):
    """TND 8-bit q/k (fp8 e4m3 or int8) with per-token-head dequant scales."""
    N1, D = 64, 128
    T = int(sum(lens))
    g = _gen(seed)
    xq = torch.randn(T, N1, D, generator=g, dtype=torch.float32)
    xk = torch.randn(T, 1, D, generator=g, dtype=torch.float32)
    w = torch.randn(T, N1, generator=g, dtype=torch.float32).to(DTYPES[dtype_w])
    q, qs = QUANTIZERS[qdtype](xq)
    k, ks = QUANTIZERS[qdtype](xk)
    qs, ks = qs.to(DTYPES[dtype_scale]), ks.to(DTYPES[dtype_scale])
    cum = torch.tensor(lens, dtype=torch.int64).cumsum(0).to(torch.int32)
    p = Problem(layout_q="TND", layout_k="TND", dtype_qk=qdtype, dtype_w=dtype_w,
                dtype_scale=dtype_scale, quant=True, B=len(lens), T1=T, T2=T, N1=N1, N2=1,
                D=D, sparse_count=sparse_count, sparse_mode=3, return_value=return_value,
                max_seqlen_k=int(max(lens)))
    return p, dict(query=q, key=k, weights=w, q_scale=qs, k_scale=ks,
                   act_q=cum.clone(), act_k=cum.clone())


def make_dsa_prefill_window(seed: int = 7, return_value: int = 1, init_num: int = 16,
                            local_num: int = 512):
    """dsa_prefill with sink tokens and a local window (values not from the
    pages, which name the attributes only): the first 16 and the last 512
    visible keys of every row are always selected."""
    p, inp = make_dsa_prefill(seed=seed, return_value=return_value)
    p.init_num = init_num
    p.local_num = local_num
    return p, inp


def make_v2_compressed(seed: int = 8, return_value: int = 1):
    """The CANN LightningIndexerV2 guide's call example (section 调用示例):
    B=2, S1=64, S2=130 original key tokens compressed by cmp_ratio=4 into
    32 keys with 2 residual tokens per batch, N1=16, D=128, topk=32,
    mask_mode 3, fp16 q/k, fp32 weights, all N(0,1)."""
    B, S1, S2, r, N1, D = 2, 64, 130, 4, 16, 128
    g = _gen(seed)
    q = _normal(g, (B, S1, N1, D), "fp16")
    k = _normal(g, (B, S2 // r, 1, D), "fp16")
    w = torch.randn(B, S1, N1, generator=g, dtype=torch.float32)
    p = Problem(layout_q="BSND", layout_k="BSND", dtype_qk="fp16", dtype_w="fp32",
                B=B, S1=S1, S2=S2 // r, N1=N1, N2=1, D=D, sparse_count=32, sparse_mode=3,
                return_value=return_value, cmp_ratio=r)
    return p, dict(query=q, key=k, weights=w,
                   cmp_residual_k=torch.full((B,), S2 % r, dtype=torch.int32))


def make_quant_varlen_int8(seed: int = 6, return_value: int = 0):
    """quant_varlen with int8 q/k, fp16 scales and fp16 weights."""
    return make_quant_varlen(seed=seed, return_value=return_value, qdtype="int8",
                             dtype_scale="fp16", dtype_w="fp16")


def make_quant_int8_pa(seed: int = 5, B: int = 24, S1: int = 4, S2: int = 512,
                       block_size: int = 128, sparse_count: int = 512, sparse_mode: int = 0,
                       return_value: int = 1):
    """The README's A3 example call: int8 q/k over the int8 range, fp16 scales
    in [0, 10), fp16 weights in [0, 0.01), PA_BSND keys whose block table maps
    logical block j of batch b to physical block b*max_blocks + j.

    Draw order: key, key scales, query, query scales, weights.
    """
    N1, D = 64, 128
    g = _gen(seed)
    mb = (S2 + block_size - 1) // block_size
    table = torch.arange(B * mb, dtype=torch.int32).reshape(B, mb)
    key = torch.randint(-128, 128, (B * mb, block_size, 1, D), generator=g, dtype=torch.int64).to(torch.int8)
    ks = (torch.rand(B * mb, block_size, 1, generator=g) * 10).to(torch.float16)
    q = torch.randint(-128, 128, (B, S1, N1, D), generator=g, dtype=torch.int64).to(torch.int8)
    qs = (torch.rand(B, S1, N1, generator=g) * 10).to(torch.float16)
    w = (torch.rand(B, S1, N1, generator=g) * 0.01).to(torch.float16)
    p = Problem(layout_q="BSND", layout_k="PA_BSND", dtype_qk="int8", dtype_w="fp16",
                dtype_scale="fp16", quant=True, B=B, S1=S1, S2=0, N1=N1, N2=1, D=D,
                num_blocks=B * mb, block_size=block_size, max_blocks_per_seq=mb,
                sparse_count=sparse_count, sparse_mode=sparse_mode, return_value=return_value,
                max_seqlen_k=S2)
    lens = torch.full((B,), S2, dtype=torch.int32)
    return p, dict(query=q, key=key, weights=w, q_scale=qs, k_scale=ks, act_q=torch.full((B,), S1, dtype=torch.int32),
                   act_k=lens, block_table=table)


WORKLOADS = {
    "tiny": make_tiny,
    "cfg2": make_cfg2,
    "dsa_prefill": make_dsa_prefill,
    "paged_decode": make_paged_decode,
    "quant_varlen": make_quant_varlen,
    "quant_varlen_int8": make_quant_varlen_int8,
    "quant_int8_pa": make_quant_int8_pa,
    "dsa_prefill_window": make_dsa_prefill_window,
    "v2_compressed": make_v2_compressed,
}


# --------------------------------------------------------------------------
# Small randomised cases for parity sweeps
# --------------------------------------------------------------------------

def make_random(seed: int, *, layout_q="BSND", layout_k="BSND", dtype_qk="bf16",
                dtype_w="bf16", B=2, S1=40, S2=300, N1=8, D=128, sparse_count=64,
                sparse_mode=3, return_value=1, ragged=True, block_size=64,
                quant=False, empty_rows=False, key_block_pad=0, quant_dtype="e4m3",
                dtype_scale="fp32", init_num=0, local_num=0, cmp_ratio=1):
    """A random problem of the given layout; lengths are ragged when asked.

    BSND: actual lengths in [1, S] (or S when not ragged).  TND: per-sequence
    lengths drawn in [1, S1] / [1, S2] and passed as prefix sums.  PA_BSND:
    keys live in a shuffled block pool; ``key_block_pad`` extra rows between
    blocks make the pool non-contiguous along axis 0.
    """
    g = _gen(seed)
    N2 = 1
    qdt = dtype_qk
    if layout_q == "BSND":
        if ragged:
            lq = torch.randint(0 if empty_rows else 1, S1 + 1, (B,), generator=g)
        else:
            lq = torch.full((B,), S1, dtype=torch.int64)
    else:
        lq = torch.randint(0 if empty_rows else 1, S1 + 1, (B,), generator=g)
    if ragged or layout_k == "PA_BSND":
        lk = torch.randint(1, S2 + 1, (B,), generator=g)
    else:
        lk = torch.full((B,), S2, dtype=torch.int64)
    if layout_k == "TND" and layout_q == "TND" and sparse_mode == 3 and not ragged:
        lk = lq.clone()

    inputs: Dict[str, Optional[torch.Tensor]] = {}
    p = Problem(layout_q=layout_q, layout_k=layout_k, dtype_qk=qdt, dtype_w=dtype_w,
                quant=quant, B=B, N1=N1, N2=N2, D=D, sparse_count=sparse_count,
                sparse_mode=sparse_mode, return_value=return_value, init_num=init_num,
                local_num=local_num, cmp_ratio=cmp_ratio)
    if cmp_ratio > 1 and sparse_mode == 3:
        # leftover original tokens per batch, each below cmp_ratio
        inputs["cmp_residual_k"] = torch.randint(0, cmp_ratio, (B,), generator=g).to(torch.int32)
    # query
    if layout_q == "BSND":
        p.S1 = S1
        qshape = (B, S1, N1, D)
        wshape = (B, S1, N1)
        if ragged:
            inputs["act_q"] = lq.to(torch.int32)
    else:
        if int(lq.sum()) == 0:
            lq[0] = 1
        p.T1 = int(lq.sum())
        qshape = (p.T1, N1, D)
        wshape = (p.T1, N1)
        inputs["act_q"] = lq.cumsum(0).to(torch.int32)
    xq = torch.randn(*qshape, generator=g, dtype=torch.float32)
    # key
    if layout_k == "BSND":
        p.S2 = S2
        kshape = (B, S2, N2, D)
        if ragged:
            inputs["act_k"] = lk.to(torch.int32)
    elif layout_k == "TND":
        p.T2 = int(lk.sum())
        kshape = (p.T2, N2, D)
        inputs["act_k"] = lk.cumsum(0).to(torch.int32)
    else:
        nblk = (lk + block_size - 1) // block_size
        pool = int(nblk.sum()) + 1          # one spare block nobody maps
        p.num_blocks = pool
        p.block_size = block_size
        p.max_blocks_per_seq = int(nblk.max()) + 1
        p.max_seqlen_k = int(lk.max())
        kshape = (pool, block_size + key_block_pad, N2, D)
        inputs["act_k"] = lk.to(torch.int32)
    xk = torch.randn(*kshape, generator=g, dtype=torch.float32)
    w = torch.randn(*wshape, generator=g, dtype=torch.float32).to(DTYPES[dtype_w])
    if layout_k == "PA_BSND":
        perm = torch.randperm(p.num_blocks, generator=g)
        table = torch.full((B, p.max_blocks_per_seq), -1, dtype=torch.int32)
        off = 0
        for b in range(B):
            n = int(nblk[b])
            table[b, :n] = perm[off:off + n].to(torch.int32)
            off += n
        inputs["block_table"] = table
        if key_block_pad:
            p.key_block_stride = (block_size + key_block_pad) * N2 * D
    if quant:
        q, qs = QUANTIZERS[quant_dtype](xq)
        k, ks = QUANTIZERS[quant_dtype](xk)
        inputs["q_scale"] = qs.to(DTYPES[dtype_scale])
        if layout_k == "PA_BSND":
            ks = ks[:, :block_size].contiguous()      # [blocks, block_size, N2]
        inputs["k_scale"] = ks.to(DTYPES[dtype_scale])
        p.dtype_qk = quant_dtype
        p.dtype_scale = dtype_scale
    else:
        q = xq.to(DTYPES[qdt])
        k = xk.to(DTYPES[qdt])
    inputs["query"] = q
    inputs["key"] = k
    inputs["weights"] = w
    return p, inputs
