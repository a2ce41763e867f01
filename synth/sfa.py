"""Seeded synthetic inputs for the sparse attention consumer.

The consumer of the indexer's output attends, for every query row, over the
keys and values its selected indices name (the CANN TileLang LightningIndexer
guide, section "LightningIndexer 在稀疏注意力中的地位": the index tensor names
the key/value subset of every query token; the open-sourcing issue lists the
forward output as the input of Sparse FlashAttention).  This module only draws
and lays out tensors -- no dot product, softmax or weighting happens here.

The index rows follow the structure of the indexer's own output: under
right-down causal masking a row sees ``nvis`` keys; when ``nvis <= K`` all of
them are selected (in random order), otherwise K distinct ones drawn uniformly;
the remaining slots hold -1.  A fraction of rows can also get -1 holes inside
the row and out-of-range entries (``junk``), which the consumer must skip.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

from . import DTYPES, _gen


@dataclasses.dataclass
class SfaProblem:
    """Static description of one sparse attention call."""

    layout_q: str = "BSND"          # BSND | TND
    layout_kv: str = "BSND"         # BSND | TND | PA_BSND
    dtype: str = "bf16"             # bf16 | fp16 (query, key, value, output)
    B: int = 1
    S1: int = 0
    S2: int = 0
    T1: int = 0
    T2: int = 0
    N1: int = 64
    D: int = 128
    Dv: int = 128
    num_blocks: int = 0
    block_size: int = 0
    max_blocks_per_seq: int = 0
    sparse_count: int = 2048
    softmax_scale: float = 0.0      # 0 = 1/sqrt(D)

    @property
    def rows(self) -> int:
        return self.B * self.S1 if self.layout_q == "BSND" else self.T1

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else self.D ** -0.5


def _index_rows(g, Sq: int, Sk: int, K: int, causal: bool, holes: float, junk: float):
    """[Sq, K] int32 index rows of one batch (see the module docstring)."""
    rows = torch.full((Sq, K), -1, dtype=torch.int32)
    for i in range(Sq):
        nvis = min(Sk, max(0, i + 1 + Sk - Sq)) if causal else Sk
        if nvis <= 0:
            continue
        if nvis <= K:
            sel = torch.randperm(nvis, generator=g)
        else:
            sel = torch.randperm(nvis, generator=g)[:K]
        rows[i, :sel.numel()] = sel.to(torch.int32)
        if holes > 0 and torch.rand((), generator=g) < holes:
            # move a few valid entries behind -1 holes inside the row
            pos = torch.randperm(K, generator=g)[: max(1, K // 8)]
            rows[i] = rows[i][torch.argsort(torch.rand(K, generator=g))]
            rows[i, pos[: max(1, pos.numel() // 2)]] = -1
        if junk > 0 and torch.rand((), generator=g) < junk:
            j = int(torch.randint(0, K, (1,), generator=g))
            rows[i, j] = Sk + int(torch.randint(0, 7, (1,), generator=g))   # beyond the keys
    return rows


def make_sfa(seed: int, *, layout_q: str = "BSND", layout_kv: str = "BSND", dtype: str = "bf16",
             B: int = 1, S1: int = 64, S2: int = 256, q_lens: Optional[Sequence[int]] = None,
             k_lens: Optional[Sequence[int]] = None, N1: int = 64, D: int = 128, Dv: int = 128,
             K: int = 128, block_size: int = 64, causal: bool = True, holes: float = 0.0,
             junk: float = 0.0, softmax_scale: float = 0.0):
    """A random sparse attention problem.

    Draw order: q, k, v, index rows (batch by batch), PA block permutation.
    ``q_lens``/``k_lens`` give ragged per-batch lengths (TND prefix sums are
    built from them; BSND uses them as actual lengths inside S1/S2).
    """
    g = _gen(seed)
    q_lens = list(q_lens) if q_lens is not None else [S1] * B
    k_lens = list(k_lens) if k_lens is not None else [S2] * B
    assert len(q_lens) == B and len(k_lens) == B
    p = SfaProblem(layout_q=layout_q, layout_kv=layout_kv, dtype=dtype, B=B, N1=N1, D=D, Dv=Dv,
                   sparse_count=K, softmax_scale=softmax_scale)
    inputs = {}
    if layout_q == "BSND":
        p.S1 = S1
        qshape = (B, S1, N1, D)
        if q_lens != [S1] * B:
            inputs["act_q"] = torch.tensor(q_lens, dtype=torch.int32)
    else:
        p.T1 = sum(q_lens)
        qshape = (p.T1, N1, D)
        inputs["act_q"] = torch.tensor(q_lens, dtype=torch.int64).cumsum(0).to(torch.int32)
    if layout_kv == "BSND":
        p.S2 = S2
        kshape, vshape = (B, S2, 1, D), (B, S2, 1, Dv)
        if k_lens != [S2] * B:
            inputs["act_k"] = torch.tensor(k_lens, dtype=torch.int32)
    elif layout_kv == "TND":
        p.T2 = sum(k_lens)
        kshape, vshape = (p.T2, 1, D), (p.T2, 1, Dv)
        inputs["act_k"] = torch.tensor(k_lens, dtype=torch.int64).cumsum(0).to(torch.int32)
    else:
        p.block_size = block_size
        nblk = [(L + block_size - 1) // block_size for L in k_lens]
        p.num_blocks = sum(nblk)
        p.max_blocks_per_seq = max(1, max(nblk))
        kshape = (p.num_blocks, block_size, 1, D)
        vshape = (p.num_blocks, block_size, 1, Dv)
        inputs["act_k"] = torch.tensor(k_lens, dtype=torch.int32)
    dt = DTYPES[dtype]
    inputs["query"] = torch.randn(*qshape, generator=g, dtype=torch.float32).to(dt)
    inputs["key"] = torch.randn(*kshape, generator=g, dtype=torch.float32).to(dt)
    inputs["value"] = torch.randn(*vshape, generator=g, dtype=torch.float32).to(dt)
    idx_rows = []
    for b in range(B):
        Sq_alloc = S1 if layout_q == "BSND" else q_lens[b]
        r = _index_rows(g, q_lens[b], k_lens[b], K, causal, holes, junk)
        if Sq_alloc > q_lens[b]:                       # BSND padding rows: all -1
            r = torch.cat([r, torch.full((Sq_alloc - q_lens[b], K), -1, dtype=torch.int32)])
        idx_rows.append(r)
    inputs["sparse_indices"] = torch.cat(idx_rows).reshape(p.rows, 1, K).contiguous()
    if layout_kv == "PA_BSND":
        perm = torch.randperm(p.num_blocks, generator=g)
        table = torch.full((B, p.max_blocks_per_seq), -1, dtype=torch.int32)
        off = 0
        for b in range(B):
            n = (k_lens[b] + block_size - 1) // block_size
            table[b, :n] = perm[off:off + n].to(torch.int32)
            off += n
        inputs["block_table"] = table
    return p, inputs


def make_sfa_prefill(seed: int = 9, S: int = 8192, N1: int = 64, K: int = 2048):
    """The consumer of the DSA prefill workload: S query rows of N1 heads over
    the same causal key range, K selected keys per row, D = Dv = 128, bf16."""
    return make_sfa(seed, B=1, S1=S, S2=S, N1=N1, K=K)


def make_sfa_decode(seed: int = 10, B: int = 64, lo: int = 4096, hi: int = 65536, N1: int = 64,
                    K: int = 2048, block_size: int = 128):
    """The consumer of the paged decode workload: one query token per batch
    over a PA_BSND key/value pool, K selected keys, D = Dv = 128, bf16."""
    g = _gen(seed)
    lens = torch.randint(lo, hi + 1, (B,), generator=g).tolist()
    return make_sfa(seed, layout_kv="PA_BSND", B=B, S1=1, S2=max(lens), q_lens=[1] * B,
                    k_lens=lens, N1=N1, K=K, block_size=block_size)
