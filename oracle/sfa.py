"""fp64 CPU oracle of the sparse attention consumer (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this module; it shares nothing with the CUDA library.

What it computes (the CANN TileLang LightningIndexer guide, section
"LightningIndexer 在稀疏注意力中的地位": attention whose key/value set for
each query token is the one its index row names, so its cost is O(N*S)
instead of O(N^2)).  The pages give no formula of their own for the consumer;
the plainest reading, taken here and listed in the design notes, is scaled
dot-product attention restricted to the selected keys, with one key/value head
shared by all query heads (the indexer's own key has a single head):

  for query row r (batch b) and head h, with J = the entries j of the row's
  index list that name a key of batch b (0 <= j < Sk_b; -1 and anything out of
  range are skipped):
      l_j   = scale * sum_d q[r,h,d] * k[b,j,d]
      out   = sum_j softmax(l)_j * v[b,j,:]
      lse   = log sum_j exp(l_j)
  with out = 0 and lse = -inf when J is empty (and for BSND padding rows).

Evaluated in float64 from the exact values of the stored bf16/fp16 bits, with
numpy primitives (a matrix product and exp/log), one row at a time.

``mutation`` (0 in every real use) plants one deliberate mistake so that the
tests can show each pin catches it:
  1 the softmax scale is dropped
  2 the softmax skips subtracting the maximum (overflows on large logits)
  3 -1 entries are read as key 0 instead of skipped
  4 the weighted sum uses the keys instead of the values
  5 the softmax runs over the heads instead of the keys
  6 TND key offsets start one token late
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch


def _f64(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    return None if t is None else t.detach().to("cpu").to(torch.float64).numpy()


def _batch_geometry(p, inputs):
    """Per batch: (first query row, query length, allocated query rows) and
    (key offset, key length); TND lengths are prefix sums."""
    B = p.B
    aq, ak = inputs.get("act_q"), inputs.get("act_k")
    if p.layout_q == "BSND":
        q_len = aq.tolist() if aq is not None else [p.S1] * B
        q_first = [b * p.S1 for b in range(B)]
        q_alloc = [p.S1] * B
    else:
        c = [0] + aq.tolist()
        q_len = [c[b + 1] - c[b] for b in range(B)]
        q_first = c[:B]
        q_alloc = q_len
    if p.layout_kv == "BSND":
        k_len = ak.tolist() if ak is not None else [p.S2] * B
        k_off = [b * p.S2 for b in range(B)]
    elif p.layout_kv == "TND":
        c = [0] + ak.tolist()
        k_len = [c[b + 1] - c[b] for b in range(B)]
        k_off = c[:B]
    else:
        k_len = ak.tolist()
        k_off = [0] * B
    return q_first, q_len, q_alloc, k_off, k_len


def _key_rows(p, inputs, b: int, k_off: int, pos: np.ndarray, mutation: int) -> np.ndarray:
    """Row numbers (in the flattened key/value tensors) of batch b's keys `pos`."""
    if p.layout_kv == "PA_BSND":
        table = inputs["block_table"][b].numpy().astype(np.int64)
        return table[pos // p.block_size] * p.block_size + pos % p.block_size
    off = k_off + (1 if (mutation == 6 and p.layout_kv == "TND") else 0)
    return off + pos


def run(p, inputs, rows: Optional[Sequence[int]] = None, mutation: int = 0):
    """out [n, N1, Dv] float64 and lse [n, N1] float64 for the given rows."""
    q = _f64(inputs["query"]).reshape(p.rows, p.N1, p.D)
    k = _f64(inputs["key"]).reshape(-1, p.D)
    v = _f64(inputs["value"]).reshape(-1, p.Dv)
    idx = inputs["sparse_indices"].numpy().reshape(p.rows, p.sparse_count).astype(np.int64)
    q_first, q_len, q_alloc, k_off, k_len = _batch_geometry(p, inputs)
    rows = list(range(p.rows)) if rows is None else list(rows)
    scale = 1.0 if mutation == 1 else float(p.scale)
    out = np.zeros((len(rows), p.N1, p.Dv))
    lse = np.full((len(rows), p.N1), -np.inf)
    for n, r in enumerate(rows):
        b = next(bb for bb in range(p.B) if q_first[bb] <= r < q_first[bb] + q_alloc[bb])
        i = r - q_first[b]
        if i >= q_len[b]:
            continue                                   # padding row
        sel = idx[r]
        if mutation == 3:
            sel = np.where(sel == -1, 0, sel)
        sel = sel[(sel >= 0) & (sel < k_len[b])]
        if sel.size == 0:
            continue
        kr = _key_rows(p, inputs, b, k_off[b], sel, mutation)
        logits = scale * (q[r] @ k[kr].T)              # [N1, m]
        axis = 0 if mutation == 5 else 1
        if mutation == 2:
            e = np.exp(logits)
            tot = e.sum(axis=axis, keepdims=True)
            w = e / tot
            lse[n] = np.log(e.sum(axis=1))
        else:
            mx = logits.max(axis=axis, keepdims=True)
            e = np.exp(logits - mx)
            tot = e.sum(axis=axis, keepdims=True)
            w = e / tot
            m1 = logits.max(axis=1, keepdims=True)
            lse[n] = (m1 + np.log(np.exp(logits - m1).sum(axis=1, keepdims=True)))[:, 0]
        vals = k[kr] if mutation == 4 else v[kr]
        out[n] = w @ vals
    return dict(out=out, lse=lse)
