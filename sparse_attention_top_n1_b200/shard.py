"""Splitting one indexer problem over several GPUs by query rows.

Every query row of the LightningIndexer is independent of the others: its
score row depends only on its own query, weights and scales and on the keys
it may see (mindspore.ops.lightning_indexer page, ".. math::"; CANN
LightningIndexerV2 guide, "三步计算流程").  So one problem shards over ranks
with no exchange at all: each rank takes a contiguous range of output rows,
keeps its own copy of the (small) key tensor, and writes its rows of
sparse_indices / sparse_values.  The ranges are balanced by visible
(query, key) pairs, which is what the score kernel's time follows.

A range becomes one to three calls ("pieces") of the ordinary entry points.
Rows keep their answers because the actual lengths of each piece are
rewritten so that every row keeps its causal diagonal:

* rows [i0, i1) of a batch with Sq query and Sk key tokens become a batch of
  Sq' = min(i1, Sq) - i0 query rows whose key length is
  Sk' = Sk - Sq + min(i1, Sq): then i' + Sk' - Sq' = i + Sk - Sq for
  i' = i - i0, the right-down causal bound of the guide's sparse_mode 3.
  With compressed keys (cmp_ratio r, residual res) the same holds for the
  original-token count Sk*r + res, split back into Sk' and res'.  Keys cut
  off this way are invisible to every row of the piece.  Mode 0 keeps Sk.
* BSND queries: a range that starts or ends inside a batch gives a one-batch
  piece for that part; the whole batches between them form one piece.
* TND queries: one piece, with prefix sums rebuilt for the batches it
  touches and the key rows starting at its first batch's keys.
* Paged keys need no key offset: the piece takes its batches' rows of
  block_table and actual_seq_lengths_key.

This module is host logic only; it neither launches nor allocates.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

_LAYOUT_NAMES = {0: "BSND", 1: "TND", 2: "PA_BSND"}


def _layout(x) -> str:
    return _LAYOUT_NAMES.get(x, x) if isinstance(x, int) else x


def _np(t) -> Optional[np.ndarray]:
    if t is None:
        return None
    if hasattr(t, "detach"):
        t = t.detach().cpu().numpy()
    return np.asarray(t, dtype=np.int64)


@dataclasses.dataclass
class Piece:
    """One call covering output rows [r0, r1) of the whole problem.

    ``fields`` are the problem attributes that differ from the whole
    problem's (B, S1, T1, T2); ``q_row0`` is the first query token row (rows
    of query, weights and q_scale), ``b0``/``nb`` the batches it spans
    (rows of block_table), ``k_row0`` the first key token row (BSND/TND keys
    and k_scale; 0 for paged keys), ``k_rows`` how many key token rows the
    piece may touch.  act_q / act_k / cmp_res are the rewritten lengths
    (int32 arrays, or None where the whole problem passes none).
    """

    r0: int
    r1: int
    fields: Dict[str, int]
    q_row0: int
    b0: int
    nb: int
    k_row0: int
    k_rows: int
    act_q: Optional[np.ndarray]
    act_k: Optional[np.ndarray]
    cmp_res: Optional[np.ndarray]


class _Lengths:
    """Per-batch query/key lengths and offsets of the whole problem."""

    def __init__(self, p, act_q, act_k, cmp_res):
        self.lq, self.lk = _layout(p.layout_q), _layout(p.layout_k)
        B = p.B
        aq, ak = _np(act_q), _np(act_k)
        if self.lq == "TND":
            cq = np.concatenate([[0], aq])
            self.q_off = cq[:-1]
            self.Sq = np.diff(cq)
        else:
            self.q_off = np.arange(B, dtype=np.int64) * p.S1
            self.Sq = aq.copy() if aq is not None else np.full(B, p.S1, dtype=np.int64)
            self.Sq = np.clip(self.Sq, 0, p.S1)
        if self.lk == "TND":
            ck = np.concatenate([[0], ak])
            self.k_off = ck[:-1]
            self.Sk = np.diff(ck)
        elif self.lk == "BSND":
            self.k_off = np.arange(B, dtype=np.int64) * p.S2
            self.Sk = ak.copy() if ak is not None else np.full(B, p.S2, dtype=np.int64)
        else:
            self.k_off = np.zeros(B, dtype=np.int64)
            self.Sk = ak.copy()
        r = int(getattr(p, "cmp_ratio", 1) or 1)
        self.r = r if r > 1 else 1
        self.mode = p.sparse_mode
        cr = _np(cmp_res)
        self.res = cr.copy() if (cr is not None and self.r > 1 and self.mode == 3) else np.zeros(B, dtype=np.int64)
        self.act_q_given = act_q is not None
        self.act_k_given = act_k is not None

    def visible(self, b: int, i: np.ndarray) -> np.ndarray:
        """Visible keys of rows i of batch b (the scheduler's rule)."""
        Sq, Sk = int(self.Sq[b]), int(self.Sk[b])
        if self.mode != 3:
            return np.where(i < Sq, Sk, 0)
        v = np.floor_divide(i + 1 - Sq + Sk * self.r + int(self.res[b]), self.r)
        return np.where(i < Sq, np.clip(v, 0, Sk), 0)

    def cut_key(self, b: int, end: int):
        """(Sk', res') for a piece of batch b whose last row is end - 1."""
        Sq, Sk, res = int(self.Sq[b]), int(self.Sk[b]), int(self.res[b])
        if self.mode != 3:
            return Sk, res
        e = min(end, Sq)
        x = Sk * self.r + res - (Sq - e)
        if x <= 0:
            return 0, 0
        return x // self.r, x % self.r


def row_costs(p, act_q=None, act_k=None, cmp_res=None) -> np.ndarray:
    """Visible keys of every output row (int64 [rows]): the balancing weight."""
    L = _Lengths(p, act_q, act_k, cmp_res)
    rows = p.B * p.S1 if L.lq == "BSND" else p.T1
    cost = np.zeros(rows, dtype=np.int64)
    for b in range(p.B):
        n = int(L.Sq[b]) if L.lq == "TND" else p.S1
        if n <= 0:
            continue
        o = int(L.q_off[b])
        cost[o:o + n] = L.visible(b, np.arange(n, dtype=np.int64))
    return cost


def split_rows(cost: Sequence[int], world: int, row_weight: int = 64) -> List[tuple]:
    """Contiguous row ranges [r0, r1), one per rank, with near-equal sums of
    ``cost + row_weight`` (the constant covers a row's Top-k and output
    write, so ranges of empty rows are not free)."""
    c = np.asarray(cost, dtype=np.int64) + row_weight
    rows = c.size
    cum = np.concatenate([[0], np.cumsum(c)])
    total = int(cum[-1])
    cuts = [0]
    for j in range(1, world):
        cuts.append(int(np.searchsorted(cum, total * j / world, side="left")))
    cuts.append(rows)
    cuts = [min(max(x, 0), rows) for x in cuts]
    for j in range(1, len(cuts)):
        cuts[j] = max(cuts[j], cuts[j - 1])
    return [(cuts[j], cuts[j + 1]) for j in range(world)]


def _bsnd_piece(p, L: _Lengths, b: int, i0: int, i1: int) -> Piece:
    sq = max(0, min(i1, int(L.Sq[b])) - i0)
    sk, res = L.cut_key(b, i1)
    fields = {"B": 1, "S1": i1 - i0}
    return Piece(r0=b * p.S1 + i0, r1=b * p.S1 + i1, fields=fields, q_row0=b * p.S1 + i0,
                 b0=b, nb=1, k_row0=int(L.k_off[b]), k_rows=p.S2 if L.lk == "BSND" else 0,
                 act_q=np.array([sq], dtype=np.int32),
                 act_k=np.array([sk], dtype=np.int32),
                 cmp_res=np.array([res], dtype=np.int32) if L.r > 1 and L.mode == 3 else None)


def _bsnd_whole(p, L: _Lengths, act_q, act_k, cmp_res, b0: int, b1: int) -> Piece:
    nb = b1 - b0
    sl = lambda a: None if a is None else np.ascontiguousarray(_np(a)[b0:b1].astype(np.int32))
    return Piece(r0=b0 * p.S1, r1=b1 * p.S1, fields={"B": nb}, q_row0=b0 * p.S1, b0=b0, nb=nb,
                 k_row0=int(L.k_off[b0]), k_rows=nb * p.S2 if L.lk == "BSND" else 0,
                 act_q=sl(act_q), act_k=sl(act_k),
                 cmp_res=sl(cmp_res) if L.r > 1 and L.mode == 3 else None)


def _tnd_piece(p, L: _Lengths, r0: int, r1: int) -> Piece:
    B = p.B
    hi_q = L.q_off + L.Sq
    # batches whose rows meet [r0, r1)
    bs = [b for b in range(B) if L.Sq[b] > 0 and L.q_off[b] < r1 and hi_q[b] > r0]
    if not bs:
        # only rows past the last prefix sum: one empty batch, every row padding
        b = min(B - 1, int(np.searchsorted(L.q_off, r0, side="right")) - 1)
        bs_first, bs_last = max(b, 0), max(b, 0)
        sqs, sks, ress = [0], [0], [0]
    else:
        bs_first, bs_last = bs[0], bs[-1]
        sqs, sks, ress = [], [], []
        for b in range(bs_first, bs_last + 1):
            s = max(r0, int(L.q_off[b])) - int(L.q_off[b])
            e = min(r1, int(hi_q[b])) - int(L.q_off[b])
            sqs.append(max(0, e - s))
            sk, res = L.cut_key(b, e)
            sks.append(sk)
            ress.append(res)
    # rows before the first batch's first row in the range cannot exist (the
    # first batch starts at or before r0 unless r0 is in a gap of empty batches)
    q_row0 = r0
    first_row = max(r0, int(L.q_off[bs_first])) if bs else r0
    assert first_row == r0 or not bs, "TND rows are consecutive across batches"
    k0 = int(L.k_off[bs_first])
    k_end = int(L.k_off[bs_last] + L.Sk[bs_last])
    nb = bs_last - bs_first + 1
    t2 = max(1, k_end - k0)
    return Piece(r0=r0, r1=r1, fields={"B": nb, "T1": r1 - r0, "T2": t2}, q_row0=q_row0,
                 b0=bs_first, nb=nb, k_row0=k0, k_rows=t2,
                 act_q=np.cumsum(sqs).astype(np.int32),
                 act_k=np.cumsum(sks).astype(np.int32) if L.lk == "TND" else np.array(sks, dtype=np.int32),
                 cmp_res=np.array(ress, dtype=np.int32) if L.r > 1 and L.mode == 3 else None)


def pieces_for_range(p, r0: int, r1: int, act_q=None, act_k=None, cmp_res=None) -> List[Piece]:
    """The calls that compute output rows [r0, r1) of problem ``p``."""
    if r1 <= r0:
        return []
    L = _Lengths(p, act_q, act_k, cmp_res)
    if L.lq == "TND":
        return [_tnd_piece(p, L, r0, r1)]
    S1 = p.S1
    b_first, i0 = divmod(r0, S1)
    b_last, i_end = divmod(r1 - 1, S1)
    i1 = i_end + 1
    if b_first == b_last:
        if i0 == 0 and i1 == S1:
            return [_bsnd_whole(p, L, act_q, act_k, cmp_res, b_first, b_first + 1)]
        return [_bsnd_piece(p, L, b_first, i0, i1)]
    out = []
    wb0 = b_first
    if i0 > 0:
        out.append(_bsnd_piece(p, L, b_first, i0, S1))
        wb0 = b_first + 1
    wb1 = b_last + 1 if i1 == S1 else b_last
    if wb1 > wb0:
        out.append(_bsnd_whole(p, L, act_q, act_k, cmp_res, wb0, wb1))
    if i1 < S1:
        out.append(_bsnd_piece(p, L, b_last, 0, i1))
    return out


def shard(p, world: int, act_q=None, act_k=None, cmp_res=None) -> List[List[Piece]]:
    """Per rank, the pieces of its contiguous, pair-balanced row range."""
    cost = row_costs(p, act_q, act_k, cmp_res)
    return [pieces_for_range(p, r0, r1, act_q, act_k, cmp_res)
            for (r0, r1) in split_rows(cost, world)]


def piece_inputs(piece: Piece, p, inputs: Dict[str, object], to=None) -> Dict[str, object]:
    """The piece's views of the whole problem's tensors (torch, any device).

    Query-side tensors (query, weights, q_scale) start at token row
    ``q_row0``; BSND/TND key-side tensors (key, k_scale) at ``k_row0``; paged
    pools are passed whole with the piece's rows of block_table.  The
    rewritten lengths are new int32 tensors made with ``to`` (a function
    mapping a numpy array to a tensor; torch.from_numpy when None).
    """
    import torch
    conv = to or (lambda a: torch.from_numpy(np.ascontiguousarray(a)))
    lq, lk = _layout(p.layout_q), _layout(p.layout_k)
    out = {}
    n_q_tokens = piece.r1 - piece.r0

    def q_side(t):
        if t is None:
            return None
        if lq == "BSND":
            flat = t.reshape((p.B * p.S1,) + tuple(t.shape[2:]))
            v = flat.narrow(0, piece.q_row0, n_q_tokens)
            return v.reshape((piece.fields.get("B", 1), n_q_tokens // piece.fields.get("B", 1)) + tuple(t.shape[2:]))
        return t.narrow(0, piece.q_row0, n_q_tokens)

    def k_side(t):
        if t is None:
            return None
        if lk == "PA_BSND":
            return t
        if lk == "BSND":
            return t.narrow(0, piece.b0, piece.nb)
        return t.narrow(0, piece.k_row0, min(piece.k_rows, t.shape[0] - piece.k_row0))

    out["query"] = q_side(inputs["query"])
    out["weights"] = q_side(inputs["weights"])
    out["q_scale"] = q_side(inputs.get("q_scale"))
    out["key"] = k_side(inputs["key"])
    out["k_scale"] = k_side(inputs.get("k_scale"))
    bt = inputs.get("block_table")
    out["block_table"] = None if bt is None else bt.narrow(0, piece.b0, piece.nb)
    out["act_q"] = None if piece.act_q is None else conv(piece.act_q)
    out["act_k"] = None if piece.act_k is None else conv(piece.act_k)
    out["cmp_residual_k"] = None if piece.cmp_res is None else conv(piece.cmp_res)
    return {k: v for k, v in out.items() if v is not None}
