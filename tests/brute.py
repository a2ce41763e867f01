"""Independent numpy brute force used to pin the oracle.

It re-expresses the golden recipe of the CANN TileLang LightningIndexer guide
(section "Golden 参考实现": einsum of query and key, ReLU, multiply by the
weights, sum over the group axis, sorted Top-k) in float64 numpy, one batch at
a time.  It shares nothing with ``oracle/li_oracle.c``: inputs are decoded with
torch's own dtype conversions, the dot products are an ``einsum``, and the
ordering is a ``lexsort`` on (-score, key index).
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(t):
    if t is None:
        return None
    return t.to(torch.float32).to(torch.float64).numpy()


def brute(p, inputs):
    q = _f64(inputs["query"])
    k = _f64(inputs["key"])
    w = _f64(inputs["weights"])
    qs = _f64(inputs.get("q_scale"))
    ks = _f64(inputs.get("k_scale"))
    aq = inputs.get("act_q")
    ak = inputs.get("act_k")
    bt = inputs.get("block_table")
    kk = p.sparse_count
    R = p.rows
    idx = np.full((R, kk), -1, dtype=np.int64)
    val = np.full((R, kk), -np.inf)
    if p.layout_q == "BSND":
        q = q.reshape(p.B * p.S1, p.N1, p.D)
        w = w.reshape(p.B * p.S1, p.N1)
        if qs is not None:
            qs = qs.reshape(p.B * p.S1, p.N1)
    for b in range(p.B):
        if p.layout_q == "BSND":
            q0, Sq = b * p.S1, (int(aq[b]) if aq is not None else p.S1)
        else:
            q0 = int(aq[b - 1]) if b else 0
            Sq = int(aq[b]) - q0
        if p.layout_k == "BSND":
            Sk = int(ak[b]) if ak is not None else p.S2
            K = k[b, :Sk, 0, :]
            KS = ks[b, :Sk, 0] if ks is not None else None
        elif p.layout_k == "TND":
            k0 = int(ak[b - 1]) if b else 0
            Sk = int(ak[b]) - k0
            K = k[k0:k0 + Sk, 0, :]
            KS = ks[k0:k0 + Sk, 0] if ks is not None else None
        else:
            Sk = int(ak[b])
            bs = p.block_size
            rows_k = [k[int(bt[b, t // bs]), t % bs, 0, :] for t in range(Sk)]
            K = np.stack(rows_k) if Sk else np.zeros((0, p.D))
            KS = (np.array([ks[int(bt[b, t // bs]), t % bs, 0] for t in range(Sk)])
                  if ks is not None else None)
        if Sq <= 0 or Sk <= 0:
            continue
        Q = q[q0:q0 + Sq]                                  # [Sq, N1, D]
        W = w[q0:q0 + Sq]                                  # [Sq, N1]
        logits = np.einsum("shd,td->sht", Q, K)            # [Sq, N1, Sk]
        if p.quant:
            logits = logits * qs[q0:q0 + Sq][:, :, None] * KS[None, None, :]
        score = (np.maximum(logits, 0.0) * W[:, :, None]).sum(axis=1)   # [Sq, Sk]
        t_all = np.arange(Sk)
        r = max(1, getattr(p, "cmp_ratio", 1))
        res = int(inputs["cmp_residual_k"][b]) if (r > 1 and p.sparse_mode == 3) else 0
        for i in range(Sq):
            if p.sparse_mode == 3:
                # compressed key t covers original tokens [t*r, (t+1)*r); the
                # original keys number Sk*r + res; count the visible ones
                nvis = max(0, min(Sk, (i + 1 - Sq + Sk * r + res) // r))
                vis = t_all < nvis
            else:
                vis = np.ones(Sk, dtype=bool)
            tv = t_all[vis]
            sv = score[i, vis]
            init_num = getattr(p, "init_num", 0)
            local_num = getattr(p, "local_num", 0)
            if init_num or local_num:
                # sink tokens and the local window are kept whatever their
                # score; the best of the other visible keys fill the rest
                nv = len(tv)
                forced = (tv < init_num) | (tv >= nv - local_num)
                others = np.flatnonzero(~forced)
                others = others[np.lexsort((tv[others], -sv[others]))]
                keep = np.concatenate([np.flatnonzero(forced),
                                       others[:max(0, min(kk, nv) - int(forced.sum()))]])
                tv, sv = tv[keep], sv[keep]
            order = np.lexsort((tv, -sv))
            n = min(kk, len(order))
            idx[q0 + i, :n] = tv[order[:n]]
            val[q0 + i, :n] = sv[order[:n]]
    return idx, val
