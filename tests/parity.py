"""Element-by-element comparison of the CUDA path with the fp64 oracle.

The rule (tolerance |g - o| <= atol + rtol*|o|; bf16/fp16/int8: rtol 2e-3, atol
1e-4; fp8: rtol 5e-2, atol 1e-4):
  * slots past min(k, visible) hold index -1 and value -inf, bit for bit;
  * the valid indices are distinct and visible (0 <= t < nvis);
  * values are non-increasing, each within tolerance of the oracle's score of
    that key and of the oracle's value in the same slot;
  * every key whose oracle score exceeds s_k + tol(s_k) is selected, and every
    selected key has an oracle score >= s_k - tol(s_k), where s_k is the
    oracle's k-th value: swaps are allowed only inside the tolerance band
    around the k-th score;
  * with sink tokens / a local window, the forced keys (the first init_num and
    last local_num visible keys) are all selected, and the band rule above
    applies to the other keys, with s_k the oracle's k'-th best other score
    (k' = min(k, visible) - number of forced keys).
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

TOL = {"bf16": (2e-3, 1e-4), "fp16": (2e-3, 1e-4), "e4m3": (5e-2, 1e-4), "int8": (2e-3, 1e-4)}
NEG_INF_BITS = np.float32(-np.inf).view(np.uint32)


def to_device(inputs, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


def compare_rows(p, gpu_idx, gpu_val, orc, rows_label=None, rtol=None, atol=None):
    """gpu_idx/gpu_val: numpy [n, k] for the rows the oracle evaluated (orc)."""
    if rtol is None:
        rtol, atol = TOL[p.dtype_qk]
    k = p.sparse_count
    scores = orc["scores"]
    for r in range(gpu_idx.shape[0]):
        label = rows_label[r] if rows_label is not None else r
        nv = int(orc["nvis"][r])
        m = min(k, nv)
        gi = gpu_idx[r]
        assert np.all(gi[m:] == -1), "row %s: padding indices" % label
        if gpu_val is not None:
            gv = gpu_val[r]
            assert np.all(gv[m:].view(np.uint32) == NEG_INF_BITS), "row %s: padding values" % label
        if m == 0:
            continue
        sel = gi[:m].astype(np.int64)
        assert np.all(sel >= 0) and np.all(sel < nv), "row %s: index out of the visible range" % label
        assert len(np.unique(sel)) == m, "row %s: duplicate indices" % label
        s = scores[r]
        os_sorted = orc["v64"][r][:m]
        got_s = s[sel]
        assert np.all(np.isfinite(got_s)), "row %s: selected an invisible key" % label
        init_num, local_num = getattr(p, "init_num", 0), getattr(p, "local_num", 0)
        forced = np.zeros(nv, dtype=bool)
        forced[:min(init_num, nv)] = True
        forced[max(0, nv - local_num):] = True
        f_idx = np.nonzero(forced)[0]
        missing_forced = np.setdiff1d(f_idx, sel)
        assert missing_forced.size == 0, "row %s: forced keys not kept %s" % (label, missing_forced[:8])
        kk = m - f_idx.size                              # slots for the other keys
        if kk > 0:
            others = np.nonzero(~forced)[0]
            s_oth = np.sort(s[others])[::-1]
            s_k = s_oth[kk - 1]
            tol_k = atol + rtol * abs(s_k)
            sel_oth = sel[~forced[sel]]
            assert np.all(s[sel_oth] >= s_k - tol_k), (
                "row %s: selected key below the k-th score band (min %.6g < %.6g)"
                % (label, s[sel_oth].min(), s_k - tol_k))
            must = others[s[others] > s_k + tol_k]
            missing = np.setdiff1d(must, sel)
            assert missing.size == 0, "row %s: missed keys %s" % (label, missing[:8])
        if gpu_val is not None:
            gv = gpu_val[r][:m].astype(np.float64)
            assert np.all(np.diff(gv) <= 0), "row %s: values not non-increasing" % label
            err_key = np.abs(gv - got_s) - (atol + rtol * np.abs(got_s))
            assert np.all(err_key <= 0), "row %s: value vs key score off by %.3g (slot %d)" % (
                label, np.abs(gv - got_s)[np.argmax(err_key)], int(np.argmax(err_key)))
            err_slot = np.abs(gv - os_sorted) - (atol + rtol * np.abs(os_sorted))
            assert np.all(err_slot <= 0), "row %s: value vs sorted oracle off by %.3g (slot %d)" % (
                label, np.abs(gv - os_sorted)[np.argmax(err_slot)], int(np.argmax(err_slot)))


def check_against_oracle(p, inputs, gpu_idx, gpu_val, rows=None, nthreads=0):
    """Run the oracle on `rows` (all when None) and compare. gpu_* are full [R, k]."""
    gi = gpu_idx.reshape(p.rows, p.sparse_count)
    gv = gpu_val.reshape(p.rows, p.sparse_count) if gpu_val is not None else None
    orc = oracle.run(p, inputs, rows=rows, want_scores=True, nthreads=nthreads)
    if rows is not None:
        gi = gi[np.asarray(rows)]
        gv = gv[np.asarray(rows)] if gv is not None else None
    compare_rows(p, gi, gv, orc, rows_label=rows)
    return orc


def check_all_rows(p, inputs, gpu_idx, gpu_val, chunk=2048):
    """check_against_oracle on every row, `chunk` rows at a time (the oracle's
    full score rows of a chunk are held in fp64), on all host cores."""
    nthreads = os.cpu_count() or 1
    for r0 in range(0, p.rows, chunk):
        check_against_oracle(p, inputs, gpu_idx, gpu_val, rows=list(range(r0, min(p.rows, r0 + chunk))),
                             nthreads=nthreads)


def sample_rows(p, n_random=256, seed=0, edge=64):
    """First/last rows, rows around index k and a seeded random sample."""
    R = p.rows
    k = p.sparse_count
    rs = set(range(min(edge, R))) | set(range(max(0, R - edge), R))
    rs |= set(range(max(0, k - 8), min(R, k + 8)))
    g = np.random.default_rng(seed)
    rs |= set(g.integers(0, R, size=min(n_random, R)).tolist())
    return sorted(rs)
