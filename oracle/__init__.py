"""fp64 CPU oracle for the LightningIndexer forward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never touches it, and it never touches the product path: the
C source ``li_oracle.c`` is compiled on its own into ``liboracle.so`` and
shares no header, helper or table with the CUDA library.

``run(problem, inputs, rows=...)`` evaluates the indexer for the given query
rows exactly as the pages define it (see the header comment of
``li_oracle.c`` for the formula, its sources and the readings taken where the
pages are silent).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "li_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DT = {"bf16": 0, "fp16": 1, "fp32": 2, "e4m3": 3, "int8": 4}
LAYOUT = {"BSND": 0, "TND": 1, "PA_BSND": 2}


class OrProblem(ctypes.Structure):
    _fields_ = [
        ("layout_q", ctypes.c_int32), ("layout_k", ctypes.c_int32),
        ("dtype_qk", ctypes.c_int32), ("dtype_w", ctypes.c_int32),
        ("dtype_scale", ctypes.c_int32), ("quant", ctypes.c_int32),
        ("B", ctypes.c_int32), ("S1", ctypes.c_int32), ("S2", ctypes.c_int32),
        ("T1", ctypes.c_int32), ("T2", ctypes.c_int32), ("N1", ctypes.c_int32),
        ("N2", ctypes.c_int32), ("D", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("key_block_stride", ctypes.c_int64),
        ("sparse_count", ctypes.c_int32), ("sparse_mode", ctypes.c_int32),
        ("return_value", ctypes.c_int32), ("mutation", ctypes.c_int32),
        ("init_num", ctypes.c_int32), ("local_num", ctypes.c_int32),
        ("cmp_ratio", ctypes.c_int32), ("cmp_residual_k", ctypes.c_void_p),
    ]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.li_oracle_rows.restype = ctypes.c_int
        L.li_oracle_rows.argtypes = [
            ctypes.POINTER(OrProblem)] + [ctypes.c_void_p] * 9 + [
            ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int]
        L.li_oracle_decode.restype = ctypes.c_double
        L.li_oracle_decode.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int]
        _lib = L
    return _lib


def _raw(t: Optional[torch.Tensor]):
    """Contiguous CPU numpy view of a tensor's stored bits (kept alive by caller)."""
    if t is None:
        return None
    t = t.detach().to("cpu").contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def _ptr(a):
    return None if a is None else a.ctypes.data


def make_problem(p, mutation: int = 0, cmp_res=None) -> OrProblem:
    """cmp_res: int32 numpy array [B] of residual original tokens (kept alive by the caller)."""
    return OrProblem(
        layout_q=LAYOUT[p.layout_q], layout_k=LAYOUT[p.layout_k],
        dtype_qk=DT[p.dtype_qk], dtype_w=DT[p.dtype_w], dtype_scale=DT[p.dtype_scale],
        quant=int(bool(p.quant)), B=p.B, S1=p.S1, S2=p.S2, T1=p.T1, T2=p.T2, N1=p.N1,
        N2=p.N2, D=p.D, num_blocks=p.num_blocks, block_size=p.block_size,
        max_blocks_per_seq=p.max_blocks_per_seq, key_block_stride=p.key_block_stride,
        sparse_count=p.sparse_count, sparse_mode=p.sparse_mode,
        return_value=p.return_value, mutation=mutation,
        init_num=getattr(p, "init_num", 0), local_num=getattr(p, "local_num", 0),
        cmp_ratio=getattr(p, "cmp_ratio", 1),
        cmp_residual_k=None if cmp_res is None else cmp_res.ctypes.data)


def max_key_len(p, inputs) -> int:
    """Largest per-batch key length (host-side, from the length tensors)."""
    ak = inputs.get("act_k")
    if p.layout_k == "BSND":
        return int(ak.max()) if ak is not None else p.S2
    if p.layout_k == "TND":
        c = ak.to(torch.int64)
        d = torch.diff(torch.cat([torch.zeros(1, dtype=torch.int64), c]))
        return int(d.max())
    return int(ak.max())


def run(p, inputs, rows: Optional[Sequence[int]] = None, want_scores: bool = False,
        nthreads: int = 0, mutation: int = 0):
    """Evaluate the oracle on query rows ``rows`` (all rows when None).

    Returns a dict with ``idx`` [n,k] int32, ``val`` [n,k] float32 (fp64
    scores rounded once), ``v64`` [n,k] float64, ``nvis`` [n] int64 and, when
    asked, ``scores`` [n, ld] float64 (NaN where a key is not visible).
    """
    L = lib()
    cmp_res = inputs.get("cmp_residual_k")
    cmp_res = None if cmp_res is None else np.ascontiguousarray(cmp_res.numpy().astype(np.int32))
    prob = make_problem(p, mutation, cmp_res)
    k = p.sparse_count
    if rows is None:
        rows_arr = None
        n = p.rows
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = len(rows_arr)
    a = {name: _raw(inputs.get(name)) for name in
         ("query", "key", "weights", "q_scale", "k_scale", "act_q", "act_k", "block_table")}
    for name in ("act_q", "act_k", "block_table"):
        if a[name] is not None:
            a[name] = np.ascontiguousarray(a[name].astype(np.int32))
    idx = np.empty((n, k), dtype=np.int32)
    val = np.empty((n, k), dtype=np.float32)
    v64 = np.empty((n, k), dtype=np.float64)
    nvis = np.empty((n,), dtype=np.int64)
    ld = max_key_len(p, inputs) if want_scores else 0
    scores = np.empty((n, ld), dtype=np.float64) if want_scores else None
    rc = L.li_oracle_rows(
        ctypes.byref(prob), _ptr(a["query"]), _ptr(a["key"]), _ptr(a["weights"]),
        _ptr(a["q_scale"]), _ptr(a["k_scale"]), _ptr(a["act_q"]), _ptr(a["act_k"]),
        _ptr(a["block_table"]), _ptr(rows_arr), n, _ptr(idx), _ptr(val), _ptr(v64),
        _ptr(scores), ld, _ptr(nvis), nthreads)
    if rc != 0:
        raise RuntimeError("li_oracle_rows failed (bad arguments)")
    out = dict(idx=idx, val=val, v64=v64, nvis=nvis)
    if want_scores:
        out["scores"] = scores
    return out


def decode(t: torch.Tensor) -> np.ndarray:
    """Decode every element of ``t`` with the oracle's own format decoders."""
    a = _raw(t)
    code = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2,
            torch.float8_e4m3fn: 3, torch.int8: 4}[t.dtype]
    flat = a.reshape(-1)
    L = lib()
    return np.array([L.li_oracle_decode(_ptr(flat), i, code) for i in range(flat.size)])
