"""Python binding of libli, the B200 LightningIndexer (C ABI in include/li.h).

The binding only marshals arguments: every step of the indexer and of the
sparse attention that consumes its output runs in the CUDA kernels of
``libli.so``.  Functions keep the C names (``li_indexer``,
``li_quant_indexer``, ``li_topk``, ``li_sparse_attention``,
``li_output_shape``, ``li_workspace_size``, ``li_read_device_status``, ...)
and take torch CUDA tensors, passing their device pointers and the current
CUDA stream.  ``indexer(...)`` and ``sparse_attention(...)`` are convenience
wrappers that allocate the outputs (and the indexer's workspace) with torch.

There is no fallback: if ``libli.so`` is missing or fails to load, importing
the functions raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libli.so")

LI_OK = 0
STATUS_NAMES = {0: "LI_OK", 1: "LI_ERR_NULL", 2: "LI_ERR_SHAPE", 3: "LI_ERR_DTYPE",
                4: "LI_ERR_LAYOUT", 5: "LI_ERR_UNSUPPORTED", 6: "LI_ERR_WORKSPACE",
                7: "LI_ERR_CUDA", 8: "LI_ERR_DEVICE"}
DTYPE = {"bf16": 0, "fp16": 1, "fp32": 2, "e4m3": 3, "int8": 4}
LAYOUT = {"BSND": 0, "TND": 1, "PA_BSND": 2}
DEV_BAD_QLEN, DEV_BAD_KLEN, DEV_BAD_BLOCK, DEV_NEG_SCALE, DEV_TIMEOUT = 1, 2, 4, 8, 16
DEV_BAD_INDEX = 32
INT64_MAX = (1 << 63) - 1
# LI_NOALLOC_SCRATCH_BYTES of include/li.h: the scratch li_indexer_noalloc holds
NOALLOC_SCRATCH_BYTES = 32 << 20

EXPORTS = ("li_output_shape", "li_workspace_size", "li_indexer", "li_quant_indexer", "li_topk",
           "li_last_error", "li_read_device_status", "li_selftest_bounded_wait",
           "li_last_launch_count", "li_set_profile_events", "li_indexer_noalloc",
           "li_sparse_attention")


class LiError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, str(status)), msg))
        self.status = status


class Params(ctypes.Structure):
    """Mirror of li_params."""
    _fields_ = [
        ("layout_q", ctypes.c_int32), ("layout_k", ctypes.c_int32),
        ("dtype_qk", ctypes.c_int32), ("dtype_w", ctypes.c_int32),
        ("dtype_scale", ctypes.c_int32),
        ("B", ctypes.c_int32), ("S1", ctypes.c_int32), ("S2", ctypes.c_int32),
        ("T1", ctypes.c_int32), ("T2", ctypes.c_int32), ("N1", ctypes.c_int32),
        ("N2", ctypes.c_int32), ("D", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("key_block_stride", ctypes.c_int64),
        ("sparse_count", ctypes.c_int32), ("sparse_mode", ctypes.c_int32),
        ("pre_tokens", ctypes.c_int64), ("next_tokens", ctypes.c_int64),
        ("return_value", ctypes.c_int32), ("max_seqlen_k", ctypes.c_int32),
        ("init_num", ctypes.c_int32), ("local_num", ctypes.c_int32),
        ("cmp_ratio", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("cmp_residual_k", ctypes.c_void_p),
    ]


class SfaParams(ctypes.Structure):
    """Mirror of li_sfa_params (sparse attention over the selected keys)."""
    _fields_ = [
        ("layout_q", ctypes.c_int32), ("layout_kv", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("B", ctypes.c_int32), ("S1", ctypes.c_int32), ("S2", ctypes.c_int32),
        ("T1", ctypes.c_int32), ("T2", ctypes.c_int32),
        ("N1", ctypes.c_int32), ("D", ctypes.c_int32), ("Dv", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32), ("sparse_count", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float), ("reserved", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libli.so (loudly failing when it is absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libli.so is not built (run python -m sparse_attention_top_n1_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        P = ctypes.POINTER(Params)
        sig = {
            "li_output_shape": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(i32)]),
            "li_workspace_size": (ctypes.c_int, [P, ctypes.POINTER(sz)]),
            "li_indexer": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "li_quant_indexer": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "li_topk": (ctypes.c_int, [vp, i64, vp, i32, i32, vp, vp, vp]),
            "li_last_error": (ctypes.c_char_p, []),
            "li_read_device_status": (ctypes.c_int, [vp, vp, ctypes.POINTER(i32)]),
            "li_selftest_bounded_wait": (ctypes.c_int, [vp, i64, vp]),
            "li_last_launch_count": (i32, []),
            "li_set_profile_events": (None, [ctypes.POINTER(ctypes.c_void_p), i32]),
            "li_indexer_noalloc": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
            "li_sparse_attention": (ctypes.c_int, [ctypes.POINTER(SfaParams), vp, vp, vp, vp, vp,
                                                   vp, vp, vp, vp, vp, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != LI_OK:
        raise LiError(status, lib().li_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def make_params(problem=None, **kw) -> Params:
    """Build li_params from an object with the attribute names of li_params
    (layouts and dtypes given as strings) and/or keyword overrides."""
    f = {}
    if problem is not None:
        for name, _ in Params._fields_:
            if hasattr(problem, name):
                f[name] = getattr(problem, name)
    f.update(kw)
    f.setdefault("N2", 1)
    f.setdefault("pre_tokens", INT64_MAX)
    f.setdefault("next_tokens", INT64_MAX)
    f.setdefault("dtype_scale", "fp32")
    for name in ("layout_q", "layout_k"):
        if isinstance(f.get(name), str):
            f[name] = LAYOUT[f[name]]
    for name in ("dtype_qk", "dtype_w", "dtype_scale"):
        if isinstance(f.get(name), str):
            f[name] = DTYPE[f[name]]
    return Params(**{k: v for k, v in f.items() if k in dict(Params._fields_)})


# ---------------------------------------------------------------- C-ABI calls

def li_output_shape(params: Params):
    dims = (ctypes.c_int64 * 4)()
    nd = ctypes.c_int32()
    _check(lib().li_output_shape(ctypes.byref(params), dims, ctypes.byref(nd)))
    return tuple(dims[i] for i in range(nd.value))


def li_workspace_size(params: Params) -> int:
    n = ctypes.c_size_t()
    _check(lib().li_workspace_size(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def li_indexer(params, query, key, weights, act_seq_q, act_seq_k, block_table, sparse_indices,
               sparse_values, workspace, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().li_indexer(ctypes.byref(params), _ptr(query), _ptr(key), _ptr(weights),
                            _ptr(act_seq_q), _ptr(act_seq_k), _ptr(block_table),
                            _ptr(sparse_indices), _ptr(sparse_values), _ptr(workspace),
                            workspace_bytes, _stream(stream)))


def li_quant_indexer(params, query, key, weights, q_scale, k_scale, act_seq_q, act_seq_k,
                     block_table, sparse_indices, sparse_values, workspace,
                     workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().li_quant_indexer(ctypes.byref(params), _ptr(query), _ptr(key), _ptr(weights),
                                  _ptr(q_scale), _ptr(k_scale), _ptr(act_seq_q),
                                  _ptr(act_seq_k), _ptr(block_table), _ptr(sparse_indices),
                                  _ptr(sparse_values), _ptr(workspace), workspace_bytes,
                                  _stream(stream)))


def li_topk(scores, ld, row_len, rows, k, sparse_indices, sparse_values=None, stream=None):
    _check(lib().li_topk(_ptr(scores), ld, _ptr(row_len), rows, k, _ptr(sparse_indices),
                         _ptr(sparse_values), _stream(stream)))


def li_indexer_noalloc(params, query, key, weights, act_seq_q, act_seq_k, block_table,
                       sparse_indices, sparse_values, stream=None):
    """li_indexer with the library's built-in scratch instead of a workspace
    (see include/li.h: for callers that cannot allocate device memory)."""
    _check(lib().li_indexer_noalloc(ctypes.byref(params), _ptr(query), _ptr(key), _ptr(weights),
                                    _ptr(act_seq_q), _ptr(act_seq_k), _ptr(block_table),
                                    _ptr(sparse_indices), _ptr(sparse_values), _stream(stream)))


def make_sfa_params(problem=None, **kw) -> SfaParams:
    """li_sfa_params from an object with its field names (layouts and dtype as
    strings; softmax_scale 0 or absent = 1/sqrt(D)) and/or keyword overrides."""
    f = {}
    if problem is not None:
        for name, _ in SfaParams._fields_:
            if hasattr(problem, name):
                f[name] = getattr(problem, name)
    f.update(kw)
    for name in ("layout_q", "layout_kv"):
        if isinstance(f.get(name), str):
            f[name] = LAYOUT[f[name]]
    if isinstance(f.get("dtype"), str):
        f["dtype"] = DTYPE[f["dtype"]]
    if not f.get("softmax_scale"):
        f["softmax_scale"] = f.get("D", 128) ** -0.5
    return SfaParams(**{k: v for k, v in f.items() if k in dict(SfaParams._fields_)})


def li_sparse_attention(params: SfaParams, query, key, value, sparse_indices, act_seq_q, act_seq_k,
                        block_table, out, lse=None, status=None, stream=None):
    _check(lib().li_sparse_attention(ctypes.byref(params), _ptr(query), _ptr(key), _ptr(value),
                                     _ptr(sparse_indices), _ptr(act_seq_q), _ptr(act_seq_k),
                                     _ptr(block_table), _ptr(out), _ptr(lse), _ptr(status),
                                     _stream(stream)))


def sparse_attention(params: SfaParams, query, key, value, sparse_indices, *, act_seq_q=None,
                     act_seq_k=None, block_table=None, want_lse=True, status=None, stream=None):
    """Run li_sparse_attention, allocating out [rows, N1, Dv] (the query's dtype)
    and, when asked, lse [rows, N1] fp32.  Returns (out, lse or None)."""
    import torch
    rows = params.B * params.S1 if params.layout_q == LAYOUT["BSND"] else params.T1
    out = torch.empty((rows, params.N1, params.Dv), dtype=query.dtype, device=query.device)
    lse = torch.empty((rows, params.N1), dtype=torch.float32, device=query.device) if want_lse else None
    li_sparse_attention(params, query, key, value, sparse_indices, act_seq_q, act_seq_k, block_table,
                        out, lse, status, stream)
    return out, lse


def li_read_device_status(workspace, stream=None) -> int:
    """SYNCHRONISING: the LI_DEV_* bits left by the last call on `workspace`."""
    flags = ctypes.c_int32()
    st = lib().li_read_device_status(_ptr(workspace), _stream(stream), ctypes.byref(flags))
    if st not in (LI_OK, 8):
        _check(st)
    return flags.value


def li_selftest_bounded_wait(status_word, timeout_ns: int, stream=None):
    _check(lib().li_selftest_bounded_wait(_ptr(status_word), timeout_ns, _stream(stream)))


def li_last_launch_count() -> int:
    return lib().li_last_launch_count()


def li_set_profile_events(events):
    """Record per-stage CUDA events in later calls (list of 4 torch.cuda.Event
    created with enable_timing=True), or turn it off with None."""
    if not events:
        lib().li_set_profile_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    lib().li_set_profile_events(arr, len(events))


def li_last_error() -> str:
    return lib().li_last_error().decode()


# ---------------------------------------------------------------- convenience

def alloc_workspace(params: Params, device="cuda"):
    import torch
    n = li_workspace_size(params)
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def indexer(params: Params, query, key, weights, *, act_seq_q=None, act_seq_k=None,
            block_table=None, q_scale=None, k_scale=None, cmp_residual_k=None, workspace=None,
            out=None, stream=None):
    """Run li_indexer / li_quant_indexer, allocating outputs (and workspace).

    cmp_residual_k (int32 [B] on the device) is stored into params before the
    call.  Returns (sparse_indices, sparse_values); sparse_values is an empty
    (0,) tensor when return_value is 0, as the CANN guide's output rule says.
    """
    import torch
    if cmp_residual_k is not None:
        params.cmp_residual_k = _ptr(cmp_residual_k)
    shape = li_output_shape(params)
    dev = query.device
    if out is None:
        idx = torch.empty(shape, dtype=torch.int32, device=dev)
        val = (torch.empty(shape, dtype=torch.float32, device=dev) if params.return_value
               else torch.empty((0,), dtype=torch.float32, device=dev))
    else:
        idx, val = out
    if workspace is None:
        workspace = alloc_workspace(params, dev)
    vptr = val if params.return_value else None
    if params.dtype_qk == DTYPE["e4m3"] or params.dtype_qk == DTYPE["int8"]:
        li_quant_indexer(params, query, key, weights, q_scale, k_scale, act_seq_q, act_seq_k,
                         block_table, idx, vptr, workspace, stream=stream)
    else:
        li_indexer(params, query, key, weights, act_seq_q, act_seq_k, block_table, idx, vptr,
                   workspace, stream=stream)
    return idx, val
