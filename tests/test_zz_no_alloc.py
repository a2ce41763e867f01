"""The allocation-free entry point, li_indexer_noalloc.

It exists for callers that cannot give the library device memory: an
operator interface that hands a kernel only its inputs and outputs, or a
serving loop that keeps cudaMalloc off its hot path.  Instead of a workspace
it uses a scratch array compiled into the library.  These tests call it
through the C ABI, twice in a row (the second call finds the first call's
data in the shared scratch), and check its output against li_indexer with a
workspace, within the parity tolerance of the other GPU tests.  They also
check that a problem larger than the scratch is refused before any launch.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_top_n1_b200 as li
import synth
from parity import TOL, to_device

pytestmark = pytest.mark.gpu


def _run_noalloc(pr, d, shape, return_value):
    idx = torch.full(shape, 12345, dtype=torch.int32, device="cuda")
    val = torch.full(shape, 7.0, dtype=torch.float32, device="cuda") if return_value else None
    li.li_indexer_noalloc(pr, d["query"], d["key"], d["weights"], d.get("act_q"),
                          d.get("act_k"), d.get("block_table"), idx, val)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), (val.cpu().numpy() if val is not None else None)


@pytest.mark.parametrize("make", [synth.make_tiny, synth.make_cfg2,
                                  lambda: synth.make_random(3, layout_k="PA_BSND", block_size=64,
                                                            B=3, S1=33, S2=700, N1=64,
                                                            sparse_count=128, return_value=1)])
def test_noalloc_matches_workspace_entry_point(make):
    p, inp = make()
    d = to_device(inp)
    pr = li.make_params(p)
    assert li.li_workspace_size(pr) <= li.NOALLOC_SCRATCH_BYTES
    ref_idx, ref_val = li.indexer(pr, d["query"], d["key"], d["weights"],
                                  act_seq_q=d.get("act_q"), act_seq_k=d.get("act_k"),
                                  block_table=d.get("block_table"))
    torch.cuda.synchronize()
    ref_idx = ref_idx.cpu().numpy()
    ref_val = ref_val.cpu().numpy() if p.return_value else None
    rtol, atol = TOL[p.dtype_qk]
    shape = li.li_output_shape(pr)
    for _ in range(2):                      # two calls in a row on the shared scratch
        idx, val = _run_noalloc(pr, d, shape, p.return_value)
        np.testing.assert_array_equal(idx, ref_idx)
        if p.return_value:
            fin = np.isfinite(ref_val)
            np.testing.assert_array_equal(np.isfinite(val), fin)
            np.testing.assert_allclose(val[fin], ref_val[fin], rtol=rtol, atol=atol)


def test_noalloc_refuses_problems_beyond_its_scratch():
    p, _ = synth.make_dsa_prefill(S=8192)            # needs ~256 MiB of score rows
    pr = li.make_params(p)
    assert li.li_workspace_size(pr) > li.NOALLOC_SCRATCH_BYTES
    st = li.lib().li_indexer_noalloc(ctypes.byref(pr), None, None, None, None, None, None,
                                     None, None, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_WORKSPACE"
    assert "bytes of scratch" in li.li_last_error()


def _edge_problem(over: bool):
    """A BSND problem whose workspace is the largest at or under the scratch
    size (over=False) or the smallest above it (over=True): rows grow one at
    a time at a fixed key length (each row adds one fp32 score row)."""
    S2 = 4096

    def size(S1):
        p, inp = synth.make_random(17, B=1, S1=S1, S2=S2, N1=8, sparse_count=64, ragged=False,
                                   sparse_mode=0)
        return li.li_workspace_size(li.make_params(p)), p, inp

    lo, hi = 1, 4096                       # size(lo) <= limit < size(hi)
    assert size(hi)[0] > li.NOALLOC_SCRATCH_BYTES
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if size(mid)[0] <= li.NOALLOC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return size(hi if over else lo)


def test_noalloc_at_the_limit_runs_and_one_row_more_is_refused():
    need, p, inp = _edge_problem(over=False)
    assert need <= li.NOALLOC_SCRATCH_BYTES
    d = to_device(inp)
    pr = li.make_params(p)
    ref_idx, ref_val = li.indexer(pr, d["query"], d["key"], d["weights"],
                                  act_seq_q=d.get("act_q"), act_seq_k=d.get("act_k"))
    idx, val = _run_noalloc(pr, d, li.li_output_shape(pr), p.return_value)
    np.testing.assert_array_equal(idx, ref_idx.cpu().numpy())
    np.testing.assert_array_equal(val, ref_val.cpu().numpy())
    need, p, inp = _edge_problem(over=True)
    assert need > li.NOALLOC_SCRATCH_BYTES
    d = to_device(inp)
    pr = li.make_params(p)
    shape = li.li_output_shape(pr)
    idx = torch.full(shape, 5, dtype=torch.int32, device="cuda")
    val = torch.full(shape, 5.0, dtype=torch.float32, device="cuda")
    with pytest.raises(li.LiError) as ei:
        li.li_indexer_noalloc(pr, d["query"], d["key"], d["weights"], d.get("act_q"),
                              d.get("act_k"), None, idx, val)
    assert ei.value.status == 6                          # LI_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((idx == 5).all())                        # nothing was launched
