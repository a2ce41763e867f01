"""Guard bands around every buffer the kernels write.

Each output (indices, values, the workspace, the attention output and its
log-sum-exp) is carved out of a larger device buffer whose head and tail are
filled with a canary pattern.  After the call the canaries must be intact and
the outputs must still match the oracle, so no kernel writes a byte outside
the buffers the caller handed it.  The inputs use ragged lengths, paged keys
with -1 table entries and rows with nothing visible, which are the cases
where an off-by-one in a bound would land outside the outputs.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.sfa as osfa
import sparse_attention_top_n1_b200 as li
import synth
from parity import check_against_oracle, to_device
from synth import sfa as ssfa

pytestmark = pytest.mark.gpu

GUARD = 4096                       # bytes of canary before and after each buffer
PATTERN = 0x5A


def guarded(nbytes, device="cuda"):
    """(whole buffer, uint8 view of the payload); the payload is 256-byte aligned."""
    whole = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=device)
    return whole, whole[GUARD:GUARD + nbytes]


def intact(whole, nbytes):
    h = whole[:GUARD].cpu()
    t = whole[GUARD + nbytes:].cpu()
    return bool(torch.all(h == PATTERN)) and bool(torch.all(t == PATTERN))


@pytest.mark.parametrize("layout_k,quant", [("BSND", False), ("TND", False), ("PA_BSND", False),
                                            ("PA_BSND", True)])
def test_indexer_writes_only_its_buffers(layout_k, quant):
    layout_q = "TND" if layout_k == "TND" else "BSND"
    p, x = synth.make_random(50, layout_q=layout_q, layout_k=layout_k, B=3, S1=37, S2=300, N1=24,
                             sparse_count=96, sparse_mode=3, empty_rows=True, quant=quant,
                             return_value=1)
    d = to_device(x)
    pr = li.make_params(p)
    shape = li.li_output_shape(pr)
    n = int(np.prod(shape))
    iw, ib = guarded(n * 4)
    vw, vb = guarded(n * 4)
    wsn = li.li_workspace_size(pr)
    ww, wb = guarded(wsn)
    idx = ib.view(torch.int32).reshape(shape)
    val = vb.view(torch.float32).reshape(shape)
    li.indexer(pr, d["query"], d["key"], d["weights"], act_seq_q=d.get("act_q"),
               act_seq_k=d.get("act_k"), block_table=d.get("block_table"), q_scale=d.get("q_scale"),
               k_scale=d.get("k_scale"), workspace=wb, out=(idx, val))
    flags = li.li_read_device_status(wb)
    torch.cuda.synchronize()
    assert flags == 0
    assert intact(iw, n * 4) and intact(vw, n * 4), "an output guard band was written"
    assert intact(ww, wsn), "a workspace guard band was written"
    check_against_oracle(p, x, idx.cpu().numpy(), val.cpu().numpy())


@pytest.mark.parametrize("kw", [
    dict(seed=51, B=2, S1=20, S2=200, q_lens=[20, 9], N1=64, K=96, holes=0.3, junk=0.2),
    dict(seed=52, layout_kv="PA_BSND", B=3, S1=4, k_lens=[300, 64, 129], N1=16, K=128, block_size=64),
    dict(seed=53, layout_q="TND", layout_kv="TND", dtype="fp16", B=2, q_lens=[7, 0], k_lens=[50, 20],
         N1=128, K=64),
])
def test_sparse_attention_writes_only_its_buffers(kw):
    p, x = ssfa.make_sfa(**kw)
    d = to_device(x)
    pr = li.make_sfa_params(p)
    nout = p.rows * p.N1 * p.Dv * 2
    nlse = p.rows * p.N1 * 4
    ow, ob = guarded(nout)
    lw, lb = guarded(nlse)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ob.view(d["query"].dtype).reshape(p.rows, p.N1, p.Dv)
    lse = lb.view(torch.float32).reshape(p.rows, p.N1)
    li.li_sparse_attention(pr, d["query"], d["key"], d["value"], d["sparse_indices"], d.get("act_q"),
                           d.get("act_k"), d.get("block_table"), out, lse, st)
    torch.cuda.synchronize()
    assert intact(ow, nout) and intact(lw, nlse), "a guard band was written"
    ref = osfa.run(p, x)
    u = 2.0 ** -9 if p.dtype == "bf16" else 2.0 ** -12
    vmax = float(x["value"].float().abs().max())
    got = out.float().cpu().numpy()
    assert np.all(np.abs(got - ref["out"]) <= 2 * u * vmax + 2 * u * np.abs(ref["out"]) + 1e-6)


def test_topk_stage_writes_only_its_buffers():
    g = torch.Generator().manual_seed(54)
    rows, ld, k = 37, 300, 64
    scores = torch.randn(rows, ld, generator=g).cuda()
    lens = torch.randint(0, ld + 1, (rows,), generator=g).to(torch.int32).cuda()
    iw, ib = guarded(rows * k * 4)
    vw, vb = guarded(rows * k * 4)
    li.li_topk(scores, ld, lens, rows, k, ib.view(torch.int32), vb.view(torch.float32))
    torch.cuda.synchronize()
    assert intact(iw, rows * k * 4) and intact(vw, rows * k * 4)
    idx = ib.view(torch.int32).reshape(rows, k).cpu().numpy()
    for r in range(rows):
        n = int(lens[r])
        m = min(n, k)
        assert np.all(idx[r, m:] == -1)
        assert len(set(idx[r, :m].tolist())) == m and (m == 0 or idx[r, :m].max() < n)
