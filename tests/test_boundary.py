"""Host-side tests of the C-ABI boundary (no GPU needed, no kernel launched).

* libli.so loads and exports every entry point include/li.h declares;
* li_output_shape follows the pages' output-shape rule on the shapes the
  pages print (tests/golden/output_shapes.json);
* argument checks reject what the pages' constraints forbid, before anything
  touches a device;
* the oracle and the CUDA library share no source.
"""
from __future__ import annotations

import ctypes
import subprocess
import json
import os
import re

import pytest
import torch

import sparse_attention_top_n1_b200 as li
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 1 << 20          # a 16-byte aligned fake pointer; never dereferenced in these tests


def header_entry_points():
    src = open(os.path.join(ROOT, "include", "li.h")).read()
    return re.findall(r"LI_API\s+[\w\s\*]+?\b(li_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    names = header_entry_points()
    assert len(names) >= 9
    L = li.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(li.EXPORTS)


def test_params_struct_matches_header_layout(tmp_path):
    """The binding's li_params mirror has the C header's size and offsets
    (checked by compiling a probe against include/li.h with the host C compiler)."""
    fields = [name for name, _ in li.Params._fields_]
    src = tmp_path / "probe.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"li.h\"\n"
                   "int main(void) {\n  printf(\"%zu\\n\", sizeof(li_params));\n" +
                   "".join('  printf("%%zu\\n", offsetof(li_params, %s));\n' % f for f in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "probe"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    out = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    assert out[0] == ctypes.sizeof(li.Params)
    for f, off in zip(fields, out[1:]):
        assert getattr(li.Params, f).offset == off, f


@pytest.mark.parametrize("case", json.load(open(os.path.join(ROOT, "tests", "golden",
                                                             "output_shapes.json")))["cases"])
def test_output_shape_golden(case):
    pr = li.make_params(**case["params"])
    assert list(li.li_output_shape(pr)) == case["sparse_indices"]
    vals = list(li.li_output_shape(pr)) if pr.return_value else [0]
    assert vals == case["sparse_values"]


def test_workspace_size_covers_score_rows():
    p, _ = synth.make_dsa_prefill(S=8192)
    n = li.li_workspace_size(li.make_params(p))
    assert n >= 8192 * 8192 * 4
    p2, _ = synth.make_paged_decode(B=64)
    n2 = li.li_workspace_size(li.make_params(p2))
    assert n2 >= 64 * p2.max_seqlen_k * 4
    assert n2 < 64 * 65536 * 4 + (1 << 20)


def _base(**kw):
    d = dict(layout_q="BSND", layout_k="BSND", dtype_qk="bf16", dtype_w="bf16", B=2, S1=8,
             S2=64, N1=8, N2=1, D=128, sparse_count=16, sparse_mode=3, return_value=0)
    d.update(kw)
    return li.make_params(**d)


BAD = [
    (dict(B=0), li.STATUS_NAMES[2]),                                   # empty tensor
    (dict(S1=0), "LI_ERR_SHAPE"),
    (dict(N2=2), "LI_ERR_SHAPE"),
    (dict(N1=0), "LI_ERR_SHAPE"),
    (dict(N1=65), "LI_ERR_SHAPE"),
    (dict(D=96), "LI_ERR_SHAPE"),
    (dict(sparse_count=0), "LI_ERR_SHAPE"),
    (dict(sparse_count=8193), "LI_ERR_SHAPE"),
    (dict(sparse_mode=1), "LI_ERR_SHAPE"),
    (dict(pre_tokens=5), "LI_ERR_SHAPE"),
    (dict(next_tokens=0), "LI_ERR_SHAPE"),
    (dict(layout_q="TND", layout_k="BSND", T1=8, T2=64), "LI_ERR_LAYOUT"),
    (dict(layout_k="TND", T2=64), "LI_ERR_LAYOUT"),
    (dict(layout_k="PA_BSND", num_blocks=4, block_size=8, max_blocks_per_seq=8), "LI_ERR_SHAPE"),
    (dict(layout_k="PA_BSND", num_blocks=4, block_size=1040, max_blocks_per_seq=1), "LI_ERR_SHAPE"),
    (dict(layout_k="PA_BSND", num_blocks=4, block_size=40, max_blocks_per_seq=2), "LI_ERR_SHAPE"),
    (dict(layout_k="PA_BSND", num_blocks=0, block_size=64, max_blocks_per_seq=2), "LI_ERR_SHAPE"),
    (dict(dtype_qk="fp32"), "LI_ERR_DTYPE"),
    (dict(dtype_qk="e4m3"), "LI_ERR_DTYPE"),
    (dict(dtype_w="int8"), "LI_ERR_DTYPE"),
    (dict(init_num=-1), "LI_ERR_SHAPE"),
    (dict(cmp_ratio=3), "LI_ERR_SHAPE"),
    (dict(cmp_ratio=256), "LI_ERR_SHAPE"),
    (dict(init_num=10, local_num=7, sparse_count=16), "LI_ERR_SHAPE"),
    (dict(return_value=2), "LI_ERR_SHAPE"),
]


@pytest.mark.parametrize("kw,err", BAD)
def test_indexer_rejects_before_launch(kw, err):
    pr = _base(**kw)
    st = li.lib().li_indexer(ctypes.byref(pr), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None,
                             FAKE, 1 << 40, None)
    assert li.STATUS_NAMES[st] == err, li.li_last_error()
    assert li.li_last_launch_count() == 0
    assert li.li_last_error()


def test_quant_checks():
    L = li.lib()
    pr = _base(dtype_qk="bf16")
    st = L.li_quant_indexer(ctypes.byref(pr), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                            FAKE, None, FAKE, 1 << 40, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_DTYPE"
    pr = _base(dtype_qk="int8", D=64)
    st = L.li_quant_indexer(ctypes.byref(pr), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                            FAKE, None, FAKE, 1 << 40, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_SHAPE"
    pr = _base(dtype_qk="int8", dtype_scale="bf16")
    st = L.li_quant_indexer(ctypes.byref(pr), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                            FAKE, None, FAKE, 1 << 40, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_DTYPE"
    pr = _base(dtype_qk="e4m3", D=64)
    st = L.li_quant_indexer(ctypes.byref(pr), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                            FAKE, None, FAKE, 1 << 40, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_SHAPE"
    pr = _base(dtype_qk="e4m3")
    st = L.li_quant_indexer(ctypes.byref(pr), FAKE, FAKE, FAKE, None, FAKE, None, None, None,
                            FAKE, None, FAKE, 1 << 40, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_NULL"


def test_pointer_and_workspace_checks():
    L = li.lib()
    pr = _base()
    args = [FAKE, FAKE, FAKE, None, None, None, FAKE, None, FAKE, 1 << 40, None]
    # missing sparse_values with return_value=1
    pr1 = _base(return_value=1)
    assert li.STATUS_NAMES[L.li_indexer(ctypes.byref(pr1), *args)] == "LI_ERR_NULL"
    # sparse_values given with return_value=0
    a2 = list(args)
    a2[7] = FAKE
    assert li.STATUS_NAMES[L.li_indexer(ctypes.byref(pr), *a2)] == "LI_ERR_NULL"
    # TND without prefix sums
    prt = _base(layout_q="TND", layout_k="TND", T1=8, T2=64)
    assert li.STATUS_NAMES[L.li_indexer(ctypes.byref(prt), *args)] == "LI_ERR_NULL"
    # PA without block table
    prp = _base(layout_k="PA_BSND", num_blocks=4, block_size=64, max_blocks_per_seq=2)
    a3 = list(args)
    a3[4] = FAKE
    assert li.STATUS_NAMES[L.li_indexer(ctypes.byref(prp), *a3)] == "LI_ERR_NULL"
    # misaligned query
    a4 = list(args)
    a4[0] = FAKE + 8
    assert li.STATUS_NAMES[L.li_indexer(ctypes.byref(pr), *a4)] == "LI_ERR_SHAPE"
    # workspace too small / misaligned
    a5 = list(args)
    a5[9] = 16
    assert li.STATUS_NAMES[L.li_indexer(ctypes.byref(pr), *a5)] == "LI_ERR_WORKSPACE"
    a6 = list(args)
    a6[8] = FAKE + 16
    assert li.STATUS_NAMES[L.li_indexer(ctypes.byref(pr), *a6)] == "LI_ERR_WORKSPACE"


def test_topk_checks():
    L = li.lib()
    assert li.STATUS_NAMES[L.li_topk(FAKE, 6, None, 2, 4, FAKE, None, None)] == "LI_ERR_SHAPE"
    assert li.STATUS_NAMES[L.li_topk(FAKE, 8, None, 2, 0, FAKE, None, None)] == "LI_ERR_SHAPE"
    assert li.STATUS_NAMES[L.li_topk(FAKE, 8, None, 2, 8193, FAKE, None, None)] == "LI_ERR_SHAPE"
    assert li.STATUS_NAMES[L.li_topk(None, 8, None, 2, 4, FAKE, None, None)] == "LI_ERR_NULL"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error():
    pr = _base()
    st = li.lib().li_indexer(ctypes.byref(pr), FAKE, FAKE, FAKE, None, None, None, FAKE, None,
                             FAKE, 1 << 40, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_CUDA"


def test_oracle_and_cuda_path_share_no_source():
    """The oracle includes nothing of the CUDA library and vice versa."""
    orc = open(os.path.join(ROOT, "oracle", "li_oracle.c")).read()
    assert "li.h" not in orc and "csrc" not in orc
    for inc in re.findall(r'#include\s+[<"]([^>"]+)[>"]', orc):
        assert inc in ("math.h", "stdint.h", "stdlib.h", "string.h", "omp.h"), inc
    csrc = os.path.join(ROOT, "sparse_attention_top_n1_b200", "csrc")
    for f in os.listdir(csrc):
        txt = open(os.path.join(csrc, f)).read()
        assert "oracle" not in txt.lower(), f
    pkg = open(os.path.join(ROOT, "sparse_attention_top_n1_b200", "__init__.py")).read()
    assert "import oracle" not in pkg and "from oracle" not in pkg
    for f in ("sfa.py", "__init__.py"):
        src = open(os.path.join(ROOT, "oracle", f)).read()
        assert "sparse_attention_top_n1_b200" not in src, f
        assert "csrc" not in src, f
    for f in os.listdir(os.path.join(ROOT, "synth")):
        if f.endswith(".py"):
            src = open(os.path.join(ROOT, "synth", f)).read()
            assert "import oracle" not in src and "sparse_attention_top_n1_b200" not in src, f


# ---------------------------------------------------------------- sparse attention

def test_sfa_params_struct_matches_header_layout(tmp_path):
    fields = [name for name, _ in li.SfaParams._fields_]
    src = tmp_path / "probe_sfa.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"li.h\"\n"
                   "int main(void) {\n  printf(\"%zu\\n\", sizeof(li_sfa_params));\n" +
                   "".join('  printf("%%zu\\n", offsetof(li_sfa_params, %s));\n' % f for f in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "probe_sfa"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    out = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    assert out[0] == ctypes.sizeof(li.SfaParams)
    for f, off in zip(fields, out[1:]):
        assert getattr(li.SfaParams, f).offset == off, f


def _sfa_base(**kw):
    f = dict(layout_q="BSND", layout_kv="BSND", dtype="bf16", B=2, S1=16, S2=64, N1=64, D=128,
             Dv=128, sparse_count=32)
    f.update(kw)
    return li.make_sfa_params(**f)


@pytest.mark.parametrize("kw,err", [
    (dict(N1=48), "LI_ERR_SHAPE"), (dict(N1=256), "LI_ERR_SHAPE"),
    (dict(D=64), "LI_ERR_UNSUPPORTED"), (dict(Dv=256), "LI_ERR_UNSUPPORTED"),
    (dict(dtype="fp32"), "LI_ERR_DTYPE"), (dict(dtype="e4m3"), "LI_ERR_DTYPE"),
    (dict(sparse_count=0), "LI_ERR_SHAPE"), (dict(sparse_count=65537), "LI_ERR_SHAPE"),
    (dict(softmax_scale=-1.0), "LI_ERR_SHAPE"), (dict(softmax_scale=float("inf")), "LI_ERR_SHAPE"),
    (dict(reserved=1), "LI_ERR_SHAPE"), (dict(layout_kv="TND"), "LI_ERR_LAYOUT"),
    (dict(layout_q="PA_BSND"), "LI_ERR_LAYOUT"), (dict(B=0), "LI_ERR_SHAPE"),
    (dict(S1=-1), "LI_ERR_SHAPE"), (dict(B=70000, S2=70000), "LI_ERR_SHAPE"),
])
def test_sfa_rejects_before_launch(kw, err):
    pr = _sfa_base(**kw)
    st = li.lib().li_sparse_attention(ctypes.byref(pr), FAKE, FAKE, FAKE, FAKE, None, None, None,
                                      FAKE, None, None, None)
    assert li.STATUS_NAMES[st] == err, li.li_last_error()


def test_sfa_pointer_checks():
    L = li.lib()
    pr = _sfa_base()
    call = lambda q=FAKE, k=FAKE, v=FAKE, i=FAKE, aq=None, ak=None, bt=None, o=FAKE, lse=None, p=pr, st=None: \
        li.STATUS_NAMES[L.li_sparse_attention(ctypes.byref(p), q, k, v, i, aq, ak, bt, o, lse, st, None)]
    assert call(q=None) == "LI_ERR_NULL"
    assert call(v=None) == "LI_ERR_NULL"
    assert call(i=None) == "LI_ERR_NULL"
    assert call(o=None) == "LI_ERR_NULL"
    assert call(k=FAKE + 8) == "LI_ERR_SHAPE"           # 16-byte alignment
    assert call(o=FAKE + 4) == "LI_ERR_SHAPE"
    assert call(st=FAKE + 2) == "LI_ERR_SHAPE"           # the status word takes atomics: 4-byte aligned
    assert call(lse=FAKE + 2) == "LI_ERR_SHAPE"
    tnd = _sfa_base(layout_q="TND", layout_kv="TND", T1=8, T2=8)
    assert call(p=tnd) == "LI_ERR_NULL"                  # TND needs the prefix sums
    pa = _sfa_base(layout_kv="PA_BSND", num_blocks=4, block_size=16, max_blocks_per_seq=2)
    assert call(p=pa, ak=FAKE) == "LI_ERR_NULL"          # PA needs the block table
    assert call(p=_sfa_base(S1=0)) == "LI_OK"            # nothing to do, nothing launched
    assert li.li_last_launch_count() == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_sfa_valid_call_without_device_reports_cuda_error():
    pr = _sfa_base()
    st = li.lib().li_sparse_attention(ctypes.byref(pr), FAKE, FAKE, FAKE, FAKE, None, None, None,
                                      FAKE, None, None, None)
    assert li.STATUS_NAMES[st] == "LI_ERR_CUDA"


def test_noalloc_scratch_size_matches_the_header():
    import re
    hdr = open(os.path.join(ROOT, "include", "li.h")).read()
    m = re.search(r"#define LI_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m, "LI_NOALLOC_SCRATCH_BYTES not found"
    assert li.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
