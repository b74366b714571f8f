"""The C-ABI library loads and exports what include/attn.h declares; host-side
argument checks return their error codes (no GPU needed: every call below is
rejected before any CUDA call)."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def A():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_attn_build", os.path.join(ROOT, "attention_varlen_gqa_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import attention_varlen_gqa_b200
    return attention_varlen_gqa_b200


def header_functions():
    with open(os.path.join(ROOT, "include", "attn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(A):
    names = header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(A.lib, n), f"{n} declared in attn.h but not exported"
    assert set(names) == set(A.EXPORTS), "binding and header disagree"


def test_no_torch_in_signatures():
    with open(os.path.join(ROOT, "include", "attn.h")) as f:
        text = f.read()
    code = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    for word in ("torch", "at::", "Tensor", "c10"):
        assert word not in code, word


def test_config(A):
    cfg = A.attn_get_config()
    assert cfg == dict(prefill_block_m=128, prefill_block_n=128, skip_tile=32, decode_splits=32,
                       decode_split_tile=128, decode_page_size=16, smallseq_max_s_kv=16)
    assert A.lib.attn_get_config(None) == -1


def test_status_strings(A):
    assert A.lib.attn_status_string(0) == b"ATTN_OK"
    assert A.lib.attn_status_string(-5) == b"ATTN_E_THRESHOLD"
    assert A.lib.attn_status_string(-99) == b"ATTN_E_UNKNOWN"


def test_workspace_query(A):
    def align(x):
        return (x + 255) // 256 * 256
    for B, h, d in ((64, 32, 128), (1, 1, 64), (7, 3, 128)):
        rows = B * h * 32
        assert A.attn_paged_decode_workspace_size(B, h, d) == align(rows * d * 4) + align(rows * 8)
        # skip mode, two passes: + scores (key slots rounded up to 64), tile maxima, split maxima
        for maxp in (1, 5, 2048):
            slots = (maxp * 16 + 63) // 64 * 64
            tiles = (maxp * 16 + 31) // 32
            want = align(rows * d * 4) + align(rows * 8) + align(B * h * slots * 4) + align(B * h * tiles * 4) \
                + align(rows * 4)
            assert A.lib.attn_paged_decode_workspace_size_ex(B, h, d, maxp, 0.1) == want
            assert A.lib.attn_paged_decode_workspace_size_ex(B, h, d, maxp, 0.0) == \
                A.attn_paged_decode_workspace_size(B, h, d)


FAKE = 1 << 20          # a 16-byte aligned fake address, never dereferenced


def varlen(A, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cq=FAKE, ck=FAKE, batch=2, tq=10, tk=10, mq=5, mk=5, hq=4, hkv=2,
             d=64, causal=1, scale=0.125, thr=0.0, mask=None, counts=None, out=FAKE, lse=None, stream=None)
    a.update(kw)
    return A.lib.attn_varlen_fwd_ex(a["q"], a["k"], a["v"], a["cq"], a["ck"], a["batch"], a["tq"], a["tk"],
                                    a["mq"], a["mk"], a["hq"], a["hkv"], a["d"], a["causal"], a["scale"],
                                    a["thr"], a["mask"], a["counts"], a["out"], a["lse"], a["stream"])


def test_varlen_argument_errors(A):
    assert varlen(A, hq=3) == -3
    assert varlen(A, hkv=0) == -3
    assert varlen(A, d=96) == -4
    assert varlen(A, thr=-0.1) == -5
    assert varlen(A, thr=1.5) == -5
    assert varlen(A, thr=float("nan")) == -5
    assert varlen(A, scale=float("inf")) == -10
    assert varlen(A, scale=0.0) == -10
    assert varlen(A, scale=-0.5) == -10
    assert varlen(A, q=None) == -1
    assert varlen(A, out=None) == -1
    assert varlen(A, k=FAKE + 8) == -2
    assert varlen(A, mq=0) == -8
    assert varlen(A, batch=-1) == -8
    assert varlen(A, mq=1 << 25, mk=1 << 25) == -13


def paged_prefill(A, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cu=FAKE, sl=FAKE, batch=2, tq=64, mq=32, mk=64, pages=8, maxp=4,
             ps=16, hq=8, hkv=2, d=128, causal=1, scale=0.1, thr=0.0, mask=None, counts=None, out=FAKE, lse=None,
             stream=None)
    a.update(kw)
    return A.lib.attn_paged_prefill(a["q"], a["kc"], a["vc"], a["bt"], a["cu"], a["sl"], a["batch"], a["tq"],
                                    a["mq"], a["mk"], a["pages"], a["maxp"], a["ps"], a["hq"], a["hkv"], a["d"],
                                    a["causal"], a["scale"], a["thr"], a["mask"], a["counts"], a["out"],
                                    a["lse"], a["stream"])


def test_paged_prefill_argument_errors(A):
    assert paged_prefill(A, ps=32) == -6
    assert paged_prefill(A, hq=7) == -3
    assert paged_prefill(A, d=96) == -4
    assert paged_prefill(A, thr=1.5) == -5
    assert paged_prefill(A, scale=0.0) == -10
    assert paged_prefill(A, bt=None) == -1
    assert paged_prefill(A, sl=None) == -1
    assert paged_prefill(A, kc=FAKE + 8) == -2
    assert paged_prefill(A, pages=0) == -8
    assert paged_prefill(A, mq=0) == -8
    assert paged_prefill(A, mq=1 << 25) == -13


def decode(A, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, batch=2, pages=4, maxp=2, ps=16, hq=8, hkv=2, d=128,
             thr=0.0, scale=0.1, mask=None, counts=None, out=FAKE, lse=None, ws=FAKE, wsb=1 << 30, stream=None)
    a.update(kw)
    return A.lib.attn_paged_decode_ex(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["batch"], a["pages"],
                                      a["maxp"], a["ps"], a["hq"], a["hkv"], a["d"], a["thr"], a["scale"],
                                      a["mask"], a["counts"], a["out"], a["lse"], a["ws"], a["wsb"], a["stream"])


def test_decode_argument_errors(A):
    assert decode(A, ps=32) == -6
    assert decode(A, hq=7) == -3
    assert decode(A, hq=64, hkv=2) == -3          # group of 32 > 16
    assert decode(A, d=256) == -4
    assert decode(A, thr=2.0) == -5
    assert decode(A, scale=float("nan")) == -10
    assert decode(A, scale=0.0) == -10
    assert decode(A, bt=None) == -1
    assert decode(A, ws=None) == -9
    assert decode(A, wsb=100) == -9
    assert decode(A, ws=FAKE + 4) == -2
    assert decode(A, pages=0) == -8
    # skip mode: a workspace selects the two-pass schedule and must be large enough
    assert decode(A, thr=0.1, wsb=100) == -9
    assert decode(A, thr=0.1, ws=FAKE + 4) == -2


def smallseq(A, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cu=FAKE, batch=3, tk=9, h=2, d=128, maxs=4, scale=0.1, out=FAKE, w=None,
             stream=None)
    a.update(kw)
    return A.lib.attn_smallseq_fwd(a["q"], a["k"], a["v"], a["cu"], a["batch"], a["tk"], a["h"], a["d"],
                                   a["maxs"], a["scale"], a["out"], a["w"], a["stream"])


def test_smallseq_argument_errors(A):
    assert smallseq(A, maxs=0) == -7
    assert smallseq(A, maxs=17) == -7
    assert smallseq(A, d=32) == -4
    assert smallseq(A, h=0) == -3
    assert smallseq(A, cu=None) == -1
    assert smallseq(A, w=FAKE + 1) == -2
    assert smallseq(A, scale=-math.inf) == -10


def smallseq_bwd(A, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, do=FAKE, w=FAKE, cu=FAKE, batch=3, tk=9, h=2, d=128, maxs=4, scale=0.1,
             dq=FAKE, dk=FAKE, dv=FAKE, stream=None)
    a.update(kw)
    return A.lib.attn_smallseq_bwd(a["q"], a["k"], a["v"], a["do"], a["w"], a["cu"], a["batch"], a["tk"], a["h"],
                                   a["d"], a["maxs"], a["scale"], a["dq"], a["dk"], a["dv"], a["stream"])


def test_smallseq_bwd_argument_errors(A):
    assert smallseq_bwd(A, maxs=0) == -7
    assert smallseq_bwd(A, maxs=17) == -7
    assert smallseq_bwd(A, d=32) == -4
    assert smallseq_bwd(A, h=0) == -3
    assert smallseq_bwd(A, batch=-1) == -8
    assert smallseq_bwd(A, w=None) == -1
    assert smallseq_bwd(A, do=None) == -1
    assert smallseq_bwd(A, dk=None) == -1
    assert smallseq_bwd(A, w=FAKE + 1) == -2
    assert smallseq_bwd(A, dq=FAKE + 8) == -2
    assert smallseq_bwd(A, scale=0.0) == -10


def varlen_bwd(A, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, do=FAKE, lse=FAKE, cq=FAKE, ck=FAKE, batch=2, tq=10, tk=10, mq=5, mk=5,
             hq=4, hkv=2, d=64, causal=1, scale=0.125, dq=FAKE, dk=FAKE, dv=FAKE, ws=FAKE, wsb=1 << 20, stream=None)
    a.update(kw)
    return A.lib.attn_varlen_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["cq"], a["ck"], a["batch"],
                                 a["tq"], a["tk"], a["mq"], a["mk"], a["hq"], a["hkv"], a["d"], a["causal"],
                                 a["scale"], a["dq"], a["dk"], a["dv"], a["ws"], a["wsb"], a["stream"])


def test_varlen_bwd_argument_errors(A):
    assert varlen_bwd(A, hq=3) == -3
    assert varlen_bwd(A, d=96) == -4
    assert varlen_bwd(A, scale=0.0) == -10
    assert varlen_bwd(A, batch=-1) == -8
    assert varlen_bwd(A, lse=None) == -1
    assert varlen_bwd(A, do=None) == -1
    assert varlen_bwd(A, dk=None) == -1
    assert varlen_bwd(A, dq=FAKE + 8) == -2
    assert varlen_bwd(A, lse=FAKE + 2) == -2
    assert varlen_bwd(A, ws=None) == -9
    assert varlen_bwd(A, wsb=8) == -9
    assert varlen_bwd(A, mk=1 << 25) == -13
    assert A.lib.attn_varlen_bwd_workspace_size(10, 4) == 256
    assert A.lib.attn_varlen_bwd_workspace_size(1000, 32) == 1000 * 32 * 4


def static_decode(A, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, batch=2, pages=4, maxp=2, ps=16, hq=8, hkv=2, d=128,
             thr=0.0, scale=0.1, out=FAKE, lse=None, stream=None)
    a.update(kw)
    return A.lib.attn_paged_decode_static(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["batch"], a["pages"],
                                          a["maxp"], a["ps"], a["hq"], a["hkv"], a["d"], a["thr"], a["scale"],
                                          a["out"], a["lse"], a["stream"])


@pytest.mark.parametrize("bad", [
    dict(ps=32), dict(hq=7), dict(hq=0), dict(hkv=0), dict(hq=64, hkv=2), dict(d=256), dict(d=0),
    dict(thr=2.0), dict(thr=-1e-3), dict(thr=float("nan")), dict(scale=float("nan")), dict(scale=0.0),
    dict(q=None), dict(kc=None), dict(vc=None), dict(bt=None), dict(sl=None), dict(out=None),
    dict(q=FAKE + 8), dict(kc=FAKE + 2), dict(vc=FAKE + 4), dict(out=FAKE + 8), dict(pages=0), dict(maxp=0),
    dict(batch=-1), dict(maxp=1 << 27)])
def test_static_decode_argument_errors_match_workspace_entry(A, bad):
    """attn_paged_decode_static checks its arguments like attn_paged_decode_ex
    and returns the same codes (all before any CUDA call)."""
    rc = static_decode(A, **bad)
    assert rc < 0
    assert rc == decode(A, **bad)


def test_static_decode_too_large_after_argument_checks(A):
    # batch * h_q = 3025 at d = 128 is one row over the 48 MiB scratch array
    assert A.lib.attn_paged_decode_workspace_size(3024, 1, 128) <= 48 << 20
    assert A.lib.attn_paged_decode_workspace_size(3025, 1, 128) > 48 << 20
    assert A.lib.attn_paged_decode_workspace_size(5957, 1, 64) <= 48 << 20
    assert A.lib.attn_paged_decode_workspace_size(5958, 1, 64) > 48 << 20
    assert static_decode(A, batch=3025, hq=1, hkv=1) == -13
    assert static_decode(A, batch=5958, hq=1, hkv=1, d=64) == -13
    # a bad argument is reported as such even when the shape is too large
    assert static_decode(A, batch=3025, hq=1, hkv=1, d=96) == -4
    assert static_decode(A, batch=3025, hq=1, hkv=1, q=None) == -1


def decode_qdq(A, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, batch=2, pages=4, maxp=2, ps=16, hq=8, hkv=2, d=128,
             thr=0.0, scale=0.1, pf=1, pa=1.0, vf=1, va=1.0, mask=None, counts=None, out=FAKE, lse=None, ws=FAKE,
             wsb=1 << 30, stream=None)
    a.update(kw)
    return A.lib.attn_paged_decode_qdq(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["batch"], a["pages"],
                                       a["maxp"], a["ps"], a["hq"], a["hkv"], a["d"], a["thr"], a["scale"], a["pf"],
                                       a["pa"], a["vf"], a["va"], a["mask"], a["counts"], a["out"], a["lse"], a["ws"],
                                       a["wsb"], a["stream"])


def test_decode_qdq_argument_errors(A):
    assert decode_qdq(A, pf=2) == -14
    assert decode_qdq(A, vf=-1) == -14
    for bad in (0.0, -1.0, float("nan"), float("inf"), 2.0 ** 70, 2.0 ** -70):
        assert decode_qdq(A, pa=bad) == -14
        assert decode_qdq(A, va=bad) == -14
    # an unused amax is not checked
    assert decode_qdq(A, pf=0, pa=float("nan"), wsb=100) == -9
    # the decode's own checks come first
    assert decode_qdq(A, hq=7) == -3
    assert decode_qdq(A, d=96) == -4
    assert decode_qdq(A, thr=1.5) == -5
    # with QDQ on, a workspace selects the two-pass skip schedule at any threshold
    need = A.lib.attn_paged_decode_qdq_workspace_size(2, 8, 128, 2)
    assert need == A.lib.attn_paged_decode_workspace_size_ex(2, 8, 128, 2, 0.5)
    assert need > A.lib.attn_paged_decode_workspace_size(2, 8, 128)
    assert decode_qdq(A, wsb=need - 1) == -9
    assert decode_qdq(A, ws=FAKE + 4) == -2
    assert A.lib.attn_status_string(-14) == b"ATTN_E_QDQ"
