"""GPU parity of the two plain entry points whose argument lists the method's
interface fixes (attn_varlen_fwd and attn_paged_decode), called through the C
ABI with raw device pointers -- not through the binding, which uses their
``_ex`` forms -- and compared with the fp64 oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import assert_close_bf16, assert_close_lse, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    import attention_varlen_gqa_b200 as A
    A.attn_get_last_device_error()
    return A


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("with_lse", [True, False])
def test_plain_varlen_fwd_tiny(A, with_lse):
    """The tiny varlen prefill (lengths {37, 64}, h_q 4, h_kv 2, d 64, causal)."""
    data = W.tiny_prefill(seed=0)
    q, k, v = (dev_bf16(data[n]) for n in ("q", "k", "v"))
    cu_q, cu_k = dev_i32(data["cu_seqlens_q"]), dev_i32(data["cu_seqlens_k"])
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda") if with_lse else None
    rc = A.lib.attn_varlen_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_q), _ptr(cu_k), 2, q.shape[0], k.shape[0],
                               data["max_q"], data["max_k"], 4, 2, 64, 1, float(data["scale"]), _ptr(out),
                               _ptr(lse), _stream())
    assert rc == 0
    assert A.attn_get_last_device_error() == 0
    ro, rl, _ = oracle.varlen_attention(data["q"], data["k"], data["v"], data["cu_seqlens_q"],
                                        data["cu_seqlens_k"], 4, 2, True, data["scale"])
    assert_close_bf16(out, ro)
    if with_lse:
        assert_close_lse(lse, rl)


def test_plain_varlen_fwd_noncausal_ragged(A):
    """s_q != s_k, an empty sequence and several 128-row blocks, non-causal."""
    data = W.varlen_prefill([130, 0, 77, 300], [64, 5, 0, 513], h_q=8, h_kv=2, d=128, causal=False, seed=3)
    q, k, v = (dev_bf16(data[n]) for n in ("q", "k", "v"))
    cu_q, cu_k = dev_i32(data["cu_seqlens_q"]), dev_i32(data["cu_seqlens_k"])
    out = torch.full_like(q, float("nan"))
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    rc = A.lib.attn_varlen_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_q), _ptr(cu_k), 4, q.shape[0], k.shape[0],
                               data["max_q"], data["max_k"], 8, 2, 128, 0, float(data["scale"]), _ptr(out),
                               _ptr(lse), _stream())
    assert rc == 0
    assert A.attn_get_last_device_error() == 0
    ro, rl, _ = oracle.varlen_attention(data["q"], data["k"], data["v"], data["cu_seqlens_q"],
                                        data["cu_seqlens_k"], 8, 2, False, data["scale"])
    assert_close_bf16(out, ro)
    assert_close_lse(lse, rl)


DECODE_LENS = [0, 1, 15, 16, 17, 33, 127, 128, 129, 1000, 4097]


def _decode_call(A, t, data, thr, workspace):
    q = t["q"]
    batch, h_q, d = q.shape
    out = torch.full_like(q, float("nan"))
    lse = torch.full((batch, h_q), float("nan"), dtype=torch.float32, device="cuda")
    ws_bytes = 0 if workspace is None else workspace.numel()
    rc = A.lib.attn_paged_decode(_ptr(q), _ptr(t["k_cache"]), _ptr(t["v_cache"]), _ptr(t["block_table"]),
                                 _ptr(t["seq_lens"]), batch, data["num_pages"], data["max_pages_per_seq"], 16,
                                 h_q, data["h_kv"], d, float(thr), float(data["scale"]), _ptr(out), _ptr(lse),
                                 _ptr(workspace), ws_bytes, _stream())
    return rc, out, lse


@pytest.mark.parametrize("thr,schedule", [(0.0, "split"), (0.1, "split"), (0.1, "sequential")])
def test_plain_paged_decode_ragged(A, thr, schedule):
    """Ragged decode lengths (empty, single-token, page and tile edges), dense
    split-KV with its workspace, and skip mode with a workspace (two passes)
    or without one (one sequential split)."""
    data = W.paged_decode(DECODE_LENS, h_q=8, h_kv=2, d=128, seed=11)
    t = {n: dev_bf16(data[n]) for n in ("q", "k_cache", "v_cache")}
    t["block_table"] = dev_i32(data["block_table"])
    t["seq_lens"] = dev_i32(data["seq_lens"])
    ws = None
    if schedule == "split":
        need = A.attn_paged_decode_workspace_size(len(DECODE_LENS), 8, 128, data["max_pages_per_seq"], thr)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    rc, out, lse = _decode_call(A, t, data, thr, ws)
    assert rc == 0
    assert A.attn_get_last_device_error() == 0
    ro, rl, rec = oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"], data["block_table"],
                                      data["seq_lens"], 8, 2, data["scale"], threshold=thr)
    if thr > 0:
        # no unit of this draw lies in the ambiguity band of the decision test
        amb = (rec.max_ratio > thr * (1 - 1e-3)) & (rec.max_ratio < thr * (1 + 1e-3)) & rec.visited
        assert not amb.any()
    assert_close_bf16(out, ro)
    assert_close_lse(lse, rl)
    # the empty sequence: zeros and -inf
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


def test_plain_paged_decode_workspace_errors(A):
    data = W.paged_decode([40, 50], h_q=4, h_kv=2, d=64, seed=1)
    t = {n: dev_bf16(data[n]) for n in ("q", "k_cache", "v_cache")}
    t["block_table"] = dev_i32(data["block_table"])
    t["seq_lens"] = dev_i32(data["seq_lens"])
    need = A.attn_paged_decode_workspace_size(2, 4, 64)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    assert _decode_call(A, t, data, 0.0, None)[0] == -9      # dense mode needs a workspace
    assert _decode_call(A, t, data, 0.0, small)[0] == -9
