"""GPU check of attn_paged_decode_static, the decode entry point for callers
that cannot allocate device memory (for example a serving runtime whose
memory pool owns the whole GPU, or a plug-in interface without a workspace
argument).  It keeps the split-KV partials in the library's own device
scratch array instead of a caller workspace.

The entry point is called through the C ABI (ctypes, raw pointers) twice in a
row on different inputs, and each result is compared with what
attn_paged_decode (caller-provided workspace) returns for the same inputs,
within the bf16 tolerance every parity test here uses.  This file is
collected last so that a failure here leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from tests.parity import assert_close_bf16, assert_close_lse, dev_i32

pytestmark = pytest.mark.gpu

TOO_LARGE = -13


@pytest.fixture(scope="module")
def A():
    import attention_varlen_gqa_b200 as A
    return A


def _device_inputs(data):
    t = {}
    for n in ("q", "k_cache", "v_cache"):
        x = data[n]
        if not isinstance(x, torch.Tensor):
            x = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
        t[n] = x
    t["block_table"] = dev_i32(data["block_table"])
    t["seq_lens"] = dev_i32(data["seq_lens"])
    return t


def _call_static(A, t, out, lse, scale):
    """attn_paged_decode_static through the C ABI with raw device pointers."""
    q, kc = t["q"], t["k_cache"]
    batch, h_q, d = q.shape
    num_pages, page, h_kv, _ = kc.shape
    ptr = lambda x: ctypes.c_void_p(x.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return A.lib.attn_paged_decode_static(
        ptr(q), ptr(kc), ptr(t["v_cache"]), ptr(t["block_table"]), ptr(t["seq_lens"]), batch, num_pages,
        t["block_table"].shape[1], page, h_q, h_kv, d, 0.0, scale, ptr(out), ptr(lse), stream)


def test_static_scratch_matches_workspace_path_twice(A):
    first = W.dense_decode(seed=0, where="device")                       # batch 64, h 32/8, d 128
    second = W.paged_decode([0, 1, 17, 129, 3000, 9000], h_q=8, h_kv=2, d=64, seed=5)
    results = []
    for data in (first, second):
        t = _device_inputs(data)
        out = torch.empty_like(t["q"])
        lse = torch.empty(t["q"].shape[:2], dtype=torch.float32, device="cuda")
        assert _call_static(A, t, out, lse, float(data["scale"])) == 0
        results.append((data, t, out, lse))
    torch.cuda.synchronize()
    assert A.attn_get_last_device_error() == 0
    # compare both results, taken back to back, with the workspace entry point
    for data, t, out, lse in results:
        ref_out, ref_lse = A.attn_paged_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                               t["seq_lens"], scale=float(data["scale"]))
        torch.cuda.synchronize()
        assert_close_bf16(out, ref_out.float().cpu().double().numpy())
        assert_close_lse(lse, ref_lse.cpu().double().numpy())


def test_static_scratch_rejects_oversized_shapes(A):
    need = A.attn_paged_decode_workspace_size(4096, 32, 128)
    assert need > A.STATIC_WORKSPACE_BYTES
    fake = ctypes.c_void_p(1 << 20)
    rc = A.lib.attn_paged_decode_static(fake, fake, fake, fake, fake, 4096, 16, 1, 16, 32, 8, 128,
                                        0.0, 0.1, fake, None, None)
    assert rc == TOO_LARGE
