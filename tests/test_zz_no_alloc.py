"""GPU check of attn_paged_decode_static, the decode entry point for callers
that cannot allocate device memory (for example a serving runtime whose
memory pool owns the whole GPU, or a plug-in interface without a workspace
argument).  It keeps the split-KV partials in the library's own device
scratch array instead of a caller workspace.

The entry point is called through the C ABI (ctypes, raw pointers) twice in a
row on different inputs, and each result is compared with what
attn_paged_decode (caller-provided workspace) returns for the same inputs,
within the bf16 tolerance every parity test here uses.  In skip mode both of
its schedules are checked against the fp64 oracle and, bit for bit, against
attn_paged_decode running the same schedule, each after a dense call has left
its partials in the scratch array: the two-pass schedule inside the array (a
small shape whose workspace fits) and the sequential one (the batch-32 x
32768-key shape, whose two-pass workspace does not fit).  This file is
collected last so that a failure here leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
import oracle
from tests.parity import assert_close_bf16, assert_close_lse, dev_i32, host_bits, unpack_bits

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


def _call_static(A, t, out, lse, scale, thr=0.0):
    """attn_paged_decode_static through the C ABI with raw device pointers."""
    q, kc = t["q"], t["k_cache"]
    batch, h_q, d = q.shape
    num_pages, page, h_kv, _ = kc.shape
    ptr = lambda x: ctypes.c_void_p(x.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return A.lib.attn_paged_decode_static(
        ptr(q), ptr(kc), ptr(t["v_cache"]), ptr(t["block_table"]), ptr(t["seq_lens"]), batch, num_pages,
        t["block_table"].shape[1], page, h_q, h_kv, d, float(thr), scale, ptr(out), ptr(lse), stream)


def _static(A, t, scale, thr):
    out = torch.empty_like(t["q"])
    lse = torch.empty(t["q"].shape[:2], dtype=torch.float32, device="cuda")
    assert _call_static(A, t, out, lse, scale, thr) == 0
    return out, lse


def _fill_scratch_with_dense_partials(A):
    """A dense call: leaves split partials of another shape in the scratch array."""
    other = W.paged_decode([3000, 700, 5000, 64], h_q=32, h_kv=8, d=128, seed=9)
    t = _device_inputs(other)
    _static(A, t, float(other["scale"]), 0.0)


def _peaked(lens, h_q=8, h_kv=2, d=128, seed=0):
    """Keys of a few tiles per sequence aligned with the group's summed query,
    so that the skip sets are neither empty nor everything."""
    data = W.paged_decode(lens, h_q=h_q, h_kv=h_kv, d=d, seed=seed)
    qf = W.bf16_bits_to_f32(data["q"]).astype(np.float64)
    kc = W.bf16_bits_to_f32(data["k_cache"])
    bt = data["block_table"]
    G = h_q // h_kv
    for b, L in enumerate(lens):
        pos = np.asarray([p for p in list(range(4)) + list(range(96, 100)) + list(range(L - 40, L - 36))
                          if 0 <= p < L], dtype=np.int64)
        for hk in range(h_kv):
            qs = qf[b, hk * G:(hk + 1) * G].sum(axis=0)
            kc[bt[b, pos // 16], pos % 16, hk] += (4.0 * qs / np.linalg.norm(qs)).astype(np.float32)
    data["k_cache"] = W.f32_to_bf16_bits(kc)
    return data


def _decisions(A, t, data, thr, schedule):
    """attn_paged_decode with a skip mask: its output and decisions."""
    B = t["q"].shape[0]
    kt = -(-t["block_table"].shape[1] * 16 // 32)
    words = -(-(B * data["h_kv"] * kt) // 32)
    mask = torch.zeros(max(words, 1), dtype=torch.int32, device="cuda")
    out, lse = A.attn_paged_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                                   skip_threshold=thr, skip_mask=mask, skip_schedule=schedule)
    bits = unpack_bits(mask, mask.numel() * 32)

    def forced(b_list):
        return {(i, hk): bits[(b * data["h_kv"] + hk) * kt:(b * data["h_kv"] + hk + 1) * kt]
                for i, b in enumerate(b_list) for hk in range(data["h_kv"])}
    return out, lse, forced


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


@pytest.mark.parametrize("thr", [1e-2, 0.1, 0.5])
def test_static_skip_two_pass_in_scratch(A, thr):
    """Skip mode on a shape whose two-pass workspace fits the scratch array:
    the two-pass schedule runs inside it.  Checked against the oracle (with the
    decisions of attn_paged_decode's same schedule) and bit for bit against
    attn_paged_decode with a caller workspace."""
    data = _peaked([1, 31, 33, 200, 700, 2048, 3000])
    need = A.attn_paged_decode_workspace_size(7, 8, 128, data["block_table"].shape[1], thr)
    assert need <= A.STATIC_WORKSPACE_BYTES
    t = _device_inputs(data)
    _fill_scratch_with_dense_partials(A)
    out, lse = _static(A, t, float(data["scale"]), thr)
    ref_out, ref_lse, forced = _decisions(A, t, data, thr, "split")
    torch.cuda.synchronize()
    assert A.attn_get_last_device_error() == 0
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    ro, rl, rec = oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"], data["block_table"],
                                      data["seq_lens"], 8, 2, data["scale"], threshold=thr,
                                      forced_skip=forced(range(7)))
    assert rec.skipped.any() or thr < 0.1
    assert_close_bf16(out, ro)
    assert_close_lse(lse, rl)


@pytest.mark.parametrize("thr", [1e-3, 0.1])
def test_static_skip_sequential_when_too_large(A, thr):
    """Skip mode on batch 32 x 32768 keys (h_q 32, h_kv 8, d 128, sink and
    window peaks), whose two-pass workspace exceeds the scratch array: the
    sequential schedule runs.  Bit for bit equal to attn_paged_decode's
    sequential schedule; 3 sampled sequences against the oracle."""
    data = W.skip_decode(seed=0, where="device")
    need = A.attn_paged_decode_workspace_size(32, 32, 128, data["block_table"].shape[1], thr)
    assert need > A.STATIC_WORKSPACE_BYTES
    t = _device_inputs(data)
    _fill_scratch_with_dense_partials(A)
    out, lse = _static(A, t, float(data["scale"]), thr)
    ref_out, ref_lse, forced = _decisions(A, t, data, thr, "sequential")
    torch.cuda.synchronize()
    assert A.attn_get_last_device_error() == 0
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    batches = [0, 13, 31]
    bt, sl = data["block_table"], data["seq_lens"]
    npg = [-(-int(sl[b]) // 16) for b in batches]
    idx = torch.as_tensor(np.concatenate([bt[b, :n] for b, n in zip(batches, npg)]), device="cuda",
                          dtype=torch.long)
    bt_sub = np.zeros((len(batches), max(npg)), dtype=np.int32)
    off = 0
    for i, n in enumerate(npg):
        bt_sub[i, :n] = np.arange(off, off + n)
        off += n
    qh = host_bits(t["q"][torch.as_tensor(batches, device="cuda")])
    ro, rl, _ = oracle.paged_decode(qh, host_bits(t["k_cache"][idx]), host_bits(t["v_cache"][idx]), bt_sub,
                                    sl[batches], 32, 8, data["scale"], threshold=thr, forced_skip=forced(batches))
    sel = torch.as_tensor(batches, device="cuda")
    assert_close_bf16(out[sel], ro)
    assert_close_lse(lse[sel], rl)
