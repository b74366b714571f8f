"""GPU parity: small-seq cross attention (s_q = 1, s_kv <= 16) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import assert_close_bf16, dev_bf16, dev_i32, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    import attention_varlen_gqa_b200 as A
    A.attn_get_last_device_error()
    return A


def _run(A, s, max_s, want_weights=True):
    q, k, v = (dev_bf16(s[n]) for n in ("q", "k", "v"))
    cu = dev_i32(s["cu_seqlens_kv"])
    return A.attn_smallseq_fwd(q, k, v, cu, max_s, want_weights=want_weights)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("max_s", list(range(1, 17)))
def test_every_bucket(A, d, max_s):
    rng = np.random.default_rng(max_s)
    lens = rng.integers(0, max_s + 1, 97).astype(np.int32)
    lens[0], lens[1] = max_s, 0
    s = W.smallseq(seed=max_s, h=3, d=d, lens=lens)
    out, wts = _run(A, s, max_s)
    ro, rw = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], 3, s["scale"], max_s)
    assert_close_bf16(out, ro)
    assert_close_bf16(wts, rw)
    assert torch.all(out[1] == 0) and torch.all(wts[1] == 0)
    assert A.attn_get_last_device_error() == 0


def test_without_weights(A):
    s = W.smallseq(seed=3, batch=50, h=4, d=128)
    out, wts = _run(A, s, s["max_s_kv"], want_weights=False)
    assert wts is None
    ro, _ = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], 4, s["scale"], s["max_s_kv"])
    assert_close_bf16(out, ro)


def test_large_scores(A):
    """Scores far from zero (scale 1, |q.k| ~ 100): the max subtraction matters."""
    s = W.smallseq(seed=4, batch=64, h=2, d=128)
    q, k, v = (dev_bf16(s[n]) for n in ("q", "k", "v"))
    cu = dev_i32(s["cu_seqlens_kv"])
    out, wts = A.attn_smallseq_fwd(q, k, v, cu, s["max_s_kv"], scale=1.0)
    ro, rw = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], 2, 1.0, s["max_s_kv"])
    assert_close_bf16(out, ro)
    assert_close_bf16(wts, rw)


def test_row_longer_than_max_sets_error(A):
    lens = np.array([3, 9, 2], dtype=np.int32)
    s = W.smallseq(seed=5, h=2, d=64, lens=lens)
    out, wts = _run(A, s, 4)
    assert A.attn_get_last_device_error() == 8          # ATTN_DEVERR_SMALLSEQ_LEN
    assert torch.all(out[1] == 0) and torch.all(wts[1] == 0)
    ro, rw = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], 2, s["scale"], 4,
                                       batches=[0, 2])
    assert_close_bf16(out, ro, where=np.s_[[0, 2]])
    assert A.attn_get_last_device_error() == 0


def test_full_size_sampled(A):
    """30720 sequences x 16 heads, s_kv from {2,4,6,8,12,16}, d = 128; device-generated
    values, 400 sampled sequences checked against the oracle."""
    s = W.smallseq(seed=0, where="device")
    cu = dev_i32(s["cu_seqlens_kv"])
    out, wts = A.attn_smallseq_fwd(s["q"], s["k"], s["v"], cu, s["max_s_kv"])
    assert A.attn_get_last_device_error() == 0
    rng = np.random.default_rng(1)
    bs = np.sort(rng.choice(s["batch"], 400, replace=False))
    cu_h = s["cu_seqlens_kv"]
    rows = np.concatenate([np.arange(cu_h[b], cu_h[b + 1]) for b in bs])
    sub_cu = W.cu_from_lens(cu_h[bs + 1] - cu_h[bs])
    idx = torch.as_tensor(rows, device="cuda")
    qh = host_bits(s["q"][torch.as_tensor(bs, device="cuda")])
    kh, vh = host_bits(s["k"][idx]), host_bits(s["v"][idx])
    ro, rw = oracle.smallseq_attention(qh, kh, vh, sub_cu, 16, s["scale"], 16)
    bsel = torch.as_tensor(bs, device="cuda")
    assert_close_bf16(out[bsel], ro)
    assert_close_bf16(wts[bsel], rw)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("h", [17, 40])
def test_heads_in_several_groups(A, d, h):
    """More than 16 heads: a token's rows travel as groups of 16 heads (the last
    one partial), each key's rows of a group as their own copy."""
    s = W.smallseq(seed=h + d, batch=300, h=h, d=d)
    out, wts = _run(A, s, s["max_s_kv"])
    ro, rw = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], h, s["scale"], s["max_s_kv"])
    assert_close_bf16(out, ro)
    assert_close_bf16(wts, rw)
    assert A.attn_get_last_device_error() == 0


def test_bad_key_ranges_write_zeros(A):
    """cu_seqlens_kv = [0, 4, 3, 22, 30, total + 3, total]: row 1 ends before
    it starts, row 2 spans 19 keys (> max_s_kv), row 4 runs past the keys and
    row 5 starts past them.  Those rows are zero, both error bits are raised,
    rows 0 and 3 are exact."""
    lens = np.array([4, 16, 2, 8, 6, 12], dtype=np.int32)
    s = W.smallseq(seed=11, h=16, d=128, lens=lens)
    total = int(s["cu_seqlens_kv"][-1])
    cu_bad = s["cu_seqlens_kv"].copy()
    cu_bad[2] = 3
    cu_bad[5] = total + 3
    q, k, v = (dev_bf16(s[n]) for n in ("q", "k", "v"))
    out, wts = A.attn_smallseq_fwd(q, k, v, dev_i32(cu_bad), 16)
    assert A.attn_get_last_device_error() == 1 | 8      # ATTN_DEVERR_CU_SEQLENS | ATTN_DEVERR_SMALLSEQ_LEN
    for b in (1, 2, 4, 5):
        assert torch.all(out[b] == 0) and torch.all(wts[b] == 0)
    good = [0, 3]
    ro, rw = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], 16, s["scale"], 16,
                                       batches=good)
    assert_close_bf16(out, ro, where=np.s_[good])
    assert_close_bf16(wts, rw, where=np.s_[good])


@pytest.mark.parametrize("pattern", ["mostly_empty", "all_sixteen", "one_token"])
def test_uneven_and_full_ring(A, pattern):
    """Token ranges split by bytes when most rows are empty; back-to-back
    16-key tokens (the largest units, the ring full); a batch of one."""
    rng = np.random.default_rng(7)
    if pattern == "mostly_empty":
        lens = np.where(rng.random(5000) < 0.02, 16, 0).astype(np.int32)
    elif pattern == "all_sixteen":
        lens = np.full(3000, 16, dtype=np.int32)
    else:
        lens = np.array([9], dtype=np.int32)
    s = W.smallseq(seed=8, h=16, d=128, lens=lens)
    out, wts = _run(A, s, 16)
    assert A.attn_get_last_device_error() == 0
    pick = np.unique(np.concatenate([np.nonzero(lens)[0][:200], np.arange(min(50, len(lens)))]))
    ro, rw = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], 16, s["scale"], 16,
                                       batches=pick)
    assert_close_bf16(out, ro, where=np.s_[pick])
    assert_close_bf16(wts, rw, where=np.s_[pick])
    empty = torch.as_tensor(np.nonzero(lens == 0)[0], device="cuda")
    assert torch.all(out[empty] == 0) and torch.all(wts[empty] == 0)
