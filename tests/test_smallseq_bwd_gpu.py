"""GPU parity: small-seq backward (grad_V, grad_attn, softmax backward,
grad_Q / grad_K from the saved attention weights) against the oracle.

Tolerance: the gradients are not bounded by the inputs' range as the forward
output is (dQ sums up to 16 scaled key rows), so a bf16 output may sit a
whole unit in the last place away from the oracle's rounding at any
magnitude: element-wise |gpu - ref| <= 2e-2 max(1, |ref|) (bf16 keeps 8
significant bits, so one unit is at most 2^-7 |ref|, and the fp32
accumulation adds ~1e-6 relative), mean-abs <= 2e-3 mean(max(1, |ref|)).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import dev_bf16, dev_i32, host_bits, to_f64, record_headroom

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    import attention_varlen_gqa_b200 as A
    A.attn_get_last_device_error()
    return A


def assert_close_grad(gpu, ref, where=None):
    g = to_f64(gpu)
    r = oracle.round_f64_to_bf16(np.asarray(ref, dtype=np.float64))
    if where is not None:
        g, r = g[where], r[where]
    mask = ~np.isnan(r)
    assert mask.any(), "nothing to compare"
    assert np.all(np.isfinite(g[mask])), "non-finite GPU output"
    scale = np.maximum(1.0, np.abs(r[mask]))
    err = np.abs(g[mask] - r[mask])
    record_headroom("small-seq backward", float((err / scale).max()), 2e-2,
                    float(err.mean() / scale.mean()), 2e-3)
    assert np.all(err <= 2e-2 * scale), f"max scaled error {(err / scale).max():.3e}"
    assert err.mean() <= 2e-3 * scale.mean(), f"mean-abs {err.mean():.3e}"


def _oracle_weights(s, max_s):
    """The forward's weights as the oracle gives them, rounded to bf16 bits."""
    _, w = oracle.smallseq_attention(s["q"], s["k"], s["v"], s["cu_seqlens_kv"], s["h"], s["scale"], max_s)
    return W.f32_to_bf16_bits(oracle.round_f64_to_bf16(np.nan_to_num(w)).astype(np.float32))


def _run(A, s, dout, weights, max_s):
    q, k, v = (dev_bf16(s[n]) for n in ("q", "k", "v"))
    return A.attn_smallseq_bwd(q, k, v, dev_bf16(dout), dev_bf16(weights), dev_i32(s["cu_seqlens_kv"]),
                               max_s, scale=s["scale"])


def _check(s, dout, weights, dq, dk, dv, batches=None):
    rq, rk, rv = oracle.smallseq_backward(s["q"], s["k"], s["v"], dout, weights, s["cu_seqlens_kv"], s["h"],
                                          s["scale"], batches=batches)
    assert_close_grad(dq, rq)
    assert_close_grad(dk, rk)
    assert_close_grad(dv, rv)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("max_s", [1, 2, 3, 4, 5, 8, 9, 12, 16])
def test_every_bucket(A, d, max_s):
    """Saved weights from the oracle's forward; every key-count code path."""
    rng = np.random.default_rng(100 + max_s)
    lens = rng.integers(0, max_s + 1, 97).astype(np.int32)
    lens[0], lens[1] = max_s, 0
    s = W.smallseq(seed=max_s + d, h=3, d=d, lens=lens)
    g = W.smallseq_grad_inputs(s, seed=max_s)
    w = _oracle_weights(s, max_s)
    dq, dk, dv = _run(A, s, g["dout"], w, max_s)
    assert A.attn_get_last_device_error() == 0
    _check(s, g["dout"], w, dq, dk, dv)
    assert torch.all(dq[1] == 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("h", [16, 17, 40])
def test_head_groups(A, d, h):
    """16 heads (a token's K and V rows as one copy each) and more than 16
    (groups of 16, one copy per key), with synthetic saved weights."""
    s = W.smallseq(seed=h + d, batch=200, h=h, d=d)
    g = W.smallseq_grad_inputs(s, seed=h)
    dq, dk, dv = _run(A, s, g["dout"], g["weights"], s["max_s_kv"])
    assert A.attn_get_last_device_error() == 0
    _check(s, g["dout"], g["weights"], dq, dk, dv)


def test_chained_with_forward(A):
    """The GPU forward's weights fed to the GPU backward, against the oracle
    backward on the oracle forward's weights."""
    s = W.smallseq(seed=21, batch=300, h=16, d=128)
    g = W.smallseq_grad_inputs(s, seed=21)
    q, k, v = (dev_bf16(s[n]) for n in ("q", "k", "v"))
    cu = dev_i32(s["cu_seqlens_kv"])
    _, wts = A.attn_smallseq_fwd(q, k, v, cu, 16, scale=s["scale"])
    dq, dk, dv = A.attn_smallseq_bwd(q, k, v, dev_bf16(g["dout"]), wts, cu, 16, scale=s["scale"])
    assert A.attn_get_last_device_error() == 0
    _check(s, g["dout"], _oracle_weights(s, 16), dq, dk, dv)


def test_bad_rows(A):
    """cu_seqlens_kv = [0, 4, 3, 22, 30, total + 3, total]: rows 1, 4, 5 have bad
    ranges, row 2 is longer than max_s_kv; their dq is zero, both error bits
    are raised, and the keys of rows 0 and 3 get exact gradients."""
    lens = np.array([4, 16, 2, 8, 6, 12], dtype=np.int32)
    s = W.smallseq(seed=22, h=16, d=128, lens=lens)
    g = W.smallseq_grad_inputs(s, seed=22)
    total = int(s["cu_seqlens_kv"][-1])
    cu_bad = s["cu_seqlens_kv"].copy()
    cu_bad[2] = 3
    cu_bad[5] = total + 3
    q, k, v = (dev_bf16(s[n]) for n in ("q", "k", "v"))
    dk0 = torch.full_like(k, 7.0)
    dq, dk, dv = A.attn_smallseq_bwd(q, k, v, dev_bf16(g["dout"]), dev_bf16(g["weights"]), dev_i32(cu_bad), 16,
                                     scale=s["scale"], dk=dk0)
    assert A.attn_get_last_device_error() == 1 | 8
    for b in (1, 2, 4, 5):
        assert torch.all(dq[b] == 0)
    good = [0, 3]
    rq, rk, rv = oracle.smallseq_backward(s["q"], s["k"], s["v"], g["dout"], g["weights"], s["cu_seqlens_kv"],
                                          16, s["scale"], batches=good)
    assert_close_grad(dq, rq, where=np.s_[good])
    keys = np.r_[0:4, 22:30]
    assert_close_grad(dk, rk, where=np.s_[keys])
    assert_close_grad(dv, rv, where=np.s_[keys])
    # keys 4..21 belong to no valid row: untouched
    assert torch.all(dk[4:22] == 7.0)


def test_full_size_sampled(A):
    """30720 tokens x 16 heads, s_kv from {2,4,6,8,12,16}, d = 128, device
    values and synthetic saved weights; 300 sampled tokens against the oracle."""
    s = W.smallseq(seed=0, where="device")
    g = W.smallseq_grad_inputs(s, seed=0, where="device")
    cu = dev_i32(s["cu_seqlens_kv"])
    dq, dk, dv = A.attn_smallseq_bwd(s["q"], s["k"], s["v"], g["dout"], g["weights"], cu, 16, scale=s["scale"])
    assert A.attn_get_last_device_error() == 0
    rng = np.random.default_rng(2)
    bs = np.sort(rng.choice(s["batch"], 300, replace=False))
    cu_h = s["cu_seqlens_kv"]
    rows = np.concatenate([np.arange(cu_h[b], cu_h[b + 1]) for b in bs])
    sub_cu = W.cu_from_lens(cu_h[bs + 1] - cu_h[bs])
    bsel = torch.as_tensor(bs, device="cuda")
    idx = torch.as_tensor(rows, device="cuda")
    rq, rk, rv = oracle.smallseq_backward(host_bits(s["q"][bsel]), host_bits(s["k"][idx]), host_bits(s["v"][idx]),
                                          host_bits(g["dout"][bsel]), host_bits(g["weights"][bsel]), sub_cu, 16,
                                          s["scale"])
    assert_close_grad(dq[bsel], rq)
    assert_close_grad(dk[idx], rk)
    assert_close_grad(dv[idx], rv)
