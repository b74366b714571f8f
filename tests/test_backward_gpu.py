"""GPU parity: varlen GQA backward (dQ, dK, dV) against the oracle.

The oracle recomputes the forward in fp64 from q, k, v and dO; the kernels
read the forward's output and log-sum-exp, taken here from the oracle
(rounded as the forward stores them) or, where noted, from the GPU forward.
Tolerance: as for the small-seq backward, a bf16 gradient may sit one unit
in the last place from the oracle's rounding at any magnitude, and dK, dV sum
over every query (and q-head) that sees the key: element-wise
|gpu - ref| <= 2e-2 max(1, |ref|), mean-abs <= 2e-3 mean(max(1, |ref|)).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import dev_bf16, dev_i32, host_bits, record_headroom, to_f64

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
    record_headroom("varlen backward", float((err / scale).max()), 2e-2,
                    float(err.mean() / scale.mean()), 2e-3)
    assert np.all(err <= 2e-2 * scale), f"max scaled error {(err / scale).max():.3e}"
    assert err.mean() <= 2e-3 * scale.mean(), f"mean-abs {err.mean():.3e}"


def _forward_from_oracle(w):
    o, lse, _ = oracle.varlen_attention(w["q"], w["k"], w["v"], w["cu_seqlens_q"], w["cu_seqlens_k"], w["h_q"],
                                        w["h_kv"], w["causal"], w["scale"])
    o = np.nan_to_num(o)
    out = W.f32_to_bf16_bits(oracle.round_f64_to_bf16(o).astype(np.float32))
    return out, np.where(np.isnan(lse), -np.inf, lse).astype(np.float32)


def _run(A, w, out, lse, dout):
    t = {n: dev_bf16(w[n]) for n in ("q", "k", "v")}
    return A.attn_varlen_bwd(t["q"], t["k"], t["v"], dev_bf16(out), dev_bf16(dout),
                             torch.from_numpy(lse).cuda(), dev_i32(w["cu_seqlens_q"]), dev_i32(w["cu_seqlens_k"]),
                             w["max_q"], w["max_k"], causal=w["causal"], scale=w["scale"])


CASES = [
    ([37, 64], None, 4, 2, 64),
    ([1, 130, 257, 0, 128], None, 4, 2, 128),
    ([200, 64, 129], [300, 64, 500], 8, 2, 128),      # s_q < s_k: bottom-right causal
    ([300, 17], [100, 40], 6, 2, 64),                 # s_q > s_k: rows that see no key
    ([255, 3], None, 8, 8, 128),                      # MHA
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-{c[1]}-h{c[2]}/{c[3]}-d{c[4]}" for c in CASES])
def test_against_oracle(A, case, causal):
    lens_q, lens_k, h_q, h_kv, d = case
    w = W.varlen_prefill(lens_q, lens_k, h_q=h_q, h_kv=h_kv, d=d, causal=causal, seed=sum(lens_q) + d)
    dout = W.output_grad(w, seed=7)
    out, lse = _forward_from_oracle(w)
    dq, dk, dv = _run(A, w, out, lse, dout)
    assert A.attn_get_last_device_error() == 0
    rq, rk, rv = oracle.varlen_backward(w["q"], w["k"], w["v"], dout, w["cu_seqlens_q"], w["cu_seqlens_k"], h_q,
                                        h_kv, causal, w["scale"])
    assert_close_grad(dq, rq)
    assert_close_grad(dk, rk)
    assert_close_grad(dv, rv)


def test_chained_with_forward_and_deterministic(A):
    """The GPU forward's output and log-sum-exp feed the backward; two runs give
    identical bits (no atomics)."""
    w = W.varlen_prefill([513, 190, 1024], h_q=8, h_kv=2, d=128, causal=True, seed=3)
    dout = W.output_grad(w, seed=3)
    t = {n: dev_bf16(w[n]) for n in ("q", "k", "v")}
    cq, ck = dev_i32(w["cu_seqlens_q"]), dev_i32(w["cu_seqlens_k"])
    o, lse = A.attn_varlen_fwd(t["q"], t["k"], t["v"], cq, ck, w["max_q"], w["max_k"], causal=True)
    g1 = A.attn_varlen_bwd(t["q"], t["k"], t["v"], o, dev_bf16(dout), lse, cq, ck, w["max_q"], w["max_k"])
    g2 = A.attn_varlen_bwd(t["q"], t["k"], t["v"], o, dev_bf16(dout), lse, cq, ck, w["max_q"], w["max_k"])
    assert A.attn_get_last_device_error() == 0
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    rq, rk, rv = oracle.varlen_backward(w["q"], w["k"], w["v"], dout, w["cu_seqlens_q"], w["cu_seqlens_k"], 8, 2,
                                        True, w["scale"])
    assert_close_grad(g1[0], rq)
    assert_close_grad(g1[1], rk)
    assert_close_grad(g1[2], rv)


def test_bad_cu_seqlens(A):
    """Sequence 1's range runs past the tokens: the error bit is raised, its rows
    are not written, the other sequence is exact."""
    w = W.varlen_prefill([64, 100], h_q=4, h_kv=2, d=64, causal=True, seed=4)
    dout = W.output_grad(w, seed=4)
    out, lse = _forward_from_oracle(w)
    cq = w["cu_seqlens_q"].copy()
    cq[2] = cq[2] + 50
    t = {n: dev_bf16(w[n]) for n in ("q", "k", "v")}
    dq0 = torch.full_like(t["q"], 5.0)
    dq, dk, dv = A.attn_varlen_bwd(t["q"], t["k"], t["v"], dev_bf16(out), dev_bf16(dout), torch.from_numpy(lse).cuda(),
                                   dev_i32(cq), dev_i32(w["cu_seqlens_k"]), w["max_q"], w["max_k"], dq=dq0)
    assert A.attn_get_last_device_error() & 1
    assert torch.all(dq[64:] == 5.0)
    rq, rk, rv = oracle.varlen_backward(w["q"], w["k"], w["v"], dout, w["cu_seqlens_q"], w["cu_seqlens_k"], 4, 2,
                                        True, w["scale"], batches=[0])
    assert_close_grad(dq, rq, where=np.s_[:64])
    assert_close_grad(dk, rk, where=np.s_[:64])
    assert_close_grad(dv, rv, where=np.s_[:64])


def test_full_size_sampled(A):
    """The GQA prefill workload (8 sequences, 24 900 tokens, h 32/8, d 128,
    causal) with the GPU forward's output and LSE; the two shortest sequences
    checked against the oracle."""
    w = W.gqa_prefill(seed=0, where="device")
    dout = W.output_grad(w, seed=0, where="device")
    cq, ck = dev_i32(w["cu_seqlens_q"]), dev_i32(w["cu_seqlens_k"])
    o, lse = A.attn_varlen_fwd(w["q"], w["k"], w["v"], cq, ck, w["max_q"], w["max_k"], causal=True)
    dq, dk, dv = A.attn_varlen_bwd(w["q"], w["k"], w["v"], o, dout, lse, cq, ck, w["max_q"], w["max_k"])
    assert A.attn_get_last_device_error() == 0
    lens = np.asarray(w["lens_q"])
    pick = [int(x) for x in np.argsort(lens)[:2]]
    cu = w["cu_seqlens_q"]
    rows = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in pick])
    idx = torch.as_tensor(rows, device="cuda")
    sub = W.cu_from_lens(lens[pick])
    hb = {n: host_bits(x[idx]) for n, x in (("q", w["q"]), ("k", w["k"]), ("v", w["v"]), ("do", dout))}
    rq, rk, rv = oracle.varlen_backward(hb["q"], hb["k"], hb["v"], hb["do"], sub, sub, 32, 8, True, w["scale"])
    assert_close_grad(dq[idx], rq)
    assert_close_grad(dk[idx], rk)
    assert_close_grad(dv[idx], rv)
