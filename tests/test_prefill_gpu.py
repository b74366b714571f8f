"""GPU parity: varlen GQA prefill (tcgen05 kernel) against the fp64 oracle."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import (assert_close_bf16, assert_close_lse, compare_skip_sets, dev_bf16, dev_i32,
                          host_bits, unpack_bits)

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def A():
    import attention_varlen_gqa_b200 as A
    A.attn_get_last_device_error()
    return A


def _dev(data):
    t = {n: (data[n] if isinstance(data[n], torch.Tensor) else dev_bf16(data[n])) for n in ("q", "k", "v")}
    t["cu_q"] = dev_i32(data["cu_seqlens_q"])
    t["cu_k"] = dev_i32(data["cu_seqlens_k"])
    return t


def _run(A, data, thr=0.0, t=None):
    t = t or _dev(data)
    B = len(data["cu_seqlens_q"]) - 1
    words, qb, kt = A.prefill_skip_mask_words(B, data["max_q"], data["max_k"], data["h_q"])
    mask = torch.zeros(max(words, 1), dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    out, lse = A.attn_varlen_fwd(t["q"], t["k"], t["v"], t["cu_q"], t["cu_k"], data["max_q"], data["max_k"],
                                 causal=data["causal"], scale=data["scale"], skip_threshold=thr,
                                 skip_mask=mask, skip_counts=counts)
    return out, lse, mask, counts, qb, kt


def _check_full(A, data, thr=0.0):
    out, lse, mask, counts, qb, kt = _run(A, data, thr)
    assert A.attn_get_last_device_error() == 0
    args = (data["q"], data["k"], data["v"], data["cu_seqlens_q"], data["cu_seqlens_k"], data["h_q"],
            data["h_kv"], data["causal"], data["scale"])
    ro, rl, rec = oracle.varlen_attention(*args, threshold=thr)
    if thr > 0:
        bits = unpack_bits(mask, mask.numel() * 32)

        def gpu(grp, T):
            b, hq, r = grp
            base = ((b * qb + r) * data["h_q"] + hq) * kt
            return bits[base:base + T]
        vis, skipped, forced = compare_skip_sets(gpu, rec, None, thr)
        assert int(counts[0]) == vis and int(counts[1]) == skipped, (counts.tolist(), vis, skipped)
        if forced:
            ro, rl, _ = oracle.varlen_attention(*args, threshold=thr, forced_skip=forced)
    else:
        assert int(counts[1]) == 0
    # rows that are not part of any sequence stay untouched; compare the packed rows
    assert_close_bf16(out, ro)
    assert_close_lse(lse, rl)
    return int(counts[0]), int(counts[1])


def test_tiny_dense(A):
    _check_full(A, W.tiny_prefill(), 0.0)


def test_tiny_skip(A):
    vis, skipped = _check_full(A, W.tiny_prefill(), 0.1)
    assert vis > 0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("heads", [(1, 1), (2, 1), (4, 2), (8, 8), (12, 3)])
@pytest.mark.parametrize("causal", [True, False])
def test_ragged(A, d, heads, causal):
    rng = np.random.default_rng(d + heads[0] * 7 + causal)
    lens = [int(x) for x in rng.integers(1, 300, 5)] + [128, 129, 1]
    data = W.varlen_prefill(lens, h_q=heads[0], h_kv=heads[1], d=d, causal=causal, seed=d + heads[0])
    _check_full(A, data)


@pytest.mark.parametrize("causal", [True, False])
def test_unequal_q_k_lengths(A, causal):
    """s_q != s_k per sequence: bottom-right causal alignment; rows with no
    visible key (s_q > s_k) give 0 and LSE -inf; sequences with no keys too."""
    lens_q = [5, 200, 130, 64, 300, 7]
    lens_k = [300, 129, 0, 64, 17, 7]
    data = W.varlen_prefill(lens_q, lens_k, h_q=4, h_kv=2, d=128, causal=causal, seed=11)
    _check_full(A, data)


def test_zero_length_sequence_golden(A):
    with open(os.path.join(GOLDEN, "zero_length_sequence.json")) as f:
        g = json.load(f)
    B, T, H, D = g["B"], g["T"], g["H"], g["D"]
    data = W.varlen_prefill([T] * B, g["seq_lengths"], h_q=H, h_kv=H, d=D, causal=True, seed=0)
    _check_full(A, data)
    out, lse, _, _, _, _ = _run(A, data)
    cu = data["cu_seqlens_q"]
    for b, L in enumerate(g["seq_lengths"]):
        pad = slice(int(cu[b]), int(cu[b]) + T - L)
        assert torch.all(out[pad].float() == g["expected_padded_output"])
        assert torch.all(torch.isneginf(lse[pad]))


def test_empty_and_single_sequences(A):
    data = W.varlen_prefill([0, 1, 0, 3], [0, 1, 4, 0], h_q=2, h_kv=1, d=64, causal=False, seed=2)
    _check_full(A, data)


@pytest.mark.parametrize("thr", [1e-3, 1e-2, 0.1, 0.5, 0.9, 1.0])
def test_skip_sets(A, thr):
    data = W.skip_parity_prefill([700, 300, 129], h_q=4, h_kv=2, d=128, seed=1)
    vis, skipped = _check_full(A, data, thr)
    assert vis > 0
    if thr >= 1e-2:
        assert skipped > 0


@pytest.mark.parametrize("thr", [1e-2, 0.5])
def test_skip_sets_odd_group(A, thr):
    """Groups of 3 query heads: a work item is two consecutive query blocks of
    one head, whose causal key ranges end one tile apart, so one tile of the
    item stops a step early while the other's steps still skip."""
    data = W.skip_parity_prefill([700, 300, 129], h_q=3, h_kv=1, d=128, seed=5)
    vis, skipped = _check_full(A, data, thr)
    assert vis > 0 and skipped > 0


def test_skip_threshold_zero_equals_dense(A):
    data = W.skip_parity_prefill([400, 250], h_q=4, h_kv=2, d=64, seed=3)
    t = _dev(data)
    o0, l0, _, c0, _, _ = _run(A, data, 0.0, t)
    o1, l1, _, c1, _, _ = _run(A, data, 1e-30, t)
    assert int(c1[1]) == 0 and int(c1[0]) > 0
    assert torch.equal(o0, o1)


def test_bad_cu_seqlens(A):
    data = W.varlen_prefill([50, 60], h_q=2, h_kv=1, d=64, seed=4)
    t = _dev(data)
    t["cu_q"] = dev_i32([0, 80, 110])      # first sequence (80 rows) is longer than max_q = 60
    A.attn_varlen_fwd(t["q"], t["k"], t["v"], t["cu_q"], t["cu_k"], 60, 60, causal=True)
    assert A.attn_get_last_device_error() & 1


def _sampled_subproblem(data, seqs, hk):
    """Host copies of the listed sequences restricted to kv-head hk and its G q-heads."""
    G = data["h_q"] // data["h_kv"]
    cu_q, cu_k = data["cu_seqlens_q"], data["cu_seqlens_k"]
    qi = np.concatenate([np.arange(cu_q[b], cu_q[b + 1]) for b in seqs])
    ki = np.concatenate([np.arange(cu_k[b], cu_k[b + 1]) for b in seqs])
    qt = torch.as_tensor(qi, device="cuda")
    kt = torch.as_tensor(ki, device="cuda")
    sub = dict(q=host_bits(data["q"][qt][:, hk * G:(hk + 1) * G]),
               k=host_bits(data["k"][kt][:, hk:hk + 1]), v=host_bits(data["v"][kt][:, hk:hk + 1]),
               cu_seqlens_q=W.cu_from_lens([cu_q[b + 1] - cu_q[b] for b in seqs]),
               cu_seqlens_k=W.cu_from_lens([cu_k[b + 1] - cu_k[b] for b in seqs]),
               h_q=G, h_kv=1, causal=data["causal"], scale=data["scale"])
    return sub, qi


def _check_sampled(A, data, thr, seqs, hk, blocks_per_seq=3):
    out, lse, mask, counts, qb, kt = _run(A, data, thr)
    assert A.attn_get_last_device_error() == 0
    sub, qi = _sampled_subproblem(data, seqs, hk)
    G = data["h_q"] // data["h_kv"]
    rows = []
    cu = sub["cu_seqlens_q"]
    for si in range(len(seqs)):
        s_q = int(cu[si + 1] - cu[si])
        nb = -(-s_q // 128)
        for r in sorted({0, nb // 2, nb - 1})[:blocks_per_seq]:
            for g in range(G):
                rows.append((int(cu[si]) + r * 128, g))
    args = (sub["q"], sub["k"], sub["v"], sub["cu_seqlens_q"], sub["cu_seqlens_k"], G, 1, sub["causal"],
            sub["scale"])
    ro, rl, rec = oracle.varlen_attention(*args, threshold=thr, rows=rows)
    if thr > 0:
        bits = unpack_bits(mask, mask.numel() * 32)

        def gpu(grp, T):
            si, g, r = grp
            base = ((seqs[si] * qb + r) * data["h_q"] + hk * G + g) * kt
            return bits[base:base + T]
        _, _, forced = compare_skip_sets(gpu, rec, None, thr)
        if forced:
            ro, rl, _ = oracle.varlen_attention(*args, threshold=thr, rows=rows, forced_skip=forced)
    qsel = torch.as_tensor(qi, device="cuda")
    g_out = out[qsel][:, hk * G:(hk + 1) * G]
    g_lse = lse[qsel][:, hk * G:(hk + 1) * G]
    assert_close_bf16(g_out, ro)
    assert_close_lse(g_lse, rl)
    return counts


def test_full_size_gqa_prefill_sampled(A):
    """8 sequences U[512, 8192] (seed 0), h_q=32, h_kv=8, d=128, causal; three
    q-blocks of the longest and the shortest sequence, kv-heads 0 and 7."""
    data = W.gqa_prefill(seed=0, where="device")
    lens = data["lens_q"]
    seqs = [int(np.argmax(lens)), int(np.argmin(lens))]
    for hk in (0, 7):
        _check_sampled(A, data, 0.0, seqs, hk)


@pytest.mark.parametrize("thr", [1e-3, 1e-2, 0.1])
def test_full_size_skip_prefill_sampled(A, thr):
    """4 x 16384 causal with sink and window peaks; sequence 2, kv-head 3."""
    data = W.skip_prefill(seed=0, where="device")
    counts = _check_sampled(A, data, thr, [2], 3)
    assert int(counts[0]) > 0


@pytest.mark.parametrize("thr", [1e-3, 1e-2])
def test_full_size_sink_prefill_sampled(A, thr):
    """4 x 16384 causal with strong attention sinks, where most units are
    skipped; sequence 1, kv-head 5."""
    data = W.sink_prefill(seed=0, where="device")
    counts = _check_sampled(A, data, thr, [1], 5)
    assert int(counts[1]) > int(counts[0]) // 4


def test_concurrent_calls_and_counter_reuse(A):
    """The kernel's CTAs claim work from a per-call counter (64 per device,
    taken in turn and re-zeroed by the kernel).  Two calls in flight on two
    streams, then more calls in a row than there are counters: every result
    equals the first, single call's bit for bit."""
    d1 = W.varlen_prefill([700, 300, 129, 1000], h_q=8, h_kv=2, d=128, causal=True, seed=21)
    d2 = W.varlen_prefill([513, 64, 900], h_q=8, h_kv=2, d=128, causal=False, seed=22)
    t1, t2 = _dev(d1), _dev(d2)

    def call(d, t):
        return A.attn_varlen_fwd(t["q"], t["k"], t["v"], t["cu_q"], t["cu_k"], d["max_q"], d["max_k"],
                                 causal=d["causal"], scale=d["scale"])

    r1, r2 = call(d1, t1), call(d2, t2)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(4):
        with torch.cuda.stream(s1):
            o1 = call(d1, t1)
        with torch.cuda.stream(s2):
            o2 = call(d2, t2)
        outs.append((o1, o2))
    torch.cuda.synchronize()
    for o1, o2 in outs:
        assert torch.equal(o1[0], r1[0]) and torch.equal(o1[1], r1[1])
        assert torch.equal(o2[0], r2[0]) and torch.equal(o2[1], r2[1])
    again = [call(d1, t1) for _ in range(70)]
    torch.cuda.synchronize()
    for o in again:
        assert torch.equal(o[0], r1[0]) and torch.equal(o[1], r1[1])
    assert A.attn_get_last_device_error() == 0


def test_many_overlapping_calls_share_claim_slots(A):
    """160 calls on four streams with no ordering between the streams, more
    than the 64 work-claim slots: calls that meet on a slot take it in turn
    (a launch tags its slot and frees it with its last claim), so every result
    equals the single call's bit for bit and no error bit is raised."""
    data = [W.varlen_prefill([300, 129, 64], h_q=8, h_kv=2, d=64, causal=True, seed=31),
            W.varlen_prefill([1000, 17], h_q=4, h_kv=4, d=128, causal=False, seed=32),
            W.varlen_prefill([513], h_q=16, h_kv=2, d=128, causal=True, seed=33),
            W.varlen_prefill([40, 80, 120, 160], h_q=2, h_kv=1, d=64, causal=True, seed=34)]
    devs = [_dev(d) for d in data]

    def call(d, t):
        return A.attn_varlen_fwd(t["q"], t["k"], t["v"], t["cu_q"], t["cu_k"], d["max_q"], d["max_k"],
                                 causal=d["causal"], scale=d["scale"])

    refs = [call(d, t) for d, t in zip(data, devs)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in data]
    outs = [[] for _ in data]
    for _ in range(40):
        for i, (d, t) in enumerate(zip(data, devs)):
            with torch.cuda.stream(streams[i]):
                outs[i].append(call(d, t))
    torch.cuda.synchronize()
    assert A.attn_get_last_device_error() == 0
    for ref, lst in zip(refs, outs):
        for o in lst:
            assert torch.equal(o[0], ref[0]) and torch.equal(o[1], ref[1])
