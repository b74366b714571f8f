"""GPU parity: paged one-token decode (dense split-KV + combine, and the
skip-softmax schedules: the split schedule in one pass or, when a split's
scores do not fit one CTA, two passes; or one sequential split) against the
oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import (assert_close_bf16, assert_close_lse, compare_skip_sets, dev_bf16, dev_i32,
                          host_bits, unpack_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    import attention_varlen_gqa_b200 as A
    A.attn_get_last_device_error()
    return A


def _dev(data):
    t = {}
    for n in ("q", "k_cache", "v_cache"):
        x = data[n]
        t[n] = x if isinstance(x, torch.Tensor) else dev_bf16(x)
    t["block_table"] = dev_i32(data["block_table"])
    t["seq_lens"] = dev_i32(data["seq_lens"])
    return t


SCHEDULES = ["split", "sequential"]


def _run(A, data, thr, t=None, schedule="split"):
    t = t or _dev(data)
    B = len(data["seq_lens"])
    kt = -(-data["block_table"].shape[1] * 16 // 32)
    words = -(-(B * data["h_kv"] * kt) // 32)
    mask = torch.zeros(max(words, 1), dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    out, lse = A.attn_paged_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                                   skip_threshold=thr, skip_mask=mask, skip_counts=counts, skip_schedule=schedule)
    return out, lse, mask, counts, kt


def _gpu_decisions(mask, kt, h_kv):
    bits = unpack_bits(mask, mask.numel() * 32)

    def get(grp, T):
        b, hk = grp
        base = (b * h_kv + hk) * kt
        return bits[base:base + T]
    return get


def _check(A, data, thr, t=None, batches=None, host=None, schedule="split"):
    """Run on the GPU and compare with the oracle (optionally on sampled batches,
    with ``host`` giving host copies of the sampled sub-problem)."""
    out, lse, mask, counts, kt = _run(A, data, thr, t, schedule)
    assert A.attn_get_last_device_error() == 0
    h_q, h_kv = data["h_q"], data["h_kv"]
    if host is None:
        ro, rl, rec = oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"], data["block_table"],
                                          data["seq_lens"], h_q, h_kv, data["scale"], threshold=thr)
        sel = np.s_[:]
        get = _gpu_decisions(mask, kt, h_kv)
    else:
        ro, rl, rec = host(thr)
        sel = torch.as_tensor(batches, device="cuda")
        full = _gpu_decisions(mask, kt, h_kv)

        def get(grp, T):
            return full((batches[grp[0]], grp[1]), T)
    g_out, g_lse = out[sel], lse[sel]
    if thr > 0:
        vis, skipped, forced = compare_skip_sets(get, rec, None, thr)
        if forced:
            ro, rl, _ = host(thr, forced) if host else oracle.paged_decode(
                data["q"], data["k_cache"], data["v_cache"], data["block_table"], data["seq_lens"],
                h_q, h_kv, data["scale"], threshold=thr, forced_skip=forced)
        if host is None:
            assert int(counts[0]) == vis and int(counts[1]) == skipped
    else:
        assert int(counts[1]) == 0
    assert_close_bf16(g_out, ro)
    assert_close_lse(g_lse, rl)
    return int(counts[0]), int(counts[1])


LENS = [0, 1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 1000, 4097, 5000]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("heads", [(8, 2), (4, 4), (32, 8), (8, 1), (24, 2), (16, 1)])
def test_dense_ragged(A, d, heads):
    h_q, h_kv = heads
    data = W.paged_decode(LENS, h_q=h_q, h_kv=h_kv, d=d, seed=h_q + d)
    _check(A, data, 0.0)


def _peaked(lens, h_q=8, h_kv=2, d=128, seed=0):
    """Keys of the first 4 tokens and of 2 later tiles aligned with the group's
    summed query, so the skip sets are non-trivial."""
    data = W.paged_decode(lens, h_q=h_q, h_kv=h_kv, d=d, seed=seed)
    qf = W.bf16_bits_to_f32(data["q"]).astype(np.float64)
    kc = W.bf16_bits_to_f32(data["k_cache"])
    bt = data["block_table"]
    G = h_q // h_kv
    for b, L in enumerate(lens):
        pos = [p for p in list(range(4)) + list(range(96, 100)) + list(range(L - 40, L - 36)) if 0 <= p < L]
        pos = np.asarray(pos, dtype=np.int64)
        for hk in range(h_kv):
            qs = qf[b, hk * G:(hk + 1) * G].sum(axis=0)
            kc[bt[b, pos // 16], pos % 16, hk] += (4.0 * qs / np.linalg.norm(qs)).astype(np.float32)
    data["k_cache"] = W.f32_to_bf16_bits(kc)
    return data


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("thr", [1e-3, 1e-2, 0.1, 0.5, 0.9, 1.0])
def test_skip_sets(A, thr, schedule):
    data = _peaked([1, 31, 33, 200, 700, 2048, 3000])
    vis, skipped = _check(A, data, thr, schedule=schedule)
    assert vis > 0
    if thr >= 0.1:
        assert skipped > 0


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("heads", [(8, 1), (24, 2), (16, 1)])
def test_skip_sets_wide_groups(A, heads, schedule):
    """Groups of 8, 12 and 16 query heads: one full, one partial and two full
    8-head column tiles of the decode MMAs."""
    data = _peaked([1, 33, 700, 3000], h_q=heads[0], h_kv=heads[1], seed=heads[0])
    vis, _ = _check(A, data, 0.1, schedule=schedule)
    assert vis > 0


@pytest.mark.parametrize("d", [64, 128])
def test_schedules_agree(A, d):
    """The two skip schedules take identical decisions (same mask and counts)
    and give the same output within bf16 rounding, on long ragged sequences
    whose splits span many tiles."""
    data = _peaked([5, 64, 1000, 4097, 9000, 20000], d=d, seed=d)
    t = _dev(data)
    for thr in (0.05, 0.5):
        o1, l1, m1, c1, _ = _run(A, data, thr, t, "split")
        o2, l2, m2, c2, _ = _run(A, data, thr, t, "sequential")
        assert A.attn_get_last_device_error() == 0
        assert torch.equal(m1, m2) and torch.equal(c1, c2)
        if thr >= 0.5:
            assert int(c1[1]) > 0
        assert torch.allclose(o1.float(), o2.float(), atol=2e-2, rtol=0)
        assert torch.allclose(l1, l2, atol=1e-3, rtol=0)


@pytest.mark.parametrize("thr", [1e-2, 0.5])
def test_split_schedule_two_pass_form(A, thr):
    """A group of 16 heads with a 50 000-token sequence: a split's scores
    (1664 keys x 16 heads in fp32, 104 KB) no longer fit the one-pass CTA, so
    the split schedule runs as two passes for the whole batch; checked
    against the oracle, skip sets included."""
    data = _peaked([1, 33, 700, 3000, 50000], h_q=16, h_kv=1, d=64, seed=16)
    vis, skipped = _check(A, data, thr)
    assert vis > 0
    if thr >= 0.5:
        assert skipped > 0


def test_split_schedule_concurrent_streams(A):
    """Skip-mode decodes over the split schedule on two streams at once, each
    call with its own workspace: a call's work counter and published split
    maxima are its own, so every result equals the same call run alone (the
    kernels are deterministic: bit-equal outputs, masks and counts)."""
    runs = [_peaked([700, 3000, 9000], seed=21), _peaked([64, 5000, 20000, 1], h_q=16, h_kv=4, seed=22)]
    devs = [_dev(d) for d in runs]
    ref = [_run(A, d, 0.05, t) for d, t in zip(runs, devs)]
    torch.cuda.synchronize()
    assert A.attn_get_last_device_error() == 0
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    got = []
    for _ in range(4):
        for d, t, s in zip(runs, devs, streams):
            with torch.cuda.stream(s):
                got.append(_run(A, d, 0.05, t))
    torch.cuda.synchronize()
    assert A.attn_get_last_device_error() == 0
    for i, g in enumerate(got):
        r = ref[i % 2]
        for a, b in zip(g[:4], r[:4]):
            assert torch.equal(a, b)


def test_skip_threshold_zero_is_dense(A):
    data = _peaked([100, 1000])
    t = _dev(data)
    o0, l0, _, _, _ = _run(A, data, 0.0, t)
    _check(A, data, 0.0, t)
    # a tiny positive threshold runs the sequential schedule and skips nothing here
    o1, l1, _, c1, _ = _run(A, data, 1e-30, t)
    assert int(c1[1]) == 0
    assert torch.allclose(o0.float(), o1.float(), atol=2e-2)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_bad_block_table_entry(A, schedule):
    data = W.paged_decode([40, 50], h_q=4, h_kv=2, d=128, seed=3)
    bt = data["block_table"].copy()
    bt[1, 2] = data["num_pages"] + 5
    data["block_table"] = bt
    for thr in (0.0, 0.1):
        out, lse, _, _, _ = _run(A, data, thr, schedule=schedule)
        assert A.attn_get_last_device_error() & 4
        assert torch.all(out[1] == 0)
        assert torch.all(torch.isneginf(lse[1]))
        ro, rl, _ = oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"], bt, data["seq_lens"],
                                        4, 2, data["scale"], threshold=thr, batches=[0])
        assert_close_bf16(out[0], ro[0])


def test_seq_len_beyond_table(A):
    data = W.paged_decode([40, 50], h_q=4, h_kv=2, d=64, seed=4)
    sl = data["seq_lens"].copy()
    sl[0] = data["block_table"].shape[1] * 16 + 1
    data["seq_lens"] = sl
    out, lse, _, _, _ = _run(A, data, 0.0)
    assert A.attn_get_last_device_error() & 2
    assert torch.all(out[0] == 0)


def _sampled_host(data, batches):
    """Host copies of the pages of the sampled sequences, renumbered 0..n-1."""
    bt = data["block_table"]
    sl = data["seq_lens"]
    pages, tables = [], []
    off = 0
    npg = [(-(-int(sl[b]) // 16)) for b in batches]
    width = max(npg)
    for b, n in zip(batches, npg):
        pages.append(bt[b, :n])
        row = np.zeros(width, dtype=np.int32)
        row[:n] = np.arange(off, off + n)
        tables.append(row)
        off += n
    idx = torch.as_tensor(np.concatenate(pages), device="cuda", dtype=torch.long)
    kh = host_bits(data["k_cache"][idx])
    vh = host_bits(data["v_cache"][idx])
    qh = host_bits(data["q"][torch.as_tensor(batches, device="cuda")])
    bt_sub = np.stack(tables)
    sl_sub = sl[batches]

    def host(thr, forced=None):
        return oracle.paged_decode(qh, kh, vh, bt_sub, sl_sub, data["h_q"], data["h_kv"], data["scale"],
                                   threshold=thr, forced_skip=forced)
    return host


def test_full_size_dense_sampled(A):
    """Batch 64, lengths U[1024, 32768], 16-token pages from a permuted pool,
    h_q=32, h_kv=8, d=128, dense split-KV; 4 sampled sequences vs the oracle."""
    data = W.dense_decode(seed=0, where="device")
    batches = [0, 5, int(np.argmax(data["seq_lens"])), int(np.argmin(data["seq_lens"]))]
    _check(A, data, 0.0, t=_dev(data), batches=batches, host=_sampled_host(data, batches))


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("thr", [1e-3, 1e-2, 0.1])
def test_full_size_skip_sampled(A, thr, schedule):
    """Batch 32 at 32768 keys with sink and window peaks; 3 sampled sequences
    vs the oracle, skip sets included."""
    data = W.skip_decode(seed=0, where="device")
    batches = [0, 13, 31]
    _check(A, data, thr, t=_dev(data), batches=batches, host=_sampled_host(data, batches), schedule=schedule)


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("thr", [1e-3, 1e-2])
def test_full_size_sink_sampled(A, thr, schedule):
    """Batch 32 at 32768 keys with strong attention sinks, where nearly every
    tile is skipped; 2 sampled sequences vs the oracle, skip sets included."""
    data = W.sink_decode(seed=0, where="device")
    batches = [3, 30]
    vis, skipped = _check(A, data, thr, t=_dev(data), batches=batches, host=_sampled_host(data, batches),
                          schedule=schedule)
    assert skipped > vis // 2
