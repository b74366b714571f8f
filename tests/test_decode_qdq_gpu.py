"""GPU parity of the one-token paged decode with NVFP4 quantise-dequantise of
P and / or V (attn_paged_decode_qdq) against the oracle (oracle.nvfp4), in
both 32-key skip schedules (two passes with a workspace, one sequential split
without), at thresholds 0 to 0.1, skip sets included.

P's codes come from the kernel's fp32 exponentials, which differ from the
oracle's by a few roundings: an element whose scaled value sits next to an
E2M1 rounding midpoint (or a block whose scale product sits next to an E4M3
one) may round the other way, and the oracle bounds the output change such
an element can cause; elsewhere the usual bf16 tolerances hold.  V's codes
are decided from the same bf16 inputs by the same fp32 operations on both
sides: a case built so that every later step is exact checks them bit for
bit, E2M1 ties included."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import nvfp4 as N
from tests.parity import (assert_close_bf16_bound, assert_close_lse, dev_bf16, dev_i32, host_bits,
                          unpack_bits)

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


def _peaked(lens, h_q=8, h_kv=2, d=128, seed=0):
    """Keys of a few tiles aligned with the group's summed query: non-trivial
    skip sets and rows whose P has large entries."""
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


def _run(A, data, t, thr, schedule, p_amax, v_amax):
    B = t["q"].shape[0]
    kt = -(-data["block_table"].shape[1] * 16 // 32)
    words = -(-(B * data["h_kv"] * kt) // 32)
    mask = torch.zeros(max(words, 1), dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    out, lse = A.attn_paged_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                                   skip_threshold=thr, skip_mask=mask, skip_counts=counts, skip_schedule=schedule,
                                   p_qdq="nvfp4" if p_amax else None, p_qdq_amax=p_amax or 1.0,
                                   v_qdq="nvfp4" if v_amax else None, v_qdq_amax=v_amax or 1.0)
    return out, lse, mask, counts, kt


def _check(A, data, thr, schedule, p_amax, v_amax, t=None, batches=None, host=None):
    t = t or _dev(data)
    out, lse, mask, counts, kt = _run(A, data, t, thr, schedule, p_amax, v_amax)
    assert A.attn_get_last_device_error() == 0
    h_kv = data["h_kv"]
    bits = unpack_bits(mask, mask.numel() * 32)
    bl = list(range(len(data["seq_lens"]))) if batches is None else batches
    forced = {(i if host else b, hk): bits[(b * h_kv + hk) * kt:(b * h_kv + hk + 1) * kt]
              for i, b in enumerate(bl) for hk in range(h_kv)}
    if host is None:
        ro, rl, rec, flip = N.paged_decode_qdq(data["q"], data["k_cache"], data["v_cache"], data["block_table"],
                                               data["seq_lens"], data["h_q"], h_kv, data["scale"], threshold=thr,
                                               p_amax=p_amax, v_amax=v_amax, forced_skip=forced)
        sel = np.s_[:]
    else:
        ro, rl, rec, flip = host(thr, p_amax, v_amax, forced)
        sel = torch.as_tensor(batches, device="cuda")
    # the decisions of the plain decode (QDQ does not change them)
    _, _, rec0 = (oracle.paged_decode(data["q"], data["k_cache"], data["v_cache"], data["block_table"],
                                      data["seq_lens"], data["h_q"], h_kv, data["scale"], threshold=thr)
                  if host is None else host(thr, None, None, None, plain=True))
    if thr > 0:
        diff = rec.skipped != rec0.skipped
        amb = (rec0.max_ratio > thr * (1 - 1e-3)) & (rec0.max_ratio < thr * (1 + 1e-3))
        assert not (diff & ~amb).any()
    else:
        assert int(counts[1]) == 0
    if host is None:
        assert int(counts[0]) == int(rec.visited.sum()) and int(counts[1]) == int(rec.skipped.sum())
    mx, mean, n_amb = assert_close_bf16_bound(out[sel], ro, flip)
    assert_close_lse(lse[sel], rl)
    return out, rec, n_amb


COMBOS = [(1.0, None), (None, 3.0), (1.0, 3.0), (1.0, 1.0)]


@pytest.mark.parametrize("schedule", ["split", "sequential"])
@pytest.mark.parametrize("p_amax,v_amax", COMBOS)
@pytest.mark.parametrize("thr", [0.0, 0.1])
def test_qdq_parity_ragged(A, thr, p_amax, v_amax, schedule):
    data = _peaked([1, 15, 16, 17, 31, 33, 200, 700, 2048, 3000])
    _check(A, data, thr, schedule, p_amax, v_amax)


@pytest.mark.parametrize("thr", [1e-3, 1e-2, 0.5])
@pytest.mark.parametrize("heads,d", [((8, 2), 64), ((24, 2), 128), ((16, 1), 64), ((4, 4), 128)])
def test_qdq_parity_heads_and_thresholds(A, heads, d, thr):
    """Groups of 4, 12, 16 and 1 query heads (one or two 8-head MMA column
    tiles), d 64 and 128, both schedules."""
    data = _peaked([5, 64, 1000, 4097], h_q=heads[0], h_kv=heads[1], d=d, seed=heads[0] + d)
    t = _dev(data)
    outs = []
    for schedule in ("split", "sequential"):
        out, rec, _ = _check(A, data, thr, schedule, 1.0, 2.5, t=t)
        outs.append(out)
    # the two schedules take the same decisions and the same walk maxima
    assert torch.allclose(outs[0].float(), outs[1].float(), atol=2e-2, rtol=0)


def test_qdq_changes_the_output(A):
    """For every operand combination the kernel lands far closer to the QDQ
    oracle than the unquantised result does, so a kernel that ignored the
    quantisation (or quantised the wrong operand) would fail."""
    data = _peaked([33, 200, 700])
    t = _dev(data)
    args = (data["q"], data["k_cache"], data["v_cache"], data["block_table"], data["seq_lens"], data["h_q"],
            data["h_kv"], data["scale"])
    plain, _, _ = oracle.paged_decode(*args)
    for p_amax, v_amax in COMBOS:
        out, _, _, _, _ = _run(A, data, t, 0.0, "split", p_amax, v_amax)
        ref, _, _, flip = N.paged_decode_qdq(*args, p_amax=p_amax, v_amax=v_amax)
        ok = flip.max(axis=-1) == 0
        g = out.float().cpu().double().numpy()
        gap = np.abs(ref - plain)[ok].max()
        err = np.abs(g - oracle.round_f64_to_bf16(ref))[ok].max()
        assert err < gap / 4, (p_amax, v_amax, err, gap)


@pytest.mark.parametrize("schedule", ["split", "sequential"])
@pytest.mark.parametrize("d", [64, 128])
def test_v_codes_bit_exact_with_ties(A, schedule, d):
    """q = 0, so every p is 1 and O is the mean of the dequantised V.  With
    v_amax = 5.25 (g = 512) and blocks whose max is 0.75 (scale 64, ratio 8)
    every step after the codes is exact, so the bf16 output must equal the
    oracle's bit for bit; the blocks hold values that land on every E2M1
    rounding midpoint (ties to even), negatives, and a second block per
    channel with values beyond amax (saturation)."""
    L, G = 64, 4            # 64 keys: the normaliser is a power of two, so the division is exact
    rng = np.random.default_rng(d)
    ties = np.array([0.03125, 0.09375, 0.15625, 0.21875, 0.3125, 0.4375, 0.625], np.float32)
    V = np.zeros((L, d), np.float32)
    for c in range(d):
        for blk0 in (0, 48):
            blk = np.concatenate([[0.75], rng.choice(np.concatenate([ties, -ties]), 15)])
            V[blk0:blk0 + 16, c] = rng.permutation(blk)
        V[16:32, c] = rng.choice([-7.0, 6.5, 2.0, 0.25, -0.5], 16)
        V[32:48, c] = np.round(rng.standard_normal(16) * 8) / 8
    npg = L // 16
    vc = np.zeros((npg, 16, 1, d), np.float32)
    vc[:, :, 0] = V.reshape(npg, 16, d)
    data = dict(q=W.f32_to_bf16_bits(np.zeros((1, G, d), np.float32)),
                k_cache=W.f32_to_bf16_bits(rng.standard_normal((npg, 16, 1, d)).astype(np.float32)),
                v_cache=W.f32_to_bf16_bits(vc), block_table=np.arange(npg, dtype=np.int32)[None, :],
                seq_lens=np.array([L], np.int32), h_q=G, h_kv=1, scale=1.0 / math.sqrt(d))
    t = _dev(data)
    out, lse, _, _, _ = _run(A, data, t, 0.0, schedule, None, 5.25)
    assert A.attn_get_last_device_error() == 0
    ro, rl, _, flip = N.paged_decode_qdq(data["q"], data["k_cache"], data["v_cache"], data["block_table"],
                                         data["seq_lens"], G, 1, data["scale"], v_amax=5.25)
    assert not flip.any()
    want = oracle.round_f64_to_bf16(ro)
    got = out.float().cpu().double().numpy()
    assert np.array_equal(got, want), np.argwhere(got != want)[:4].tolist()


def _sampled_host(data, batches):
    bt, sl = data["block_table"], data["seq_lens"]
    npg = [-(-int(sl[b]) // 16) for b in batches]
    idx = torch.as_tensor(np.concatenate([bt[b, :n] for b, n in zip(batches, npg)]), device="cuda",
                          dtype=torch.long)
    bt_sub = np.zeros((len(batches), max(npg)), dtype=np.int32)
    off = 0
    for i, n in enumerate(npg):
        bt_sub[i, :n] = np.arange(off, off + n)
        off += n
    kh, vh = host_bits(data["k_cache"][idx]), host_bits(data["v_cache"][idx])
    qh = host_bits(data["q"][torch.as_tensor(batches, device="cuda")])
    sl_sub = sl[batches]

    def host(thr, p_amax, v_amax, forced, plain=False):
        if plain:
            return oracle.paged_decode(qh, kh, vh, bt_sub, sl_sub, data["h_q"], data["h_kv"], data["scale"],
                                       threshold=thr)
        return N.paged_decode_qdq(qh, kh, vh, bt_sub, sl_sub, data["h_q"], data["h_kv"], data["scale"],
                                  threshold=thr, p_amax=p_amax, v_amax=v_amax, forced_skip=forced)
    return host


@pytest.mark.parametrize("schedule", ["split", "sequential"])
@pytest.mark.parametrize("thr", [0.0, 1e-2])
def test_qdq_full_size_sampled(A, thr, schedule):
    """Batch 32 at 32768 keys (h_q 32, h_kv 8, d 128, sink and window peaks),
    p and v amax 1 as in the page's usage example; 3 sampled sequences."""
    data = W.skip_decode(seed=0, where="device")
    batches = [0, 13, 31]
    _check(A, data, thr, schedule, 1.0, 1.0, t=_dev(data), batches=batches, host=_sampled_host(data, batches))


@pytest.mark.parametrize("schedule", ["split", "sequential"])
def test_qdq_bad_block_table_entry(A, schedule):
    """A block-table entry outside the pool sets ATTN_DEVERR_BLOCK_TABLE and
    zeroes that sequence's output, with QDQ on as without; the other
    sequence still matches the oracle."""
    data = W.paged_decode([40, 50], h_q=4, h_kv=2, d=128, seed=3)
    bt = data["block_table"].copy()
    bt[1, 2] = data["num_pages"] + 5
    data["block_table"] = bt
    t = _dev(data)
    for thr in (0.0, 0.1):
        out, lse, _, _, _ = _run(A, data, t, thr, schedule, 1.0, 2.0)
        assert A.attn_get_last_device_error() & 4
        assert torch.all(out[1] == 0)
        assert torch.all(torch.isneginf(lse[1]))
        ro, rl, _, flip = N.paged_decode_qdq(data["q"], data["k_cache"], data["v_cache"], bt, data["seq_lens"], 4,
                                             2, data["scale"], threshold=thr, p_amax=1.0, v_amax=2.0, batches=[0])
        assert_close_bf16_bound(out[0], ro[0], flip[0])


def test_qdq_seq_len_beyond_table(A):
    data = W.paged_decode([40, 50], h_q=4, h_kv=2, d=64, seed=4)
    sl = data["seq_lens"].copy()
    sl[0] = data["block_table"].shape[1] * 16 + 1
    data["seq_lens"] = sl
    out, lse, _, _, _ = _run(A, data, _dev(data), 0.0, "split", 1.0, None)
    assert A.attn_get_last_device_error() & 2
    assert torch.all(out[0] == 0)
