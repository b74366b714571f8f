"""Checks that pin the NVFP4 QDQ oracle (``oracle.nvfp4``) to facts fixed
outside it: the FP4 E2M1 grid enumerated from its bit layout, torch's FP8
E4M3 cast (a library routine), hand-computed closed forms, invariants of the
recipe, and decode cases whose result follows by hand.

Each ``pin_*`` raises AssertionError on a disagreement.  They run in
``test_nvfp4_oracle.py``, directly and against planted mistakes.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from oracle import nvfp4 as N
from workloads import f32_to_bf16_bits


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _fp4_codes():
    """The 16 FP4 E2M1 codes from the format's bit layout: sign, 2 exponent
    bits (bias 1; 0 = subnormal), 1 mantissa bit.  Returns (values, mantissa bits)."""
    vals, mbits = [], []
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
        vals.append(-mag if s else mag)
        mbits.append(m)
    return np.array(vals), np.array(mbits)


def _fp4_brute(y):
    """Nearest FP4 value by exhaustive search; ties to the code whose mantissa
    bit is 0; magnitudes beyond the largest finite value saturate."""
    vals, mbits = _fp4_codes()
    out = []
    for v in np.asarray(y, dtype=np.float64).ravel():
        if abs(v) >= 6.0:
            out.append(math.copysign(6.0, v))
            continue
        d = np.abs(vals - v)
        best = d.min()
        cand = [i for i in range(16) if d[i] == best]
        even = [i for i in cand if mbits[i] == 0]
        pick = vals[(even or cand)[0]]
        out.append(0.0 if pick == 0 else pick)
    return np.array(out)


def pin_e2m1_brute_force():
    rng = np.random.default_rng(0)
    vals, _ = _fp4_codes()
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    ys = np.concatenate([
        rng.uniform(-8, 8, 4000), vals, mids, -mids,
        np.nextafter(mids.astype(np.float32), np.float32(0)), np.nextafter(mids.astype(np.float32), np.float32(9)),
        [0.0, 6.0, 6.5, 100.0, -7.0, 1e-30]]).astype(np.float32)
    got = N.e2m1_round(ys).astype(np.float64)
    want = _fp4_brute(ys)
    assert np.array_equal(np.abs(got), np.abs(want)), np.flatnonzero(got != want)[:5]
    assert np.array_equal(np.sign(got)[got != 0], np.sign(want)[want != 0])


def pin_e4m3_against_torch():
    """FP8 E4M3 rounding equals torch's float8_e4m3fn cast where that cast is
    finite (|x| <= 464), and saturates at 448 above it."""
    rng = np.random.default_rng(1)
    xs = np.concatenate([
        np.exp2(rng.uniform(-12, 8.85, 6000)), rng.uniform(0, 1e-3, 500),
        # ties: midpoints between neighbouring E4M3 values, normal and subnormal
        [2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875, 17.0, 19.0, 232.0, 464.0, 0.0]]).astype(np.float32)
    xs = np.concatenate([xs, -xs])
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).float().numpy()
    got = N.e4m3_round(xs)
    assert np.array_equal(got, want), (xs[got != want][:5], got[got != want][:5], want[got != want][:5])
    big = np.array([465.0, 480.0, 1e6, -1e9], dtype=np.float32)
    assert np.array_equal(N.e4m3_round(big), np.array([448, 448, 448, -448], dtype=np.float32))


def pin_qdq_closed_forms():
    # a block whose max equals amax: scale 448, ratio g/s = 1 when amax = 6
    x = np.zeros(16, np.float32)
    x[0], x[1], x[2] = 6.0, 1.5, -3.0
    dq, codes, s, g = N.qdq_blocks(x, 6.0)
    assert s.tolist() == [448.0] and g == np.float32(448.0)
    assert dq.tolist() == x.astype(np.float64).tolist()
    # saturation: a value beyond amax comes back as amax (the block's max)
    y = np.array([10.0, 0.5, -0.25] + [0.0] * 13, np.float32)
    dq, codes, s, _ = N.qdq_blocks(y, 1.0)
    assert s.tolist() == [448.0]                              # 10 * 448 saturates
    assert dq[:3].tolist() == [1.0, 0.5, -0.25]              # codes 6, 3, -1.5 at 1/6 each
    # an all-zero block stays zero; so does a block whose scale underflows E4M3
    assert np.all(N.qdq_blocks(np.zeros(16, np.float32), 1.0)[0] == 0)
    assert np.all(N.qdq_blocks(np.full(16, 1e-7, np.float32), 1.0)[0] == 0)
    # ties of the element rounding at g = 512 (amax = 5.25), scale 64 (ratio 8):
    # y = 8 x lands on every E2M1 midpoint and goes to the even neighbour
    t = np.array([0.75, 0.03125, 0.09375, 0.15625, 0.21875, 0.3125, 0.4375, 0.625,
                  -0.09375, -0.625, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0], np.float32)
    dq, codes, s, g = N.qdq_blocks(t, 5.25)
    assert g == np.float32(512.0) and s.tolist() == [64.0]
    assert codes[:10].tolist() == [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -1.0, -4.0]
    assert dq[:10].tolist() == [c * 64 / 512 for c in [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -1.0, -4.0]]


def pin_qdq_invariants():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((5, 48)) * np.exp2(rng.integers(-6, 6, (5, 1)))).astype(np.float32)
    for amax in (1.0, 3.5, 40.0):
        dq, codes, s, g = N.qdq_blocks(x, amax)
        # idempotent: a dequantised block quantises to itself
        assert np.array_equal(N.qdq_blocks(dq.astype(np.float32), amax)[0], dq)
        # odd: -x gives -QDQ(x)
        assert np.array_equal(N.qdq_blocks(-x, amax)[0], -dq)
        # blocks are independent: each 16-value block alone gives the same values
        for j in range(3):
            assert np.array_equal(N.qdq_blocks(x[:, 16 * j:16 * j + 16], amax)[0], dq[:, 16 * j:16 * j + 16])
        # scaling x and amax by a power of two scales the result by it
        for e in (-3, 5):
            assert np.array_equal(N.qdq_blocks(x * np.float32(2.0 ** e), amax * 2.0 ** e)[0], dq * 2.0 ** e)
        # error of a value no larger than amax: at most one E2M1 unit (half the
        # 4-to-6 gap) of its block's scale, i.e. |x - dq| <= s / g
        xb = x.reshape(5, 3, 16)
        err = np.abs(dq.reshape(5, 3, 16) - xb)
        bound = (s.astype(np.float64) / np.float64(g))[..., None] * 1.0000001
        ok = np.abs(xb).max(axis=-1, keepdims=True) <= amax
        assert np.all((err <= bound) | ~ok)
        assert np.all(np.abs(codes) <= 6) and np.all(np.isin(np.abs(codes), N._E2M1_GRID))


def _decode_case(Ks, Vs, qv, scale=1.0):
    """One sequence, one head, keys Ks [L, d], values Vs [L, d], query qv [d]
    as bf16 bits in the decode layout (pages of 16)."""
    L, d = Ks.shape
    npg = -(-L // 16)
    kc = np.zeros((npg * 16, 1, d), np.float32)
    vc = np.zeros((npg * 16, 1, d), np.float32)
    kc[:L, 0], vc[:L, 0] = Ks, Vs
    return (bf(np.asarray(qv, np.float32).reshape(1, 1, d)), bf(kc.reshape(npg, 16, 1, d)),
            bf(vc.reshape(npg, 16, 1, d)), np.arange(npg, dtype=np.int32)[None, :], np.array([L]))


def pin_qdq_decode_running_max():
    """Two 32-key tiles: tile 0 scores 0, tile 1 key 32 scores 2, the rest 0.
    P is taken against the running max after its tile (0 for tile 0, 2 for
    tile 1), quantised in 16-key blocks with p_amax = 1 (scale 448 for a block
    holding p = 1): tile 0's p are 1 (exact); keys 33-47 have p = e^-2, scaled
    6 e^-2 = 0.81 -> E2M1 1 -> 1/6; keys 48-63 form a block of e^-2 alone:
    e^-2 * 448 = 60.6 -> E4M3 60, ratio 2688/60 = 44.8, 6.06 -> 6 -> 6*60/2688.
    The normaliser sums the unquantised p."""
    d = 2
    L = 64
    Ks = np.zeros((L, d), np.float32)
    Ks[32] = [2.0, 0.0]
    rng = np.random.default_rng(3)
    Vs = np.round(rng.standard_normal((L, d)) * 4) / 4
    q, kc, vc, bt, sl = _decode_case(Ks, Vs, [1.0, 0.0])
    out, lse, _, _ = N.paged_decode_qdq(q, kc, vc, bt, sl, 1, 1, 1.0, p_amax=1.0)
    e2 = math.exp(-2.0)
    w = np.zeros(L)
    w[:32] = e2                       # p = 1 at the tile's running max 0, weight e^(0 - 2)
    w[32] = 1.0
    w[33:48] = 1.0 / 6.0
    w[48:] = 6.0 * 60.0 / 2688.0
    lsum = 32 * e2 + 1.0 + 31 * e2
    want = (w @ Vs.astype(np.float64)) / lsum
    assert np.allclose(out[0, 0], want, rtol=0, atol=1e-12), (out[0, 0], want)
    assert abs(lse[0, 0] - (2.0 + math.log(lsum))) < 1e-12
    # without QDQ the same call is the plain decode
    o2, l2, _, _ = N.paged_decode_qdq(q, kc, vc, bt, sl, 1, 1, 1.0)
    o3, l3, _ = oracle.paged_decode(q, kc, vc, bt, sl, 1, 1, 1.0)
    assert np.allclose(o2, o3, rtol=0, atol=1e-13) and np.allclose(l2, l3, rtol=0, atol=1e-13)


def pin_qdq_decode_v_blocks_along_keys():
    """q = 0: every p is 1, so O is the mean of the dequantised V over the 16
    keys.  Channel 0 = [6, 1, 0, ...] with v_amax = 6: scale 448, ratio 1,
    exact.  Channel 1 = 0.1 on every key: 0.1 * 448/6 = 7.47 -> E4M3 7.5,
    ratio 448/7.5, 5.97 -> 6 -> 6 * 7.5 / 448 each (blocks along keys; blocks
    along channels would give other values)."""
    L, d = 16, 2
    Vs = np.zeros((L, d), np.float32)
    Vs[0, 0], Vs[1, 0] = 6.0, 1.0
    bf16_tenth = 0.10009765625                       # 0.1 rounded to bf16
    Vs[:, 1] = bf16_tenth
    q, kc, vc, bt, sl = _decode_case(np.zeros((L, d), np.float32), Vs, [0.0, 0.0])
    out, _, _, _ = N.paged_decode_qdq(q, kc, vc, bt, sl, 1, 1, 1.0, v_amax=6.0)
    s1 = 7.5                                         # E4M3 of 0.10009765625 * 74.666...
    assert abs(np.float32(bf16_tenth) * (np.float32(448.0) / np.float32(6.0)) - 7.47) < 0.01
    assert np.allclose(out[0, 0], [7.0 / 16.0, 6.0 * s1 / 448.0], rtol=0, atol=1e-12), out[0, 0]
    # with P QDQ too (p = 1 is exact) nothing changes; one key gives V itself
    out2, _, _, _ = N.paged_decode_qdq(q, kc, vc, bt, sl, 1, 1, 1.0, p_amax=1.0, v_amax=6.0)
    assert np.array_equal(out2, out)
    q1, kc1, vc1, bt1, sl1 = _decode_case(np.zeros((1, d), np.float32), Vs[1:2] * 3, [0.5, 0.0])
    o1, l1, _, _ = N.paged_decode_qdq(q1, kc1, vc1, bt1, sl1, 1, 1, 1.0, p_amax=1.0)
    assert np.allclose(o1[0, 0], oracle.bf16_bits_to_f64(vc1[0, 0, 0]), rtol=0, atol=0)
    assert l1[0, 0] == 0.0


def pin_qdq_decode_skip_and_gqa():
    """Skip mode with QDQ: the decisions are the plain decode's and the LSE is
    unchanged (the normaliser is unquantised); and GQA equals one decode per
    query head on the shared K/V with the group's decisions forced, since each
    head's P is quantised over its own row and V's blocks do not depend on
    the heads."""
    rng = np.random.default_rng(4)
    L, d, G = 100, 8, 2
    Ks = rng.standard_normal((L, d)).astype(np.float32)
    Ks[:4] += 8.0 * np.ones(d, np.float32) / math.sqrt(d)
    Vs = rng.standard_normal((L, d)).astype(np.float32)
    qv = np.ones((G, d), np.float32) / math.sqrt(d) * np.array([[1.0], [0.5]], np.float32)
    npg = -(-L // 16)
    kc = np.zeros((npg * 16, 1, d), np.float32)
    vc = np.zeros((npg * 16, 1, d), np.float32)
    kc[:L, 0], vc[:L, 0] = Ks, Vs
    q, kc, vc = bf(qv.reshape(1, G, d)), bf(kc.reshape(npg, 16, 1, d)), bf(vc.reshape(npg, 16, 1, d))
    bt, sl = np.arange(npg, dtype=np.int32)[None, :], np.array([L])
    for thr in (0.0, 0.5):
        o, l, rec, _ = N.paged_decode_qdq(q, kc, vc, bt, sl, G, 1, 1.0, threshold=thr, p_amax=1.0, v_amax=4.0)
        o0, l0, rec0 = oracle.paged_decode(q, kc, vc, bt, sl, G, 1, 1.0, threshold=thr)
        assert np.array_equal(rec.skipped, rec0.skipped)
        assert np.allclose(l, l0, rtol=0, atol=1e-12)
        assert not np.allclose(o, o0, rtol=0, atol=1e-3)          # QDQ changes the output
        if thr > 0:
            assert rec.skipped.any() and not rec.skipped.all()
        for h in range(G):
            oh, lh, _, _ = N.paged_decode_qdq(q[:, h:h + 1], kc, vc, bt, sl, 1, 1, 1.0, threshold=thr,
                                             p_amax=1.0, v_amax=4.0, forced_skip={(0, 0): rec.skipped[0]})
            assert np.allclose(oh[0, 0], o[0, h], rtol=0, atol=1e-13)
            assert np.allclose(lh[0, 0], l[0, h], rtol=0, atol=1e-13)


ALL_PINS = [pin_e2m1_brute_force, pin_e4m3_against_torch, pin_qdq_closed_forms, pin_qdq_invariants,
            pin_qdq_decode_running_max, pin_qdq_decode_v_blocks_along_keys, pin_qdq_decode_skip_and_gqa]
