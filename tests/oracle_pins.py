"""Checks that pin the fp64 oracle to facts fixed outside itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a
closed form, an invariant, a library routine or brute force.  They are called
by ``test_oracle_pins.py`` and, against deliberately broken copies of oracle
primitives, by ``test_oracle_mutations.py``.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from oracle import attention as A
from workloads import cu_from_lens, f32_to_bf16_bits


def bf(x):
    """Exact small values as bf16 bit patterns."""
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def close(a, b, tol=1e-12):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    same_inf = (np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b)))
    with np.errstate(invalid="ignore"):
        diff = np.where(same_inf, 0.0, np.abs(a - b))
    assert np.all(diff <= tol * np.maximum(1.0, np.abs(np.where(same_inf, 0, b)))), \
        f"max diff {np.nanmax(diff)}"


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def pin_two_by_two():
    """q=(1,0), k=((1,0),(0,1)), v=((1,2),(3,4)): p = (e^s, 1)/(e^s + 1), s = scale."""
    for scale in (1.0, 0.5):
        q = bf([[[1.0, 0.0]]])                         # [1, 1, 2]
        k = bf([[[1.0, 0.0]], [[0.0, 1.0]]])           # [2, 1, 2]
        v = bf([[[1.0, 2.0]], [[3.0, 4.0]]])
        out, lse, _ = oracle.varlen_attention(q, k, v, [0, 1], [0, 2], 1, 1, False, scale)
        e = math.exp(scale)
        p0, p1 = e / (e + 1), 1 / (e + 1)
        close(out[0, 0], [p0 * 1 + p1 * 3, p0 * 2 + p1 * 4])
        close(lse[0, 0], math.log(e + 1))
        # same numbers through the small-seq and the paged-decode entry points
        o2, w2 = oracle.smallseq_attention(q, k, v, [0, 2], 1, scale, 2)
        close(o2[0, 0], out[0, 0])
        close(w2[0, 0, 0], [p0, p1])
        kc = k.reshape(1, 2, 1, 2)                     # one page of 2 slots
        o3, l3, _ = oracle.paged_decode(q, kc, v.reshape(1, 2, 1, 2), np.array([[0]]),
                                        np.array([2]), 1, 1, scale, page_size=2)
        close(o3[0, 0], out[0, 0])
        close(l3[0, 0], lse[0, 0])


def pin_causal_two_by_two():
    """Causal, s_q = s_k = 2: row 0 sees key 0 only (O = v0, LSE = s00)."""
    q = bf([[[1.0, 0.0]], [[1.0, 0.0]]])
    k = bf([[[1.0, 0.0]], [[0.0, 1.0]]])
    v = bf([[[1.0, 2.0]], [[3.0, 4.0]]])
    out, lse, _ = oracle.varlen_attention(q, k, v, [0, 2], [0, 2], 1, 1, True, 1.0)
    close(out[0, 0], [1.0, 2.0])
    close(lse[0, 0], 1.0)
    e = math.e
    close(out[1, 0], [(e * 1 + 3) / (e + 1), (e * 2 + 4) / (e + 1)])
    close(lse[1, 0], math.log(e + 1))


def pin_single_key():
    """s_kv = 1: O = V, weight 1, LSE = the only score."""
    rng = np.random.default_rng(5)
    q = bf(rng.standard_normal((3, 2, 8)))
    k = bf(rng.standard_normal((3, 2, 8)))
    v = bf(rng.standard_normal((3, 2, 8)))
    out, w = oracle.smallseq_attention(q, k, v, [0, 1, 2, 3], 2, 0.3, 4)
    vf = oracle.bf16_bits_to_f64(v)
    close(out, vf)
    close(w[:, :, 0, 0], np.ones((3, 2)))
    close(w[:, :, 0, 1:], np.zeros((3, 2, 3)))
    o2, l2, _ = oracle.varlen_attention(q, k, v, [0, 1, 2, 3], [0, 1, 2, 3], 2, 2, True, 0.3)
    close(o2, vf)
    qf, kf = oracle.bf16_bits_to_f64(q), oracle.bf16_bits_to_f64(k)
    close(l2, 0.3 * np.einsum("thd,thd->th", qf, kf))


def pin_uniform_scores():
    """Q = 0 makes every score 0: O = mean of the allowed V, LSE = ln(count).

    Uses s_q != s_k so the causal alignment matters (bottom-right: row i sees
    keys j <= i + s_k - s_q), with one sequence whose early rows see nothing.
    """
    rng = np.random.default_rng(1)
    lens_q, lens_k = [5, 7, 3], [9, 4, 3]
    cu_q, cu_k = cu_from_lens(lens_q), cu_from_lens(lens_k)
    h_q, h_kv, d = 4, 2, 6
    q = bf(np.zeros((cu_q[-1], h_q, d)))
    k = bf(rng.standard_normal((cu_k[-1], h_kv, d)))
    v = bf(rng.standard_normal((cu_k[-1], h_kv, d)))
    vf = oracle.bf16_bits_to_f64(v)
    for causal in (False, True):
        out, lse, _ = oracle.varlen_attention(q, k, v, cu_q, cu_k, h_q, h_kv, causal, 0.7)
        for b in range(3):
            for i in range(lens_q[b]):
                n = lens_k[b] if not causal else max(0, min(lens_k[b], i + lens_k[b] - lens_q[b] + 1))
                for hq in range(h_q):
                    hk = hq // (h_q // h_kv)
                    row = cu_q[b] + i
                    if n == 0:
                        close(out[row, hq], np.zeros(d))
                        assert lse[row, hq] == -math.inf
                    else:
                        close(out[row, hq], vf[cu_k[b]:cu_k[b] + n, hk].mean(axis=0))
                        close(lse[row, hq], math.log(n))


# ---------------------------------------------------------------------------
# library routine: torch scaled_dot_product_attention in fp64 on the CPU
# ---------------------------------------------------------------------------

def _sdpa_reference(q, k, v, cu_q, cu_k, h_q, h_kv, causal, scale):
    """Mask-based attention through torch's SDPA, per sequence, fp64."""
    qf, kf, vf = (torch.from_numpy(oracle.bf16_bits_to_f64(x)) for x in (q, k, v))
    out = torch.zeros_like(qf)
    G = h_q // h_kv
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        s_q, s_k = q1 - q0, k1 - k0
        if s_q == 0 or s_k == 0:
            continue
        mask = torch.ones(s_q, s_k, dtype=torch.bool)
        if causal:
            mask = torch.ones(s_q, s_k, dtype=torch.bool).tril(diagonal=s_k - s_q)
        qq = qf[q0:q1].permute(1, 0, 2)                          # [h_q, s_q, d]
        kk = kf[k0:k1].permute(1, 0, 2).repeat_interleave(G, 0)  # [h_q, s_k, d]
        vv = vf[k0:k1].permute(1, 0, 2).repeat_interleave(G, 0)
        o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
        live = mask.any(dim=1)
        o[:, ~live] = 0.0
        out[q0:q1] = o.permute(1, 0, 2)
    return out.numpy()


def pin_dense_matches_sdpa():
    rng = np.random.default_rng(2)
    for causal in (False, True):
        lens_q, lens_k = [1, 40, 77, 0, 33], [1, 40, 90, 5, 20]
        cu_q, cu_k = cu_from_lens(lens_q), cu_from_lens(lens_k)
        h_q, h_kv, d = 8, 2, 16
        q = bf(rng.standard_normal((cu_q[-1], h_q, d)))
        k = bf(rng.standard_normal((cu_k[-1], h_kv, d)))
        v = bf(rng.standard_normal((cu_k[-1], h_kv, d)))
        out, _, _ = oracle.varlen_attention(q, k, v, cu_q, cu_k, h_q, h_kv, causal, 0.25)
        ref = _sdpa_reference(q, k, v, cu_q, cu_k, h_q, h_kv, causal, 0.25)
        close(out, ref, tol=1e-10)


def pin_gqa_equals_repeated_mha():
    """GQA with h_kv heads == MHA whose K/V heads are repeat-interleaved G times."""
    rng = np.random.default_rng(3)
    lens = [50, 17]
    cu = cu_from_lens(lens)
    h_q, h_kv, d = 6, 2, 8
    q = bf(rng.standard_normal((cu[-1], h_q, d)))
    k = bf(rng.standard_normal((cu[-1], h_kv, d)))
    v = bf(rng.standard_normal((cu[-1], h_kv, d)))
    G = h_q // h_kv
    k_rep = np.repeat(k, G, axis=1)
    v_rep = np.repeat(v, G, axis=1)
    for thr in (0.0, 0.3):
        o1, l1, _ = oracle.varlen_attention(q, k, v, cu, cu, h_q, h_kv, True, 0.4,
                                            threshold=thr, block_m=16, tile_n=8)
        o2, l2, _ = oracle.varlen_attention(q, k_rep, v_rep, cu, cu, h_q, h_q, True, 0.4,
                                            threshold=thr, block_m=16, tile_n=8)
        close(o1, o2)
        close(l1, l2)


# ---------------------------------------------------------------------------
# paged == contiguous; split + combine == unsplit
# ---------------------------------------------------------------------------

def pin_paged_equals_contiguous():
    rng = np.random.default_rng(4)
    page = 4
    lens = np.array([9, 1, 16, 0, 7])
    B, h_q, h_kv, d = len(lens), 4, 2, 8
    pages_per = (lens + page - 1) // page
    pool = int(pages_per.sum()) + 3
    perm = rng.permutation(pool)
    bt = np.zeros((B, int(pages_per.max())), dtype=np.int32)
    off = 0
    for b in range(B):
        bt[b, :pages_per[b]] = perm[off:off + pages_per[b]]
        off += pages_per[b]
    kc = bf(rng.standard_normal((pool, page, h_kv, d)))
    vc = bf(rng.standard_normal((pool, page, h_kv, d)))
    q = bf(rng.standard_normal((B, h_q, d)))
    out, lse, _ = oracle.paged_decode(q, kc, vc, bt, lens, h_q, h_kv, 0.5, page_size=page)
    # the test's own gather, token by token
    kcont, vcont = [], []
    for b in range(B):
        for t in range(lens[b]):
            kcont.append(kc[bt[b, t // page], t % page])
            vcont.append(vc[bt[b, t // page], t % page])
    kcont = np.array(kcont).reshape(-1, h_kv, d)
    vcont = np.array(vcont).reshape(-1, h_kv, d)
    o2, l2, _ = oracle.varlen_attention(q, kcont, vcont, np.arange(B + 1), cu_from_lens(lens),
                                        h_q, h_kv, False, 0.5)
    close(out, o2)
    close(lse, l2)
    assert np.all(out[3] == 0) and np.all(lse[3] == -math.inf)


def pin_paged_prefill():
    """Paged prefill == varlen forward on the test's own token-by-token gather
    (causal, s_q < s_k, an empty sequence, a sequence with no queries), and
    with one query per sequence == the decode oracle (two independent paths)."""
    rng = np.random.default_rng(5)
    page = 4
    lens_k = np.array([9, 0, 13, 5])
    lens_q = np.array([3, 0, 13, 0])
    B, h_q, h_kv, d = len(lens_k), 4, 2, 8
    pages_per = (lens_k + page - 1) // page
    pool = int(pages_per.sum()) + 2
    perm = rng.permutation(pool)
    bt = np.zeros((B, int(pages_per.max())), dtype=np.int32)
    off = 0
    for b in range(B):
        bt[b, :pages_per[b]] = perm[off:off + pages_per[b]]
        off += pages_per[b]
    kc = bf(rng.standard_normal((pool, page, h_kv, d)))
    vc = bf(rng.standard_normal((pool, page, h_kv, d)))
    q = bf(rng.standard_normal((int(lens_q.sum()), h_q, d)))
    cu_q = cu_from_lens(lens_q)
    out, lse, _ = oracle.paged_prefill(q, kc, vc, bt, cu_q, lens_k, h_q, h_kv, True, 0.5, page_size=page)
    kcont, vcont = [], []
    for b in range(B):
        for t in range(lens_k[b]):
            kcont.append(kc[bt[b, t // page], t % page])
            vcont.append(vc[bt[b, t // page], t % page])
    kcont = np.array(kcont).reshape(-1, h_kv, d)
    vcont = np.array(vcont).reshape(-1, h_kv, d)
    o2, l2, _ = oracle.varlen_attention(q, kcont, vcont, cu_q, cu_from_lens(lens_k), h_q, h_kv, True, 0.5)
    close(out, o2)
    close(lse, l2)
    # one query per sequence, causal: the last position sees the whole context
    q1 = bf(rng.standard_normal((B, h_q, d)))
    o3, l3, _ = oracle.paged_prefill(q1, kc, vc, bt, np.arange(B + 1), lens_k, h_q, h_kv, True, 0.5,
                                     page_size=page)
    o4, l4, _ = oracle.paged_decode(q1, kc, vc, bt, lens_k, h_q, h_kv, 0.5, page_size=page)
    close(o3, o4)
    close(l3, l4)
    assert np.all(o3[1] == 0) and np.all(l3[1] == -math.inf)


def pin_split_combine():
    rng = np.random.default_rng(6)
    for n, splits, tile in ((1000, 32, 16), (37, 32, 4), (5, 8, 2), (300, 3, 128)):
        S = rng.standard_normal((3, n)) * 3
        V = rng.standard_normal((n, 5))
        parts = oracle.split_partials(S, V, splits, tile)
        O, lse = oracle.combine_partials(parts)
        O2, lse2, _ = oracle.softmax_over_kept(S, np.ones_like(S, dtype=bool), V)
        close(O, O2, 1e-12)
        close(lse, lse2, 1e-12)
        # closed form of the log-sum-exp
        close(lse, np.log(np.exp(S).sum(axis=1)), 1e-12)


# ---------------------------------------------------------------------------
# the tile-skip rule
# ---------------------------------------------------------------------------

def _peaked_group(first, second, n_per_tile=32):
    S = np.array([[first] * n_per_tile + [second] * n_per_tile], dtype=np.float64)
    return S, np.ones_like(S, dtype=bool), np.eye(2 * n_per_tile)[:, :3]


def pin_peaked_decisions():
    """Tile 0 scores 10, tile 1 scores 0: ratio exp(-10) = 4.54e-5."""
    S, al, V = _peaked_group(10.0, 0.0)
    for thr, expect in ((1e-4, True), (4e-5, False), (0.0, False), (1.0, True)):
        for fn in (oracle.group_attention, oracle.literal_group_attention):
            O, L, vis, sk, mr = fn(S.tolist() if fn is oracle.literal_group_attention else S,
                                   al.tolist() if fn is oracle.literal_group_attention else al,
                                   V.tolist() if fn is oracle.literal_group_attention else V,
                                   thr, 32)
            assert list(vis) == [True, True]
            assert list(sk) == [False, expect], (fn.__name__, thr, list(sk))
            close(mr[1], math.exp(-10.0))
            n_kept = 32 if expect else 64
            close(L[0], 10.0 + math.log(32 + (0 if expect else 32 * math.exp(-10.0))))
            assert n_kept in (32, 64)


def pin_strict_threshold():
    """A ratio exactly equal to the threshold is kept (the test is strict)."""
    S, al, V = _peaked_group(2.0, 0.0)
    thr = math.exp(0.0 - 2.0)
    for fn in (oracle.group_attention, oracle.literal_group_attention):
        args = (S, al, V) if fn is oracle.group_attention else (S.tolist(), al.tolist(), V.tolist())
        _, _, _, sk, _ = fn(*args, thr, 32)
        assert list(sk) == [False, False], fn.__name__
        _, _, _, sk, _ = fn(*args, math.nextafter(thr, 1.0), 32)
        assert list(sk) == [False, True], fn.__name__


def pin_causal_dead_rows_vote_skip():
    """Rows without an allowed key in a tile vote skip; a tile no row may see
    is not visited.  s_q = s_k = 64 causal, one 64-row block, 32-key tiles:
    in tile 1 rows 0..31 see nothing, rows 32..63 decide."""
    s = 64
    S = np.zeros((s, s))
    S[:, :32] = 8.0                     # every row's max lives in tile 0
    al = A.allowed_mask(s, s, True)
    V = np.random.default_rng(0).standard_normal((s, 4))
    for fn in (oracle.group_attention, oracle.literal_group_attention):
        args = (S, al, V) if fn is oracle.group_attention else (S.tolist(), al.tolist(), V.tolist())
        _, _, vis, sk, _ = fn(*args, 1e-3, 32)
        assert list(vis) == [True, True]
        assert list(sk) == [False, True], fn.__name__
    # a block of rows 0..31 only: tile 1 is never visited
    _, _, vis, sk, _ = oracle.group_attention(S[:32], al[:32], V, 1e-3, 32)
    assert list(vis) == [True, False] and list(sk) == [False, False]


def pin_threshold_zero_is_dense():
    rng = np.random.default_rng(7)
    lens = [70, 129, 3]
    cu = cu_from_lens(lens)
    q = bf(rng.standard_normal((cu[-1], 4, 8)))
    k = bf(rng.standard_normal((cu[-1], 2, 8)))
    v = bf(rng.standard_normal((cu[-1], 2, 8)))
    o0, l0, rec = oracle.varlen_attention(q, k, v, cu, cu, 4, 2, True, 0.35, threshold=0.0,
                                          block_m=32, tile_n=8)
    ref = _sdpa_reference(q, k, v, cu, cu, 4, 2, True, 0.35)
    close(o0, ref, 1e-10)
    assert rec.skipped.sum() == 0


def pin_threshold_one():
    """thr = 1 skips exactly the visited tiles whose every row has tmax < m_prev
    (brute force over rows and tiles)."""
    rng = np.random.default_rng(8)
    R, n, tile = 5, 100, 8
    S = rng.standard_normal((R, n)) * 2
    al = rng.random((R, n)) < 0.8
    V = rng.standard_normal((n, 3))
    _, _, vis, sk, _ = oracle.group_attention(S, al, V, 1.0, tile)
    T = (n + tile - 1) // tile
    for t in range(T):
        cols = range(t * tile, min(n, (t + 1) * tile))
        visited = any(al[r, j] for r in range(R) for j in cols)
        all_below = True
        for r in range(R):
            tmax = max([S[r, j] for j in cols if al[r, j]], default=-math.inf)
            prev = max([S[r, j] for j in range(t * tile) if al[r, j]], default=-math.inf)
            if tmax == -math.inf:
                continue
            if not (prev > -math.inf and tmax < prev):
                all_below = False
        assert vis[t] == visited
        assert sk[t] == (visited and all_below), t


def pin_literal_equals_vectorised():
    """Sequential online recurrence == prefix-max vectorisation on random tiny
    groups, with and without forced decisions."""
    rng = np.random.default_rng(9)
    for trial in range(40):
        R = int(rng.integers(1, 6))
        n = int(rng.integers(1, 70))
        tile = int(rng.choice([4, 8, 32]))
        S = rng.standard_normal((R, n)) * rng.choice([0.5, 2.0, 6.0])
        al = rng.random((R, n)) < rng.choice([0.5, 0.9, 1.0])
        if trial % 3 == 0:
            al = np.tril(np.ones((R, n), dtype=bool), k=n - R)
        V = rng.standard_normal((n, 3))
        thr = float(rng.choice([0.0, 1e-3, 0.05, 0.3, 0.9, 1.0]))
        T = (n + tile - 1) // tile
        forced = None if trial % 4 else rng.random(T) < 0.5
        O1, L1, v1, s1, r1 = oracle.literal_group_attention(S.tolist(), al.tolist(), V.tolist(),
                                                           thr, tile, forced)
        O2, L2, v2, s2, r2 = oracle.group_attention(S, al, V, thr, tile, forced)
        assert list(v1) == list(v2)
        assert list(s1) == list(s2), (trial, s1, list(s2))
        close(np.array(O1), O2, 1e-12)
        close(np.array(L1), L2, 1e-12)
        if forced is None:
            close(np.array(r1), r2, 1e-12)


def pin_probabilities_sum_to_one():
    rng = np.random.default_rng(10)
    lens = np.array([2, 16, 5, 1, 12])
    cu = cu_from_lens(lens)
    q = bf(rng.standard_normal((5, 3, 8)))
    k = bf(rng.standard_normal((cu[-1], 3, 8)))
    v = bf(rng.standard_normal((cu[-1], 3, 8)))
    out, w = oracle.smallseq_attention(q, k, v, cu, 3, 0.5, 16)
    close(w.sum(axis=3), np.ones((5, 3, 1)))
    vf = oracle.bf16_bits_to_f64(v)
    for b in range(5):
        assert np.all(w[b, :, 0, lens[b]:] == 0)
        for h in range(3):
            close(out[b, h], w[b, h, 0, :lens[b]] @ vf[cu[b]:cu[b + 1], h])
    # the same sums hold over kept entries when tiles are skipped
    S = rng.standard_normal((4, 90)) * 4
    al = np.ones_like(S, dtype=bool)
    _, _, _, kept = oracle.tile_decisions(S, al, 0.2, 8)
    _, _, P = oracle.softmax_over_kept(S, kept, rng.standard_normal((90, 2)))
    close(P.sum(axis=1), np.ones(4))
    assert np.all(P[~kept] == 0)


def pin_bf16_codec():
    close(oracle.bf16_bits_to_f64(np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000], np.uint16)),
          [1.0, -2.0, 1.0 + 2 ** -7, 0.0, -0.0])
    r = oracle.round_f64_to_bf16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8 + 2 ** -30),
                                           3.0, 1e-3]))
    close(r[:4], [1.0, 1 + 2 ** -6, -(1 + 2 ** -7), 3.0])
    assert abs(r[4] - 1e-3) <= 2 ** -10 * 2 ** -8


def pin_smallseq_equals_varlen():
    """Small-seq == varlen forward with one query per sequence (non-causal)."""
    rng = np.random.default_rng(11)
    lens = np.array([3, 16, 1, 8, 0, 12])
    cu = cu_from_lens(lens)
    B, h, d = len(lens), 4, 16
    q = bf(rng.standard_normal((B, h, d)))
    k = bf(rng.standard_normal((cu[-1], h, d)))
    v = bf(rng.standard_normal((cu[-1], h, d)))
    out, w = oracle.smallseq_attention(q, k, v, cu, h, 0.3, 16)
    o2, _, _ = oracle.varlen_attention(q, k, v, np.arange(B + 1), cu, h, h, False, 0.3)
    close(out, o2)
    assert np.all(out[4] == 0) and np.all(w[4] == 0)


def pin_decode_skip_matches_literal():
    """Decode skip mode: units (b, kv-head, 32-key tile) over the G heads of the
    group, against the literal recurrence on the test's own score matrix."""
    rng = np.random.default_rng(12)
    page, h_q, h_kv, d = 16, 4, 2, 8
    lens = np.array([100, 64, 7])
    B = len(lens)
    pages_per = (lens + page - 1) // page
    pool = int(pages_per.sum())
    bt = np.zeros((B, int(pages_per.max())), dtype=np.int32)
    perm = rng.permutation(pool)
    off = 0
    for b in range(B):
        bt[b, :pages_per[b]] = perm[off:off + pages_per[b]]
        off += pages_per[b]
    kc = rng.standard_normal((pool, page, h_kv, d))
    for b in range(B):
        kc[bt[b, 0], :4] += 3.0                        # the first 4 tokens dominate
    kc = bf(kc)
    vc = bf(rng.standard_normal((pool, page, h_kv, d)))
    q = bf(np.abs(rng.standard_normal((B, h_q, d))))
    thr = 0.05
    out, lse, rec = oracle.paged_decode(q, kc, vc, bt, lens, h_q, h_kv, 0.5, threshold=thr,
                                        page_size=page, tile_n=32)
    qf, kf, vf = (oracle.bf16_bits_to_f64(x) for x in (q, kc, vc))
    n_skipped = 0
    for gi, (b, hk) in enumerate(rec.groups):
        L = int(lens[b])
        K = np.array([kf[bt[b, t // page], t % page, hk] for t in range(L)])
        Vv = np.array([vf[bt[b, t // page], t % page, hk] for t in range(L)])
        heads = list(range(hk * (h_q // h_kv), (hk + 1) * (h_q // h_kv)))
        S = 0.5 * (qf[b, heads] @ K.T)
        O, Ls, vis, sk, _ = oracle.literal_group_attention(
            S.tolist(), np.ones_like(S, dtype=bool).tolist(), Vv.tolist(), thr, 32)
        close(out[b, heads], np.array(O), 1e-12)
        close(lse[b, heads], np.array(Ls), 1e-12)
        T = len(sk)
        assert list(rec.skipped[gi, :T]) == list(sk)
        n_skipped += sum(sk)
    assert n_skipped > 0



# ---------------------------------------------------------------------------
# small-seq backward
# ---------------------------------------------------------------------------

def _smallseq_case(seed, lens, h, d):
    rng = np.random.default_rng(seed)
    cu = cu_from_lens(np.asarray(lens))
    B = len(lens)
    q = rng.standard_normal((B, h, d))
    k = rng.standard_normal((int(cu[-1]), h, d))
    v = rng.standard_normal((int(cu[-1]), h, d))
    do = rng.standard_normal((B, h, d))
    return cu, q, k, v, do


def pin_smallseq_backward_autograd():
    """With the exact softmax as the saved weights, the backward equals torch
    autograd (fp64) of L = sum dO . O through scores, softmax and P V."""
    lens = [3, 16, 1, 8, 0, 5]
    h, d, scale = 3, 8, 0.4
    cu, q, k, v, do = _smallseq_case(13, lens, h, d)
    B, max_s = len(lens), 16
    W = np.zeros((B, h, 1, max_s))
    dq_t, dk_t, dv_t = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        k0, k1 = int(cu[b]), int(cu[b + 1])
        for hh in range(h):
            qt = torch.tensor(q[b, hh], requires_grad=True)
            kt = torch.tensor(k[k0:k1, hh], requires_grad=True)
            vt = torch.tensor(v[k0:k1, hh], requires_grad=True)
            P = torch.softmax(scale * (kt @ qt), dim=0)
            (torch.tensor(do[b, hh]) * (P @ vt)).sum().backward()
            W[b, hh, 0, :k1 - k0] = P.detach().numpy()
            dq_t[b, hh] = qt.grad.numpy() if k1 > k0 else 0.0
            dk_t[k0:k1, hh] = kt.grad.numpy()
            dv_t[k0:k1, hh] = vt.grad.numpy()
    dq, dk, dv = oracle.smallseq_backward(q, k, v, do, W, cu, h, scale)
    close(dq, dq_t)
    close(dk, dk_t)
    close(dv, dv_t)
    assert np.all(dq[4] == 0)


def pin_smallseq_backward_finite_differences():
    """Central differences of sum dO . O, with O from the oracle's own masked
    softmax, match the backward in a few coordinates of q, k and v."""
    lens = [4, 7]
    h, d, scale, eps = 2, 6, 0.7, 1e-5
    cu, q, k, v, do = _smallseq_case(14, lens, h, d)

    def loss(q, k, v):
        qq, kk, vv = q, k, v
        tot = 0.0
        for b in range(len(lens)):
            k0, k1 = int(cu[b]), int(cu[b + 1])
            for hh in range(h):
                S = scale * (qq[b, hh][None, :] @ kk[k0:k1, hh].T)
                O, _, _ = oracle.softmax_over_kept(S, np.ones_like(S, dtype=bool), vv[k0:k1, hh])
                tot += float(do[b, hh] @ O[0])
        return tot

    W = np.zeros((len(lens), h, 1, 16))
    for b in range(len(lens)):
        k0, k1 = int(cu[b]), int(cu[b + 1])
        for hh in range(h):
            S = scale * (q[b, hh][None, :] @ k[k0:k1, hh].T)
            W[b, hh, 0, :k1 - k0] = oracle.softmax_over_kept(S, np.ones_like(S, dtype=bool), v[k0:k1, hh])[2][0]
    dq, dk, dv = oracle.smallseq_backward(q, k, v, do, W, cu, h, scale)
    rng = np.random.default_rng(15)
    for which, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(4):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            fd = (loss(**{**args, which: plus}) - loss(**{**args, which: minus})) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def pin_smallseq_backward_single_key():
    """One key: P = 1 whatever the score, so dQ = dK = 0 and dV = dO."""
    cu, q, k, v, do = _smallseq_case(16, [1, 1], 2, 4)
    W = np.ones((2, 2, 1, 1))
    dq, dk, dv = oracle.smallseq_backward(bf(q), bf(k), bf(v), bf(do), W, cu, 2, 0.9)
    close(dq, np.zeros_like(dq))
    close(dk, np.zeros_like(dk))
    close(dv, oracle.bf16_bits_to_f64(bf(do)))


# ---------------------------------------------------------------------------
# varlen backward
# ---------------------------------------------------------------------------

def _varlen_case(seed, lens_q, lens_k, h_q, h_kv, d):
    rng = np.random.default_rng(seed)
    cq, ck = cu_from_lens(np.asarray(lens_q)), cu_from_lens(np.asarray(lens_k))
    q = rng.standard_normal((int(cq[-1]), h_q, d))
    k = rng.standard_normal((int(ck[-1]), h_kv, d))
    v = rng.standard_normal((int(ck[-1]), h_kv, d))
    do = rng.standard_normal((int(cq[-1]), h_q, d))
    return cq, ck, q, k, v, do


def pin_varlen_backward_autograd():
    """= torch autograd in fp64 of sum dO . O through the masked softmax, GQA
    heads sharing one K/V leaf, causal (bottom-right, s_q < s_k included) and
    not."""
    h_q, h_kv, d, scale = 4, 2, 8, 0.35
    lens_q, lens_k = [3, 9, 1, 6], [5, 9, 4, 6]
    cq, ck, q, k, v, do = _varlen_case(17, lens_q, lens_k, h_q, h_kv, d)
    for causal in (True, False):
        dq, dk, dv = oracle.varlen_backward(q, k, v, do, cq, ck, h_q, h_kv, causal, scale)
        qt = torch.tensor(q, requires_grad=True)
        kt = torch.tensor(k, requires_grad=True)
        vt = torch.tensor(v, requires_grad=True)
        loss = 0.0
        for b in range(len(lens_q)):
            q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
            s_q, s_k = q1 - q0, k1 - k0
            i = torch.arange(s_q)[:, None]
            j = torch.arange(s_k)[None, :]
            mask = (j <= i + (s_k - s_q)) if causal else torch.ones(s_q, s_k, dtype=torch.bool)
            for hq in range(h_q):
                hk = hq // (h_q // h_kv)
                S = scale * (qt[q0:q1, hq] @ kt[k0:k1, hk].T)
                P = torch.softmax(S.masked_fill(~mask, float("-inf")), dim=1)
                loss = loss + (torch.tensor(do[q0:q1, hq]) * (P @ vt[k0:k1, hk])).sum()
        loss.backward()
        close(dq, qt.grad.numpy())
        close(dk, kt.grad.numpy())
        close(dv, vt.grad.numpy())


def pin_varlen_backward_gqa_is_summed_mha():
    """GQA gradients = MHA gradients on K/V repeated per q-head, with dK and dV
    summed over each group's heads."""
    h_q, h_kv, d, scale = 6, 2, 4, 0.5
    cq, ck, q, k, v, do = _varlen_case(18, [7, 4], [7, 4], h_q, h_kv, d)
    G = h_q // h_kv
    dq, dk, dv = oracle.varlen_backward(q, k, v, do, cq, ck, h_q, h_kv, True, scale)
    dq2, dk2, dv2 = oracle.varlen_backward(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), do, cq, ck,
                                           h_q, h_q, True, scale)
    close(dq, dq2)
    close(dk, dk2.reshape(dk2.shape[0], h_kv, G, d).sum(axis=2))
    close(dv, dv2.reshape(dv2.shape[0], h_kv, G, d).sum(axis=2))


def pin_varlen_backward_finite_differences():
    """Central differences of sum dO . O (O from the oracle's masked softmax)."""
    h_q, h_kv, d, scale, eps = 2, 1, 5, 0.6, 1e-5
    cq, ck, q, k, v, do = _varlen_case(19, [6], [8], h_q, h_kv, d)
    allowed = A.allowed_mask(6, 8, True)

    def loss(q, k, v):
        tot = 0.0
        for hq in range(h_q):
            O, _, _ = oracle.softmax_over_kept(scale * (q[:, hq] @ k[:, 0].T), allowed, v[:, 0])
            tot += float((do[:, hq] * O).sum())
        return tot

    dq, dk, dv = oracle.varlen_backward(q, k, v, do, cq, ck, h_q, h_kv, True, scale)
    rng = np.random.default_rng(20)
    for which, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(5):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            fd = (loss(**{**args, which: plus}) - loss(**{**args, which: minus})) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def pin_varlen_backward_dead_rows():
    """Causal with s_q > s_k: the first s_q - s_k rows see no key, so their dQ
    is zero and they add nothing to dK or dV; an empty sequence gives zeros."""
    h_q, h_kv, d = 2, 2, 4
    cq, ck, q, k, v, do = _varlen_case(21, [6, 0], [2, 3], h_q, h_kv, d)
    dq, dk, dv = oracle.varlen_backward(q, k, v, do, cq, ck, h_q, h_kv, True, 0.5)
    close(dq[:4], np.zeros_like(dq[:4]))
    dq2, dk2, dv2 = oracle.varlen_backward(q[4:6], k[:2], v[:2], do[4:6], [0, 2], [0, 2], h_q, h_kv, True, 0.5)
    close(dk[:2], dk2)
    close(dv[:2], dv2)
    close(dq[4:6], dq2)
    close(dk[2:], np.zeros_like(dk[2:]))

ALL_PINS = [
    pin_bf16_codec, pin_two_by_two, pin_causal_two_by_two, pin_single_key, pin_uniform_scores,
    pin_dense_matches_sdpa, pin_gqa_equals_repeated_mha, pin_paged_equals_contiguous, pin_paged_prefill,
    pin_split_combine, pin_peaked_decisions, pin_strict_threshold, pin_causal_dead_rows_vote_skip,
    pin_threshold_zero_is_dense, pin_threshold_one, pin_literal_equals_vectorised,
    pin_probabilities_sum_to_one, pin_smallseq_equals_varlen, pin_decode_skip_matches_literal,
    pin_smallseq_backward_autograd, pin_smallseq_backward_finite_differences, pin_smallseq_backward_single_key,
    pin_varlen_backward_autograd, pin_varlen_backward_gqa_is_summed_mha, pin_varlen_backward_finite_differences,
    pin_varlen_backward_dead_rows,
]
