"""fp64 CPU oracle for fused scaled-dot-product attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may call it.  It shares no code with the CUDA library.

What it computes (the plain definition, written out):

  s_ij  = scale * <q_i, k_j>                      (fp64, from bf16 bit patterns)
  allowed(i, j) = j < s_k, and for causal masking j <= i + (s_k - s_q)
  O_i   = sum_j p_ij v_j,  p_ij = exp(s_ij - M_i) / l_i over the *kept* keys
  LSE_i = M_i + ln l_i    (natural log)

  Sources:
  * NVIDIA/Model-Optimizer PR 1034 "Add Triton unified attention kernel with
    HuggingFace integration", description: flash attention with
    variable-length batching, GQA and causal/non-causal masking.
  * NovaSky-AI/SkyRL PR 879 "[tx] Add cuDNN flash attention", Summary: the
    mask-based attention used as the expected value, and the review
    suggestion that a fully padded (zero-length) sequence gives zero output.

Skip-softmax tile rule (NVIDIA/TensorRT-LLM PR 9821 "Skip Softmax Attention",
Description: a dynamic-sparsity add-on to flash-attention kernels;
NVIDIA/Model-Optimizer PR 1941 "Add split-k decode kernel for skip softmax",
What does this PR do?, first bullet: tiles are visited in order so that the
skip decision follows the running softmax maximum; fourth bullet: the
threshold is a validated runtime argument):

  keys are cut into tiles of ``tile_n`` keys, visited in increasing order.
  For every row r served by a unit and tile t:
     tmax_r(t) = max of the row's allowed scores in tile t  (-inf if none)
     m_r(t)    = running max of the row over the tiles before t (-inf at first)
  The unit (row group, tile) is SKIPPED iff every row r it serves has
     exp(tmax_r(t) - m_r(t)) < threshold          (strict)
  with exp(-inf - x) = 0 and exp(x - (-inf)) = +inf.  Skipped entries add
  nothing to the numerator or the denominator.

Readings where the pages are silent (each is listed in the design notes):
  * causal masking is bottom-right aligned (j <= i + s_k - s_q);
  * q-head hq reads kv-head hq // (h_q / h_kv) (consecutive grouping);
  * the threshold domain is [0, 1];
  * a row with no allowed key gives O = 0 and LSE = -inf;
  * a unit is "visited" when at least one (row, key) pair in it is allowed;
    tiles with no allowed pair are neither visited nor skipped.

Two independent evaluations of the skip rule live here:
  * ``literal_group_attention``: the sequential online-softmax recurrence,
    tile by tile, one scalar at a time (tiny inputs only);
  * ``group_attention``: the vectorised form.  For threshold <= 1 a skipped
    tile never raises the running max of any row it serves (all its rows have
    tmax < m), so m_r(t) is the prefix max of tile maxima whatever the
    decisions are; the decisions for all tiles can then be taken at once.
The two are checked against each other by the tests.
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -math.inf


# ---------------------------------------------------------------------------
# bf16 <-> fp64 (exact decode, round-to-nearest-even encode)
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) to fp64 exactly."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), kept as fp64.

    bf16 keeps 8 significant bits.  Rounding is done directly on the fp64
    significand so there is no double rounding through fp32.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    finite = np.isfinite(x) & (x != 0)
    if not np.any(finite):
        return out
    xf = x[finite]
    mant, expo = np.frexp(np.abs(xf))          # |x| = mant * 2**expo, mant in [0.5, 1)
    # bf16 normal range has the fp32 exponent range; below 2**-126 the
    # spacing is fixed at 2**-133.
    q_exp = np.maximum(expo - 8, -133)           # spacing of the bf16 grid at |x|
    scaled = np.ldexp(np.abs(xf), -q_exp)        # integer grid units, exact in fp64
    rounded = np.rint(scaled)                    # numpy rint rounds half to even
    res = np.ldexp(rounded, q_exp) * np.sign(xf)
    res[np.abs(res) > 3.3895313892515355e38] = np.inf * np.sign(res[np.abs(res) > 3.3895313892515355e38])
    out[finite] = res
    return out


# ---------------------------------------------------------------------------
# Mask, GQA mapping and the tile test (the method's primitives)
# ---------------------------------------------------------------------------

def kv_head_of(hq: int, h_q: int, h_kv: int) -> int:
    """GQA: q-head ``hq`` reads kv-head ``hq // (h_q / h_kv)``."""
    group = h_q // h_kv
    return hq // group


def allowed_mask(s_q: int, s_k: int, causal: bool) -> np.ndarray:
    """Boolean [s_q, s_k]: which keys each query row may attend to.

    Causal masking is bottom-right aligned: row i sees keys j <= i + (s_k - s_q).
    """
    i = np.arange(s_q)[:, None]
    j = np.arange(s_k)[None, :]
    if causal:
        return j <= i + (s_k - s_q)
    return np.ones((s_q, s_k), dtype=bool)


def tile_ratio(tmax: float, m_prev: float) -> float:
    """exp(tmax - m_prev) with the conventions of the tile test."""
    if tmax == NEG_INF:
        return 0.0
    if m_prev == NEG_INF:
        return math.inf
    return math.exp(tmax - m_prev)


def unit_skipped(ratios, threshold: float) -> bool:
    """A unit is skipped iff every row it serves has ratio < threshold (strict)."""
    return all(r < threshold for r in ratios)


# ---------------------------------------------------------------------------
# Literal sequential evaluation (tiny inputs; pure Python scalar loops)
# ---------------------------------------------------------------------------

def literal_group_attention(S, allowed, V, threshold, tile_n, forced_skip=None):
    """Online-softmax recurrence over key tiles for one row group.

    S: [R][n] scores, allowed: [R][n] bools, V: [n][d] values (sequences of
    Python floats).  Returns (O [R][d], lse [R], visited [T], skipped [T],
    max_ratio [T]).  Every row keeps a running max m, a running sum l and an
    unnormalised accumulator; a kept tile rescales them by exp(m_old - m_new)
    as in any flash-attention forward.
    """
    R = len(S)
    n = len(V)
    d = len(V[0]) if n else 0
    T = (n + tile_n - 1) // tile_n
    m = [NEG_INF] * R
    l = [0.0] * R
    acc = [[0.0] * d for _ in range(R)]
    visited, skipped, max_ratio = [], [], []
    for t in range(T):
        lo, hi = t * tile_n, min(n, (t + 1) * tile_n)
        tmax = []
        for r in range(R):
            best = NEG_INF
            for j in range(lo, hi):
                if allowed[r][j] and S[r][j] > best:
                    best = S[r][j]
            tmax.append(best)
        vis = any(allowed[r][j] for r in range(R) for j in range(lo, hi))
        ratios = [tile_ratio(tmax[r], m[r]) for r in range(R)]
        if vis:
            skip = unit_skipped(ratios, threshold)
            if forced_skip is not None:
                skip = bool(forced_skip[t])
        else:
            skip = False
        visited.append(vis)
        skipped.append(skip and vis)
        max_ratio.append(max(ratios) if R else 0.0)
        if not vis or skip:
            continue
        for r in range(R):
            m_new = max(m[r], tmax[r])
            if m_new == NEG_INF:
                continue
            alpha = 0.0 if m[r] == NEG_INF else math.exp(m[r] - m_new)
            l[r] *= alpha
            for c in range(d):
                acc[r][c] *= alpha
            for j in range(lo, hi):
                if allowed[r][j]:
                    p = math.exp(S[r][j] - m_new)
                    l[r] += p
                    for c in range(d):
                        acc[r][c] += p * V[j][c]
            m[r] = m_new
    O, lse = [], []
    for r in range(R):
        if l[r] == 0.0:
            O.append([0.0] * d)
            lse.append(NEG_INF)
        else:
            O.append([a / l[r] for a in acc[r]])
            lse.append(m[r] + math.log(l[r]))
    return O, lse, visited, skipped, max_ratio


# ---------------------------------------------------------------------------
# Vectorised evaluation (prefix max of tile maxima)
# ---------------------------------------------------------------------------

def tile_decisions(S, allowed, threshold, tile_n, forced_skip=None):
    """Tile test for one row group, all tiles at once.

    Returns (visited [T], skipped [T], max_ratio [T], kept [R, n]).
    """
    S = np.asarray(S, dtype=np.float64)
    allowed = np.asarray(allowed, dtype=bool)
    R, n = S.shape
    T = (n + tile_n - 1) // tile_n
    if T == 0:
        empty = np.zeros(0, dtype=bool)
        return empty, empty, np.zeros(0), np.zeros((R, n), dtype=bool)
    pad = T * tile_n - n
    Sm = np.where(allowed, S, NEG_INF)
    if pad:
        Sm = np.concatenate([Sm, np.full((R, pad), NEG_INF)], axis=1)
        al = np.concatenate([allowed, np.zeros((R, pad), dtype=bool)], axis=1)
    else:
        al = allowed
    tmax = Sm.reshape(R, T, tile_n).max(axis=2)                     # [R, T]
    run = np.maximum.accumulate(tmax, axis=1)                        # max over tiles <= t
    m_prev = np.concatenate([np.full((R, 1), NEG_INF), run[:, :-1]], axis=1)
    with np.errstate(invalid="ignore", over="ignore"):
        ratio = np.exp(tmax - m_prev)                                # nan where both -inf
    ratio = np.where(tmax == NEG_INF, 0.0, ratio)
    ratio = np.where((m_prev == NEG_INF) & (tmax != NEG_INF), np.inf, ratio)
    visited = al.reshape(R, T, tile_n).any(axis=(0, 2))
    max_ratio = ratio.max(axis=0) if R else np.zeros(T)
    skipped = visited & np.all(ratio < threshold, axis=0)
    if forced_skip is not None:
        skipped = visited & np.asarray(forced_skip, dtype=bool)[:T]
    kept_tiles = ~skipped
    kept = allowed & np.repeat(kept_tiles, tile_n)[None, :n]
    return visited, skipped, max_ratio, kept


def softmax_over_kept(S, kept, V):
    """O, LSE of a masked softmax over the ``kept`` entries (fp64).

    Rows without a kept entry give O = 0 and LSE = -inf.
    """
    S = np.asarray(S, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Sm = np.where(kept, S, NEG_INF)
    M = Sm.max(axis=1) if Sm.shape[1] else np.full(Sm.shape[0], NEG_INF)
    empty = M == NEG_INF
    Msafe = np.where(empty, 0.0, M)
    P = np.where(kept, np.exp(Sm - Msafe[:, None]), 0.0)
    l = P.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        O = (P @ V) / np.where(empty, 1.0, l)[:, None]
        lse = np.where(empty, NEG_INF, Msafe + np.log(np.where(empty, 1.0, l)))
    O[empty] = 0.0
    return O, lse, P / np.where(empty, 1.0, l)[:, None]


def group_attention(S, allowed, V, threshold=0.0, tile_n=32, forced_skip=None):
    """Vectorised form of ``literal_group_attention`` for one row group."""
    visited, skipped, max_ratio, kept = tile_decisions(S, allowed, threshold, tile_n, forced_skip)
    O, lse, _ = softmax_over_kept(S, kept, V)
    return O, lse, visited, skipped, max_ratio


# ---------------------------------------------------------------------------
# Varlen (packed THD) prefill
# ---------------------------------------------------------------------------

class SkipRecord:
    """Per-unit tile-test results.

    ``visited``, ``skipped`` and ``max_ratio`` are arrays indexed
    [unit_group, tile]; the unit groups are listed in ``groups`` as tuples.
    """

    def __init__(self, groups, visited, skipped, max_ratio):
        self.groups = groups
        self.visited = visited
        self.skipped = skipped
        self.max_ratio = max_ratio

    def counts(self):
        return int(self.visited.sum()), int(self.skipped.sum())


def varlen_attention(q, k, v, cu_seqlens_q, cu_seqlens_k, h_q, h_kv, causal, scale,
                     threshold=0.0, block_m=128, tile_n=32, forced_skip=None,
                     rows=None):
    """Packed variable-length GQA attention forward.

    q: [total_q, h_q, d] bf16 bits, k/v: [total_k, h_kv, d] bf16 bits,
    cu_seqlens_*: [B + 1] exclusive prefix sums.  Units for the tile test are
    (sequence b, q-head, q-block of ``block_m`` rows) x (key tile of ``tile_n``).
    ``forced_skip`` maps (b, hq, r) -> bool array of tile decisions.
    ``rows``: optional set of (token, q-head) pairs; only blocks holding one
    of them are evaluated (sampled checks on large inputs).

    Returns (out fp64 [total_q, h_q, d], lse fp64 [total_q, h_q], SkipRecord).
    Rows not evaluated are NaN.
    """
    qf = bf16_bits_to_f64(q)
    kf = bf16_bits_to_f64(k)
    vf = bf16_bits_to_f64(v)
    total_q, _, d = qf.shape
    cu_q = np.asarray(cu_seqlens_q, dtype=np.int64)
    cu_k = np.asarray(cu_seqlens_k, dtype=np.int64)
    B = len(cu_q) - 1
    out = np.full((total_q, h_q, d), np.nan)
    lse = np.full((total_q, h_q), np.nan)
    groups, vis_l, skip_l, ratio_l = [], [], [], []
    want = None
    if rows is not None:
        want = {}
        for (tok, hq) in rows:
            want.setdefault(hq, set()).add(int(tok))
    for b in range(B):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        s_q, s_k = q1 - q0, k1 - k0
        if s_q == 0:
            continue
        allowed_full = allowed_mask(s_q, s_k, causal)
        for hq in range(h_q):
            hk = kv_head_of(hq, h_q, h_kv)
            Kb = kf[k0:k1, hk, :]
            Vb = vf[k0:k1, hk, :]
            for r in range((s_q + block_m - 1) // block_m):
                i0, i1 = r * block_m, min(s_q, (r + 1) * block_m)
                if want is not None:
                    toks = want.get(hq, ())
                    if not any(q0 + i0 <= t < q0 + i1 for t in toks):
                        continue
                S = scale * (qf[q0 + i0:q0 + i1, hq, :] @ Kb.T)
                al = allowed_full[i0:i1]
                fs = None if forced_skip is None else forced_skip.get((b, hq, r))
                O, L, vis, sk, mr = group_attention(S, al, Vb, threshold, tile_n, fs)
                out[q0 + i0:q0 + i1, hq, :] = O
                lse[q0 + i0:q0 + i1, hq] = L
                groups.append((b, hq, r))
                vis_l.append(vis)
                skip_l.append(sk)
                ratio_l.append(mr)
    T = max((len(x) for x in vis_l), default=0)

    def stack(lst, fill, dtype):
        arr = np.full((len(lst), T), fill, dtype=dtype)
        for i, x in enumerate(lst):
            arr[i, :len(x)] = x
        return arr

    rec = SkipRecord(groups, stack(vis_l, False, bool), stack(skip_l, False, bool),
                     stack(ratio_l, 0.0, np.float64))
    return out, lse, rec


# ---------------------------------------------------------------------------
# Paged one-token decode
# ---------------------------------------------------------------------------

def gather_paged(cache, block_table_row, seq_len, page_size):
    """Contiguous [seq_len, h_kv, d] view of one sequence of a paged cache.

    cache: [num_pages, page_size, h_kv, d]; token t lives in page
    block_table_row[t // page_size] at slot t % page_size.
    """
    t = np.arange(seq_len)
    pages = np.asarray(block_table_row)[t // page_size]
    return cache[pages, t % page_size]


def paged_decode(q, k_cache, v_cache, block_table, seq_lens, h_q, h_kv, scale,
                 threshold=0.0, page_size=16, tile_n=32, forced_skip=None,
                 batches=None):
    """One-token decode against a paged KV cache.

    q: [B, h_q, d] bf16 bits; caches: [num_pages, page_size, h_kv, d] bf16 bits;
    block_table: [B, max_pages] int; seq_lens: [B] int.
    threshold 0 is the dense softmax over all L keys.  threshold > 0 applies the
    tile test with units (b, kv-head, key tile of ``tile_n``) whose rows are the
    G = h_q / h_kv query heads of the group, tiles visited in key order
    (NVIDIA/Model-Optimizer PR 1941, first bullet).
    ``forced_skip`` maps (b, hk) -> bool array of tile decisions.
    Returns (out fp64 [B, h_q, d], lse fp64 [B, h_q], SkipRecord).
    """
    qf = bf16_bits_to_f64(q)
    B, _, d = qf.shape
    G = h_q // h_kv
    out = np.full((B, h_q, d), np.nan)
    lse = np.full((B, h_q), np.nan)
    groups, vis_l, skip_l, ratio_l = [], [], [], []
    for b in (range(B) if batches is None else batches):
        L = int(seq_lens[b])
        Kb = bf16_bits_to_f64(gather_paged(k_cache, block_table[b], L, page_size))
        Vb = bf16_bits_to_f64(gather_paged(v_cache, block_table[b], L, page_size))
        for hk in range(h_kv):
            heads = [hq for hq in range(h_q) if kv_head_of(hq, h_q, h_kv) == hk]
            S = scale * (qf[b, heads, :] @ Kb[:, hk, :].T)          # [G, L]
            al = np.ones_like(S, dtype=bool)
            fs = None if forced_skip is None else forced_skip.get((b, hk))
            O, Lse, vis, sk, mr = group_attention(S, al, Vb[:, hk, :], threshold, tile_n, fs)
            out[b, heads, :] = O
            lse[b, heads] = Lse
            groups.append((b, hk))
            vis_l.append(vis)
            skip_l.append(sk)
            ratio_l.append(mr)
    T = max((len(x) for x in vis_l), default=0)

    def stack(lst, fill, dtype):
        arr = np.full((len(lst), T), fill, dtype=dtype)
        for i, x in enumerate(lst):
            arr[i, :len(x)] = x
        return arr

    assert G * h_kv == h_q
    rec = SkipRecord(groups, stack(vis_l, False, bool), stack(skip_l, False, bool),
                     stack(ratio_l, 0.0, np.float64))
    return out, lse, rec


def paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k, h_q, h_kv, causal, scale,
                  threshold=0.0, page_size=16, block_m=128, tile_n=32, forced_skip=None, rows=None):
    """Varlen GQA attention forward whose keys and values live in a paged cache
    (chunked prefill / multi-token decode against the cache).

    NVIDIA/Model-Optimizer PR 1941 "Add split-k decode kernel for skip
    softmax", What does this PR do?, fifth bullet: prefill and multi-token
    decode over the paged cache are attention over the same cache with
    several query tokens per sequence.  The result is that of
    ``varlen_attention`` on the sequence's keys and values gathered from its
    pages: sequence b has the queries cu_seqlens_q[b]:cu_seqlens_q[b+1] and
    the s_k = seq_lens_k[b] cached tokens; causal masking is bottom-right
    aligned (the queries are the last s_q positions of the context).
    Returns (out, lse, SkipRecord) like ``varlen_attention``.
    """
    lens = [int(x) for x in seq_lens_k]
    kf, vf = [], []
    for b, L in enumerate(lens):
        kf.append(gather_paged(k_cache, block_table[b], L, page_size))
        vf.append(gather_paged(v_cache, block_table[b], L, page_size))
    shape = (0,) + tuple(np.asarray(k_cache).shape[2:])
    k = np.concatenate(kf) if sum(lens) else np.zeros(shape, dtype=np.asarray(k_cache).dtype)
    v = np.concatenate(vf) if sum(lens) else np.zeros(shape, dtype=np.asarray(v_cache).dtype)
    cu_k = np.zeros(len(lens) + 1, dtype=np.int64)
    cu_k[1:] = np.cumsum(lens)
    return varlen_attention(q, k, v, cu_seqlens_q, cu_k, h_q, h_kv, causal, scale, threshold=threshold,
                            block_m=block_m, tile_n=tile_n, forced_skip=forced_skip, rows=rows)


def split_partials(S, V, n_splits, tile):
    """Split-KV partial results for one row group (dense, no skipping).

    Keys are cut into ceil(n / tile) tiles; split s owns the contiguous tile
    range [s * per, (s + 1) * per) with per = ceil(n_tiles / n_splits).  Each
    split returns its own running max m_s, sum l_s = sum exp(s - m_s) and
    unnormalised o_s = sum exp(s - m_s) v.  An empty split has m = -inf, l = 0.
    (NVIDIA/Model-Optimizer PR 1941, second bullet: the 32-split, 128-token
    schedule; how tiles are dealt to splits is not printed, this is a reading.)
    """
    S = np.asarray(S, dtype=np.float64)
    R, n = S.shape
    n_tiles = (n + tile - 1) // tile
    per = (n_tiles + n_splits - 1) // n_splits if n_tiles else 0
    parts = []
    for s in range(n_splits):
        lo = min(n, s * per * tile)
        hi = min(n, (s + 1) * per * tile)
        if hi <= lo:
            parts.append((np.full(R, NEG_INF), np.zeros(R), np.zeros((R, V.shape[1]))))
            continue
        Ss = S[:, lo:hi]
        m = Ss.max(axis=1)
        P = np.exp(Ss - m[:, None])
        parts.append((m, P.sum(axis=1), P @ V[lo:hi]))
    return parts


def combine_partials(parts):
    """Log-sum-exp combine of split partials.

    M = max_s m_s; L = sum_s l_s exp(m_s - M); O = sum_s exp(m_s - M) o_s / L;
    LSE = M + ln L.  Splits with m = -inf contribute nothing.
    """
    ms = np.stack([p[0] for p in parts])           # [S, R]
    ls = np.stack([p[1] for p in parts])
    os_ = np.stack([p[2] for p in parts])          # [S, R, d]
    M = ms.max(axis=0)
    empty = M == NEG_INF
    Msafe = np.where(empty, 0.0, M)
    w = np.where(ms == NEG_INF, 0.0, np.exp(np.where(ms == NEG_INF, 0.0, ms) - Msafe[None, :]))
    L = (w * ls).sum(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        O = (w[:, :, None] * os_).sum(axis=0) / np.where(empty, 1.0, L)[:, None]
        lse = np.where(empty, NEG_INF, Msafe + np.log(np.where(empty, 1.0, L)))
    O[empty] = 0.0
    return O, lse


# ---------------------------------------------------------------------------
# Small-sequence cross attention (s_q = 1, s_kv <= 16)
# ---------------------------------------------------------------------------

def smallseq_attention(q, k, v, cu_seqlens_kv, h, scale, max_s_kv, batches=None):
    """Batched one-query cross attention with short, variable key lists.

    ROCm/TransformerEngine PR 461 "Integrate CK varlen cross attention for
    small-seq (s_q=1, s_kv<=16)", description bullets: the batch counts query
    tokens (one per sequence), every sequence has its own number of keys
    from cu_seqlens_kv, h_q = h_kv, non-causal; the attention weights
    [B, h, 1, max_s_kv] are returned in the input dtype.

    q: [B, h, d] bf16 bits; k/v: [total_kv, h, d] bf16 bits.
    Returns (out fp64 [B, h, d], weights fp64 [B, h, 1, max_s_kv]).
    Weights beyond a row's own s_kv are 0 (reading: padding is silent on
    the page).  O is computed from the unrounded probabilities.
    """
    qf = bf16_bits_to_f64(q)
    kf = bf16_bits_to_f64(k)
    vf = bf16_bits_to_f64(v)
    B, _, d = qf.shape
    cu = np.asarray(cu_seqlens_kv, dtype=np.int64)
    out = np.full((B, h, d), np.nan)
    w = np.full((B, h, 1, max_s_kv), np.nan)
    for b in (range(B) if batches is None else batches):
        k0, k1 = int(cu[b]), int(cu[b + 1])
        n = k1 - k0
        for hh in range(h):
            S = scale * (qf[b, hh, :][None, :] @ kf[k0:k1, hh, :].T)     # [1, n]
            O, _, P = softmax_over_kept(S, np.ones_like(S, dtype=bool), vf[k0:k1, hh, :])
            out[b, hh] = O[0]
            w[b, hh, 0, :] = 0.0
            w[b, hh, 0, :n] = P[0]
    return out, w


def _as_f64(x):
    """bf16 bit patterns (uint16) decoded exactly; any other array taken as values."""
    x = np.asarray(x)
    return bf16_bits_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)


def smallseq_backward(q, k, v, dout, weights, cu_seqlens_kv, h, scale, batches=None):
    """Gradients of ``smallseq_attention`` from the attention weights it returned.

    ROCm/TransformerEngine PR 461 "Integrate CK varlen cross attention for
    small-seq (s_q=1, s_kv<=16)", description bullets: the backward runs as
    grad_V, grad_attn, softmax backward and grad_Q / grad_K, and it reads the
    attention weights the forward wrote into the reused auxiliary buffer
    (forward write, backward read) rather than recomputing them.

    For one (token b, head hh) with keys j = k0 .. k1-1 and P_j the saved
    weight of key j, the steps in the page's order:
      grad_V:       dV_j = P_j dO
      grad_attn:    dP_j = <dO, v_j>
      softmax bwd:  dS_j = P_j (dP_j - sum_i P_i dP_i)
      grad_Q:       dQ   = scale * sum_j dS_j k_j
      grad_K:       dK_j = scale * dS_j q
    (the forward's scores are scale * <q, k_j>, so the chain rule puts the
    scale on dQ and dK).  Rows with no key give dQ = 0.

    q, dout: [B, h, d]; k, v: [total_kv, h, d]; weights: [B, h, 1, >= s_kv]
    -- bf16 bit patterns (uint16) or float values.  Returns fp64 dq [B, h, d]
    and dk, dv [total_kv, h, d]; rows and keys outside ``batches`` are NaN.
    """
    qf, kf, vf, of = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    wf = _as_f64(weights)
    B, _, d = qf.shape
    cu = np.asarray(cu_seqlens_kv, dtype=np.int64)
    dq = np.full((B, h, d), np.nan)
    dk = np.full(kf.shape, np.nan)
    dv = np.full(vf.shape, np.nan)
    for b in (range(B) if batches is None else batches):
        k0, k1 = int(cu[b]), int(cu[b + 1])
        n = k1 - k0
        for hh in range(h):
            P = wf[b, hh, 0, :n]                                  # [n] saved weights
            dO = of[b, hh]                                        # [d]
            dv[k0:k1, hh] = P[:, None] * dO[None, :]              # grad_V
            dP = vf[k0:k1, hh] @ dO                               # grad_attn
            dS = P * (dP - np.dot(P, dP))                         # softmax backward
            dq[b, hh] = scale * (dS @ kf[k0:k1, hh]) if n else 0.0   # grad_Q
            dk[k0:k1, hh] = scale * dS[:, None] * qf[b, hh][None, :]  # grad_K
    return dq, dk, dv


def varlen_backward(q, k, v, dout, cu_seqlens_q, cu_seqlens_k, h_q, h_kv, causal, scale, batches=None):
    """Gradients of ``varlen_attention`` (dense, no skipping) w.r.t. q, k and v.

    NVIDIA/Model-Optimizer PR 1034 "Add Triton unified attention kernel with
    HuggingFace integration", description: the kernel serves training through
    autograd, which needs the backward of the same masked softmax(Q K^T) V.
    With P the row softmax over the allowed keys (recomputed here in fp64) and
    dO the output gradient, the chain rule gives, per sequence and q-head
    (kv-head hk = the q-head's group):
      dV_hk += P^T dO                   dP = dO V^T
      dS = P * (dP - rowsum(P * dP))    (rowsum(P * dP) = <dO_i, O_i>)
      dQ = scale * dS K                 dK_hk += scale * dS^T Q
    Rows with no allowed key have P = 0 and contribute nothing.

    q, dout: [total_q, h_q, d]; k, v: [total_k, h_kv, d] (bf16 bits or float
    values).  Returns fp64 dq, dk, dv; with ``batches`` only those sequences
    are evaluated and the rest are NaN.
    """
    qf, kf, vf, of = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    cu_q = np.asarray(cu_seqlens_q, dtype=np.int64)
    cu_k = np.asarray(cu_seqlens_k, dtype=np.int64)
    B = len(cu_q) - 1
    dq = np.full(qf.shape, np.nan)
    dk = np.full(kf.shape, np.nan)
    dv = np.full(vf.shape, np.nan)
    for b in (range(B) if batches is None else batches):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        s_q, s_k = q1 - q0, k1 - k0
        dk[k0:k1] = 0.0
        dv[k0:k1] = 0.0
        dq[q0:q1] = 0.0
        if s_q == 0 or s_k == 0:
            continue
        allowed = allowed_mask(s_q, s_k, causal)
        for hq in range(h_q):
            hk = kv_head_of(hq, h_q, h_kv)
            Q, K, V, dO = qf[q0:q1, hq], kf[k0:k1, hk], vf[k0:k1, hk], of[q0:q1, hq]
            _, _, P = softmax_over_kept(scale * (Q @ K.T), allowed, V)
            dv[k0:k1, hk] += P.T @ dO
            dP = dO @ V.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dq[q0:q1, hq] = scale * (dS @ K)
            dk[k0:k1, hk] += scale * (dS.T @ Q)
    return dq, dk, dv
