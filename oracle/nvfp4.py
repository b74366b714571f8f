"""NVFP4 quantise-dequantise (QDQ) of the decode's P and V, and the one-token
paged decode with it -- plain CPU code.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may call it.  It shares no code with the CUDA library.

Source: NVIDIA/Model-Optimizer PR 1941 "Add split-k decode kernel for skip
softmax", What does this PR do?, third bullet (skip-softmax works together
with NVFP4 QDQ of P and V) and Usage (``p_qdq="nvfp4"``, ``p_qdq_amax``,
``v_qdq="nvfp4"``, ``v_qdq_amax``).  The page names the format and the
arguments but prints no recipe.  The reading used here (each item is also
listed in the design notes):

  * NVFP4 is NVIDIA's published 4-bit format: FP4 E2M1 values (sign, 2-bit
    exponent with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4,
    6), one FP8 E4M3 scale per block of 16 consecutive values, and one fp32
    tensor scale derived from the tensor's amax (the ``*_qdq_amax`` argument).
  * Blocks run along the key axis for both operands of P V, its contraction
    axis (where a block-scaled FP4 GEMM keeps its scales): P in blocks of 16
    consecutive keys of one query head's row, V in blocks of 16 consecutive
    keys (one 16-token page) of one channel of one kv-head.
  * Per block of values x (all arithmetic steps below are fp32, round to
    nearest even, as the kernel takes them, since they decide the codes):
        k = 448 / amax,  g = 2688 / amax           (2688 = 6 * 448)
        b = max |x_i|
        s = E4M3(b * k)        (round to nearest even, saturating at 448)
        r = g / s   (0 when s = 0)
        q_i = E2M1(x_i * r)    (round to nearest even, saturating at 6)
        x_dq_i = q_i * s / g   (the dequantised value, exact in fp64)
  * P is the exponential against the running maximum of the sequential
    32-key walk after the key's tile is taken in: p_j = exp(s_j - M_t(j)),
    M_t the max over the kept tiles up to and including t (skipped tiles
    never raise it).  QDQ applies to the operands of P V only: the softmax
    normaliser l sums the unquantised p, so the LSE output does not change.
  * With QDQ on, the decode always takes 32-key tiles in order (at threshold
    0 none is skipped), so P is defined by the same walk whatever the
    threshold.
"""
from __future__ import annotations

import numpy as np

from .attention import NEG_INF, SkipRecord, bf16_bits_to_f64, gather_paged, kv_head_of, tile_decisions

E2M1_MAX = 6.0
E4M3_MAX = 448.0
BLOCK = 16

# E2M1 magnitudes in code order (code = 2 * exponent field + mantissa bit)
_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_E2M1_MIDS = (_E2M1_GRID[:-1] + _E2M1_GRID[1:]) / 2          # 0.25, 0.75, ..., 5


def e2m1_round(y):
    """Round fp32 values to the FP4 E2M1 grid: nearest, ties to the even
    mantissa (even code), magnitudes above 6 saturate to 6.  Returns fp32."""
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y).astype(np.float64)
    idx = np.searchsorted(_E2M1_MIDS, a, side="left")            # midpoints strictly below |y|
    at_mid = (idx < len(_E2M1_MIDS)) & (a == _E2M1_MIDS[np.minimum(idx, len(_E2M1_MIDS) - 1)])
    idx = np.where(at_mid & (idx % 2 == 1), idx + 1, idx)        # a tie goes to the even code
    return (np.sign(y) * _E2M1_GRID[idx]).astype(np.float32)


def e4m3_round(x):
    """Round fp32 values to the FP8 E4M3 grid (bias 7, 3 mantissa bits, no
    infinities, largest finite 448, subnormal step 2**-9): nearest, ties to
    even, magnitudes beyond 448 saturate to 448.  Returns fp32."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float64)
    out = np.zeros_like(a)
    nz = a > 0
    _, expo = np.frexp(a[nz])                                   # a = m * 2**expo, m in [0.5, 1)
    step_exp = np.maximum(expo - 1 - 3, -9)                     # 3 mantissa bits; subnormals at 2**-9
    out[nz] = np.ldexp(np.rint(np.ldexp(a[nz], -step_exp)), step_exp)
    out = np.minimum(out, E4M3_MAX)
    return (np.sign(x) * out).astype(np.float32)


def tensor_scales(amax):
    """(k, g) = (448 / amax, 2688 / amax) in fp32 for a finite amax > 0."""
    a = np.float32(amax)
    if not (np.isfinite(a) and a > 0):
        raise ValueError("amax must be finite and > 0")
    return np.float32(448.0) / a, np.float32(2688.0) / a


def qdq_blocks(x, amax):
    """NVFP4 QDQ of fp32 values x whose LAST axis is cut into blocks of 16
    (a shorter last block takes the remaining values).  Returns (x_dq fp64,
    codes fp32 in [-6, 6], block scales fp32 [..., n_blocks], g)."""
    x = np.asarray(x, dtype=np.float32)
    k, g = tensor_scales(amax)
    n = x.shape[-1]
    nb = (n + BLOCK - 1) // BLOCK
    pad = nb * BLOCK - n
    xp = np.concatenate([x, np.zeros(x.shape[:-1] + (pad,), np.float32)], axis=-1) if pad else x
    xb = xp.reshape(x.shape[:-1] + (nb, BLOCK))
    bmax = np.abs(xb).max(axis=-1)                               # exact
    s = e4m3_round(bmax * k)                                     # fp32 product, then E4M3
    with np.errstate(divide="ignore"):
        r = np.where(s > 0, g / np.where(s > 0, s, np.float32(1)), np.float32(0)).astype(np.float32)
    q = e2m1_round(xb * r[..., None])                            # fp32 product, then E2M1
    xdq = q.astype(np.float64) * s.astype(np.float64)[..., None] / np.float64(g)
    codes = q.reshape(xp.shape)[..., :n]
    return xdq.reshape(xp.shape)[..., :n], codes, s, g


def _neighbour_gap(y):
    """For fp32 values y on the E2M1 scale: the magnitude change if y rounded
    to the other side of its nearest rounding midpoint (0 if none near)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    idx = np.clip(np.searchsorted(_E2M1_MIDS, a), 0, len(_E2M1_MIDS) - 1)
    lo = np.clip(idx - 1, 0, len(_E2M1_MIDS) - 1)
    near = np.where(np.abs(a - _E2M1_MIDS[idx]) < np.abs(a - _E2M1_MIDS[lo]), idx, lo)
    gap = _E2M1_GRID[near + 1] - _E2M1_GRID[near]
    return _E2M1_MIDS[near], gap


def p_flip_bound(p32, amax, rel=2e-5):
    """Per-element bound on how far the kernel's dequantised P may sit from
    the one computed here, for P in fp32 blocks along the last axis.

    The kernel's p carries the rounding of its fp32 score and exponential
    (relative error far below ``rel``); an element whose scaled value lies
    within ``rel`` of an E2M1 rounding midpoint, or whose block scale's
    product lies within ``rel`` of an E4M3 one, may round the other way
    there.  Returns an fp64 array like p32: the largest change of that
    element's dequantised value (a whole block's values when its scale is
    the ambiguous one)."""
    p32 = np.asarray(p32, dtype=np.float32)
    k, g = tensor_scales(amax)
    n = p32.shape[-1]
    nb = (n + BLOCK - 1) // BLOCK
    pad = nb * BLOCK - n
    xp = np.concatenate([p32, np.zeros(p32.shape[:-1] + (pad,), np.float32)], axis=-1) if pad else p32
    xb = xp.reshape(p32.shape[:-1] + (nb, BLOCK)).astype(np.float64)
    bmax = xb.max(axis=-1)
    raw = bmax * np.float64(k)
    s = e4m3_round((bmax * k).astype(np.float32)).astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(s[..., None] > 0, xb * (np.float64(g) / np.where(s > 0, s, 1.0))[..., None], 0.0)
    mid, gap = _neighbour_gap(y)
    elem = np.where(np.abs(y - mid) <= rel * np.maximum(mid, 1e-30), gap, 0.0) * s[..., None] / np.float64(g)
    # the block scale's product next to an E4M3 midpoint: under either scale
    # a value is at most one E2M1 unit (half the widest gap, 4 to 6) from x,
    # so the two dequantised values differ by at most two units of the
    # larger scale
    s_up = e4m3_round((raw * (1 + 4 * rel)).astype(np.float32)).astype(np.float64)
    s_dn = e4m3_round((raw * (1 - 4 * rel)).astype(np.float32)).astype(np.float64)
    scale_amb = (s_up != s) | (s_dn != s)
    blk = np.where(scale_amb[..., None], 2.0 * np.maximum(s_up, s)[..., None] / np.float64(g), 0.0)
    blk = np.broadcast_to(blk, xb.shape)
    out = np.maximum(elem, blk)
    return out.reshape(xp.shape)[..., :n]


def paged_decode_qdq(q, k_cache, v_cache, block_table, seq_lens, h_q, h_kv, scale, threshold=0.0,
                     p_amax=None, v_amax=None, page_size=16, tile_n=32, forced_skip=None, batches=None):
    """One-token paged decode with NVFP4 QDQ of P (``p_amax`` not None) and/or
    V (``v_amax`` not None), following the reading in the module docstring.

    Inputs as ``oracle.paged_decode``.  Returns (out fp64 [B, h_q, d], lse fp64
    [B, h_q], SkipRecord, flip fp64 [B, h_q, d]): ``flip`` bounds, per output
    element, how far a kernel whose p differs from this fp64 p by a few fp32
    roundings may land from ``out`` (rows without P elements near a rounding
    midpoint have 0)."""
    qf = bf16_bits_to_f64(q)
    B, _, d = qf.shape
    G = h_q // h_kv
    out = np.full((B, h_q, d), np.nan)
    lse = np.full((B, h_q), np.nan)
    flip = np.zeros((B, h_q, d))
    groups, vis_l, skip_l, ratio_l = [], [], [], []
    for b in (range(B) if batches is None else batches):
        L = int(seq_lens[b])
        Kb = bf16_bits_to_f64(gather_paged(k_cache, block_table[b], L, page_size))
        Vb = bf16_bits_to_f64(gather_paged(v_cache, block_table[b], L, page_size))
        for hk in range(h_kv):
            heads = [hq for hq in range(h_q) if kv_head_of(hq, h_q, h_kv) == hk]
            S = scale * (qf[b, heads, :] @ Kb[:, hk, :].T)            # [G, L]
            allowed = np.ones_like(S, dtype=bool)
            fs = None if forced_skip is None else forced_skip.get((b, hk))
            visited, skipped, max_ratio, kept = tile_decisions(S, allowed, threshold, tile_n, fs)
            groups.append((b, hk))
            vis_l.append(visited)
            skip_l.append(skipped)
            ratio_l.append(max_ratio)
            V = Vb[:, hk, :]                                           # [L, d]
            if L == 0 or not kept.any():
                out[b, heads, :] = 0.0
                lse[b, heads] = NEG_INF
                continue
            # running max after each tile, the walk's max (a skipped tile never
            # raises it, so over all tiles or the kept ones it is the same)
            T = (L + tile_n - 1) // tile_n
            pad = T * tile_n - L
            tmax = np.concatenate([S, np.full((G, pad), NEG_INF)], axis=1).reshape(G, T, tile_n).max(axis=2)
            run = np.maximum.accumulate(tmax, axis=1)                  # M_t per row
            Mt = np.repeat(run, tile_n, axis=1)[:, :L]                 # M_t(j) per key
            Mfin = run[:, -1]
            with np.errstate(invalid="ignore"):
                P = np.where(kept, np.exp(S - np.where(np.isfinite(Mt), Mt, 0.0)), 0.0)
            w = np.where(kept, np.exp(np.where(np.isfinite(Mt), Mt, 0.0) - Mfin[:, None]), 0.0)
            l = (P * w).sum(axis=1)                                    # unquantised normaliser
            if p_amax is not None:
                p32 = P.astype(np.float32)
                Pq, _, _, _ = qdq_blocks(p32, p_amax)
                Pflip = p_flip_bound(p32, p_amax)
            else:
                Pq, Pflip = P, np.zeros_like(P)
            if v_amax is not None:
                Vq, _, _, _ = qdq_blocks(V.astype(np.float32).T, v_amax)   # blocks along keys per channel
                Vq = Vq.T
            else:
                Vq = V
            O = ((Pq * w) @ Vq) / l[:, None]
            out[b, heads, :] = O
            lse[b, heads] = Mfin + np.log(l)
            flip[b, heads, :] = ((Pflip * w) @ np.abs(Vq)) / l[:, None]
    T = max((len(x) for x in vis_l), default=0)

    def stack(lst, fill, dtype):
        arr = np.full((len(lst), T), fill, dtype=dtype)
        for i, x in enumerate(lst):
            arr[i, :len(x)] = x
        return arr

    rec = SkipRecord(groups, stack(vis_l, False, bool), stack(skip_l, False, bool),
                     stack(ratio_l, 0.0, np.float64))
    return out, lse, rec, flip
