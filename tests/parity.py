"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances: bf16 outputs max-abs <= 2e-2 and mean-abs <= 2e-3 against the
oracle rounded to bf16; LSE abs <= 1e-3; skipped-unit sets identical except
for units whose tile test lies within 1e-3 relative of the threshold.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-3
AMBIG_REL = 1e-3


def to_f64(t):
    if isinstance(t, torch.Tensor):
        if t.dtype == torch.bfloat16:
            t = t.float()
        return t.detach().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def assert_close_bf16(gpu, ref, where=None, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    g = to_f64(gpu)
    r = oracle.round_f64_to_bf16(np.asarray(ref, dtype=np.float64))
    if where is not None:
        g, r = g[where], r[where]
    mask = ~np.isnan(r)
    assert mask.any(), "nothing to compare"
    assert np.all(np.isfinite(g[mask])), "non-finite GPU output"
    err = np.abs(g[mask] - r[mask])
    assert err.max() <= max_abs, f"max-abs {err.max():.3e} > {max_abs}"
    assert err.mean() <= mean_abs, f"mean-abs {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


def assert_close_lse(gpu, ref, where=None, tol=LSE_ABS):
    g = to_f64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    if where is not None:
        g, r = g[where], r[where]
    mask = ~np.isnan(r)
    ninf = np.isneginf(r[mask])
    assert np.array_equal(np.isneginf(g[mask]), ninf), "-inf rows differ"
    d = np.abs(g[mask][~ninf] - r[mask][~ninf])
    if d.size:
        assert d.max() <= tol, f"LSE max-abs {d.max():.3e} > {tol}"


def unpack_bits(words, n_bits):
    w = to_np_u32(words)
    bits = np.unpackbits(w.view(np.uint8), bitorder="little")
    return bits[:n_bits].astype(bool)


def to_np_u32(t):
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().numpy().view(np.uint32)
    return np.asarray(t, dtype=np.uint32)


def compare_skip_sets(gpu_skipped, rec, group_index, threshold):
    """gpu_skipped: callable (group tuple, n_tiles) -> bool array of GPU decisions.

    Returns (n_visited, n_skipped, list of groups whose decisions differ only on
    ambiguous units -> GPU decisions for those groups).  Raises on a
    difference outside the ambiguity band.
    """
    lo, hi = threshold * (1 - AMBIG_REL), threshold * (1 + AMBIG_REL)
    forced = {}
    for gi, grp in enumerate(rec.groups):
        vis = rec.visited[gi]
        T = len(vis)
        g = gpu_skipped(grp, T)
        o = rec.skipped[gi]
        diff = (g != o) & vis
        if np.any(g & ~vis):
            raise AssertionError(f"GPU skipped an unvisited unit in {grp}")
        if diff.any():
            amb = (rec.max_ratio[gi] > lo) & (rec.max_ratio[gi] < hi)
            bad = diff & ~amb
            if bad.any():
                t = int(np.flatnonzero(bad)[0])
                raise AssertionError(
                    f"skip decision differs at {grp} tile {t}: gpu={g[t]} oracle={o[t]} "
                    f"max_ratio={rec.max_ratio[gi][t]:.6g} thr={threshold}")
            forced[grp] = g.copy()
    return int(rec.visited.sum()), int(rec.skipped.sum()), forced


def dev_bf16(bits, device="cuda"):
    """uint16 bf16 bit patterns (numpy) -> bf16 CUDA tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def host_bits(t):
    """bf16 tensor -> uint16 numpy bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_i32(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def assert_close_bf16_bound(gpu, ref, bound, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    """assert_close_bf16 with a per-element allowance ``bound`` (>= 0) for
    elements whose reference rests on a rounding decision the two sides may
    take differently (a quantised code next to its rounding midpoint): such an
    element may differ by max_abs + bound; the mean over elements without an
    allowance stays under mean_abs.  Returns (max error, mean error, number
    of elements with an allowance)."""
    g = to_f64(gpu)
    r = oracle.round_f64_to_bf16(np.asarray(ref, dtype=np.float64))
    b = np.asarray(bound, dtype=np.float64)
    mask = ~np.isnan(r)
    assert mask.any(), "nothing to compare"
    assert np.all(np.isfinite(g[mask])), "non-finite GPU output"
    err = np.abs(g - r)
    bad = mask & (err > max_abs + b)
    assert not bad.any(), f"max-abs {err[bad].max():.3e} over {max_abs} + allowance at {np.argwhere(bad)[:3].tolist()}"
    strict = mask & (b == 0)
    if strict.any():
        assert err[strict].mean() <= mean_abs, f"mean-abs {err[strict].mean():.3e} > {mean_abs}"
    return float(err[mask].max()), float(err[strict].mean()) if strict.any() else 0.0, int((mask & (b > 0)).sum())


# Largest errors seen per check, against their bounds: printed at the end of
# the run (tests/conftest.py) so that a tolerance's headroom is visible.
HEADROOM = {}


def record_headroom(name, max_err, max_bound, mean_err, mean_bound):
    old = HEADROOM.get(name, (0.0, max_bound, 0.0, mean_bound))
    HEADROOM[name] = (max(old[0], max_err), max_bound, max(old[2], mean_err), mean_bound)
