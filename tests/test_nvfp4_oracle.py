"""The NVFP4 QDQ oracle against its pins, and planted mistakes in copies of
its functions that the pins must catch (CPU only)."""
import inspect
import textwrap

import pytest

from oracle import nvfp4 as N
from tests import nvfp4_pins


@pytest.mark.parametrize("pin", nvfp4_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# (function, text to replace, replacement, what the mistake is)
MUTANTS = [
    ("e2m1_round", "idx = np.where(at_mid & (idx % 2 == 1), idx + 1, idx)",
     "idx = np.where(at_mid, idx + 1, idx)", "E2M1 ties away from zero"),
    ("e2m1_round", "side=\"left\"", "side=\"right\"", "E2M1 ties toward zero"),
    ("e2m1_round", "_E2M1_GRID[idx]", "np.minimum(_E2M1_GRID[idx], 4.0)", "E2M1 saturates at 4"),
    ("e4m3_round", "expo - 1 - 3", "expo - 1 - 4", "E4M3 with 4 mantissa bits"),
    ("e4m3_round", "np.maximum(expo - 1 - 3, -9)", "np.maximum(expo - 1 - 3, -6)", "E4M3 subnormal step"),
    ("e4m3_round", "np.rint(", "np.floor(", "E4M3 truncates"),
    ("tensor_scales", "np.float32(2688.0) / a", "np.float32(448.0) / a", "tensor scale without the E2M1 max"),
    ("qdq_blocks", "bmax = np.abs(xb).max(axis=-1)", "bmax = xb.max(axis=-1)", "block max without abs"),
    ("qdq_blocks", "s = e4m3_round(bmax * k)", "s = (bmax * k).astype(np.float32)", "block scale not rounded"),
    ("qdq_blocks", "q = e2m1_round(xb * r[..., None])", "q = xb * r[..., None]", "values not rounded"),
    ("paged_decode_qdq", "Mt = np.repeat(run, tile_n, axis=1)[:, :L]",
     "Mt = np.repeat(run[:, -1:], L, axis=1)", "P against the final max"),
    ("paged_decode_qdq",
     "Mt = np.repeat(run, tile_n, axis=1)[:, :L]",
     "Mt = np.repeat(np.concatenate([run[:, :1], run[:, :-1]], axis=1), tile_n, axis=1)[:, :L]",
     "P against the max before the tile"),
    ("paged_decode_qdq", "Vq, _, _, _ = qdq_blocks(V.astype(np.float32).T, v_amax)",
     "Vq, _, _, _ = qdq_blocks(V.astype(np.float32), v_amax)", "V blocks along channels"),
    ("paged_decode_qdq", "l = (P * w).sum(axis=1)", "l = (N_qdq(P) * w).sum(axis=1)", "normaliser of quantised P"),
    ("paged_decode_qdq", "O = ((Pq * w) @ Vq) / l[:, None]", "O = ((P * w) @ Vq) / l[:, None]", "P not quantised"),
]


def _mutated(name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(N, name)))
    assert old in src, f"{old!r} not in {name}"
    ns = dict(N.__dict__)
    ns["N_qdq"] = lambda P: N.qdq_blocks(P.astype("float32"), 1.0)[0]
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns[name]


@pytest.mark.parametrize("name,old,new,what", MUTANTS, ids=[m[3] for m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, old, new, what):
    monkeypatch.setattr(N, name, _mutated(name, old, new))
    failed = []
    for pin in nvfp4_pins.ALL_PINS:
        try:
            pin()
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"mutant '{what}' in {name} passed every pin"
