"""Plant plausible mistakes in copies of oracle functions and check that the
pins catch every one of them (CPU only; the oracle itself is not modified on
disk)."""
import inspect
import textwrap

import pytest

import oracle
from oracle import attention as A
from tests import oracle_pins

# (function, text to replace, replacement, what the mistake is)
MUTANTS = [
    ("kv_head_of", "return hq // group", "return hq % h_kv", "GQA head mapping interleaved"),
    ("allowed_mask", "j <= i + (s_k - s_q)", "j <= i", "causal mask top-left aligned"),
    ("allowed_mask", "j <= i + (s_k - s_q)", "j < i + (s_k - s_q)", "causal diagonal dropped"),
    ("tile_ratio", "math.exp(tmax - m_prev)", "math.exp(m_prev - tmax)", "ratio sign flipped"),
    ("unit_skipped", "r < threshold", "r <= threshold", "non-strict tile test"),
    ("unit_skipped", "all(r < threshold", "any(r < threshold", "one row decides a unit"),
    ("tile_decisions", "run = np.maximum.accumulate(tmax, axis=1)", "run = tmax",
     "previous tile max instead of running max"),
    ("tile_decisions", "np.all(ratio < threshold, axis=0)", "np.all(ratio <= threshold, axis=0)",
     "non-strict vectorised tile test"),
    ("tile_decisions", "visited = al.reshape(R, T, tile_n).any(axis=(0, 2))",
     "visited = np.ones(T, dtype=bool)", "dead tiles counted as visited"),
    ("softmax_over_kept", "Msafe + np.log(", "np.log(", "LSE drops the max"),
    ("softmax_over_kept", "O = (P @ V)", "O = (P @ V[::-1])", "values in the wrong order"),
    ("softmax_over_kept", "P = np.where(kept, np.exp(Sm - Msafe[:, None]), 0.0)",
     "P = np.where(kept, np.exp(Sm), 0.0) * np.exp(-Msafe[:, None]) + 0.0 * Msafe[:, None]",
     "(control: same value, rearranged)"),
    ("varlen_attention", "S = scale * (", "S = (", "scale dropped"),
    ("varlen_attention", "Kb = kf[k0:k1, hk, :]", "Kb = kf[k0:k1, 0, :]", "kv head ignored"),
    ("paged_decode", "S = scale * (", "S = (", "decode scale dropped"),
    ("paged_decode", "Kb[:, hk, :].T", "Kb[:, 0, :].T", "decode kv head ignored"),
    ("gather_paged", "cache[pages, t % page_size]", "cache[pages, t // page_size % page_size]",
     "page slot index"),
    ("paged_prefill", "gather_paged(k_cache, block_table[b], L, page_size)",
     "gather_paged(k_cache, block_table[0], L, page_size)", "paged prefill reads sequence 0's pages"),
    ("paged_prefill", "cu_k, h_q, h_kv, causal, scale", "cu_k, h_q, h_kv, False, scale",
     "paged prefill drops the causal mask"),
    ("combine_partials", "L = (w * ls).sum(axis=0)", "L = ls.sum(axis=0)", "combine drops weights"),
    ("combine_partials", "Msafe + np.log(", "np.log(", "combine LSE drops the max"),
    ("split_partials", "hi = min(n, (s + 1) * per * tile)", "hi = min(n, (s + 1) * per * tile - 1)",
     "split drops a key"),
    ("smallseq_attention", "kf[k0:k1, hh, :]", "kf[k0:k1, 0, :]", "small-seq head ignored"),
    ("smallseq_attention", "w[b, hh, 0, :] = 0.0", "w[b, hh, 0, :] = 1.0", "weights padding"),
    ("smallseq_backward", "dS = P * (dP - np.dot(P, dP))", "dS = P * dP", "softmax backward drops the row term"),
    ("smallseq_backward", "dq[b, hh] = scale * (dS @ kf[k0:k1, hh])", "dq[b, hh] = (dS @ kf[k0:k1, hh])",
     "grad_Q without the scale"),
    ("smallseq_backward", "dP = vf[k0:k1, hh] @ dO", "dP = kf[k0:k1, hh] @ dO", "grad_attn reads K for V"),
    ("smallseq_backward", "scale * dS[:, None] * qf[b, hh][None, :]", "scale * dS[:, None] * of[b, hh][None, :]",
     "grad_K scales dO instead of q"),
    ("smallseq_backward", "P[:, None] * dO[None, :]", "P[::-1, None] * dO[None, :]", "grad_V keys reversed"),
    ("varlen_backward", "dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))", "dS = P * dP",
     "varlen softmax backward drops the row term"),
    ("varlen_backward", "dk[k0:k1, hk] += scale * (dS.T @ Q)", "dk[k0:k1, hk] += dS.T @ Q", "dK without the scale"),
    ("varlen_backward", "dv[k0:k1, hk] += P.T @ dO", "dv[k0:k1, hk] = P.T @ dO", "dV not summed over the group"),
    ("varlen_backward", "dq[q0:q1, hq] = scale * (dS @ K)", "dq[q0:q1, hq] = scale * (dS @ V)", "dQ from V"),
    ("literal_group_attention", "acc[r][c] *= alpha", "acc[r][c] *= 1.0", "missing O rescale"),
    ("literal_group_attention", "l[r] *= alpha", "l[r] *= 1.0", "missing l rescale"),
    ("bf16_bits_to_f64", "<< 16", "<< 15", "bf16 decode shift"),
    ("round_f64_to_bf16", "np.rint(scaled)", "np.floor(scaled)", "truncation instead of RNE"),
]


def _mutated(name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(A, name)))
    assert old in src, f"{old!r} not in {name}"
    ns = dict(A.__dict__)
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns[name]


def _pins_fail():
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin()
        except Exception:          # an assertion or a crash both count as caught
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name,old,new,what", MUTANTS, ids=[m[3] for m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, old, new, what):
    fn = _mutated(name, old, new)
    monkeypatch.setattr(A, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)
    failed = _pins_fail()
    if what.startswith("(control"):
        assert failed == [], f"equivalent rewrite flagged by {failed}"
    else:
        assert failed, f"mutant '{what}' in {name} passed every pin"
