"""The fp64 oracle against closed forms, invariants, torch's SDPA and brute force."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from tests import oracle_pins
from workloads import cu_from_lens, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_zero_length_sequence_golden():
    """The mixed-length case with one fully padded sequence: its output is zero."""
    with open(os.path.join(GOLDEN, "zero_length_sequence.json")) as f:
        g = json.load(f)
    B, T, H, D = g["B"], g["T"], g["H"], g["D"]
    lens = g["seq_lengths"]
    rng = np.random.default_rng(0)
    # left padding of T - L positions == bottom-right causal alignment with
    # s_q = T query rows and s_k = L keys: row i sees keys j <= i - (T - L)
    cu_q = cu_from_lens([T] * B)
    cu_k = cu_from_lens(lens)
    q = f32_to_bf16_bits(rng.standard_normal((B * T, H, D), dtype=np.float32))
    k = f32_to_bf16_bits(rng.standard_normal((int(cu_k[-1]), H, D), dtype=np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((int(cu_k[-1]), H, D), dtype=np.float32))
    out, lse, _ = oracle.varlen_attention(q, k, v, cu_q, cu_k, H, H, True, 1 / math.sqrt(D))
    for b, L in enumerate(lens):
        rows = slice(b * T, b * T + T - L)            # padding positions
        assert np.all(out[rows] == g["expected_padded_output"])
        assert np.all(np.isneginf(lse[rows]))
        valid = out[b * T + T - L:(b + 1) * T]
        assert np.all(np.isfinite(valid)) and (L == 0 or np.abs(valid).max() > 0)
