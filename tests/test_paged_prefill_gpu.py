"""GPU parity: varlen GQA prefill whose keys and values live in a paged cache
(chunked prefill / multi-token decode) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import (assert_close_bf16, assert_close_lse, compare_skip_sets, dev_bf16, dev_i32,
                          unpack_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    import attention_varlen_gqa_b200 as A
    A.attn_get_last_device_error()
    return A


def _dev(data):
    t = {n: dev_bf16(data[n]) for n in ("q", "k_cache", "v_cache")}
    t["bt"] = dev_i32(data["block_table"])
    t["cu_q"] = dev_i32(data["cu_seqlens_q"])
    t["sl"] = dev_i32(data["seq_lens_k"])
    return t


def _run(A, data, causal, thr=0.0, t=None):
    t = t or _dev(data)
    B = len(data["lens_q"])
    words, qb, kt = A.prefill_skip_mask_words(B, data["max_q"], data["max_k"], data["h_q"])
    mask = torch.zeros(max(words, 1), dtype=torch.int32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    out, lse = A.attn_paged_prefill(t["q"], t["k_cache"], t["v_cache"], t["bt"], t["cu_q"], t["sl"],
                                    data["max_q"], data["max_k"], causal=causal, scale=data["scale"],
                                    skip_threshold=thr, skip_mask=mask, skip_counts=counts)
    return out, lse, mask, counts, qb, kt


def _check(A, data, causal, thr=0.0):
    out, lse, mask, counts, qb, kt = _run(A, data, causal, thr)
    assert A.attn_get_last_device_error() == 0
    args = (data["q"], data["k_cache"], data["v_cache"], data["block_table"], data["cu_seqlens_q"],
            data["seq_lens_k"], data["h_q"], data["h_kv"], causal, data["scale"])
    ro, rl, rec = oracle.paged_prefill(*args, threshold=thr)
    if thr > 0:
        bits = unpack_bits(mask, mask.numel() * 32)

        def gpu(grp, T):
            b, hq, r = grp
            base = ((b * qb + r) * data["h_q"] + hq) * kt
            return bits[base:base + T]
        vis, skipped, forced = compare_skip_sets(gpu, rec, None, thr)
        assert int(counts[0]) == vis and int(counts[1]) == skipped, (counts.tolist(), vis, skipped)
        if forced:
            ro, rl, _ = oracle.paged_prefill(*args, threshold=thr, forced_skip=forced)
    else:
        assert int(counts[1]) == 0
    assert_close_bf16(out, ro)
    assert_close_lse(lse, rl)
    return out, lse


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d,heads", [(128, (8, 2)), (64, (6, 3))])
def test_chunked_prefill(A, causal, d, heads):
    """Query chunks shorter than their contexts (the last s_q positions),
    ragged lengths across pages and 128-key tiles, an empty context, a
    sequence without queries."""
    data = W.paged_prefill([100, 1, 257, 0, 64, 3], [300, 50, 257, 10, 1000, 0], h_q=heads[0],
                           h_kv=heads[1], d=d, seed=31)
    _check(A, data, causal)


@pytest.mark.parametrize("thr", [1e-2, 0.1])
@pytest.mark.parametrize("heads", [(4, 2), (3, 1)])
def test_chunked_prefill_skip(A, thr, heads):
    """Skip mode on the paged cache; with a group of 3 an item's two query
    blocks (one head) end one key tile apart."""
    data = W.paged_prefill([200, 77], [700, 333], h_q=heads[0], h_kv=heads[1], d=128, seed=32)
    _check(A, data, True, thr)


def test_paged_equals_contiguous_bit_for_bit(A):
    """The same keys gathered into a packed tensor give the contiguous
    kernel's result exactly (same arithmetic; only the copies differ)."""
    data = W.paged_prefill([257, 640, 33], [257, 640, 33], h_q=8, h_kv=2, d=128, seed=33)
    t = _dev(data)
    out, lse, *_ = _run(A, data, True, t=t)
    ks, vs = [], []
    for b, L in enumerate(data["lens_k"]):
        ks.append(oracle.gather_paged(data["k_cache"], data["block_table"][b], L, 16))
        vs.append(oracle.gather_paged(data["v_cache"], data["block_table"][b], L, 16))
    k, v = dev_bf16(np.concatenate(ks)), dev_bf16(np.concatenate(vs))
    cu_k = dev_i32(W.cu_from_lens(data["lens_k"]))
    o2, l2 = A.attn_varlen_fwd(t["q"], k, v, t["cu_q"], cu_k, data["max_q"], data["max_k"], causal=True,
                               scale=data["scale"])
    assert torch.equal(out, o2) and torch.equal(lse, l2)


def test_one_query_matches_decode(A):
    """One query per sequence against the cache: the decode kernel's result
    (different kernels, both against the same definition)."""
    lens = [17, 300, 1024, 5]
    data = W.paged_prefill([1] * len(lens), lens, h_q=8, h_kv=2, d=128, seed=34)
    t = _dev(data)
    out, lse, *_ = _run(A, data, True, t=t)
    q = t["q"].view(len(lens), 8, 128)
    o2, l2 = A.attn_paged_decode(q, t["k_cache"], t["v_cache"], t["bt"], t["sl"], scale=data["scale"])
    assert (out.view_as(o2).float() - o2.float()).abs().max().item() <= 2e-2
    assert (lse.view_as(l2) - l2).abs().max().item() <= 1e-3


def test_garbage_past_the_end_is_ignored(A):
    """Cache slots past a sequence's end in its last page hold NaN: the
    output stays finite and equal to the clean cache's."""
    data = W.paged_prefill([40, 130], [45, 131], h_q=4, h_kv=2, d=128, seed=35)
    t = _dev(data)
    clean, lse0, *_ = _run(A, data, False, t=t)
    nan = torch.tensor(float("nan"), dtype=torch.bfloat16, device="cuda")
    for b, L in enumerate(data["lens_k"]):
        assert L % 16 != 0
        page = int(data["block_table"][b][(L - 1) // 16])
        t["k_cache"][page, L % 16:] = nan
        t["v_cache"][page, L % 16:] = nan
    dirty, lse1, *_ = _run(A, data, False, t=t)
    assert A.attn_get_last_device_error() == 0
    assert torch.isfinite(dirty.float()).all()
    assert torch.equal(dirty, clean) and torch.equal(lse1, lse0)


def test_bad_block_table_entry(A):
    data = W.paged_prefill([20, 20], [40, 40], h_q=4, h_kv=2, d=64, seed=36)
    t = _dev(data)
    t["bt"][1, 1] = data["num_pages"] + 5
    _run(A, data, True, t=t)
    err = A.attn_get_last_device_error()
    assert err & 4, err                      # ATTN_DEVERR_BLOCK_TABLE


@pytest.mark.parametrize("n_seq", [31, 32, 33, 45])
def test_many_sequences(A, n_seq):
    """Work items are ranked by sequence length for batches of up to 32
    sequences and taken in batch order beyond; both sides of that limit, with
    contexts longer than the queries (sequences outermost in the item order)
    and a few empty queries or contexts."""
    rng = np.random.default_rng(40 + n_seq)
    lens_q = rng.integers(0, 150, n_seq)
    lens_k = lens_q + rng.integers(0, 400, n_seq)
    lens_k[3] = 0
    lens_q[3] = 0
    lens_q[5] = 0
    data = W.paged_prefill(lens_q.tolist(), lens_k.tolist(), h_q=4, h_kv=2, d=64, seed=50 + n_seq)
    _check(A, data, True)


def test_bad_seq_len_in_ranked_batch(A):
    """Sequences outermost and ranked (keys beyond queries, 5 sequences): one
    seq_lens_k entry beyond its block-table row is reported and its rows are
    left alone; the other sequences are exact."""
    data = W.paged_prefill([30, 64, 5, 100, 17], [200, 64, 300, 400, 17], h_q=4, h_kv=2, d=64, seed=37)
    t = _dev(data)
    bad = 2
    t["sl"][bad] = data["block_table"].shape[1] * 16 + 1
    out0 = torch.full_like(t["q"], 3.0)
    out, lse = A.attn_paged_prefill(t["q"], t["k_cache"], t["v_cache"], t["bt"], t["cu_q"], t["sl"],
                                    data["max_q"], data["block_table"].shape[1] * 16 + 1, causal=True,
                                    scale=data["scale"], out=out0)
    err = A.attn_get_last_device_error()
    assert err & 1, err                      # ATTN_DEVERR_CU_SEQLENS
    ro, rl, _ = oracle.paged_prefill(data["q"], data["k_cache"], data["v_cache"], data["block_table"],
                                     data["cu_seqlens_q"], data["seq_lens_k"], data["h_q"], data["h_kv"], True,
                                     data["scale"])
    cu = data["cu_seqlens_q"]
    good = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in range(5) if b != bad])
    gsel = torch.as_tensor(good, device="cuda")
    assert_close_bf16(out[gsel], ro[good])
    assert_close_lse(lse[gsel], rl[good])
    assert torch.all(out[int(cu[bad]):int(cu[bad + 1])] == 3.0)


def test_sequence_order_does_not_change_results(A):
    """The same sequences in reverse batch order (so the longest-first ranking
    and the claim order both change): every sequence's output and LSE are
    bit-identical to the forward order's."""
    lens_q = [40, 130, 7, 256, 65, 1]
    lens_k = [300, 130, 900, 700, 65, 1500]
    data = W.paged_prefill(lens_q, lens_k, h_q=8, h_kv=2, d=128, seed=38)
    t = _dev(data)
    out, lse, *_ = _run(A, data, True, t=t)
    order = list(range(len(lens_q)))[::-1]
    cu = data["cu_seqlens_q"]
    rows = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in order])
    ridx = torch.as_tensor(rows, device="cuda")
    cu_r = dev_i32(W.cu_from_lens([lens_q[b] for b in order]))
    bt_r = t["bt"][torch.as_tensor(order, device="cuda")].contiguous()
    sl_r = t["sl"][torch.as_tensor(order, device="cuda")].contiguous()
    out_r, lse_r = A.attn_paged_prefill(t["q"][ridx].contiguous(), t["k_cache"], t["v_cache"], bt_r, cu_r, sl_r,
                                        data["max_q"], data["max_k"], causal=True, scale=data["scale"])
    assert A.attn_get_last_device_error() == 0
    assert torch.equal(out_r, out[ridx]) and torch.equal(lse_r, lse[ridx])
