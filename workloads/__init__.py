"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and
the benchmark.

This module draws numbers and lays out buffers; it holds none of the
attention arithmetic.  Structure (sequence lengths, page permutations, key
counts) always comes from ``numpy.random.default_rng(seed)``.  Values come
from one of two sources, chosen by the caller and recorded in the returned
dict under ``"values"``:

* ``"host"``: ``default_rng`` standard normals in fp32, rounded to bf16 with
  round-to-nearest-even, returned as uint16 bit patterns (small cases that
  the oracle evaluates in full);
* ``"device"``: ``torch.Generator(device="cuda")`` normals in fp32 rounded
  to bf16 on the GPU (full-size cases; numpy would need minutes for the
  multi-GB paged caches).  The oracle then reads sampled slices copied back
  to the host, so both sides still see the same bits.

Shapes follow the workloads of the pages (packed THD tensors, a paged cache
of 16-token pages with a permuted page pool, one-query small-seq batches).
"""

from __future__ import annotations

import numpy as np

SMALLSEQ_BUCKETS = (2, 4, 6, 8, 12, 16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _host_normal(rng, shape):
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def _device_normal(shape, seed, stream):
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(int(seed) * 1000003 + int(stream))
    x = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32)
    return x.to(torch.bfloat16)


def _values(rng, shape, where, seed, stream):
    if where == "host":
        return _host_normal(rng, shape)
    if where == "device":
        return _device_normal(shape, seed, stream)
    raise ValueError(f"unknown value source {where!r}")


def cu_from_lens(lens) -> np.ndarray:
    lens = np.asarray(lens, dtype=np.int64)
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    return cu


# ---------------------------------------------------------------------------
# Prefill
# ---------------------------------------------------------------------------

def varlen_prefill(lens_q, lens_k=None, h_q=4, h_kv=2, d=64, causal=True, seed=0,
                   where="host", scale=None):
    """Packed varlen Q/K/V with the given per-sequence lengths."""
    lens_q = [int(x) for x in lens_q]
    lens_k = list(lens_q) if lens_k is None else [int(x) for x in lens_k]
    cu_q, cu_k = cu_from_lens(lens_q), cu_from_lens(lens_k)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    rng = np.random.default_rng(seed)
    q = _values(rng, (tq, h_q, d), where, seed, 1)
    k = _values(rng, (tk, h_kv, d), where, seed, 2)
    v = _values(rng, (tk, h_kv, d), where, seed, 3)
    return dict(q=q, k=k, v=v, cu_seqlens_q=cu_q, cu_seqlens_k=cu_k,
                lens_q=lens_q, lens_k=lens_k, max_q=max(lens_q, default=0),
                max_k=max(lens_k, default=0), h_q=h_q, h_kv=h_kv, d=d,
                causal=bool(causal), scale=(1.0 / np.sqrt(d)) if scale is None else scale,
                values=where, seed=seed)


def tiny_prefill(seed=0, where="host"):
    """2 sequences of lengths {37, 64}, h_q=4, h_kv=2, d=64, causal."""
    return varlen_prefill([37, 64], h_q=4, h_kv=2, d=64, causal=True, seed=seed, where=where)


def gqa_prefill_lens(seed=0, n=8, lo=512, hi=8192):
    """Sequence lengths uniform in [lo, hi] (inclusive) from ``default_rng(seed)``."""
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, n)]


def gqa_prefill(seed=0, where="device"):
    """8 sequences of lengths U[512, 8192], h_q=32, h_kv=8, d=128, causal."""
    lens = gqa_prefill_lens(seed)
    return varlen_prefill(lens, h_q=32, h_kv=8, d=128, causal=True, seed=seed, where=where)


# ---------------------------------------------------------------------------
# Paged decode
# ---------------------------------------------------------------------------

def paged_layout(seq_lens, page_size, rng):
    """Block table over a shared page pool dealt out in a random order.

    The pool holds exactly sum(ceil(L / page_size)) pages; rows of the block
    table are filled in sequence order from ``rng.permutation(pool)``; unused
    tail entries are 0 and never read.
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int64)
    pages_per = (seq_lens + page_size - 1) // page_size
    pool = int(pages_per.sum())
    perm = rng.permutation(pool).astype(np.int32)
    max_pages = int(pages_per.max()) if len(pages_per) else 0
    bt = np.zeros((len(seq_lens), max(max_pages, 1)), dtype=np.int32)
    off = 0
    for b, n in enumerate(pages_per):
        bt[b, :n] = perm[off:off + n]
        off += int(n)
    return bt, pool


def paged_decode(seq_lens, h_q=32, h_kv=8, d=128, page_size=16, seed=0, where="host"):
    """q [B, h_q, d]; caches [pool, page_size, h_kv, d]; permuted block table."""
    rng = np.random.default_rng(seed)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    bt, pool = paged_layout(seq_lens, page_size, rng)
    B = len(seq_lens)
    q = _values(rng, (B, h_q, d), where, seed, 1)
    kc = _values(rng, (max(pool, 1), page_size, h_kv, d), where, seed, 2)
    vc = _values(rng, (max(pool, 1), page_size, h_kv, d), where, seed, 3)
    return dict(q=q, k_cache=kc, v_cache=vc, block_table=bt, seq_lens=seq_lens,
                h_q=h_q, h_kv=h_kv, d=d, page_size=page_size, num_pages=max(pool, 1),
                max_pages_per_seq=bt.shape[1], scale=1.0 / np.sqrt(d), values=where, seed=seed)


def paged_prefill(lens_q, lens_k, h_q=8, h_kv=2, d=128, page_size=16, seed=0, where="host"):
    """Packed queries [sum(lens_q), h_q, d] against a paged cache holding
    lens_k[b] tokens per sequence (the block table a permutation of the pool);
    the queries of a sequence are the last lens_q[b] positions of its context."""
    rng = np.random.default_rng(seed)
    lens_q = np.asarray(lens_q, dtype=np.int32)
    lens_k = np.asarray(lens_k, dtype=np.int32)
    bt, pool = paged_layout(lens_k, page_size, rng)
    q = _values(rng, (int(lens_q.sum()), h_q, d), where, seed, 1)
    kc = _values(rng, (max(pool, 1), page_size, h_kv, d), where, seed, 2)
    vc = _values(rng, (max(pool, 1), page_size, h_kv, d), where, seed, 3)
    return dict(q=q, k_cache=kc, v_cache=vc, block_table=bt, cu_seqlens_q=cu_from_lens(lens_q),
                seq_lens_k=lens_k, lens_q=[int(x) for x in lens_q], lens_k=[int(x) for x in lens_k],
                max_q=max(int(lens_q.max()), 1), max_k=max(int(lens_k.max()), 1), h_q=h_q, h_kv=h_kv, d=d,
                page_size=page_size, num_pages=max(pool, 1), scale=1.0 / np.sqrt(d), values=where, seed=seed)


def decode_lens(seed=0, batch=64, lo=1024, hi=32768):
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, batch)]


def dense_decode(seed=0, where="device"):
    """Batch 64, KV lengths U[1024, 32768], page 16, h_q=32, h_kv=8, d=128."""
    return paged_decode(decode_lens(seed), seed=seed, where=where)


# ---------------------------------------------------------------------------
# Skip-softmax workloads (sink tokens + local window aligned to the query)
# ---------------------------------------------------------------------------

def _peak_keys_torch(k, qdir, positions, strength=3.0):
    """k[pos] += strength * qdir for the listed positions (torch tensors)."""
    import torch
    kk = k.float()
    idx = torch.as_tensor(positions, device=k.device, dtype=torch.long)
    kk[idx] += strength * qdir
    return kk.to(k.dtype)


def skip_decode(seed=0, batch=32, L=32768, h_q=32, h_kv=8, d=128, page_size=16,
                where="device", n_sink=4, window=256, strength=3.0):
    """Decode with peaked keys: 4 sink tokens and the last 256 tokens of every
    (sequence, kv-head) get k += 3 * qhat, qhat = normalize(sum of the group's
    query vectors)."""
    data = paged_decode([L] * batch, h_q=h_q, h_kv=h_kv, d=d, page_size=page_size,
                        seed=seed, where=where)
    positions = list(range(n_sink)) + list(range(L - window, L))
    G = h_q // h_kv
    if where == "host":
        qf = bf16_bits_to_f32(data["q"]).astype(np.float64)
        kc = bf16_bits_to_f32(data["k_cache"])
        bt = data["block_table"]
        pos = np.asarray(positions)
        for b in range(batch):
            for hk in range(h_kv):
                qs = qf[b, hk * G:(hk + 1) * G].sum(axis=0)
                qhat = qs / np.linalg.norm(qs)
                pages, slots = bt[b, pos // page_size], pos % page_size
                kc[pages, slots, hk] += (strength * qhat).astype(np.float32)
        data["k_cache"] = f32_to_bf16_bits(kc)
    else:
        import torch
        q = data["q"].float()
        kc = data["k_cache"]
        bt = torch.as_tensor(data["block_table"], device=kc.device, dtype=torch.long)
        pos = torch.as_tensor(positions, device=kc.device, dtype=torch.long)
        for b in range(batch):
            pages, slots = bt[b, pos // page_size], pos % page_size
            for hk in range(h_kv):
                qs = q[b, hk * G:(hk + 1) * G].sum(dim=0)
                qhat = qs / qs.norm()
                sub = kc[pages, slots, hk].float() + strength * qhat
                kc[pages, slots, hk] = sub.to(kc.dtype)
    data["peaks"] = dict(n_sink=n_sink, window=window, strength=strength)
    return data


def skip_prefill(seed=0, n_seq=4, L=16384, h_q=32, h_kv=8, d=128, where="device",
                 n_sink=4, window=256, strength=3.0):
    """4 x 16384-token causal prefill with the same peaked-key recipe; qhat
    comes from the sequence's last query token."""
    data = varlen_prefill([L] * n_seq, h_q=h_q, h_kv=h_kv, d=d, causal=True, seed=seed,
                          where=where)
    G = h_q // h_kv
    positions = list(range(n_sink)) + list(range(L - window, L))
    cu = data["cu_seqlens_q"]
    if where == "host":
        qf = bf16_bits_to_f32(data["q"]).astype(np.float64)
        kf = bf16_bits_to_f32(data["k"])
        for b in range(n_seq):
            last = int(cu[b + 1]) - 1
            rows = int(cu[b]) + np.asarray(positions)
            for hk in range(h_kv):
                qs = qf[last, hk * G:(hk + 1) * G].sum(axis=0)
                kf[rows, hk] += (strength * qs / np.linalg.norm(qs)).astype(np.float32)
        data["k"] = f32_to_bf16_bits(kf)
    else:
        import torch
        q = data["q"].float()
        k = data["k"]
        for b in range(n_seq):
            last = int(cu[b + 1]) - 1
            rows = torch.as_tensor(int(cu[b]) + np.asarray(positions), device=k.device)
            for hk in range(h_kv):
                qs = q[last, hk * G:(hk + 1) * G].sum(dim=0)
                sub = k[rows, hk].float() + strength * qs / qs.norm()
                k[rows, hk] = sub.to(k.dtype)
    data["peaks"] = dict(n_sink=n_sink, window=window, strength=strength)
    return data


def skip_parity_prefill(lens, h_q=4, h_kv=2, d=64, seed=0, spread=0.25, peak=6.0,
                        peak_tiles=(0, 3), tile_n=32):
    """Host workload with non-trivial skip sets: per q-head, every query row is
    q0 + spread * N(0,1); keys are N(0,1) except the listed 32-key tiles of
    each sequence, which get peak * q0dir added so that they dominate."""
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in lens]
    cu = cu_from_lens(lens)
    tq = int(cu[-1])
    G = h_q // h_kv
    q0 = rng.standard_normal((h_kv, d)).astype(np.float32)
    q0 /= np.linalg.norm(q0, axis=1, keepdims=True)
    q = np.repeat(q0, G, axis=0)[None, :, :] * np.sqrt(d) \
        + spread * rng.standard_normal((tq, h_q, d)).astype(np.float32)
    k = rng.standard_normal((tq, h_kv, d)).astype(np.float32)
    v = rng.standard_normal((tq, h_kv, d)).astype(np.float32)
    for b in range(len(lens)):
        for t in peak_tiles:
            lo = int(cu[b]) + t * tile_n
            hi = min(int(cu[b + 1]), lo + tile_n)
            if lo < hi:
                k[lo:hi] += peak * q0[None, :, :]
    return dict(q=f32_to_bf16_bits(q), k=f32_to_bf16_bits(k), v=f32_to_bf16_bits(v),
                cu_seqlens_q=cu, cu_seqlens_k=cu, lens_q=lens, lens_k=lens,
                max_q=max(lens), max_k=max(lens), h_q=h_q, h_kv=h_kv, d=d, causal=True,
                scale=1.0 / np.sqrt(d), values="host", seed=seed)


def _sink_directions(seed, h_kv, d):
    rng = np.random.default_rng(seed + 7919)
    u = rng.standard_normal((h_kv, d))
    return (u / np.linalg.norm(u, axis=1, keepdims=True)).astype(np.float32)


def _add_rows(x, rows, heads, delta, where):
    """x[rows, heads] += delta (bf16 buffer: host uint16 bits or a device tensor)."""
    if where == "host":
        xf = bf16_bits_to_f32(x)
        xf[np.ix_(rows, heads)] += delta
        return f32_to_bf16_bits(xf)
    import torch
    r = torch.as_tensor(rows, device=x.device).view(-1, 1)
    h = torch.as_tensor(heads, device=x.device).view(1, -1)
    x[r, h] = (x[r, h].float() + torch.as_tensor(delta, device=x.device)).to(x.dtype)
    return x


def sink_prefill(seed=0, n_seq=4, L=16384, h_q=32, h_kv=8, d=128, n_sink=4, beta=12.0, where="device"):
    """Attention-sink prefill, a workload of this package (not one the pages
    measure) on which the skip rule has work to skip: per kv-head a seeded
    unit direction u; every query row is N(0, 1) + sqrt(d) u of its kv-head
    and the first ``n_sink`` keys of each sequence get k += beta u, so their
    scaled scores sit near beta while all other scores are about N(0, 2)."""
    data = varlen_prefill([L] * n_seq, h_q=h_q, h_kv=h_kv, d=d, causal=True, seed=seed, where=where)
    u = _sink_directions(seed, h_kv, d)
    G = h_q // h_kv
    rows_q = np.arange(int(data["cu_seqlens_q"][-1]))
    data["q"] = _add_rows(data["q"], rows_q, np.arange(h_q), np.repeat(u, G, axis=0)[None] * np.sqrt(d), where)
    sinks = np.concatenate([int(c) + np.arange(n_sink) for c in data["cu_seqlens_k"][:-1]])
    data["k"] = _add_rows(data["k"], sinks, np.arange(h_kv), (beta * u)[None], where)
    data["peaks"] = dict(n_sink=n_sink, beta=beta)
    return data


def sink_decode(seed=0, batch=32, L=32768, h_q=32, h_kv=8, d=128, page_size=16, n_sink=4, beta=12.0,
                where="device"):
    """The attention-sink recipe of ``sink_prefill`` on the paged decode
    shapes: q += sqrt(d) u of its kv-head, the first ``n_sink`` cache
    positions of every sequence get k += beta u."""
    data = paged_decode([L] * batch, h_q=h_q, h_kv=h_kv, d=d, page_size=page_size, seed=seed, where=where)
    u = _sink_directions(seed, h_kv, d)
    G = h_q // h_kv
    B = len(data["seq_lens"])
    q2 = data["q"].reshape(B, h_q, d) if where == "host" else data["q"]
    data["q"] = _add_rows(q2, np.arange(B), np.arange(h_q), np.repeat(u, G, axis=0)[None] * np.sqrt(d), where)
    kc = data["k_cache"]
    shape = kc.shape
    flat = kc.reshape(shape[0] * shape[1], h_kv, d)
    pos = np.arange(n_sink)
    slots = np.concatenate([data["block_table"][b, pos // page_size].astype(np.int64) * page_size
                            + pos % page_size for b in range(B)])
    flat = _add_rows(flat, slots, np.arange(h_kv), (beta * u)[None], where)
    data["k_cache"] = flat.reshape(shape)
    data["peaks"] = dict(n_sink=n_sink, beta=beta)
    return data


# ---------------------------------------------------------------------------
# Small-seq cross attention
# ---------------------------------------------------------------------------

def smallseq_lens(seed=0, batch=30720, choices=SMALLSEQ_BUCKETS):
    return np.random.default_rng(seed).choice(np.asarray(choices), batch).astype(np.int32)


def smallseq(seed=0, batch=30720, h=16, d=128, choices=SMALLSEQ_BUCKETS, where="host",
             lens=None):
    """q [B, h, d]; k/v [sum s_kv, h, d]; s_kv drawn from ``choices``."""
    rng = np.random.default_rng(seed)
    if lens is None:
        lens = rng.choice(np.asarray(choices), batch).astype(np.int32)
    else:
        lens = np.asarray(lens, dtype=np.int32)
        batch = len(lens)
    cu = cu_from_lens(lens)
    tk = int(cu[-1])
    q = _values(rng, (batch, h, d), where, seed, 1)
    k = _values(rng, (max(tk, 1), h, d), where, seed, 2)
    v = _values(rng, (max(tk, 1), h, d), where, seed, 3)
    return dict(q=q, k=k, v=v, cu_seqlens_kv=cu, lens=lens, batch=batch, h=h, d=d,
                max_s_kv=int(lens.max()) if batch else 1, scale=1.0 / np.sqrt(d),
                values=where, seed=seed)


def smallseq_grad_inputs(s, seed=0, where="host"):
    """Backward inputs for a small-seq case ``s``: dO [B, h, d] ~ N(0, 1) and
    saved weights [B, h, 1, max_s_kv] standing in for a forward's: per row,
    uniform(0.05, 1) draws over the row's own keys scaled to sum to 1, zero
    beyond; both bf16."""
    B, h, d, ms = s["batch"], s["h"], s["d"], s["max_s_kv"]
    lens = np.asarray(s["lens"])
    if where == "host":
        rng = np.random.default_rng(seed + 7919)
        dout = _host_normal(rng, (B, h, d))
        u = rng.uniform(0.05, 1.0, (B, h, 1, ms))
        u = u * (np.arange(ms)[None, None, None, :] < lens[:, None, None, None])
        tot = u.sum(axis=3, keepdims=True)
        w = np.divide(u, tot, out=np.zeros_like(u), where=tot > 0)
        return dict(dout=dout, weights=f32_to_bf16_bits(w.astype(np.float32)))
    import torch
    dout = _device_normal((B, h, d), seed, 4)
    g = torch.Generator(device="cuda")
    g.manual_seed(int(seed) * 1000003 + 5)
    u = torch.rand((B, h, 1, ms), generator=g, device="cuda") * 0.95 + 0.05
    ln = torch.as_tensor(lens, device="cuda")
    u = u * (torch.arange(ms, device="cuda")[None, None, None, :] < ln[:, None, None, None])
    tot = u.sum(dim=3, keepdim=True)
    w = torch.where(tot > 0, u / tot.clamp_min(1e-30), torch.zeros_like(u))
    return dict(dout=dout, weights=w.to(torch.bfloat16))


def output_grad(data, seed=0, where="host"):
    """dO ~ N(0, 1) (bf16) shaped like the query tensor of a prefill case."""
    shape = (int(data["cu_seqlens_q"][-1]), data["h_q"], data["d"])
    return _values(np.random.default_rng(seed + 104729), shape, where, seed, 6)
