#!/usr/bin/env python
"""Benchmark of the fused attention-forward hot path on B200.

One step = one pass over every operation of the hot path, each on its own
synthetic workload resident in HBM:
  prefill   varlen GQA causal prefill, 8 sequences with lengths U[512, 8192]
            (seed 0 -> 24 900 tokens), h_q=32, h_kv=8, d=128, fp32 LSE
  decode    paged one-token decode, batch 64, KV lengths U[1024, 32768],
            16-token pages from a permuted pool, h_q=32, h_kv=8, d=128,
            dense 32-split schedule + LSE combine
  smallseq  30 720 one-query sequences with s_kv from {2,4,6,8,12,16},
            h=16, d=128, attention weights returned
The headline `value` is the prefill throughput (TFLOP/s over the allowed
(query, key) pairs); the decode and small-seq rows report HBM GB/s.  Every
operation's inputs are larger than the 126 MB L2, so no flush is needed
between steps.  The skip-softmax workload (4 x 16384 prefill, batch 32 x
32768 decode, peaked sink/window keys) is measured after the timed steps at
thresholds {0, 1e-3, 1e-2, 0.1} and reported with its skipped-unit fraction;
so is an attention-sink workload on the same shapes (strong sink keys that
most query rows align with), on which most tiles are skipped, to show what
skipping saves.

Multi-GPU (torchrun, one rank per GPU): the operations are independent
problems, so every rank runs the same step on its own seed (weak scaling, no
data-path collective); timing is the max over ranks.

`--impl reference` times the fp64 CPU oracle instead (bounded samples of the
prefill workload on the host cores; rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL_WORKLOAD = ("varlen GQA causal prefill bf16: 8 seqs, lengths U[512,8192] (seed 0), "
                    "h_q=32, h_kv=8, d=128, fp32 LSE, threshold 0")
METRIC = "prefill TFLOP/s & decode/small-seq HBM GB/s vs B200 peak; skipped-tile %"
UNIT = "TFLOP/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "smallseq", "skip", "smallseq_bwd",
                                       "decode_skip", "decode_qdq", "varlen_bwd", "paged_prefill"],
                    default="all",
                    help="profiling aid: run a single operation (no JSON line)")
    ap.add_argument("--no-skip", action="store_true",
                    help="leave out the skip-softmax, paged-prefill and the two backward measurements")
    ap.add_argument("--no-cpu", action="store_true", help="leave out the CPU oracle baseline")
    ap.add_argument("--small", action="store_true",
                    help="profiling aid with --only: quarter-size decode / small-seq batches")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


def prefill_flops(lens_q, lens_k, h_q, d, causal):
    """4 * d * h_q * (allowed (query, key) pairs): QK^T and PV, 2 flops per MAC."""
    pairs = 0
    for sq, sk in zip(lens_q, lens_k):
        if causal:
            # row i sees min(sk, max(0, i + sk - sq + 1)) keys
            for_rows = [min(sk, max(0, i + sk - sq + 1)) for i in range(sq)] if sq != sk else None
            pairs += sum(for_rows) if for_rows is not None else sq * (sq + 1) // 2
        else:
            pairs += sq * sk
    return 4.0 * d * h_q * pairs


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "attention_varlen_gqa_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, src_hash, units_key, units):
    """Per-launch DRAM bytes from the committed ncu summary, scaled to this
    launch's units; None when the kernel source changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    if rec.get("source_sha") != src_hash:
        return None
    return rec["dram_bytes"] * units / rec[units_key]


def reduce_over_ranks(x, op, world, device):
    """All-reduce one float over the ranks ("max" or "sum"); identity at world 1."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def aggregate_ranks(local, world, device):
    """Whole-job figures from one rank's measurements.  Times are the max over
    ranks (the slowest rank ends the step); work (FLOPs, bytes) is summed, since
    every rank runs its own problems (weak scaling).  Every rank must call this
    with the same keys in the same order: each key is one collective."""
    out = {"per": {k: reduce_over_ranks(v, "max", world, device) for k, v in sorted(local["per"].items())}}
    for k in ("total_ms", "e2e_ms"):
        out[k] = reduce_over_ranks(local[k], "max", world, device)
    for k in ("flops", "dec_bytes", "ss_bytes"):
        out[k] = reduce_over_ranks(local[k], "sum", world, device)
    out["value"] = out["flops"] / (out["per"]["prefill"] * 1e-3) / 1e12
    out["e2e_value"] = out["flops"] / (out["e2e_ms"] * 1e-3) / 1e12
    return out


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix=f"clocks_rank{self.index}_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the prefill workload)
# ---------------------------------------------------------------------------

def oracle_slab(i, seed=0):
    """Run the fp64 oracle on slab i of the prefill workload: slabs are the
    (sequence, kv-head group) pairs, sequences taken longest first and cycled.
    Returns (flops, seconds, sequence length)."""
    import numpy as np

    import oracle
    import workloads as W
    lens = W.gqa_prefill_lens(seed)
    d, G = 128, 4
    order = sorted(range(len(lens)), key=lambda b: -lens[b])
    L = lens[order[i % len(order)]]
    rng = np.random.default_rng(seed + i)
    q = W.f32_to_bf16_bits(rng.standard_normal((L, G, d), dtype=np.float32))
    k = W.f32_to_bf16_bits(rng.standard_normal((L, 1, d), dtype=np.float32))
    v = W.f32_to_bf16_bits(rng.standard_normal((L, 1, d), dtype=np.float32))
    t0 = time.perf_counter()
    oracle.varlen_attention(q, k, v, [0, L], [0, L], G, 1, True, 1.0 / math.sqrt(d))
    return prefill_flops([L], [L], G, d, True), time.perf_counter() - t0, L


def oracle_sample(budget_s, seed=0):
    """Oracle slabs in order until `budget_s` seconds of CPU time have passed.
    Returns (flops, seconds, description, threads)."""
    done, flops, t_total, i = [], 0.0, 0.0, 0
    while t_total < budget_s and i < 64:
        f, t, L = oracle_slab(i, seed)
        flops += f
        t_total += t
        done.append(L)
        i += 1
    threads = len(os.sched_getaffinity(0))
    desc = (f"fp64 oracle on {len(done)} (sequence, kv-head group) slabs of the prefill workload "
            f"(lengths {done}, 4 q-heads each, causal, d=128)")
    return flops, t_total, desc, threads


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np  # noqa: F401
    per_step, lens_done = [], []
    flops_total = 0.0
    for s in range(args.warmup + args.steps):
        f, t, L = oracle_slab(s)
        if s >= args.warmup:
            per_step.append(t)
            flops_total += f
            lens_done.append(L)
    threads = len(os.sched_getaffinity(0))
    desc = (f"fp64 oracle, one (sequence, kv-head group) slab of the prefill workload per step "
            f"(4 q-heads, causal, d=128; sequence lengths {lens_done})")
    secs = sum(per_step)
    value = flops_total / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PREFILL_WORKLOAD, "sample": "bounded per step"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU path
# ---------------------------------------------------------------------------

def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import numpy as np
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    import attention_varlen_gqa_b200 as A
    import workloads as W
    stream = torch.cuda.current_stream()
    pk = peaks()
    seed = rank

    # ---------------- inputs (device-resident) ----------------
    want = {"prefill", "decode", "smallseq"} if args.only == "all" else {args.only}
    if args.only in ("decode_skip", "decode_qdq"):
        want = {"decode"}
    ops = []
    if "prefill" in want:
        pre = W.gqa_prefill(seed=seed, where="device")
        pre_cq = torch.from_numpy(pre["cu_seqlens_q"]).to(dev)
        pre_ck = torch.from_numpy(pre["cu_seqlens_k"]).to(dev)
        pre_out = torch.empty_like(pre["q"])
        pre_lse = torch.empty(pre["q"].shape[:2], dtype=torch.float32, device=dev)
        pre_flops = prefill_flops(pre["lens_q"], pre["lens_k"], 32, 128, True)

        def do_prefill():
            A.attn_varlen_fwd(pre["q"], pre["k"], pre["v"], pre_cq, pre_ck, pre["max_q"], pre["max_k"],
                              causal=True, out=pre_out, lse=pre_lse)
        ops.append(("prefill", do_prefill))

    if "decode" in want:
        dec_batch = 16 if args.small else 64
        dec = W.paged_decode(W.decode_lens(seed, batch=dec_batch), seed=seed, where="device")
        dec_bt = torch.from_numpy(dec["block_table"]).to(dev)
        dec_sl = torch.from_numpy(dec["seq_lens"]).to(dev)
        dec_out = torch.empty_like(dec["q"])
        dec_lse = torch.empty(dec["q"].shape[:2], dtype=torch.float32, device=dev)
        dec_ws = torch.empty(A.attn_paged_decode_workspace_size(dec_batch, 32, 128), dtype=torch.uint8,
                             device=dev)
        L = dec["seq_lens"].astype(np.int64)
        dec_bytes = float(L.sum() * 8 * 128 * 2 * 2 + dec_batch * 32 * 128 * 2 * 2 + dec_batch * 32 * 4 +
                          (-(-L // 16)).sum() * 4 + dec_batch * 4)

        def do_decode():
            A.attn_paged_decode(dec["q"], dec["k_cache"], dec["v_cache"], dec_bt, dec_sl, out=dec_out,
                                lse=dec_lse, workspace=dec_ws)
        ops.append(("decode", do_decode))

    if "smallseq" in want:
        ss = W.smallseq(seed=seed, batch=7680 if args.small else 30720, where="device")
        ss_cu = torch.from_numpy(ss["cu_seqlens_kv"]).to(dev)
        ss_out = torch.empty_like(ss["q"])
        ss_w = torch.empty((ss["batch"], 16, 1, 16), dtype=torch.bfloat16, device=dev)
        tk = int(ss["cu_seqlens_kv"][-1])
        ss_bytes = float(ss["batch"] * 16 * 128 * 2 * 2 + tk * 16 * 128 * 2 * 2 + ss["batch"] * 16 * 16 * 2 +
                         (ss["batch"] + 1) * 4)

        def do_smallseq():
            A.attn_smallseq_fwd(ss["q"], ss["k"], ss["v"], ss_cu, 16, out=ss_out, weights=ss_w)
        ops.append(("smallseq", do_smallseq))

    if args.only in ("decode_skip", "decode_qdq"):
        # the decode workload in skip mode (threshold 0.1) over the split
        # schedule (one pass; two with quantisation); decode_qdq adds NVFP4
        # quantise-dequantise of P and V (amax 1)
        qkw = dict(p_qdq="nvfp4", p_qdq_amax=1.0, v_qdq="nvfp4", v_qdq_amax=1.0) if args.only == "decode_qdq" else {}
        dsk_ws = torch.empty(A.attn_paged_decode_workspace_size(dec_batch, 32, 128, dec["block_table"].shape[1], 0.1),
                             dtype=torch.uint8, device=dev)
        for _ in range(args.warmup + args.steps):
            A.attn_paged_decode(dec["q"], dec["k_cache"], dec["v_cache"], dec_bt, dec_sl, skip_threshold=0.1,
                                out=dec_out, lse=dec_lse, workspace=dsk_ws, **qkw)
        torch.cuda.synchronize()
        assert A.attn_get_last_device_error() == 0
        return
    if args.only in ("prefill", "decode", "smallseq"):
        fn = dict(ops)[args.only]
        for _ in range(args.warmup + args.steps):
            fn()
        torch.cuda.synchronize()
        assert A.attn_get_last_device_error() == 0
        return
    if args.only == "skip":
        print(json.dumps(measure_skip(A, W, torch, dev, seed, pk, reps=max(1, args.steps))), flush=True)
        return
    if args.only == "paged_prefill":
        measure_paged_prefill(A, W, torch, dev, seed, pk, reps=max(1, args.steps))
        assert A.attn_get_last_device_error() == 0
        return
    if args.only == "varlen_bwd":
        measure_varlen_bwd(A, W, torch, dev, seed, pk, reps=max(1, args.steps))
        assert A.attn_get_last_device_error() == 0
        return
    if args.only == "smallseq_bwd":
        measure_smallseq_bwd(A, W, torch, dev, seed, pk, reps=max(1, args.steps),
                             batch=7680 if args.small else 30720)
        assert A.attn_get_last_device_error() == 0
        return

    def barrier():
        if world > 1:
            dist.barrier()

    # ---------------- warm-up ----------------
    for _ in range(args.warmup):
        for _, fn in ops:
            fn()
    torch.cuda.synchronize()
    assert A.attn_get_last_device_error() == 0

    # ---------------- timed steps ----------------
    ev = {name: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)] for name, _ in ops}
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start.record(stream)
    for s in range(args.steps):
        for name, fn in ops:
            a, b = ev[name][s]
            a.record(stream)
            fn()
            b.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    per = {name: sum(a.elapsed_time(b) for a, b in ev[name]) / args.steps for name, _ in ops}
    assert A.attn_get_last_device_error() == 0

    # ---------------- end to end through the public API, host buffers ----------------
    # Every step copies its q, k, v and cu_seqlens from pinned host memory,
    # runs attn_varlen_fwd and reads its output and LSE back to pinned host
    # memory.  Steps are pipelined over two device buffer sets: the copy-in
    # stream fills set k % 2 while the previous step's kernel and its
    # read-back (copy-out stream) run, the two copy directions sharing the
    # full-duplex link.  The timed region starts before the first copy and
    # ends after the last read-back.
    host = {n: torch.empty(pre[n].shape, dtype=pre[n].dtype, pin_memory=True) for n in ("q", "k", "v")}
    for n in host:
        host[n].copy_(pre[n])
    h_cq = torch.from_numpy(pre["cu_seqlens_q"]).pin_memory()
    h_ck = torch.from_numpy(pre["cu_seqlens_k"]).pin_memory()
    h_out = [torch.empty(pre_out.shape, dtype=pre_out.dtype, pin_memory=True) for _ in range(2)]
    h_lse = [torch.empty(pre_lse.shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    d_in = [{n: torch.empty_like(pre[n]) for n in ("q", "k", "v")} for _ in range(2)]
    d_cq = [torch.empty_like(pre_cq) for _ in range(2)]
    d_ck = [torch.empty_like(pre_ck) for _ in range(2)]
    d_out = [torch.empty_like(pre_out) for _ in range(2)]
    d_lse = [torch.empty_like(pre_lse) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_free = [None, None]      # kernel that last read input set b
    out_free = [None, None]     # read-back that last read output set b

    def e2e_step(k):
        b = k % 2
        with torch.cuda.stream(s_in):
            if in_free[b] is not None:
                s_in.wait_event(in_free[b])
            for n in ("q", "k", "v"):
                d_in[b][n].copy_(host[n], non_blocking=True)
            d_cq[b].copy_(h_cq, non_blocking=True)
            d_ck[b].copy_(h_ck, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(s_in)
        stream.wait_event(loaded)
        if out_free[b] is not None:
            stream.wait_event(out_free[b])
        A.attn_varlen_fwd(d_in[b]["q"], d_in[b]["k"], d_in[b]["v"], d_cq[b], d_ck[b], pre["max_q"], pre["max_k"],
                          causal=True, out=d_out[b], lse=d_lse[b], stream=stream)
        done = torch.cuda.Event()
        done.record(stream)
        in_free[b] = done
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            h_out[b].copy_(d_out[b], non_blocking=True)
            h_lse[b].copy_(d_lse[b], non_blocking=True)
            back = torch.cuda.Event()
            back.record(s_out)
            out_free[b] = back

    for k in range(args.warmup):
        e2e_step(k)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for k in range(args.steps):
        e2e_step(k)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms_local = e0.elapsed_time(e1) / args.steps
    # the result of the last step, read back to the host, against the device-timed run's
    assert torch.equal(h_out[(args.steps - 1) % 2], pre_out.cpu())
    h2d = sum(host[n].numel() * host[n].element_size() for n in host) + 2 * h_cq.numel() * 4
    d2h = h_out[0].numel() * 2 + h_lse[0].numel() * 4
    agg = aggregate_ranks({"per": per, "total_ms": total_ms, "e2e_ms": e2e_ms_local, "flops": pre_flops,
                           "dec_bytes": dec_bytes, "ss_bytes": ss_bytes}, world, dev)

    skip = paged = ssb = vbwd = None
    if not args.no_skip:
        skip = measure_skip(A, W, torch, dev, seed, pk, reps=3)
        paged = measure_paged_prefill(A, W, torch, dev, seed, pk, reps=3)
        ssb = measure_smallseq_bwd(A, W, torch, dev, seed, pk, reps=5)
        vbwd = measure_varlen_bwd(A, W, torch, dev, seed, pk, reps=5)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    # the roofline is per kernel launch on this GPU; `value` and the rows are whole-job
    src = source_hash("prefill.cu", "tcgen05.cuh", "common.cuh")
    pre_tflops = pre_flops / (per["prefill"] * 1e-3) / 1e12
    pre_traffic = recorded_traffic("prefill_gqa_causal_24900", src, "flops", pre_flops)
    roofline = {"bound": "tensor", "achieved": pre_tflops, "peak": pk["bf16"], "unit": "TFLOP/s",
                "frac": pre_tflops / pk["bf16"], "traffic": pre_traffic,
                "peak_kind": f"{pk['src']} bf16 dense (burst)",
                "frac_of_2250_datasheet": pre_tflops / 2250.0}
    P = agg["per"]
    dec_gbs = agg["dec_bytes"] / (P["decode"] * 1e-3) / 1e9 / world
    ss_gbs = agg["ss_bytes"] / (P["smallseq"] * 1e-3) / 1e9 / world
    rows = {
        "prefill": {"ms": P["prefill"], "tflops": agg["value"], "flops": agg["flops"],
                    "frac_of_measured": agg["value"] / world / pk["bf16"],
                    "frac_of_2250": agg["value"] / world / 2250.0, "lens": pre["lens_q"]},
        "decode": {"ms": P["decode"], "gbs": dec_gbs * world, "bytes": agg["dec_bytes"],
                   "frac_of_measured": dec_gbs / pk["hbm"], "frac_of_8000": dec_gbs / 8000.0,
                   "workload": "batch 64, KV U[1024,32768] seed 0, page 16, h 32/8, d 128, 32 splits",
                   "traffic": recorded_traffic("decode_dense_b64", source_hash("decode.cu", "common.cuh"),
                                               "bytes", dec_bytes)},
        "smallseq": {"ms": P["smallseq"], "gbs": ss_gbs * world, "bytes": agg["ss_bytes"],
                     "frac_of_measured": ss_gbs / pk["hbm"], "frac_of_8000": ss_gbs / 8000.0,
                     "workload": "30720 x s_kv{2..16} seed 0, h 16, d 128, + weights",
                     "traffic": recorded_traffic("smallseq_b30720", source_hash("smallseq.cu", "common.cuh"),
                                                 "bytes", ss_bytes)},
    }
    cpu = None
    if world == 1 and not args.no_cpu:
        f, t, desc, threads = oracle_sample(12.0)
        cpu = {"value": f / t / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": t}
    line = {
        "metric": METRIC, "value": agg["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": agg["total_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": PREFILL_WORKLOAD, "step": "prefill + paged decode + small-seq",
                   "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "rows": rows,
        "skip": skip,
        "paged_prefill": paged,
        "smallseq_bwd": ssb,
        "varlen_bwd": vbwd,
        "cpu_baseline": cpu,
        "e2e": {"value": agg["e2e_value"], "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": agg["e2e_ms"],
                "what": "prefill through the C entry point attn_varlen_fwd (the binding calls it when no "
                        "skip threshold, mask or counts are asked for) with q/k/v/cu_seqlens copied from pinned host "
                        "memory and out/lse copied back every step; steps pipelined over two device "
                        "buffer sets (copy-in, kernel and read-back on three streams)"},
        "gpu_launches": 4 * args.steps,
        "clocks": clock_info,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _time_ms(torch, run, reps):
    run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        run()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def _skip_prefill_sweep(A, torch, dev, sp, reps, thresholds):
    cq = torch.from_numpy(sp["cu_seqlens_q"]).to(dev)
    ck = torch.from_numpy(sp["cu_seqlens_k"]).to(dev)
    out = torch.empty_like(sp["q"])
    lse = torch.empty(sp["q"].shape[:2], dtype=torch.float32, device=dev)
    counts = torch.zeros(2, dtype=torch.int64, device=dev)
    dense_flops = prefill_flops(sp["lens_q"], sp["lens_k"], sp["h_q"], sp["d"], True)
    res = {}
    for thr in thresholds:
        def run():
            A.attn_varlen_fwd(sp["q"], sp["k"], sp["v"], cq, ck, sp["max_q"], sp["max_k"], causal=True,
                              out=out, lse=lse, skip_threshold=thr, skip_counts=counts)
        ms = _time_ms(torch, run, reps)
        vis, sk = (int(x) for x in counts.tolist())
        frac = sk / vis if vis and thr > 0 else 0.0
        # executed: QK^T over visited units always, PV only over kept ones
        executed = dense_flops * (1.0 - frac / 2.0)
        res[str(thr)] = {"ms": ms, "skipped_frac": frac, "visited_units": vis, "skipped_units": sk,
                         "dense_equiv_tflops": dense_flops / ms / 1e9, "executed_tflops_est": executed / ms / 1e9}
    return res


def _skip_decode_sweep(A, torch, dev, sd, reps, pk, runs):
    """runs: (key, threshold, schedule) triples, or (key, threshold, schedule,
    (p_amax, v_amax)) with NVFP4 quantise-dequantise of P and V."""
    import numpy as np
    bt = torch.from_numpy(sd["block_table"]).to(dev)
    sl = torch.from_numpy(sd["seq_lens"]).to(dev)
    B, h_q, d = sd["q"].shape
    h_kv = sd["k_cache"].shape[2]
    out = torch.empty_like(sd["q"])
    lse = torch.empty((B, h_q), dtype=torch.float32, device=dev)
    counts = torch.zeros(2, dtype=torch.int64, device=dev)
    kbytes = float(sd["seq_lens"].astype(np.int64).sum() * h_kv * d * 2)
    res = {}
    for run_spec in runs:
        key, thr, sched = run_spec[:3]
        qdq = run_spec[3] if len(run_spec) > 3 else None
        qkw = {} if qdq is None else dict(p_qdq="nvfp4", p_qdq_amax=qdq[0], v_qdq="nvfp4", v_qdq_amax=qdq[1])
        ws = None
        if sched == "split":
            need = (A.lib.attn_paged_decode_qdq_workspace_size(B, h_q, d, bt.shape[1]) if qdq else
                    A.attn_paged_decode_workspace_size(B, h_q, d, bt.shape[1], thr))
            ws = torch.empty(need, dtype=torch.uint8, device=dev)

        def run():
            A.attn_paged_decode(sd["q"], sd["k_cache"], sd["v_cache"], bt, sl, skip_threshold=thr,
                                out=out, lse=lse, workspace=ws, skip_counts=counts, skip_schedule=sched, **qkw)
        ms = _time_ms(torch, run, reps)
        vis, sk = (int(x) for x in counts.tolist())
        frac = sk / vis if vis and thr > 0 else 0.0
        # all of K, V of the kept tiles, q, out and lse
        alg = kbytes + kbytes * (1.0 - frac) + B * h_q * d * 2 * 2 + B * h_q * 4
        res[str(key)] = {"ms": ms, "skipped_frac": frac, "visited_tiles": vis, "skipped_tiles": sk,
                         "gbs": alg / ms / 1e6, "frac_of_measured": alg / ms / 1e6 / pk["hbm"],
                         "schedule": "dense split-KV" if thr == 0 and not qdq else
                         (("two passes over 32 splits" if qdq else "one pass over 32 splits, scores on chip")
                          if sched == "split" else "one sequential split")}
        if qdq:
            res[str(key)]["qdq"] = f"NVFP4 P (amax {qdq[0]}) and V (amax {qdq[1]})"
    return res


def measure_skip(A, W, torch, dev, seed, pk, reps=3):
    """Skip-softmax workload at thresholds {0, 1e-3, 1e-2, 0.1}, plus the
    attention-sink workload on the same shapes, on which most tiles pass the
    skip test (what skipping saves)."""
    thresholds = (0.0, 1e-3, 1e-2, 0.1)
    # skip mode runs the split schedule (workspace given: one pass, or two with
    # quantisation); "0.1/sequential" is the one-split-per-(sequence, kv-head)
    # schedule at the same threshold
    runs = [(t, t, "split") for t in thresholds] + [("0.1/sequential", 0.1, "sequential")]
    # NVFP4 quantise-dequantise of P and V (amax 1 each, the page's usage example)
    runs += [(f"qdq/{t}", t, "split", (1.0, 1.0)) for t in thresholds]
    runs += [("qdq/0.1/sequential", 0.1, "sequential", (1.0, 1.0))]
    res = {}
    sp = W.skip_prefill(seed=seed, where="device")
    res["prefill"] = _skip_prefill_sweep(A, torch, dev, sp, reps, thresholds)
    del sp
    sd = W.skip_decode(seed=seed, where="device")
    res["decode"] = _skip_decode_sweep(A, torch, dev, sd, reps, pk, runs)
    del sd
    sink = {"workload": "attention sinks (not a pages workload): the same shapes; per kv-head a unit "
                        "direction u, q += sqrt(d) u, the first 4 keys of each sequence k += 12 u"}
    sp = W.sink_prefill(seed=seed, where="device")
    sink["prefill"] = _skip_prefill_sweep(A, torch, dev, sp, reps, thresholds)
    del sp
    sd = W.sink_decode(seed=seed, where="device")
    sink["decode"] = _skip_decode_sweep(A, torch, dev, sd, reps, pk, runs)
    del sd
    res["sink"] = sink
    return res


def measure_paged_prefill(A, W, torch, dev, seed, pk, reps=3):
    """Chunked prefill against a paged cache: 16 sequences with contexts
    U[2048, 16384] (seed), the last 512 positions as queries, h_q=32, h_kv=8,
    d=128, 16-token pages, causal.  Not a step row: reported beside it."""
    import numpy as np
    rng = np.random.default_rng(1000 + seed)
    lens_k = rng.integers(2048, 16385, 16)
    lens_q = np.full(16, 512)
    d = W.paged_prefill(lens_q, lens_k, h_q=32, h_kv=8, d=128, seed=seed, where="device")
    bt = torch.from_numpy(d["block_table"]).to(dev)
    cq = torch.from_numpy(d["cu_seqlens_q"]).to(dev)
    sl = torch.from_numpy(d["seq_lens_k"]).to(dev)
    out = torch.empty_like(d["q"])
    lse = torch.empty(d["q"].shape[:2], dtype=torch.float32, device=dev)
    pairs = sum(int(sq) * (int(sk) - int(sq)) + int(sq) * (int(sq) + 1) // 2 for sq, sk in zip(lens_q, lens_k))
    flops = 4.0 * 128 * 32 * pairs

    def run():
        A.attn_paged_prefill(d["q"], d["k_cache"], d["v_cache"], bt, cq, sl, d["max_q"], d["max_k"],
                             causal=True, out=out, lse=lse)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    return {"workload": "16 sequences, contexts U[2048,16384] (seed), last 512 positions as queries, "
                        "h 32/8, d 128, page 16, causal",
            "ms": ms, "flops": flops, "tflops": flops / ms / 1e9, "frac_of_measured": flops / ms / 1e9 / pk["bf16"],
            "lens_k": [int(x) for x in lens_k]}


def measure_varlen_bwd(A, W, torch, dev, seed, pk, reps=5):
    """Varlen GQA backward on the prefill workload (8 sequences, 24 900 tokens,
    h 32/8, d 128, causal) from the GPU forward's output and LSE, dO ~ N(0, 1).
    FLOPs: 2.5 x the forward's (the five matrix products of the backward: S,
    dP, dV, dK, dQ); the kernels recompute S and dP once more.  Not a step
    row: reported beside it."""
    w = W.gqa_prefill(seed=seed, where="device")
    dout = W.output_grad(w, seed=seed, where="device")
    cq = torch.from_numpy(w["cu_seqlens_q"]).to(dev)
    ck = torch.from_numpy(w["cu_seqlens_k"]).to(dev)
    o, lse = A.attn_varlen_fwd(w["q"], w["k"], w["v"], cq, ck, w["max_q"], w["max_k"], causal=True)
    dq, dk, dv = torch.empty_like(w["q"]), torch.empty_like(w["k"]), torch.empty_like(w["v"])
    ws = torch.empty(A.lib.attn_varlen_bwd_workspace_size(w["q"].shape[0], 32), dtype=torch.uint8, device=dev)

    def run():
        A.attn_varlen_bwd(w["q"], w["k"], w["v"], o, dout, lse, cq, ck, w["max_q"], w["max_k"], causal=True,
                          dq=dq, dk=dk, dv=dv, workspace=ws)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    flops = 2.5 * prefill_flops(w["lens_q"], w["lens_k"], 32, 128, True)
    tf = flops / ms / 1e9
    return {"workload": "8 sequences U[512, 8192] seed 0 (24 900 tokens), h 32/8, d 128, causal; dO ~ N(0, 1)",
            "ms": ms, "flops": flops, "tflops": tf, "frac_of_measured": tf / pk["bf16"],
            "frac_of_2250": tf / 2250.0}


def measure_smallseq_bwd(A, W, torch, dev, seed, pk, reps=5, batch=30720):
    """Small-seq backward on the small-seq step workload (30720 tokens, s_kv
    from {2,4,6,8,12,16}, h 16, d 128) with dO ~ N(0, 1) and synthetic saved
    weights; inputs and outputs (4.4 GB) exceed L2.  Not a step row: reported
    beside it.  Bytes: q, dO, K, V, weights read; dq, dK, dV written."""
    s = W.smallseq(seed=seed, batch=batch, where="device")
    g = W.smallseq_grad_inputs(s, seed=seed, where="device")
    cu = torch.from_numpy(s["cu_seqlens_kv"]).to(dev)
    q, k, v = s["q"], s["k"], s["v"]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def run():
        A.attn_smallseq_bwd(q, k, v, g["dout"], g["weights"], cu, s["max_s_kv"], dq=dq, dk=dk, dv=dv)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    byts = (3 * q.numel() + 4 * k.numel() + g["weights"].numel()) * 2
    gbs = byts / ms / 1e6
    return {"workload": f"{batch} x s_kv{{2..16}} seed 0, h 16, d 128; dO, synthetic saved weights",
            "ms": ms, "bytes": byts, "gbs": gbs, "frac_of_measured": gbs / pk["hbm"],
            "frac_of_8000": gbs / 8000.0,
            "traffic": recorded_traffic("smallseq_bwd_b30720", source_hash("smallseq.cu", "common.cuh"),
                                        "bytes", byts)}


if __name__ == "__main__":
    main()
