"""Multi-rank host logic of the benchmark, on CPU with the gloo backend.

The hot path shards into independent problems (weak scaling, no data-path
collective); what multi-GPU runs add is host logic: the whole-job figures
(max of the ranks' times, sum of their work) and the reference arm printing
from rank 0 only.  Both are exercised here with world size 2.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _agg_worker(rank, world, port, out_path):
    import datetime

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: slower by r ms, its own amount of work
        local = {"per": {"prefill": 1.0 + rank, "decode": 0.5 + 0.25 * rank, "smallseq": 0.4 - 0.1 * rank},
                 "total_ms": 20.0 + rank, "e2e_ms": 10.0 - rank,
                 "flops": 1e12 * (rank + 1), "dec_bytes": 4e9 + rank, "ss_bytes": 2e9 * (rank + 1)}
        agg = bench.aggregate_ranks(local, world, "cpu")
        if rank == 0:
            with open(out_path, "w") as f:
                json.dump(agg, f)
    finally:
        dist.destroy_process_group()


def test_aggregate_over_two_ranks(tmp_path):
    out = tmp_path / "agg.json"
    mp.start_processes(_agg_worker, args=(2, free_port(), str(out)), nprocs=2, join=True,
                       start_method="spawn")
    agg = json.loads(out.read_text())
    assert agg["per"] == {"prefill": 2.0, "decode": 0.75, "smallseq": 0.4}
    assert agg["total_ms"] == 21.0 and agg["e2e_ms"] == 10.0
    assert agg["flops"] == 3e12 and agg["dec_bytes"] == 8e9 + 1 and agg["ss_bytes"] == 6e9
    # whole-job throughput: all ranks' work over the slowest rank's time
    assert agg["value"] == pytest.approx(3e12 / 2.0e-3 / 1e12)
    assert agg["e2e_value"] == pytest.approx(3e12 / 10.0e-3 / 1e12)


def test_aggregate_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    local = {"per": {"prefill": 1.5, "decode": 1.0, "smallseq": 0.5}, "total_ms": 3.0, "e2e_ms": 4.0,
             "flops": 3e12, "dec_bytes": 1.0, "ss_bytes": 2.0}
    agg = bench.aggregate_ranks(local, 1, "cpu")
    assert agg["per"] == local["per"] and agg["flops"] == 3e12
    assert agg["value"] == pytest.approx(2000.0)


def test_reference_arm_prints_once_under_torchrun():
    """`bench.py --impl reference` under torchrun: rank 0 alone runs the oracle
    sample and prints one JSON line; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


# ---------------------------------------------------------------------------
# one varlen batch sharded by whole sequences across ranks
# ---------------------------------------------------------------------------

def test_sequence_cost_counts_allowed_pairs():
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from attention_varlen_gqa_b200 import shard
    for s_q, s_k in ((1, 1), (5, 5), (7, 3), (3, 9), (0, 4), (4, 0), (128, 300)):
        for causal in (True, False):
            want = int(oracle.allowed_mask(s_q, s_k, causal).sum()) if s_q and s_k else 0
            assert shard.sequence_cost(s_q, s_k, causal) == want


def test_lpt_partition_properties():
    sys.path.insert(0, ROOT)
    from attention_varlen_gqa_b200 import shard
    import numpy as np
    rng = np.random.default_rng(0)
    for world in (1, 2, 3, 8):
        costs = rng.integers(0, 10_000, 37).tolist()
        parts = shard.lpt_partition(costs, world)
        assert len(parts) == world
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(costs)))                       # each sequence exactly once
        loads = [sum(costs[i] for i in p) for p in parts]
        lower = max(sum(costs) / world, max(costs))
        assert max(loads) <= (4 / 3) * lower + 1e-9                  # the list-scheduling bound
        assert parts == shard.lpt_partition(costs, world)           # deterministic
    assert shard.lpt_partition([5, 5, 5], 1) == [[0, 1, 2]]


def _shard_worker(rank, world, port, out_path):
    import datetime

    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    import workloads as W
    from attention_varlen_gqa_b200 import shard

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        lens_q = [70, 0, 129, 33, 200, 5, 64]
        lens_k = [70, 16, 150, 33, 230, 5, 64]
        data = W.varlen_prefill(lens_q, lens_k, h_q=4, h_kv=2, d=64, causal=True, seed=7)
        parts = shard.shard_varlen(lens_q, lens_k, True, world)
        mine = parts[rank]
        rq, cq = shard.shard_rows(data["cu_seqlens_q"], mine)
        rk, ck = shard.shard_rows(data["cu_seqlens_k"], mine)
        out, lse, _ = oracle.varlen_attention(data["q"][rq], data["k"][rk], data["v"][rk], cq, ck, 4, 2, True,
                                              data["scale"])
        got = [None] * world
        dist.all_gather_object(got, (mine, rq.tolist(), out, lse))
        if rank == 0:
            full_o = np.full((int(data["cu_seqlens_q"][-1]), 4, 64), np.nan)
            full_l = np.full((int(data["cu_seqlens_q"][-1]), 4), np.nan)
            for seqs, rows, o, l in got:
                full_o[rows] = o
                full_l[rows] = l
            ref_o, ref_l, _ = oracle.varlen_attention(data["q"], data["k"], data["v"], data["cu_seqlens_q"],
                                                      data["cu_seqlens_k"], 4, 2, True, data["scale"])
            same = bool(np.array_equal(full_o, ref_o, equal_nan=True) and np.array_equal(full_l, ref_l))
            with open(out_path, "w") as f:
                json.dump({"same": same, "parts": parts}, f)
    finally:
        dist.destroy_process_group()


def test_sharded_batch_equals_unsharded(tmp_path):
    """Two gloo ranks each take their LPT share of one varlen batch (whole
    sequences, heaviest first to the least-loaded rank), compute it on its own
    (here with the fp64 oracle), and the gathered results equal the unsharded
    computation exactly: the sequences are independent problems."""
    out = tmp_path / "shard.json"
    mp.start_processes(_shard_worker, args=(2, free_port(), str(out)), nprocs=2, join=True, start_method="spawn")
    res = json.loads(out.read_text())
    assert res["same"]
    assert sorted(i for p in res["parts"] for i in p) == list(range(7))
    assert all(len(p) > 0 for p in res["parts"])
