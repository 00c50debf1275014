"""The N > 1 path of bench.py on CPU: two gloo ranks own different sequences (no data
moves between them) and report the slowest rank's time; under torchrun the reference
arm runs on rank 0 only."""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from gated_delta_rule_102_b200 import synth
        wl = bench.rank_workload(synth.WORKLOADS["batch64"], rank)
        mine = synth.step_inputs(wl, 0, rows=[0])["qkv"].tobytes()[:256]
        seen = [None] * world
        dist.all_gather_object(seen, mine)
        slowest = bench.max_over_ranks(1.5 + rank, torch.device("cpu"), world)
        # ragged launches: each rank draws its own token counts; the job total is their sum
        rag = bench.rank_workload(synth.WORKLOADS["ragged_b64_t16"], rank)
        mine_tokens = float(synth.varlen_counts(rag, 0, rag.tokens).sum())
        everyone = [None] * world
        dist.all_gather_object(everyone, mine_tokens)
        total = bench.sum_over_ranks(mine_tokens, torch.device("cpu"), world)
        q.put((rank, slowest, len(set(seen)) == world, total == sum(everyone) and len(set(everyone)) == world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_sequences_and_report_the_slowest():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [2.5, 2.5]      # max over ranks on every rank
    assert all(r[2] for r in res)                 # each rank draws different sequences
    assert all(r[3] for r in res)                 # token totals are summed over ranks


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "1"]
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 3
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
