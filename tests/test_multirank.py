"""Host logic of the multi-GPU bench path, run as two gloo ranks on the CPU.

On N GPUs every rank runs its own batch (weak scaling: different seeds, no
data exchange); the only collectives are the barrier and the max-reduce of
the per-rank device times. These tests check that logic without a GPU.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from gated_delta_rule_101_b200.inputs import prefill_inputs

        # the max over ranks is what the bench reports as the job's time
        t = bench.max_over_ranks(1.5 + rank, world, "cpu")
        bench.barrier(world)
        # each rank's batch is drawn from its own seed
        p = bench.PREFILL
        inp = prefill_inputs(B=1, T=64, H=2, s0_std=p["s0_std"], la_range=p["la_range"],
                             seed=p["seed"] + 1000 * rank, device="cpu")
        mine = torch.tensor([float(inp.q.float().sum()), float(inp.log_alpha.sum())])
        allv = [torch.zeros(2) for _ in range(world)]
        dist.all_gather(allv, mine)
        out[rank] = (t, [v.tolist() for v in allv])
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduce_and_distinct_batches():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5  # max of 1.5 and 2.5 on both ranks
    sums = res[0][1]
    assert sums == res[1][1]
    assert sums[0] != sums[1], "ranks must run different batches"


def test_reference_arm_two_ranks_only_rank0_reports():
    """bench.py --impl reference under torchrun with 2 ranks: one JSON line, exit 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    import json

    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
