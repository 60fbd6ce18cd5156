"""Host logic of `bench.py --gpus N` (replicas, one process per GPU), run on CPU
with world_size-2 gloo process groups: the step time is the maximum over the
ranks, the job throughput counts every rank's tokens, and the reference arm
runs on rank 0 only. The forward needs no collective on the data path, so
the timing reduction is the only exchange between ranks."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank, expect):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(per_rank[rank], "cpu", world)
        assert got == expect, (rank, got, expect)
        # every rank agrees on the job value computed from the reduced time
        v = bench.job_tokens_per_s(1000, world, got[0])
        assert abs(v - 1000 * world / (expect[0] / 1e3)) < 1e-6 * v
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_step_time_is_the_maximum_over_two_gloo_ranks():
    world = 2
    per_rank = [[10.0, 7.5], [12.5, 3.0]]  # [step ms total, e2e ms total] per rank
    expect = [12.5, 7.5]
    mp.start_processes(_rank_main, args=(world, _free_port(), per_rank, expect), nprocs=world,
                       start_method="spawn", join=True)


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.job_tokens_per_s(16384, 1, 0.5) == pytest.approx(16384 / 0.5e-3)
    assert bench.job_tokens_per_s(16384, 8, 0.5) == pytest.approx(8 * 16384 / 0.5e-3)


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    return subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--gpus", str(world), "--steps", "1",
         "--warmup", "3", "--workload", "tiny_fp32"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_on_a_non_zero_rank_exits_quietly():
    r = _run_reference(1, 2)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_on_rank_zero_prints_one_line():
    r = _run_reference(0, 2)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_metric_names_the_block_and_the_gpu_count():
    r = _run_reference(0, 1)
    assert r.returncode == 0, r.stderr
    line = json.loads([ln for ln in r.stdout.splitlines() if ln.strip()][0])
    assert line["metric"] == "tokens/s and TFLOPS (% bf16 peak) for RoM projection block fwd, 1 B200"


def _grad_rank_main(rank, world, port):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from mixture_experts_projections_b200 import rom

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank gradients of different shapes, started in the backward's
        # order (dW_out first, the router's next, Conv / Gate last)
        g = {n: torch.full(shape, float(rank + 1)) * (i + 1)
             for i, (n, shape) in enumerate([("dw_out", (3, 4, 5)), ("dw_r", (4, 2)),
                                             ("dbias", (2,)), ("dw_conv", (3, 5, 4)),
                                             ("dw_gate", (3, 5, 4))])}
        sync = rom.GradientAllReduce()
        sync.start(g["dw_out"])
        sync.start(g["dw_r"], g["dbias"])
        sync.start(g["dw_conv"], g["dw_gate"])
        sync.finish()
        assert sync.pending == []
        total = sum(r + 1 for r in range(world))
        for i, n in enumerate(["dw_out", "dw_r", "dbias", "dw_conv", "dw_gate"]):
            assert torch.all(g[n] == total * (i + 1)), (rank, n)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_data_parallel_gradients_are_summed_over_two_gloo_ranks():
    """The data-parallel gradient exchange of the backward (GradientAllReduce,
    which rom.block_backward drives with grad_sync): every rank ends with the
    sum of all ranks' gradients, in the order they were started."""
    world = 2
    mp.start_processes(_grad_rank_main, args=(world, _free_port()), nprocs=world,
                       start_method="spawn", join=True)
