"""Host logic of bench.py's multi-rank path, on CPU: world size 2 over gloo
(the GPU runs use NCCL with the same calls), and the reference arm's
behaviour on ranks other than 0."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # rank r's step times: the slowest rank differs per entry
        mine = [1.0 + rank, 5.0 - rank, 3.0]
        got = bench.max_over_ranks(mine, "cpu", world)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(" ".join(repr(x) for x in got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        vals = [float(x) for x in (tmp_path / f"rank{r}.txt").read_text().split()]
        assert vals == [2.0, 5.0, 3.0]  # every rank sees the maximum of each entry


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([0.25, 7.0], "cpu", 1) == [0.25, 7.0]


def test_whole_job_value_is_weak_scaling_aggregate():
    flops = 2 * 4096 * 4096 * 11008 * 2.0  # one FFN step per rank
    one = bench.whole_job_tflops(flops, 1, 0.5)
    assert bench.whole_job_tflops(flops, 8, 0.5) == pytest.approx(8 * one)
    assert bench.whole_job_tflops(flops, 2, 1.0) == pytest.approx(one)  # a slower rank halves it


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1", MASTER_PORT="29555")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0 and "warmup" in r.stderr
