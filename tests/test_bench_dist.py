"""Host-side logic of bench.py's multi-rank path, run as two gloo ranks on CPU.

bench.py under torchrun runs one independent replica per GPU (data parallel over
sequences, no collective on the data path); the only collectives are the timing
barrier and the max over ranks of the measured times, and rank 0 alone prints.
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
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured (r + 1) ms for the step loop and (10 - r) ms end to end
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank], torch.device("cpu"))
        queue.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(queue.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    # every rank sees the slowest rank's times
    assert results[0] == results[1] == [2.0, 10.0, 0.5]


def test_max_over_ranks_without_process_group():
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu")) == [3.0, 4.0]


def test_job_throughput_is_whole_job_weak_scaling():
    # 16 tokens per rank per step, 100 steps, slowest rank 250 ms
    assert bench.job_throughput(1, 16, 100, 250.0) == pytest.approx(6400.0)
    assert bench.job_throughput(8, 16, 100, 250.0) == pytest.approx(8 * 6400.0)


def test_reference_arm_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_layer_copies_exceed_twice_l2():
    # the query path's weights at the V3 shape (W_DQ 22.0 MB + W_UQ 75.5 MB)
    per = (1536 * 7168 + 128 * 192 * 1536) * 2
    n = bench.layer_copies(per)
    assert n == 4 and n * per > 2 * bench.L2_BYTES and (n - 1) * per <= 2 * bench.L2_BYTES + per
    # small layers need many copies, huge ones still two
    assert bench.layer_copies(1 << 20) * (1 << 20) > 2 * bench.L2_BYTES
    assert bench.layer_copies(10 * bench.L2_BYTES) == 2
