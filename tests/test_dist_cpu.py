"""Host logic of the multi-GPU path on the CPU: two gloo ranks run the
bench's max-over-ranks timing reduction and the per-step all-reduce of the
adapter gradients (the only exchange data parallelism needs: W is frozen and
gets no gradient)."""

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t_max = bench.max_over_ranks(10.0 + rank, world, "cpu")
        # adapter gradients of 2 linears in one flat buffer, rank-dependent values
        grads = torch.arange(12, dtype=torch.float32) * (rank + 1)
        dL1 = grads[:8].view(4, 2)
        dist.all_reduce(grads)
        bench.barrier(world)
        q.put((rank, t_max, grads.tolist(), dL1.sum().item()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_timing_and_grad_allreduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    expect = [float(i * 3) for i in range(12)]  # (1 + 2) * i
    for rank, t_max, grads, view_sum in res:
        assert t_max == 11.0                     # the slowest rank's time
        assert grads == expect                   # summed over ranks, same on every rank
        assert view_sum == sum(expect[:8])       # views into the flat buffer see the reduced values


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""
