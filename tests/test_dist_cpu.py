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


# ------------------------------------------------ sharded quantisation
def test_shard_ranges_cover_whole_groups_in_order():
    sys.path.insert(0, ROOT)
    from bit_nf4_quantized_15_b200.sharded import GROUP, shard_ranges
    for n in [0, 64, 16384, 16384 * 3 - 64, 16384 * 7, 4096 * 11008, 37 * 19200]:
        for world in [1, 2, 3, 4, 8, 64]:
            rs = shard_ranges(n, world)
            assert len(rs) == world and rs[0][0] == 0 and rs[-1][1] == n
            groups = []
            for (a, b), (c, _) in zip(rs, rs[1:] + [(n, n)]):
                assert a <= b and b == c                       # contiguous, in rank order
                assert a % GROUP == 0 and (b % GROUP == 0 or b == n)   # whole groups
                groups.append((b - a + GROUP - 1) // GROUP)
            assert max(groups) - min(groups) <= 1              # balanced


def _shard_worker(rank, world, port, q, N, K):
    import datetime
    import numpy as np
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as O
    from bit_nf4_quantized_15_b200.sharded import quantize_sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(5)                       # the same weight on every rank
        a = rng.normal(0, 0.02, (N, K))
        a[:, ::97] *= 40.0
        Wb = O.f32_to_bf16_bits(a.astype(np.float32))
        W = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16)

        def oracle_share(flat):                               # the per-rank step, on the CPU
            bits = flat.view(torch.int16).numpy().view(np.uint16).reshape(1, -1)
            if bits.size == 0:
                return (torch.empty(0, dtype=torch.uint8), torch.empty(0, dtype=torch.uint8),
                        torch.empty(0, dtype=torch.float32))
            codes, c2, c1 = O.quantize(bits)
            return torch.from_numpy(codes), torch.from_numpy(c2), torch.from_numpy(c1)

        w = quantize_sharded(W, quantize_fn=oracle_share)
        codes, c2, c1 = O.quantize(Wb)
        ok = (np.array_equal(w.codes.numpy(), codes) and np.array_equal(w.c2.numpy(), c2)
              and np.array_equal(w.c1.numpy().view(np.uint32), c1.view(np.uint32)) and (w.N, w.K) == (N, K))
        q.put((rank, ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N,K", [(2, 37, 64 * 300), (3, 8, 4096)])
def test_sharded_quantize_equals_whole_weight(world, N, K):
    """Each rank quantises its run of 16384-weight groups, one all-gather per
    buffer: the result equals quantising the whole weight, bit for bit (a
    partial last group; a rank with an empty share when world > groups)."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q, N, K)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [ok for _, ok in res] == [True] * world
