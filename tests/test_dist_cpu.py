"""Host logic of the multi-GPU path on the CPU: two gloo ranks run the
bench's max-over-ranks timing reduction and the package's per-step
all-reduce of the adapter gradients (the only exchange data parallelism
needs: W is frozen and gets no gradient)."""

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
    from bit_nf4_quantized_15_b200.data_parallel import AdapterGrads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t_max = bench.max_over_ranks(10.0 + rank, world, "cpu")
        # the package's exchange: two linears' dL1/dL2 in one flat buffer,
        # written through the per-linear views with rank-dependent values
        g = AdapterGrads([(3, 2), (5, 4)], r=2, device="cpu")
        for i, (N, K) in enumerate(g.shapes):
            g.dL1[i].copy_(torch.arange(K * 2, dtype=torch.float32).view(K, 2) * (rank + 1) + i)
            g.dL2[i].copy_(torch.arange(2 * N, dtype=torch.float32).view(2, N) * (rank + 1) - i)
        g.all_reduce()
        summed = [(g.dL1[i].clone(), g.dL2[i].clone()) for i in range(2)]
        g.all_reduce(average=True)
        bench.barrier(world)
        q.put((rank, t_max, g.flat.numel(), [(a.tolist(), b.tolist()) for a, b in summed],
               [(a.tolist(), b.tolist()) for a, b in zip(g.dL1, g.dL2)]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_timing_and_grad_allreduce():
    """Two gloo ranks: the bench's max-over-ranks timing, and the package's
    adapter-gradient exchange (AdapterGrads.all_reduce) that the bench calls
    once per step."""
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
    expect_sum, expect_avg = [], []
    for i, (N, K) in enumerate([(3, 2), (5, 4)]):
        a = torch.arange(K * 2, dtype=torch.float32).view(K, 2)
        b = torch.arange(2 * N, dtype=torch.float32).view(2, N)
        s1, s2 = a * 3 + 2 * i, b * 3 - 2 * i        # (1 + 2) x + 2 i over the two ranks
        expect_sum.append((s1.tolist(), s2.tolist()))
        expect_avg.append(((s1 * 2 / 2).tolist(), (s2 * 2 / 2).tolist()))
    for rank, t_max, n, summed, averaged in res:
        assert t_max == 11.0                     # the slowest rank's time
        assert n == (2 * 2 + 2 * 3) + (4 * 2 + 2 * 5)
        assert summed == expect_sum              # summed over ranks, same on every rank, seen through the views
        assert averaged == expect_avg            # the second exchange sums the sums and divides by world


def test_adapter_grads_single_process_is_a_noop():
    sys.path.insert(0, ROOT)
    from bit_nf4_quantized_15_b200.data_parallel import AdapterGrads, adapter_grad_elems
    g = AdapterGrads([(8, 64), (16, 128)], r=4, device="cpu")
    assert g.flat.numel() == adapter_grad_elems(8, 64, 4) + adapter_grad_elems(16, 128, 4)
    assert g.dL1[1].shape == (128, 4) and g.dL2[1].shape == (4, 16)
    g.dL2[0].fill_(3.0)
    g.all_reduce()
    assert g.flat[64 * 4:64 * 4 + 32].eq(3.0).all() and g.nbytes == g.flat.numel() * 4
    with pytest.raises(ValueError):
        adapter_grad_elems(0, 64, 4)


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
