#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = forward + backward of every QLoRA linear of a LLaMA-65B
transformer block (q, k, v, o 8192x8192; gate, up 22016x8192; down
8192x22016 as nn.Linear weights [out, in]; 8192 tokens = 16 x 512; r = 64,
alpha = 16; W ~ N(0, 0.015), X ~ N(0, 1), dY ~ N(0, 1e-2)), seeded
synthetic data, weights already NF4-quantised and resident in HBM.  The
linears are not chained (attention, SwiGLU and norms are not part of the
measured path).  Multi-GPU (torchrun): data parallel, every rank its own
8192 tokens (weak scaling), the adapter gradients all-reduced (sum) over
NCCL once per step by the package's AdapterGrads.

Prints one JSON line (rank 0): whole-job algorithmic TFLOP/s of the step
(4 M K N + 6 M r (K + N) per linear; no dequantisation work counted), plus
  e2e        the same metric through the C ABI with the step's activations
             copied host->device and the adapter gradients device->host
             inside the timed region (the copies of later linears overlap
             the computation of earlier ones, on a copy stream);
  roofline   the fused dequant-GEMM launches (Y of the forward, dX of the
             backward), timed live by events the library records around
             them on the launching stream, against the measured dense-bf16
             peak (burst, or sustained when the sampled SM clock shows the
             power cap), each direction also on its own;
  cpu_baseline   the CPU oracle on a bounded sample of the same workload.
At N = 1 it adds the other workloads as extra keys: llama7b_block (the same
step on a LLaMA-7B block), linear4096_m16 (one 4096x4096 linear at 16
tokens, fwd + bwd, against its HBM roofline), gemv (few-token forward of
the LLaMA-65B FFN linears), quant / dequant / formats (the bulk 2^31-weight
round trip), adapters (adapter merge and the paged AdamW step) and
context_bf16_gemm (cuBLAS on the dequantised weight).
`--impl reference` times the oracle as the reference arm.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("fused QLoRA linear fwd+bwd TFLOP/s and % of roofline; "
          "NF4 (de)quant GB/s vs HBM peak")
WORKLOAD = "llama65b_block"
# DRAM bytes (read + write) per fused dequant-GEMM launch of the headline
# step: the mean over its 14 fused launches (Y and dX of the 7 linears) of
# dram__bytes_read.sum + dram__bytes_write.sum, one single-pass ncu capture
# of `bench.py --no-extras --no-cpu-baseline --steps 1 --warmup 1`.
FUSED_TRAFFIC_BYTES = 907.0e6
RT_WORKLOAD = ("bulk NF4 round trip of 2^31 bf16 weights (4 GiB): half N(0, 0.02), half Student-t(3) x 0.02 "
               "with 0.1% outliers x50; one launch per direction")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def linear_flops(M, N, K, r):
    return 4.0 * M * K * N + 6.0 * M * r * (K + N)


def fwd_gemm_flops(M, N, K, r):
    """Y = X.W^T + (s T).L2: the forward fused launch."""
    return 2.0 * M * K * N + 2.0 * M * r * N


def dx_gemm_flops(M, N, K, r):
    """dX = dY.W + (s dT).L1^T: the backward fused launch."""
    return 2.0 * M * K * N + 2.0 * M * r * K


def nf4_bytes(N, K):
    n = N * K
    return n // 2 + n // 64 + 4 * ((n // 64 + 255) // 256)


def quant_bytes(N, K):
    return 2 * N * K + nf4_bytes(N, K)


def dequant_bytes(N, K):
    return nf4_bytes(N, K) + 2 * N * K


def few_token_bytes(M, N, K, r):
    """Algorithmic bytes of one forward + backward at few tokens: the NF4
    weight read once per direction, the activations, adapters, T and the
    adapter gradients read or written once."""
    w = nf4_bytes(N, K)
    act = 2 * M * K + 2 * M * N          # X, Y (fwd) and dY, dX (bwd) each
    ad = 2 * (K * r + r * N)             # L1, L2
    fwd = w + act + ad + 4 * M * r
    bwd = w + act + ad + 4 * M * r + 4 * (K * r + r * N) + 2 * M * K  # + T in, dL1/dL2 out, X again
    return fwd + bwd


# ----------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples are kept for inspection: QLORA_CLOCKS_DIR, else the system temp directory
        import tempfile
        base = os.environ.get("QLORA_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(base, f"clocks_bench_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "100", "-i", str(self.gpu)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.close()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                smax.append(float(parts[2].split()[0]))
                power.append(float(parts[3].split()[0]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- CPU oracle
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_linear_state(workload: str, which: int, tokens: int):
    """Oracle inputs for one linear of a workload on `tokens` tokens: the
    weight quantised by the oracle, and X, L1, L2, dY as fp64."""
    import oracle as O
    from bit_nf4_quantized_15_b200 import workloads as WL
    wl = WL.WORKLOADS[workload]
    lin = wl.linears[which]
    t = WL.make_linear(wl, lin, seed=which, device="cpu", M=tokens)
    b = WL.bf16_bits
    codes, c2, c1 = O.quantize(b(t["W"]))
    X, L1, L2, dY = (O.bf16_bits_to_f64(b(t[k])) for k in ("X", "L1", "L2", "dY"))
    return dict(codes=codes, c2=c2, c1=c1, N=lin.N, K=lin.K, X=X, L1=L1, L2=L2, dY=dY, s=wl.s, r=wl.r,
                name=lin.name, tokens=tokens)


def oracle_linear_step(st):
    """One oracle step of a linear: dequantise the weight, then the fp64
    forward and backward (the dequantisation is part of every step, as on
    the GPU, where each GEMM dequantises on chip)."""
    import oracle as O
    What = O.bf16_bits_to_f64(O.dequant(st["codes"], st["c2"], st["c1"], st["N"], st["K"]))
    Y, T = O.linear_fwd(st["X"], What, st["L1"], st["L2"], st["s"])
    O.linear_bwd(st["dY"], st["X"], What, st["L1"], st["L2"], st["s"], T)


def time_oracle(fn, reps):
    fn()
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    return (time.perf_counter() - t0) / reps


def cpu_baseline(workload=WORKLOAD, which=0, tokens=64, reps=3):
    st = oracle_linear_state(workload, which, tokens)
    dt = time_oracle(lambda: oracle_linear_step(st), reps)
    flops = linear_flops(tokens, st["N"], st["K"], st["r"])
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"{st['name']} {st['N']}x{st['K']} of {workload}, {tokens} tokens, r={st['r']}: NF4 "
                       f"dequantise of the weight + fp64 forward + backward (numpy on the host), mean of {reps}"),
            "seconds_per_sample": dt}


def cpu_baseline_roundtrip(n=1 << 24, reps=2):
    """The oracle's quantise and dequantise on the first 2^24 weights of the
    round-trip input, in GB/s of the same algorithmic bytes as the GPU."""
    import oracle as O
    from bit_nf4_quantized_15_b200 import workloads as WL
    W = WL.bf16_bits(WL.roundtrip_weights(n, seed=0, device="cpu")).reshape(n // 4096, 4096)
    parts = O.quantize(W)
    tq = time_oracle(lambda: O.quantize(W), reps)
    td = time_oracle(lambda: O.dequant(*parts, n // 4096, 4096), reps)
    return {"quant_gbs": quant_bytes(n // 4096, 4096) / tq / 1e9,
            "dequant_gbs": dequant_bytes(n // 4096, 4096) / td / 1e9, "unit": "GB/s",
            "cores": blas_threads(), "kind": "oracle",
            "sample": f"first 2^24 weights of the round-trip input (4096-wide rows), numpy, mean of {reps}"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    tokens = 128
    st = oracle_linear_state(WORKLOAD, 0, tokens)
    flops = linear_flops(tokens, st["N"], st["K"], st["r"])
    for _ in range(args.warmup):
        oracle_linear_step(st)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_linear_step(st)
    dt = time.perf_counter() - t0
    v = flops * args.steps / dt / 1e12
    cores = blas_threads()
    sample = (f"q-projection {st['N']}x{st['K']} of {WORKLOAD}, {tokens} tokens per step: NF4 dequantise + fp64 "
              f"forward + backward")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_tokens": tokens, "linear": f"q {st['N']}x{st['K']}", "r": st["r"],
                   "alpha": 16},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- GPU workloads
class BlockStep:
    """Forward + backward of every linear of a workload (weights quantised
    and resident, one workspace, adapter gradients in one AdapterGrads)."""

    def __init__(self, q, WL, wl, dev, keep_bf16=False):
        import torch
        from bit_nf4_quantized_15_b200.data_parallel import AdapterGrads
        self.q, self.wl, self.dev = q, wl, dev
        M, r = wl.M, wl.r
        self.grads = AdapterGrads([(l.N, l.K) for l in wl.linears], r, device=dev)
        self.layers = []
        max_ws = 0
        for i, lin in enumerate(wl.linears):
            t = WL.make_linear(wl, lin, seed=i, device=dev)
            w = q.quantize(t["W"])
            L = dict(lin=lin, w=w, X=t["X"], dY=t["dY"], L1=t["L1"], L2=t["L2"],
                     Y=torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev),
                     T=torch.empty((M, r), dtype=torch.float32, device=dev),
                     dX=torch.empty((M, lin.K), dtype=torch.bfloat16, device=dev),
                     dL1=self.grads.dL1[i], dL2=self.grads.dL2[i])
            if keep_bf16:
                L["Wbf16"] = t["W"]
            self.layers.append(L)
            max_ws = max(max_ws, q.workspace_bytes(M, lin.N, lin.K, r))
        self.ws = torch.empty(max_ws, dtype=torch.uint8, device=dev)
        self.flops = sum(linear_flops(M, l.N, l.K, r) for l in wl.linears)
        self.y_flops = sum(fwd_gemm_flops(M, l.N, l.K, r) for l in wl.linears)
        self.dx_flops = sum(dx_gemm_flops(M, l.N, l.K, r) for l in wl.linears)
        # bytes the two fused launches of a linear must move: NF4 weight, the
        # activation in (X or dY), the output (Y or dX), adapters and s.T / s.dT
        self.fused_bytes = sum(2 * nf4_bytes(l.N, l.K) + 2 * 2 * M * (l.K + l.N) + 2 * 2 * r * (l.K + l.N)
                               + 2 * 2 * M * r for l in wl.linears)

    def step(self, events=None, exchange=False, before=None, after=None):
        """One forward + backward of every linear; `before(i)` / `after(i)`
        run around linear i (stream waits and event records of a caller that
        feeds the inputs from the host)."""
        q, s = self.q, self.wl.s
        for i, L in enumerate(self.layers):
            if before is not None:
                before(i)
            if events is not None:
                q.set_gemm_events(events[i][0], events[i][1])
            q.linear_fwd(L["X"], L["w"], L["L1"], L["L2"], s, ws=self.ws, Y=L["Y"], T=L["T"])
            if events is not None:
                q.set_gemm_events(events[i][2], events[i][3])
            q.linear_bwd(L["dY"], L["X"], L["T"], L["w"], L["L1"], L["L2"], s, ws=self.ws,
                         dX=L["dX"], dL1=L["dL1"], dL2=L["dL2"])
            if after is not None:
                after(i)
        if exchange:
            self.grads.all_reduce()

    def timed(self, steps, warmup, world=1, clocks=None):
        """Device time of `steps` steps (CUDA events on the launching stream,
        barrier + synchronize on both sides) and the fused launches' own
        event times per direction."""
        import torch
        q = self.q
        n = len(self.layers)
        ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)] for _ in range(steps)]
        for es in ev:
            for e4 in es:
                for e in e4:
                    e.record()
        for _ in range(max(warmup, 1)):
            self.step(exchange=world > 1)
        torch.cuda.synchronize()
        assert q.read_status(self.dev) == 0, "device status after warm-up"
        barrier(world)
        torch.cuda.synchronize()
        if clocks is not None:
            clocks.start()
            time.sleep(0.3)
        launches0 = q.kernel_launches()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for k in range(steps):
            self.step(events=ev[k], exchange=world > 1)
        t1.record()
        torch.cuda.synchronize()
        launches = q.kernel_launches() - launches0
        barrier(world)
        clk = clocks.stop() if clocks is not None else None
        y_ms = sum(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(steps) for i in range(n)) / steps
        dx_ms = sum(ev[k][i][2].elapsed_time(ev[k][i][3]) for k in range(steps) for i in range(n)) / steps
        assert q.read_status(self.dev) == 0, "device status after the timed region"
        return dict(ms=t0.elapsed_time(t1), y_ms=y_ms, dx_ms=dx_ms, launches=launches, clocks=clk)


def gemv_rates(q, WL, dev, hbm_gbs, pk_kind, copies=4, reps=20):
    """Forward of the LLaMA-65B FFN up (22016x8192) and down (8192x22016)
    linears at M = 1, 4, 16 tokens (r = 64), weights rotated over `copies`
    NF4 copies so that they stream from HBM.  Rate = NF4 weight bytes
    (codes + c2 + c1) per second of the whole forward call."""
    import torch
    wl = WL.WORKLOADS["llama65b_ffn_gemv"]
    res = {}
    for lin in wl.linears:
        t = WL.make_linear(wl, lin, seed=0, device=dev, M=16)
        ws = [q.quantize(t["W"]) for _ in range(copies)]
        del t["W"]
        nbytes = sum(q.storage_bytes(lin.N, lin.K))
        for M in (1, 4, 16):
            X = t["X"][:M].contiguous()
            wsb = torch.empty(q.workspace_bytes(M, lin.N, lin.K, wl.r), dtype=torch.uint8, device=dev)
            Y = torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev)
            T = torch.empty((M, wl.r), dtype=torch.float32, device=dev)
            for i in range(copies):
                q.linear_fwd(X, ws[i], t["L1"], t["L2"], wl.s, ws=wsb, Y=Y, T=T)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(reps):
                q.linear_fwd(X, ws[i % copies], t["L1"], t["L2"], wl.s, ws=wsb, Y=Y, T=T)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / reps
            gbs = nbytes / (us * 1e-6) / 1e9
            res[f"{lin.name}_M{M}"] = {"us": us, "weight_gbs": gbs, "frac": gbs / hbm_gbs}
        del ws
    res["peak"] = hbm_gbs
    res["peak_source"] = f"{pk_kind} HBM copy"
    res["bytes"] = "NF4 codes + c2 + c1 of the linear (0.516 B per weight)"
    res["l2"] = f"weights rotated over {copies} NF4 copies (4 x 93 MB > L2)"
    return res


def few_token_linear(q, WL, dev, hbm_gbs, pk_kind, reps=50):
    """One 4096x4096 QLoRA linear at 16 tokens (r = 16, s = 2), forward +
    backward, L2 flushed before every repetition (a 512 MB write), timed per
    repetition with CUDA events, issued directly and replayed from a CUDA
    graph (no host launch gaps).  Against its HBM roofline: the NF4 weight
    read once per direction plus activations, adapters and gradients."""
    import torch
    wl = WL.WORKLOADS["linear4096_m16"]
    lin = wl.linears[0]
    M, N, K, r, s = wl.M, lin.N, lin.K, wl.r, wl.s
    t = WL.make_linear(wl, lin, seed=0, device=dev)
    w = q.quantize(t["W"])
    ws = torch.empty(q.workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    T = torch.empty((M, r), dtype=torch.float32, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dL1 = torch.empty((K, r), dtype=torch.float32, device=dev)
    dL2 = torch.empty((r, N), dtype=torch.float32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def run():
        q.linear_fwd(t["X"], w, t["L1"], t["L2"], s, ws=ws, Y=Y, T=T)
        q.linear_bwd(t["dY"], t["X"], T, w, t["L1"], t["L2"], s, ws=ws, dX=dX, dL1=dL1, dL2=dL2)

    def per_rep(fn):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in evs:
            flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) * 1e3 for a, b in evs)

    n0 = q.kernel_launches()
    run()
    launches = q.kernel_launches() - n0
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    us_stream = per_rep(run)
    us_graph = None
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            run()
        torch.cuda.current_stream(dev).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        g.replay()
        torch.cuda.synchronize()
        us_graph = per_rep(g.replay)
        del g
    except Exception as e:  # capture unsupported: report the direct timing only
        us_graph = f"capture failed: {type(e).__name__}"
    assert q.read_status(dev) == 0
    nbytes = few_token_bytes(M, N, K, r)
    best = us_graph if isinstance(us_graph, float) else us_stream
    gbs = nbytes / (best * 1e-6) / 1e9
    return {"workload": f"one {N}x{K} linear, {M} tokens, r={r}, s={s}, fwd + bwd; L2 flushed before each rep",
            "us": best, "us_graph": us_graph, "us_stream": us_stream, "launches": launches,
            "bytes": nbytes, "gbs": gbs, "frac": gbs / hbm_gbs, "peak": hbm_gbs,
            "peak_source": f"{pk_kind} HBM copy", "roofline_us": nbytes / hbm_gbs / 1e3,
            "flops": linear_flops(M, N, K, r)}


def adapter_rates(q, WL, dev, hbm_gbs, pk_kind, reps=10):
    """Adapter merge of the LLaMA-65B gate linear (22016x8192, r = 64) and
    the paged AdamW step over all adapters of the LLaMA-65B block (state in
    paged memory, resident on the GPU), as GB/s of their algorithmic bytes
    against the HBM copy bandwidth."""
    import torch
    wl = WL.WORKLOADS["llama65b_block"]
    lin = wl.linears[4]
    t = WL.make_linear(wl, lin, seed=4, device=dev, M=1)
    w = q.quantize(t["W"])
    del t["W"]
    out = torch.empty((lin.N, lin.K), dtype=torch.bfloat16, device=dev)
    for _ in range(2):
        q.adapter_merge(w, t["L1"], t["L2"], wl.s, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        q.adapter_merge(w, t["L1"], t["L2"], wl.s, out=out)
    e1.record()
    torch.cuda.synchronize()
    m_us = e0.elapsed_time(e1) * 1e3 / reps
    m_bytes = nf4_bytes(lin.N, lin.K) + 2 * lin.N * lin.K + 2 * wl.r * (lin.N + lin.K)
    del w, out, t
    n = sum(wl.r * (l.N + l.K) for l in wl.linears)
    p = torch.randn(n, device=dev) * 0.01
    g = torch.randn(n, device=dev) * 1e-3
    pb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    mb, vb = q.paged_empty(n, dev), q.paged_empty(n, dev)
    mb.prefetch(dev.index or 0)
    vb.prefetch(dev.index or 0)
    for k in range(1, 3):
        q.adamw_step(p, g, mb.tensor, vb.tensor, k, lr=1e-4, weight_decay=0.01, p_bf16=pb)
    torch.cuda.synchronize()
    e0.record()
    for k in range(3, 3 + reps):
        q.adamw_step(p, g, mb.tensor, vb.tensor, k, lr=1e-4, weight_decay=0.01, p_bf16=pb)
    e1.record()
    torch.cuda.synchronize()
    a_us = e0.elapsed_time(e1) * 1e3 / reps
    a_bytes = n * (4 * 2 + 4 + 4 * 2 + 4 * 2 + 2)   # p r/w, g, m r/w, v r/w, bf16 copy
    assert q.read_status(dev) == 0
    del mb, vb
    return {
        "merge": {"workload": f"W^ + s (L1 L2)^T of {lin.name} {lin.N}x{lin.K}, r={wl.r}, to bf16", "us": m_us,
                  "bytes": m_bytes, "gbs": m_bytes / m_us / 1e3, "frac": m_bytes / m_us / 1e3 / hbm_gbs},
        "adamw_paged": {"workload": f"AdamW over the {n} adapter parameters of the LLaMA-65B block (r={wl.r}), "
                                    "state in paged memory resident on the GPU", "us": a_us, "bytes": a_bytes,
                        "gbs": a_bytes / a_us / 1e3, "frac": a_bytes / a_us / 1e3 / hbm_gbs},
        "peak": hbm_gbs, "peak_source": f"{pk_kind} HBM copy"}


def bf16_gemm_ms(layers, reps):
    """Mean device time per step of the two weight products of every linear,
    Y = X.W^T and dX = dY.W, done by torch.matmul (cuBLAS) on the dequantised
    bf16 weight: the 16-bit baseline the pages compare QLoRA's
    dequantise-on-the-fly with ("roughly 30-40% slower")."""
    import torch
    outs = [(torch.empty_like(L["Y"]), torch.empty_like(L["dX"])) for L in layers]

    def run():
        for L, (Y, dX) in zip(layers, outs):
            torch.matmul(L["X"], L["Wdq"].t(), out=Y)
            torch.matmul(L["dY"], L["Wdq"], out=dX)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def roundtrip_rates(q, WL, dev, hbm, reps):
    """NF4 quantise / dequantise GB/s on the bulk round trip of 2^31 weights
    (one launch per direction, viewed as a 524288 x 4096 matrix), and the
    same for the compared formats."""
    import torch
    rt_n = WL.ROUNDTRIP_WEIGHTS
    rt_N, rt_K = rt_n // 4096, 4096
    Wrt = WL.roundtrip_weights(rt_n, seed=0, device=dev).view(rt_N, rt_K)
    Wout = torch.empty_like(Wrt)
    qb, db = quant_bytes(rt_N, rt_K), dequant_bytes(rt_N, rt_K)

    def one(fmt, scale="e4m3"):
        wrt = q.NF4Weight.empty(rt_N, rt_K, dev, fmt, scale)
        for _ in range(2):
            q.quantize_into(Wrt, wrt)
            q.dequant(wrt, out=Wout)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(reps):
            q.quantize_into(Wrt, wrt)
        a1.record()
        torch.cuda.synchronize()
        qg = qb * reps / (a0.elapsed_time(a1) / 1e3) / 1e9
        a0.record()
        for _ in range(reps):
            q.dequant(wrt, out=Wout)
        a1.record()
        torch.cuda.synchronize()
        return qg, db * reps / (a0.elapsed_time(a1) / 1e3) / 1e9

    quant_gbs, dequant_gbs = one("nf4")
    formats = {}
    for fmt, scale in (("fp4", "e4m3"), ("int4", "e4m3"), ("nf4", "e5m2")):
        qg, dg = one(fmt, scale)
        formats[fmt if scale == "e4m3" else f"{fmt}_{scale}"] = {
            "quant_gbs": qg, "quant_frac": qg / hbm, "dequant_gbs": dg, "dequant_frac": dg / hbm}
    del Wrt, Wout
    assert q.read_status(dev) == 0
    return quant_gbs, dequant_gbs, qb, db, formats


# ------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import bit_nf4_quantized_15_b200 as q
    from bit_nf4_quantized_15_b200 import workloads as WL

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    pk, pk_kind = peaks()
    hbm = pk["hbm_gbs"]
    extras = world == 1 and not args.no_extras

    wl = WL.WORKLOADS[args.workload]
    M, r = wl.M, wl.r
    blk = BlockStep(q, WL, wl, dev, keep_bf16=extras)
    torch.cuda.synchronize()
    assert q.read_status(dev) == 0

    # ---- timed region: device time of K steps, fused-GEMM events per launch
    res = blk.timed(args.steps, args.warmup, world, ClockSampler(local) if rank == 0 else None)
    ms_max = max_over_ranks(res["ms"], world, dev)
    value = blk.flops * world * args.steps / (ms_max / 1e3) / 1e12
    clk = res["clocks"]
    gemm_ms = res["y_ms"] + res["dx_ms"]
    achieved = (blk.y_flops + blk.dx_flops) / (gemm_ms / 1e3) / 1e12
    y_ach = blk.y_flops / (res["y_ms"] / 1e3) / 1e12
    dx_ach = blk.dx_flops / (res["dx_ms"] / 1e3) / 1e12
    burst, sustained = pk["bf16_tflops"], pk["bf16_tflops_sustained"]
    # The burst peak applies while the SM clock holds its maximum; under the
    # power cap (the sampled clock well below it) the sustained one does.
    at_max = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz") and clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"])
    peak, peak_kind = (burst, "burst") if (at_max or not clk or not clk.get("sm_mhz")) else (sustained, "sustained")
    n_lin = len(blk.layers)
    roofline = {
        "bound": "tensor", "kernel": "fused dequant-GEMM (Y of the forward, dX of the backward)",
        "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
        "traffic": FUSED_TRAFFIC_BYTES,
        "traffic_unit": "DRAM bytes read + written per launch (ncu), mean over the step's fused launches",
        "peak_source": f"{pk_kind} {peak_kind} dense bf16 (SM clock median {clk and clk.get('sm_mhz')} MHz)",
        "frac_burst": achieved / burst, "frac_sustained": achieved / sustained,
        "launches_timed": 2 * n_lin, "ms_per_launch": gemm_ms / (2 * n_lin),
        "y": {"achieved": y_ach, "frac": y_ach / peak, "ms_per_step": res["y_ms"], "flops_per_step": blk.y_flops},
        "dx": {"achieved": dx_ach, "frac": dx_ach / peak, "ms_per_step": res["dx_ms"],
               "flops_per_step": blk.dx_flops},
        "flops_note": "algorithmic: 2 M K N + 2 M r (N or K) per launch; the dequantisation is not counted",
        "algorithmic_bytes_per_launch": blk.fused_bytes / (2 * n_lin),
    }

    line_extra = {}
    if extras:
        # context: the same two products with a plain bf16 weight (cuBLAS)
        for L in blk.layers:
            L["Wdq"] = q.dequant(L["w"])
            L.pop("Wbf16", None)
        bf16_ms = bf16_gemm_ms(blk.layers, max(args.steps, 3))
        for L in blk.layers:
            L.pop("Wdq", None)
        line_extra["context_bf16_gemm"] = {
            "what": "Y = X.W^T and dX = dY.W of the block's 7 linears per step: the fused dequant-GEMM launches "
                    "(NF4 weight, LoRA term included) against torch.matmul (cuBLAS) on the dequantised bf16 weight",
            "fused_ms_per_step": gemm_ms, "bf16_ms_per_step": bf16_ms, "fused_over_bf16": gemm_ms / bf16_ms}

    # ---- end to end through the C ABI: activations in, adapter grads out
    pin = lambda t: t.detach().cpu().pin_memory()
    hX = [pin(L["X"]) for L in blk.layers]
    hdY = [pin(L["dY"]) for L in blk.layers]
    hG = torch.empty(blk.grads.flat.numel(), dtype=torch.float32, pin_memory=True)
    h2d = sum(x.numel() * 2 + y.numel() * 2 for x, y in zip(hX, hdY))
    d2h = blk.grads.nbytes

    # The step's inputs go up on a copy stream, linear by linear, while the
    # earlier linears compute: linear i waits for its own inputs only, and its
    # buffers are refilled for the next step once this step's linear i is done.
    copy_stream = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in blk.layers]
    done = [torch.cuda.Event() for _ in blk.layers]
    begin = torch.cuda.Event()

    def e2e_step():
        cur = torch.cuda.current_stream(dev)
        begin.record(cur)                 # every copy of the step starts after the step does
        copy_stream.wait_event(begin)
        for i, L in enumerate(blk.layers):
            copy_stream.wait_event(done[i])
            with torch.cuda.stream(copy_stream):
                L["X"].copy_(hX[i], non_blocking=True)
                L["dY"].copy_(hdY[i], non_blocking=True)
            ready[i].record(copy_stream)
        blk.step(exchange=world > 1, before=lambda i: cur.wait_event(ready[i]),
                 after=lambda i: done[i].record(cur))
        hG.copy_(blk.grads.flat, non_blocking=True)

    for _ in range(max(args.warmup, 1)):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e = blk.flops * world * args.steps / (e_ms / 1e3) / 1e12
    del hX, hdY, hG
    layers_desc = [f"{l.name} {l.N}x{l.K}" for l in wl.linears]
    del blk
    torch.cuda.empty_cache()

    if extras:
        # ---- the LLaMA-7B block, same step
        if args.workload != "llama7b_block":
            b7 = BlockStep(q, WL, WL.WORKLOADS["llama7b_block"], dev)
            r7 = b7.timed(max(args.steps, 10), args.warmup)
            g7 = r7["y_ms"] + r7["dx_ms"]
            a7 = (b7.y_flops + b7.dx_flops) / (g7 / 1e3) / 1e12
            line_extra["llama7b_block"] = {
                "value": b7.flops * max(args.steps, 10) / (r7["ms"] / 1e3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": r7["ms"] / max(args.steps, 10), "fused_achieved": a7, "fused_frac_burst": a7 / burst,
                "y_achieved": b7.y_flops / (r7["y_ms"] / 1e3) / 1e12,
                "dx_achieved": b7.dx_flops / (r7["dx_ms"] / 1e3) / 1e12,
                "workload": "LLaMA-7B block, 7 linears, 4096 tokens, r=64, alpha=16"}
            del b7
            torch.cuda.empty_cache()
        # ---- one 4096x4096 linear at 16 tokens, fwd + bwd (HBM / launch bound)
        line_extra["linear4096_m16"] = few_token_linear(q, WL, dev, hbm, pk_kind)
        # ---- NF4 quantise / dequantise: the bulk round trip of 2^31 weights
        reps = max(args.steps, 3)
        quant_gbs, dequant_gbs, qb, db, formats = roundtrip_rates(q, WL, dev, hbm, reps)
        line_extra["quant"] = {"workload": RT_WORKLOAD, "value": quant_gbs, "unit": "GB/s", "frac": quant_gbs / hbm,
                               "peak": hbm, "bytes": qb, "peak_source": f"{pk_kind} HBM copy"}
        line_extra["dequant"] = {"workload": RT_WORKLOAD, "value": dequant_gbs, "unit": "GB/s",
                                 "frac": dequant_gbs / hbm, "peak": hbm, "bytes": db,
                                 "peak_source": f"{pk_kind} HBM copy"}
        line_extra["formats"] = {"workload": RT_WORKLOAD + "; FP4 = E2M1/6 and Int4 = k/7 levels (the compared "
                                                           "formats), nf4_e5m2 = NF4 with E5M2 block scales",
                                 "unit": "GB/s", **formats}
        # ---- adapter merge and the paged AdamW step
        line_extra["adapters"] = adapter_rates(q, WL, dev, hbm, pk_kind)
        # ---- few-token forward (dequant-GEMV regime): LLaMA-65B FFN up and down
        if not args.no_gemv:
            line_extra["gemv"] = gemv_rates(q, WL, dev, hbm, pk_kind)

    if rank == 0:
        base = None
        if world == 1 and not args.no_cpu_baseline:
            base = cpu_baseline()
            if extras:
                rt = cpu_baseline_roundtrip()
                line_extra["quant"]["cpu_baseline"] = {k: v for k, v in rt.items() if k != "dequant_gbs"}
                line_extra["dequant"]["cpu_baseline"] = {k: v for k, v in rt.items() if k != "quant_gbs"}
                c1 = cpu_baseline("linear4096_m16", 0, 16, reps=3)
                line_extra["linear4096_m16"]["cpu_baseline"] = c1
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "linears": layers_desc, "tokens_per_gpu": M, "r": r,
                       "alpha": wl.alpha, "global_tokens": M * world, "parallelism": f"dp{world}",
                       "l2": "inputs larger than L2: each step streams several GB of codes and activations",
                       "tokens_per_s": M * world * args.steps / (ms_max / 1e3)},
            "e2e": {"value": e2e, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "roofline": roofline,
            "cpu_baseline": base,
            "clocks": clk,
            "gpu_launches": res["launches"],
            **line_extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_profile_case(args):
    """Small cases for ncu captures, in this order: one LLaMA-65B gate linear
    (22016x8192) at 2048 tokens, quantise then two forward + backward passes
    (engine launches per pass: T, Y, dT, dX, dL1, dL2); two quantise and two
    dequantise passes of a 32768x4096 weight; few-token forwards (M = 16, 1,
    16, 1) of the LLaMA-65B FFN up linear 22016x8192; one forward + backward
    of the 4096x4096 linear at 16 tokens."""
    import torch
    import bit_nf4_quantized_15_b200 as q
    from bit_nf4_quantized_15_b200 import workloads as WL
    wl = WL.WORKLOADS[WORKLOAD]
    lin = wl.linears[4]
    t = WL.make_linear(wl, lin, seed=4, device="cuda", M=2048)
    w = q.quantize(t["W"])
    del t["W"]
    ws = torch.empty(q.workspace_bytes(2048, lin.N, lin.K, wl.r), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        Y, T = q.linear_fwd(t["X"], w, t["L1"], t["L2"], wl.s, ws=ws)
        q.linear_bwd(t["dY"], t["X"], T, w, t["L1"], t["L2"], wl.s, ws=ws)
    del t, w, ws, Y, T
    Wbig = torch.randn((32768, 4096), device="cuda", dtype=torch.float32).mul_(0.02).to(torch.bfloat16)
    wbig = q.NF4Weight.empty(32768, 4096, "cuda")
    out = torch.empty_like(Wbig)
    for _ in range(2):
        q.quantize_into(Wbig, wbig)
    for _ in range(2):
        q.dequant(wbig, out=out)
    del Wbig, wbig, out
    gw = WL.WORKLOADS["llama65b_ffn_gemv"]
    g = WL.make_linear(gw, gw.linears[0], seed=0, device="cuda", M=16)
    gq = q.quantize(g["W"])
    gws = torch.empty(q.workspace_bytes(16, gw.linears[0].N, gw.linears[0].K, gw.r), dtype=torch.uint8,
                      device="cuda")
    for _ in range(2):
        for M in (16, 1):
            q.linear_fwd(g["X"][:M].contiguous(), gq, g["L1"], g["L2"], gw.s, ws=gws)
    del g, gq, gws
    sw = WL.WORKLOADS["linear4096_m16"]
    st = WL.make_linear(sw, sw.linears[0], seed=0, device="cuda")
    sq = q.quantize(st["W"])
    Ys, Ts = q.linear_fwd(st["X"], sq, st["L1"], st["L2"], sw.s)
    q.linear_bwd(st["dY"], st["X"], Ts, sq, st["L1"], st["L2"], sw.s)
    torch.cuda.synchronize()
    assert q.read_status() == 0
    print(json.dumps({"profile_case": f"{lin.name} {lin.N}x{lin.K}", "tokens": 2048, "r": wl.r,
                      "launches": q.kernel_launches()}))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gemv", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="headline workload only")
    ap.add_argument("--profile", action="store_true", help="run the small ncu capture cases")
    args = ap.parse_args(argv)
    if args.profile:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
