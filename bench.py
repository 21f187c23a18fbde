#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = forward + backward of every QLoRA linear of a LLaMA-7B
transformer block (q, k, v, o 4096x4096; gate, up 11008x4096; down
4096x11008; 4096 tokens = 2 x 2048; r = 64, alpha = 16), seeded synthetic
data, weights already NF4-quantised and resident.  The linears are not
chained (attention, SwiGLU and norms are not part of the measured path).
Multi-GPU (torchrun): data parallel, every rank its own 4096 tokens (weak
scaling), the adapter gradients all-reduced (sum) over NCCL once per step.

Prints one JSON line (rank 0): whole-job algorithmic TFLOP/s of the step
(4 M K N + 6 M r (K + N) per linear; no dequantisation work counted), plus
  e2e        same metric through the C ABI with the step's activations
             copied host->device and the adapter gradients device->host
             inside the timed region;
  roofline   the fused dequant-GEMM launches (Y of the forward, dX of the
             backward), timed live by events the library records around
             them, against the measured sustained dense-bf16 peak;
  quant / dequant   NF4 double-quantise and dequantise GB/s of the block's
             7 weights against the measured HBM copy bandwidth;
  cpu_baseline   the CPU oracle on a bounded sample of the same workload.
`--impl reference` times that oracle as the reference arm.
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
WORKLOAD = "llama7b_block"
# DRAM bytes (read + write) per fused dequant-GEMM launch, averaged over the
# 14 launches of a LLaMA-7B block step, from one ncu capture of the current
# engine (profiles/fused_gemm_traffic_llama7b_block.md).
FUSED_TRAFFIC_BYTES = 80.7e6
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


def main_gemm_flops(M, N, K, r):
    # Y = X.W^T + (sT).L2 and dX = dY.W + (s dT).L1^T: the two fused launches
    return (2.0 * M * K * N + 2.0 * M * r * N) + (2.0 * M * K * N + 2.0 * M * r * K)


def quant_bytes(N, K):
    n = N * K
    return 2 * n + n // 2 + n // 64 + 4 * ((n // 64 + 255) // 256)


def dequant_bytes(N, K):
    n = N * K
    return n // 2 + n // 64 + 4 * ((n // 64 + 255) // 256) + 2 * n


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
                                          "-lms", "200", "-i", str(self.gpu)], stdout=self.f,
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
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                smax.append(float(parts[2].split()[0]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle
def oracle_sample_step(state):
    """One bounded oracle step: dequantise the q-projection weight and run the
    fp64 forward and backward of that linear on a sample of tokens."""
    import oracle as O
    codes, c2, c1, N, K, X, L1, L2, dY, s = state
    What = O.bf16_bits_to_f64(O.dequant(codes, c2, c1, N, K))
    Y, T = O.linear_fwd(X, What, L1, L2, s)
    O.linear_bwd(dY, X, What, L1, L2, s, T)


def oracle_state(tokens: int):
    import numpy as np
    import oracle as O
    from bit_nf4_quantized_15_b200 import workloads as WL
    wl = WL.WORKLOADS[WORKLOAD]
    lin = wl.linears[0]
    t = WL.make_linear(wl, lin, seed=0, device="cpu", M=tokens)
    b = lambda x: WL.bf16_bits(x)
    Wb = b(t["W"])
    codes, c2, c1 = O.quantize(Wb)
    X, L1, L2, dY = (O.bf16_bits_to_f64(b(t[k])) for k in ("X", "L1", "L2", "dY"))
    return (codes, c2, c1, lin.N, lin.K, X, L1, L2, dY, wl.s), linear_flops(tokens, lin.N, lin.K, wl.r)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(tokens=256, reps=3):
    state, flops = oracle_state(tokens)
    oracle_sample_step(state)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle_sample_step(state)
    dt = (time.perf_counter() - t0) / reps
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"q-projection 4096x4096 of {WORKLOAD}, {tokens} tokens, r=64: NF4 dequantise of the "
                       f"weight + fp64 forward + backward, numpy on the host, mean of {reps} reps"),
            "seconds_per_sample": dt}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    tokens = 128
    state, flops = oracle_state(tokens)
    for _ in range(args.warmup):
        oracle_sample_step(state)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(state)
    dt = time.perf_counter() - t0
    v = flops * args.steps / dt / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_tokens": tokens, "linear": "q 4096x4096", "r": 64, "alpha": 16},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"q-projection of {WORKLOAD}, {tokens} tokens per step: dequantise + fp64 fwd + bwd"},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


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
    return res


def bf16_gemm_ms(q, layers, reps):
    """Mean device time per step of the two weight products of every linear,
    Y = X.W^T and dX = dY.W, done by torch.matmul (cuBLAS) on the dequantised
    bf16 weight: the 16-bit baseline the pages compare QLoRA's
    dequantise-on-the-fly with ("roughly 30-40% slower")."""
    import torch
    Wh = [q.dequant(L["w"]) for L in layers]
    outs = [(torch.empty_like(L["Y"]), torch.empty_like(L["dX"])) for L in layers]

    def run():
        for L, W, (Y, dX) in zip(layers, Wh, outs):
            torch.matmul(L["X"], W.t(), out=Y)
            torch.matmul(L["dY"], W, out=dX)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del Wh, outs
    return ms


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

    wl = WL.WORKLOADS[args.workload]
    M, r, s = wl.M, wl.r, wl.s
    layers = []
    max_ws = 0
    for i, lin in enumerate(wl.linears):
        t = WL.make_linear(wl, lin, seed=i, device=dev)
        w = q.quantize(t["W"])
        layers.append(dict(lin=lin, Wbf16=t["W"], w=w, X=t["X"], dY=t["dY"], L1=t["L1"], L2=t["L2"],
                           Y=torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev),
                           T=torch.empty((M, r), dtype=torch.float32, device=dev),
                           dX=torch.empty((M, lin.K), dtype=torch.bfloat16, device=dev)))
        max_ws = max(max_ws, q.workspace_bytes(M, lin.N, lin.K, r))
    # adapter gradients of the block live in one flat buffer (one all-reduce per step)
    sizes = [lin.K * r + r * lin.N for lin in wl.linears]
    grads = torch.empty(sum(sizes), dtype=torch.float32, device=dev)
    off = 0
    for L, lin in zip(layers, wl.linears):
        L["dL1"] = grads[off:off + lin.K * r].view(lin.K, r)
        L["dL2"] = grads[off + lin.K * r:off + lin.K * r + r * lin.N].view(r, lin.N)
        off += lin.K * r + r * lin.N
    ws = torch.empty(max_ws, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    assert q.read_status(dev) == 0

    n_lin = len(layers)
    # per step, per linear: events around the forward and the backward fused dequant-GEMM
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_lin)]
          for _ in range(args.steps)]
    for es in ev:
        for e4 in es:
            for e in e4:
                e.record()

    def step(timed=None):
        for i, L in enumerate(layers):
            if timed is not None:
                q.set_gemm_events(timed[i][0], timed[i][1])
            q.linear_fwd(L["X"], L["w"], L["L1"], L["L2"], s, ws=ws, Y=L["Y"], T=L["T"])
            if timed is not None:
                q.set_gemm_events(timed[i][2], timed[i][3])
            q.linear_bwd(L["dY"], L["X"], L["T"], L["w"], L["L1"], L["L2"], s, ws=ws,
                         dX=L["dX"], dL1=L["dL1"], dL2=L["dL2"])
        if world > 1:
            import torch.distributed as dist
            dist.all_reduce(grads)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    assert q.read_status(dev) == 0, "device status after warm-up"

    # ---- timed region: device time of K steps, gemm events per launch
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    launches0 = q.kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    gemm_ms = 0.0
    t0.record()
    for k in range(args.steps):
        step(timed=ev[k])
    t1.record()
    torch.cuda.synchronize()
    for k in range(args.steps):
        for i in range(n_lin):
            gemm_ms += ev[k][i][0].elapsed_time(ev[k][i][1]) + ev[k][i][2].elapsed_time(ev[k][i][3])
    gemm_ms /= args.steps
    launches = q.kernel_launches() - launches0
    barrier(world)
    clk = clocks.stop() if rank == 0 else None
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, world, dev)
    assert q.read_status(dev) == 0, "device status after the timed region"

    step_flops = sum(linear_flops(M, L["lin"].N, L["lin"].K, r) for L in layers)
    value = step_flops * world * args.steps / (ms_max / 1e3) / 1e12
    gemm_flops = sum(main_gemm_flops(M, L["lin"].N, L["lin"].K, r) for L in layers)
    pk, pk_kind = peaks()
    achieved = gemm_flops / (gemm_ms / 1e3) / 1e12
    # context: the same products with a plain bf16 weight (cuBLAS)
    bf16_ms = bf16_gemm_ms(q, layers, max(args.steps, 3))

    # ---- NF4 quantise / dequantise: the bulk round trip of 2^31 weights (4 GiB
    # of bf16: half N(0, 0.02), half Student-t(3) x 0.02 with x50 outliers),
    # one launch per direction, viewed as a 524288 x 4096 matrix.
    for L in layers:
        L.pop("Wbf16", None)
    rt_n = WL.ROUNDTRIP_WEIGHTS
    rt_N, rt_K = rt_n // 4096, 4096
    Wrt = WL.roundtrip_weights(rt_n, seed=0, device=dev).view(rt_N, rt_K)
    Wout = torch.empty_like(Wrt)
    qb, db = quant_bytes(rt_N, rt_K), dequant_bytes(rt_N, rt_K)
    reps = max(args.steps, 3)

    def roundtrip(fmt, scale="e4m3"):
        """(quantise GB/s, dequantise GB/s) of one format on the round trip."""
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

    quant_gbs, dequant_gbs = roundtrip("nf4")
    # the two 4-bit formats the method is compared with (same round trip)
    formats = {}
    for fmt, scale in (("fp4", "e4m3"), ("int4", "e4m3"), ("nf4", "e5m2")):
        qg, dg = roundtrip(fmt, scale)
        formats[fmt if scale == "e4m3" else f"{fmt}_{scale}"] = {
            "quant_gbs": qg, "quant_frac": qg / pk["hbm_gbs"], "dequant_gbs": dg, "dequant_frac": dg / pk["hbm_gbs"]}
    del Wrt, Wout
    assert q.read_status(dev) == 0

    # ---- few-token forward (dequant-GEMV regime): LLaMA-65B FFN up and down
    gemv = gemv_rates(q, WL, dev, pk["hbm_gbs"], pk_kind) if not args.no_gemv else None

    # ---- end to end through the C ABI: activations in, adapter grads out
    pin = lambda t: t.detach().cpu().pin_memory()
    hX = [pin(L["X"]) for L in layers]
    hdY = [pin(L["dY"]) for L in layers]
    hG = torch.empty(grads.numel(), dtype=torch.float32, pin_memory=True)
    h2d = sum(x.numel() * 2 + y.numel() * 2 for x, y in zip(hX, hdY))
    d2h = grads.numel() * 4

    def e2e_step():
        for i, L in enumerate(layers):
            L["X"].copy_(hX[i], non_blocking=True)
            L["dY"].copy_(hdY[i], non_blocking=True)
        step()
        hG.copy_(grads, non_blocking=True)

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
    e2e = step_flops * world * args.steps / (e_ms / 1e3) / 1e12

    if rank == 0:
        base = cpu_baseline() if world == 1 and not args.no_cpu_baseline else None
        hbm = pk["hbm_gbs"]
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "linears": [f"{l.name} {l.N}x{l.K}" for l in wl.linears],
                       "tokens_per_gpu": M, "r": r, "alpha": wl.alpha, "global_tokens": M * world,
                       "parallelism": f"dp{world}",
                       "l2": "inputs larger than L2: each step streams ~0.7 GB of codes and activations",
                       "tokens_per_s": M * world * args.steps / (ms_max / 1e3)},
            "e2e": {"value": e2e, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "roofline": {"bound": "tensor", "kernel": "fused dequant-GEMM (Y forward, dX backward)",
                         "achieved": achieved, "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops_sustained"], "traffic": FUSED_TRAFFIC_BYTES,
                         "traffic_unit": "bytes per launch (DRAM read + write, ncu, mean over the step's launches)",
                         "peak_source": f"{pk_kind} sustained dense bf16",
                         "launches_timed": 2 * n_lin, "ms_per_launch": gemm_ms / (2 * n_lin)},
            "context_bf16_gemm": {
                "what": "Y = X.W^T and dX = dY.W of the 7 linears per step: the fused dequant-GEMM launches (NF4 "
                        "weight, LoRA term included) against torch.matmul (cuBLAS) on the dequantised bf16 weight",
                "fused_ms_per_step": gemm_ms, "bf16_ms_per_step": bf16_ms, "fused_over_bf16": gemm_ms / bf16_ms},
            "quant": {"workload": RT_WORKLOAD, "value": quant_gbs, "unit": "GB/s", "frac": quant_gbs / hbm, "peak": hbm,
                      "bytes": qb, "peak_source": f"{pk_kind} HBM copy"},
            "dequant": {"workload": RT_WORKLOAD, "value": dequant_gbs, "unit": "GB/s", "frac": dequant_gbs / hbm, "peak": hbm,
                        "bytes": db, "peak_source": f"{pk_kind} HBM copy"},
            "formats": {"workload": RT_WORKLOAD + "; FP4 = E2M1/6 and Int4 = k/7 levels (the compared formats), "
                                                  "nf4_e5m2 = NF4 with E5M2 block scales",
                        "unit": "GB/s", **formats},
            "gemv": gemv,
            "cpu_baseline": base,
            "clocks": clk,
            "gpu_launches": launches,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_profile_case(args):
    """One linear (gate, 11008x4096, 4096 tokens, r = 64): quantise, then two
    forward + backward passes; the second is the one to capture with ncu
    (engine launches in order: T, Y, dT, dX, dL1, dL2).  Then two quantise and
    two dequantise passes of a 32768x4096 weight, then few-token forwards
    (M = 16, 1, 16, 1) of the LLaMA-65B FFN up linear 22016x8192, then one
    forward + backward of the q (4096x4096) and down (4096x11008) linears."""
    import torch
    import bit_nf4_quantized_15_b200 as q
    from bit_nf4_quantized_15_b200 import workloads as WL
    wl = WL.WORKLOADS[WORKLOAD]
    lin = wl.linears[4]
    t = WL.make_linear(wl, lin, seed=4, device="cuda")
    w = q.quantize(t["W"])
    ws = torch.empty(q.workspace_bytes(wl.M, lin.N, lin.K, wl.r), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        Y, T = q.linear_fwd(t["X"], w, t["L1"], t["L2"], wl.s, ws=ws)
        q.linear_bwd(t["dY"], t["X"], T, w, t["L1"], t["L2"], wl.s, ws=ws)
    # then two NF4 quantise and two dequantise passes over a 256 MB bf16 weight (> L2)
    Wbig = torch.randn((32768, 4096), device="cuda", dtype=torch.float32).mul_(0.02).to(torch.bfloat16)
    wbig = q.NF4Weight.empty(32768, 4096, "cuda")
    out = torch.empty_like(Wbig)
    for _ in range(2):
        q.quantize_into(Wbig, wbig)
    for _ in range(2):
        q.dequant(wbig, out=out)
    # then few-token forwards of the 65B FFN up linear (22016x8192): M = 16, 1, 16, 1
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
    # then one forward + backward of the q (4096x4096) and down (4096x11008)
    # linears of the same block, so every fused-GEMM shape of the step appears
    for li in (0, 6):
        lt = WL.make_linear(wl, wl.linears[li], seed=li, device="cuda")
        lw = q.quantize(lt["W"])
        lws = torch.empty(q.workspace_bytes(wl.M, wl.linears[li].N, wl.linears[li].K, wl.r), dtype=torch.uint8,
                          device="cuda")
        Yl, Tl = q.linear_fwd(lt["X"], lw, lt["L1"], lt["L2"], wl.s, ws=lws)
        q.linear_bwd(lt["dY"], lt["X"], Tl, lw, lt["L1"], lt["L2"], wl.s, ws=lws)
        del lt, lw, lws, Yl, Tl
    torch.cuda.synchronize()
    assert q.read_status() == 0
    print(json.dumps({"profile_case": f"{lin.name} {lin.N}x{lin.K}", "tokens": wl.M, "r": wl.r,
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
    ap.add_argument("--profile", action="store_true", help="run the single-linear ncu capture case")
    args = ap.parse_args(argv)
    if args.profile:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
