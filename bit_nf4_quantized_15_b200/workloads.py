"""Seeded synthetic workloads (shapes and random draws only, no arithmetic
of the method).  Shared by the tests, the bench and the smoke check; both
the CUDA path and the CPU oracle consume the tensors made here.

Shapes follow LLaMA-family linears (the pages fine-tune LLaMA 7B-65B with
LoRA on every linear layer).  Weights are stored as ``nn.Linear`` weights
``[N, K]`` = (out, in).  "N(0, s)" means standard deviation ``s``.  Every
fp32 draw is rounded to bf16 (round-to-nearest-even by torch).

Recipe for adapters where a workload gives none: ``L1 ~ N(0, 1/K)``,
``L2 ~ N(0, 0.01)``, the same rule as the single-linear workload.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class LinearShape:
    name: str
    N: int          # out features
    K: int          # in features


@dataclass(frozen=True)
class Workload:
    name: str
    linears: tuple
    M: int                       # tokens
    r: int
    alpha: float
    w_std: float
    x_std: float = 1.0
    dy_std: float = 1.0
    l1_std: float | None = None  # None: 1/K
    l2_std: float = 0.01
    backward: bool = True
    note: str = ""

    @property
    def s(self) -> float:
        return self.alpha / self.r


def _llama(hidden, ffn):
    return (LinearShape("q", hidden, hidden), LinearShape("k", hidden, hidden),
            LinearShape("v", hidden, hidden), LinearShape("o", hidden, hidden),
            LinearShape("gate", ffn, hidden), LinearShape("up", ffn, hidden),
            LinearShape("down", hidden, ffn))


WORKLOADS = {
    # one 4096x4096 linear, 16 tokens, r = 16, s = 2, fwd + bwd
    "linear4096_m16": Workload("linear4096_m16", (LinearShape("w", 4096, 4096),), M=16, r=16,
                               alpha=32.0, w_std=0.02, l1_std=1.0 / 4096, l2_std=0.01),
    # LLaMA-7B block: 7 QLoRA linears, 4096 tokens (2 x 2048), r = 64, alpha = 16
    "llama7b_block": Workload("llama7b_block", _llama(4096, 11008), M=4096, r=64, alpha=16.0,
                              w_std=0.02),
    # LLaMA-65B FFN up/down as few-token forward (dequant-GEMV), r = 64, alpha = 16
    "llama65b_ffn_gemv": Workload("llama65b_ffn_gemv", (LinearShape("up", 22016, 8192),
                                                        LinearShape("down", 8192, 22016)),
                                  M=16, r=64, alpha=16.0, w_std=0.02, backward=False),
    # LLaMA-65B block: 8192 tokens (16 x 512), r = 64, alpha = 16, W ~ N(0, 0.015), dY ~ N(0, 1e-2)
    "llama65b_block": Workload("llama65b_block", _llama(8192, 22016), M=8192, r=64, alpha=16.0,
                               w_std=0.015, dy_std=1e-2),
}

ROUNDTRIP_WEIGHTS = 2 ** 31     # bulk quantise/dequantise round trip (4 GiB of bf16)


def generator(seed: int = 0, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, std, g, device="cpu"):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def make_linear(wl: Workload, lin: LinearShape, seed: int = 0, device="cpu", M: int | None = None):
    """Draw W, X, L1, L2, dY for one linear of a workload, in that order."""
    M = wl.M if M is None else M
    g = generator(seed, device)
    l1_std = wl.l1_std if wl.l1_std is not None else 1.0 / lin.K
    out = {
        "W": normal_bf16((lin.N, lin.K), wl.w_std, g, device),
        "X": normal_bf16((M, lin.K), wl.x_std, g, device),
        "L1": normal_bf16((lin.K, wl.r), l1_std, g, device),
        "L2": normal_bf16((wl.r, lin.N), wl.l2_std, g, device),
    }
    if wl.backward:
        out["dY"] = normal_bf16((M, lin.N), wl.dy_std, g, device)
    return out


def roundtrip_weights(n: int = ROUNDTRIP_WEIGHTS, seed: int = 0, device="cpu", chunk: int = 1 << 26):
    """Bulk-quantisation input: the first half ~ N(0, 0.02); the second half
    Student-t with 3 degrees of freedom times 0.02, each element of it
    multiplied by 50 with probability 0.001 (outliers that stress absmax).

    Student-t(3) = Z / sqrt(V/3) with V a sum of three squared standard
    normals.  Drawn chunk by chunk so the temporaries stay small.
    """
    g = generator(seed, device)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    half = n // 2
    for i in range(0, half, chunk):
        m = min(chunk, half - i)
        out[i:i + m] = (torch.randn(m, generator=g, device=device) * 0.02).to(torch.bfloat16)
    for i in range(half, n, chunk):
        m = min(chunk, n - i)
        z = torch.randn(m, generator=g, device=device)
        v = torch.randn((3, m), generator=g, device=device).square_().sum(0)
        t = z / torch.sqrt(v / 3.0) * 0.02
        mask = torch.rand(m, generator=g, device=device) < 0.001
        t = torch.where(mask, t * 50.0, t)
        out[i:i + m] = t.to(torch.bfloat16)
    return out


def bf16_bits(t: torch.Tensor):
    """Raw uint16 bit patterns of a bf16 tensor, as a numpy array on the host."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
