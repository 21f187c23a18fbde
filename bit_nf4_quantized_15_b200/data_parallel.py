"""Data-parallel QLoRA linears: the adapter-gradient exchange.

Under data parallelism every rank holds a replica of the frozen 4-bit
weights and runs the layer on its own tokens.  The weight gets no gradient
(nlp-lineage "QLoRA", section "The idea": only L1 and L2 receive weight
gradients; examadda "QLoRA", "The Flow": nothing flows into the 4-bit base),
so the one exchange a training step needs is the sum over ranks of every
linear's dL1 and dL2.  ``AdapterGrads`` keeps those gradients for a set of
linears in one flat fp32 buffer, hands out per-linear views for
``linear_bwd`` to write into, and reduces the whole buffer with a single
collective (NCCL between GPUs; any torch.distributed backend works, gloo in
the CPU tests).

    g = AdapterGrads([(N0, K0), (N1, K1)], r=64, device="cuda")
    dX, _, _ = linear_bwd(dY, X, T, w0, L1, L2, s, dL1=g.dL1[0], dL2=g.dL2[0])
    ...
    g.all_reduce()          # sum over ranks, in place; views see the result

No TMA multicast or peer-memory access is involved: the exchange is a plain
collective on a local buffer.
"""

from __future__ import annotations

import torch

__all__ = ["AdapterGrads", "adapter_grad_elems"]


def adapter_grad_elems(N: int, K: int, r: int) -> int:
    """fp32 elements of dL1 [K, r] plus dL2 [r, N] for one linear."""
    if N < 1 or K < 1 or r < 1:
        raise ValueError("N, K and r must be positive")
    return K * r + r * N


class AdapterGrads:
    """dL1/dL2 of several linears (weights ``[N, K]``, rank ``r``) in one
    contiguous fp32 buffer, in the order given: linear i's dL1 ``[K, r]``
    then its dL2 ``[r, N]``."""

    def __init__(self, shapes, r: int, device="cuda", dtype=torch.float32):
        self.shapes = [(int(N), int(K)) for N, K in shapes]
        self.r = int(r)
        sizes = [adapter_grad_elems(N, K, self.r) for N, K in self.shapes]
        self.flat = torch.zeros(sum(sizes), dtype=dtype, device=device)
        self.dL1, self.dL2 = [], []
        off = 0
        for (N, K), n in zip(self.shapes, sizes):
            self.dL1.append(self.flat[off:off + K * self.r].view(K, self.r))
            self.dL2.append(self.flat[off + K * self.r:off + n].view(self.r, N))
            off += n

    @property
    def nbytes(self) -> int:
        return self.flat.numel() * self.flat.element_size()

    def all_reduce(self, group=None, average: bool = False):
        """Sum (or, with ``average``, mean) the buffer over the ranks of
        ``group`` in place: one collective for every linear's gradients.  A
        no-op without an initialised process group or with a single rank."""
        import torch.distributed as dist

        if not dist.is_available() or not dist.is_initialized():
            return self
        world = dist.get_world_size(group)
        if world == 1:
            return self
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
        if average:
            self.flat.div_(world)
        return self
