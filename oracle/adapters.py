"""Adapter-side operations around the QLoRA layer: the plain CPU oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

* ``adapter_merge``: folding a trained adapter back into the weight.  The
  examadda "QLoRA" page ("Practical Notes", third bullet) warns that merging
  an adapter into a 4-bit base is lossy and says to dequantise first; so the
  merge produces the 16-bit weight W^ + s (L1 L2)^T, and quantising that
  again is a separate, lossy step (measured with ``quantize``/``dequant``).
* ``adamw_step``: the optimizer step on the adapters whose state the paged
  optimizers keep in memory that can be paged between GPU and host
  (nlp-lineage "QLoRA", section "The idea", paged-optimizers bullet; tecyfy
  "What is QLoRA", "The 3 tricks"; inferensys glossary, paged-optimizers
  paragraph).  The pages name the optimizer's memory handling, not its
  update rule; AdamW with decoupled weight decay is the reading taken (the
  optimizer the QLoRA recipe pages it for).
"""

from __future__ import annotations

import math

import numpy as np

from .nf4_oracle import bf16_bits_to_f64, f32_to_bf16_bits

__all__ = ["f64_to_bf16_bits", "adapter_merge", "adamw_scalars", "adamw_step"]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns with ONE rounding (to nearest, ties to even),
    straight from the fp64 value (going through fp32 would round twice).

    bf16 keeps 8 significant bits and fp32's exponent range: normal values
    have a quantum of 2^(e-7) for |x| in [2^e, 2^(e+1)), subnormals (below
    2^-126) a fixed quantum of 2^-133.  Values that round beyond the largest
    finite bf16 become infinities."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                              # a = f * 2^e, f in [0.5, 1)
    e = np.maximum(e - 1, -126)                     # a in [2^e, 2^(e+1)) for normals
    quantum = np.ldexp(1.0, (e - 7).astype(np.int64))
    r = np.rint(a / quantum) * quantum              # rint: ties to even; a/quantum is exact
    r = np.where(a == 0, 0.0, r)
    big = r >= 2.0 ** 128
    out = np.copysign(np.where(big, np.inf, r), x)
    with np.errstate(over="ignore"):
        f32 = out.astype(np.float32)                # exact: every bf16 value is an fp32 value
    return f32_to_bf16_bits(f32)


def adapter_merge(What_bits: np.ndarray, L1_bits: np.ndarray, L2_bits: np.ndarray, s: float) -> np.ndarray:
    """W_merged = RNbf16(W^ + s (L1 L2)^T): the dequantised weight ``[N, K]``
    (bf16 bits) plus the scaled adapter product, in fp64 with one final
    rounding to bf16.  ``L1`` is ``[K, r]``, ``L2`` ``[r, N]`` (bf16 bits), so
    (L1 L2)^T is ``[N, K]``, the nn.Linear layout of W.  Afterwards
    X W_merged^T equals the layer's forward X W^T + s X L1 L2 up to the
    rounding of the merged weight."""
    W = bf16_bits_to_f64(What_bits)
    L1 = bf16_bits_to_f64(L1_bits)
    L2 = bf16_bits_to_f64(L2_bits)
    return f64_to_bf16_bits(W + s * (L1 @ L2).T)


def adamw_scalars(lr: float, beta1: float, beta2: float, eps: float, weight_decay: float, step: int):
    """The fp32 constants of step ``step`` (1-based): lr, beta1, 1 - beta1,
    beta2, 1 - beta2, eps, weight_decay and the bias corrections
    1 - beta1^step, 1 - beta2^step, each computed in fp64 and rounded once to
    fp32 (the GPU entry point receives exactly these values)."""
    if step < 1:
        raise ValueError("step counts from 1")
    f = np.float32
    return dict(lr=f(lr), b1=f(beta1), omb1=f(1.0 - beta1), b2=f(beta2), omb2=f(1.0 - beta2), eps=f(eps),
                wd=f(weight_decay), bc1=f(1.0 - beta1 ** step), bc2=f(1.0 - beta2 ** step))


def adamw_step(p, g, m, v, c):
    """One AdamW step (decoupled weight decay) in fp32, every operation
    rounded to fp32 in this order (c: ``adamw_scalars``):

        m    = b1 m + (1 - b1) g
        v    = b2 v + ((1 - b2) g) g
        mhat = m / (1 - b1^t)           vhat = v / (1 - b2^t)
        p    = p - lr (mhat / (sqrt(vhat) + eps) + wd p)

    Returns the new (p, m, v) as float32 arrays and p rounded to bf16 bits
    (the 16-bit copy the layer multiplies with)."""
    f = np.float32
    p = np.asarray(p, np.float32)
    g = np.asarray(g, np.float32)
    m = np.asarray(m, np.float32)
    v = np.asarray(v, np.float32)
    m = (c["b1"] * m).astype(f) + (c["omb1"] * g).astype(f)
    m = m.astype(f)
    v = (c["b2"] * v).astype(f) + ((c["omb2"] * g).astype(f) * g).astype(f)
    v = v.astype(f)
    mhat = (m / c["bc1"]).astype(f)
    vhat = (v / c["bc2"]).astype(f)
    denom = (np.sqrt(vhat).astype(f) + c["eps"]).astype(f)
    upd = (mhat / denom).astype(f)
    upd = (upd + (c["wd"] * p).astype(f)).astype(f)
    p = (p - (c["lr"] * upd).astype(f)).astype(f)
    return p, m, v, f32_to_bf16_bits(p)
