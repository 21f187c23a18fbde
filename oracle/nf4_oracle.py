"""NF4 double-quantisation and QLoRA linear layer: the plain CPU oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Every function states the passage it follows.  Where the pages leave a step
open, the reading taken is stated next to the code and listed in the design
notes.  All parity pins live in ``tests/test_oracle_*.py``.

Conventions
-----------
* ``W`` is the ``nn.Linear`` weight, shape ``[N, K]`` (out x in), row-major.
  The pages' ``Y = X·W`` uses its transpose.
* Quantisation blocks are 64 consecutive elements of the flattened W
  (``K % 64 == 0``, so a block never crosses a row).
* bf16 tensors are handled as their raw ``uint16`` bit patterns.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

__all__ = [
    "BLOCK", "DQ_BLOCK", "E4M3_MAX",
    "norm_cdf", "norm_ppf", "nf4_delta", "nf4_codebook_f64", "nf4_codebook",
    "FORMATS", "fp4_codebook_f64", "int4_codebook_f64", "codebook",
    "nf4_midpoints", "nearest_level",
    "bf16_bits_to_f32", "f32_to_bf16_bits", "bf16_bits_to_f64",
    "e4m3_decode", "e4m3_encode", "e4m3_encode_exact",
    "E5M2_MAX", "SCALE_CODECS", "e5m2_decode", "e5m2_encode", "e5m2_encode_exact",
    "MEAN_CODECS", "pairwise_sum_f32",
    "block_absmax", "quantize", "dequant", "decoded_scales",
    "linear_fwd", "linear_bwd", "adapter_grads",
    "storage_bytes", "bits_per_weight",
]

BLOCK = 64          # weights per first-level block ("The idea": blocks of 64)
DQ_BLOCK = 256      # first-level scales per second-level (c1) block
E4M3_MAX = 448.0    # largest finite OCP E4M3 value
E5M2_MAX = 57344.0  # largest finite OCP E5M2 value


# ---------------------------------------------------------------------------
# Standard normal quantile (fp64).  Used only to build the NF4 codebook.
# ---------------------------------------------------------------------------

def norm_cdf(x: float) -> float:
    """Phi(x) = erfc(-x/sqrt 2)/2, the textbook closed form."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def norm_ppf(p: float) -> float:
    """Phi^{-1}(p) in fp64 by bisection on :func:`norm_cdf`.

    Slow but plainly correct: Phi is strictly increasing, so halving the
    bracket until its two ends are adjacent doubles pins the root to the
    accuracy of ``math.erfc`` (about 1e-15 here).
    """
    if not 0.0 < p < 1.0:
        raise ValueError("p must lie in (0, 1)")
    lo, hi = -40.0, 40.0
    while True:
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if norm_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    return lo if abs(norm_cdf(lo) - p) <= abs(norm_cdf(hi) - p) else hi


# ---------------------------------------------------------------------------
# NF4 codebook ("The idea", NF4 bullet: 16 values, each an equal share of
# N(0,1), with an exact zero; inferensys glossary: zero-mean normal, levels
# denser near zero).
# ---------------------------------------------------------------------------

def nf4_delta() -> float:
    """Outermost probability used for the +-1 endpoints.

    Reading (the pages give no formula): the quantiles of the 0 and 1 bin
    edges are infinite, so the endpoint probability is the mean of the
    outermost equal-share bin centres for 16 and for 15 bins,
    1 - (1/32 + 1/30)/2.
    """
    return 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


def nf4_codebook_f64() -> list:
    """The 16 NF4 levels in fp64, ascending, endpoints exactly -1 and +1.

    8 positive levels at Phi^{-1} of 8 equally spaced probabilities from
    delta down towards 1/2 (the 1/2 point itself is the zero level), 7
    negative levels mirrored from 7 equally spaced probabilities over the same
    range, the exact zero, all divided by the largest level.
    """
    d = nf4_delta()
    pos = [norm_ppf(d + i * (0.5 - d) / 8.0) for i in range(8)]
    neg = [-norm_ppf(d + i * (0.5 - d) / 7.0) for i in range(7)]
    levels = sorted(pos + [0.0] + neg)
    top = max(levels)
    return [v / top for v in levels]


def nf4_codebook() -> np.ndarray:
    """The codebook as stored and used: each fp64 level rounded to fp32."""
    return np.array(nf4_codebook_f64(), dtype=np.float32)


# ---------------------------------------------------------------------------
# The 4-bit formats NF4 is compared with (nlp-lineage "QLoRA", section "What it
# showed", third bullet: "a standard 4-bit float" and "4-bit integers").  The
# pages name them only; the readings below are the plainest ones.  Each keeps
# everything else of the method (blocks of 64, absmax scale, E4M3 double
# quantisation, nearest level with ties to the lower code) and swaps only the
# 16 levels; a code is an index into the ascending level table.
# ---------------------------------------------------------------------------

FORMATS = ("nf4", "fp4", "int4")


def fp4_codebook_f64() -> list:
    """"A standard 4-bit float", read as OCP E2M1 (1 sign bit, 2 exponent bits
    with bias 1, 1 mantissa bit: magnitudes 0, 1/2, 1, 3/2, 2, 3, 4, 6)
    divided by its largest magnitude 6, so that the block absmax maps to +-1
    as for NF4.  +0 and -0 are one level; the 16th entry is a pad level -2,
    below every x = w / absmax (its decision midpoint -3/2 is never reached),
    so the table stays 16 strictly increasing levels."""
    mags = [Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]
    pos = [m / 6 for m in mags]
    return [-2.0] + [float(-p) for p in reversed(pos)] + [0.0] + [float(p) for p in pos]


def int4_codebook_f64() -> list:
    """"4-bit integers", read as symmetric absmax integer quantisation: levels
    k/7 for k = -7 .. 7 (the block absmax maps to +-7), plus the code that
    the symmetric form leaves unused (two's-complement -8) as the pad level
    -8/7 (decision midpoint -15/14 < -1: never reached)."""
    return [float(Fraction(k, 7)) for k in range(-8, 8)]


def codebook(fmt: str = "nf4") -> np.ndarray:
    """The 16 ascending fp32 levels of a format (each rounded once from its
    exact or fp64 value)."""
    if fmt == "nf4":
        return nf4_codebook()
    if fmt == "fp4":
        return np.array(fp4_codebook_f64(), dtype=np.float32)
    if fmt == "int4":
        return np.array(int4_codebook_f64(), dtype=np.float32)
    raise ValueError(f"unknown format {fmt!r}")


def nf4_midpoints(q: np.ndarray | None = None) -> np.ndarray:
    """Exact fp64 midpoints between neighbouring fp32 levels (15 values)."""
    if q is None:
        q = nf4_codebook()
    q64 = q.astype(np.float64)
    return (q64[:-1] + q64[1:]) / 2.0  # sum of two fp32 values is exact in fp64


def nearest_level(x: np.ndarray, q: np.ndarray | None = None) -> np.ndarray:
    """Index of the codebook level nearest to each fp32 ``x``.

    Ties go to the lower index (``np.argmin`` returns the first minimum).
    Reading: the pages say "nearest" and leave ties open.  The fp64
    differences of two fp32 values in [-1, 1] are exact wherever a tie is
    possible, so the argmin is the exact nearest level.
    """
    if q is None:
        q = nf4_codebook()
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    d = np.abs(x64[..., None] - q.astype(np.float64))
    return np.argmin(d, axis=-1).astype(np.uint8)


# ---------------------------------------------------------------------------
# bf16 and OCP E4M3 codecs
# ---------------------------------------------------------------------------

def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact: append 16 zero bits)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, round-to-nearest-even; NaN -> quiet NaN 0x7FC0."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), r).astype(np.uint16)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 (bias 7, no infinities, S.1111.111 = NaN) -> fp64.

    Normal: (-1)^s 2^(e-7) (1 + m/8); subnormal (e = 0): (-1)^s 2^-6 m/8.
    """
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    nan = (c & 0x7F) == 0x7F
    return np.where(nan, np.nan, s * mag)


def _e4m3_finite_values():
    """All 127 non-negative finite E4M3 values with their codes, exact."""
    out = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        out.append((v, code))
    return out


_E4M3_TABLE = _e4m3_finite_values()


def e4m3_encode_exact(x: float) -> int:
    """Scalar E4M3 encoder from the definition, in exact rationals.

    Round to nearest, ties to the even code (mantissa LSB 0); finite values
    beyond the largest finite magnitude saturate to +-448 ("satfinite"); NaN
    encodes as 0x7F.
    """
    if math.isnan(x):
        return 0x7F
    sign = 0x80 if math.copysign(1.0, x) < 0 else 0
    if math.isinf(x):
        return sign | 0x7E
    a = Fraction(abs(x))
    if a >= Fraction(448):
        return sign | 0x7E
    best = None
    for v, code in _E4M3_TABLE:
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and (code & 1) == 0):
            best = (d, code)
    return sign | best[1]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Vectorised E4M3 encoder (same rule as :func:`e4m3_encode_exact`).

    For a finite |x| the spacing of E4M3 values around it is 2^(E-3) for
    normal binades (E = floor(log2|x|) >= -6) and 2^-9 below; |x| divided by
    that power of two is exact in fp64 and ``np.rint`` rounds half to even,
    which is the even-code rule because codes are monotone in magnitude.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    sign = np.where(np.signbit(x), 0x80, 0).astype(np.int64)
    with np.errstate(divide="ignore", invalid="ignore"):
        _, ex = np.frexp(a)                       # a = f * 2^ex, f in [0.5, 1)
        E = np.maximum(ex.astype(np.int64) - 1, -6)
        quantum = np.exp2((E - 3).astype(np.float64))
        n = np.rint(a / quantum)
        v = n * quantum
    v = np.where(np.isfinite(v), v, 448.0)
    v = np.minimum(v, 448.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        _, ev = np.frexp(v)
        Ev = ev.astype(np.int64) - 1
        sub = v < 2.0 ** -6
        code_sub = np.rint(v / 2.0 ** -9)
        mant = np.rint((v / np.exp2(Ev.astype(np.float64)) - 1.0) * 8.0)
        code_norm = ((Ev + 7) << 3) + mant.astype(np.int64)
    code = np.where(sub, code_sub.astype(np.int64), code_norm)
    code = np.where(v == 0, 0, code)
    code = (sign | code).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)


# ---------------------------------------------------------------------------
# E5M2: the other 8-bit float, for the scale-codec variant of the double
# quantisation (the pages say only "8-bit floats"; E4M3 is the method's
# reading here, E5M2 the compared alternative: two more exponent bits, one
# fewer mantissa bit).
# ---------------------------------------------------------------------------

def e5m2_decode(code: np.ndarray) -> np.ndarray:
    """OCP FP8 E5M2 (bias 15; exponent 31 holds Inf and NaN) -> fp64.

    Normal: (-1)^s 2^(e-15) (1 + m/4); subnormal (e = 0): (-1)^s 2^-14 m/4.
    """
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 2) & 0x1F
    m = (c & 0x3).astype(np.float64)
    mag = np.where(e == 0, m / 4.0 * 2.0 ** -14, (1.0 + m / 4.0) * np.exp2((e - 15).astype(np.float64)))
    mag = np.where(e == 31, np.where(m == 0, np.inf, np.nan), mag)
    return s * mag


def _e5m2_finite_values():
    """All 124 non-negative finite E5M2 values with their codes, exact."""
    out = []
    for code in range(0x7C):
        e, m = code >> 2, code & 3
        v = Fraction(m, 4) * Fraction(1, 2 ** 14) if e == 0 else (1 + Fraction(m, 4)) * Fraction(2) ** (e - 15)
        out.append((v, code))
    return out


_E5M2_TABLE = _e5m2_finite_values()


def e5m2_encode_exact(x: float) -> int:
    """Scalar E5M2 encoder in exact rationals: nearest value, ties to the even
    code, saturating to +-57344 (satfinite); NaN encodes as 0x7F."""
    if math.isnan(x):
        return 0x7F
    sign = 0x80 if math.copysign(1.0, x) < 0 else 0
    if math.isinf(x):
        return sign | 0x7B
    a = Fraction(abs(x))
    if a >= Fraction(int(E5M2_MAX)):
        return sign | 0x7B
    best = None
    for v, code in _E5M2_TABLE:
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and (code & 1) == 0):
            best = (d, code)
    return sign | best[1]


def e5m2_encode(x: np.ndarray) -> np.ndarray:
    """Vectorised E5M2 encoder (same rule as :func:`e5m2_encode_exact`): the
    spacing around |x| is 2^(E-2) in normal binades (E >= -14) and 2^-16
    below; np.rint rounds half to even."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    sign = np.where(np.signbit(x), 0x80, 0).astype(np.int64)
    with np.errstate(divide="ignore", invalid="ignore"):
        _, ex = np.frexp(a)
        E = np.maximum(ex.astype(np.int64) - 1, -14)
        quantum = np.exp2((E - 2).astype(np.float64))
        n = np.rint(a / quantum)
        v = n * quantum
    v = np.where(np.isfinite(v), v, E5M2_MAX)
    v = np.minimum(v, E5M2_MAX)
    with np.errstate(divide="ignore", invalid="ignore"):
        _, ev = np.frexp(v)
        Ev = ev.astype(np.int64) - 1
        sub = v < 2.0 ** -14
        code_sub = np.rint(v / 2.0 ** -16)
        mant = np.rint((v / np.exp2(Ev.astype(np.float64)) - 1.0) * 4.0)
        code_norm = ((Ev + 15) << 2) + mant.astype(np.int64)
    code = np.where(sub, code_sub.astype(np.int64), code_norm)
    code = np.where(v == 0, 0, code)
    code = (sign | code).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)


# scale codec -> (largest finite value, encoder, decoder)
SCALE_CODECS = {"e4m3": (E4M3_MAX, e4m3_encode, e4m3_decode), "e5m2": (E5M2_MAX, e5m2_encode, e5m2_decode),
                "e4m3_mean": (E4M3_MAX, e4m3_encode, e4m3_decode)}
# Codecs whose c1 array holds two fp32 values per group: c1_g, then the group
# mean mu_g of the block scales (the mean-centred double quantisation).
MEAN_CODECS = ("e4m3_mean",)


# ---------------------------------------------------------------------------
# Mean-centred double quantisation (a variant of the scale quantisation; the
# pages say only that the 32-bit block scales are quantised to 8-bit floats,
# inferensys glossary, double-quantisation paragraph).  Reading: all block
# scales are non-negative, so before the 8-bit step each group of 256 is
# centred on its mean and the signed residuals use the sign bit of E4M3:
#   mu_g = RN32(S_g / n_g), S_g the fp32 sum of the group's scales taken as a
#          pairwise tree over 256 slots (adjacent pairs first, empty slots of
#          a partial group are zeros), n_g the number of blocks in the group
#   d_b  = RN32(c_b - mu_g);  c1_g = RN32(max_b |d_b| / 448)
#   c2_b = E4M3_RNE_sat(RN32(d_b / c1_g)), signed; 0 when c1_g = 0
#   c^_b = RN32(RN32(dec(c2_b) * c1_g) + mu_g)
# ---------------------------------------------------------------------------

def pairwise_sum_f32(v: np.ndarray, slots: int = DQ_BLOCK) -> np.float32:
    """fp32 sum of ``v`` (at most ``slots`` values, zero-padded) as a pairwise
    tree: slot 2i + slot 2i+1 first, then pairs of those sums, ... ; every
    addition rounded to fp32."""
    a = np.zeros(slots, np.float32)
    a[: len(v)] = np.asarray(v, np.float32)
    while len(a) > 1:
        a = (a[0::2] + a[1::2]).astype(np.float32)
    return np.float32(a[0])


# ---------------------------------------------------------------------------
# Quantiser ("The idea": blocks of 64, 32-bit scale per block, scales
# quantised again to 8 bits; inferensys: block-wise absmax, 8-bit floats).
# ---------------------------------------------------------------------------

def block_absmax(W_bits: np.ndarray) -> np.ndarray:
    """c_b = max |w| over each 64-weight block, as fp32 (exact)."""
    w = bf16_bits_to_f32(np.asarray(W_bits).reshape(-1, BLOCK))
    return np.abs(w).max(axis=1).astype(np.float32)


def _check_shape(N: int, K: int):
    if K % BLOCK != 0 or N < 1 or K < 1:
        raise ValueError("W must be [N, K] with K a multiple of 64")


def quantize(W_bits: np.ndarray, chunk_blocks: int = 1 << 16, fmt: str = "nf4", scale: str = "e4m3"):
    """NF4 double quantisation of a bf16 weight ``[N, K]`` (``fmt`` swaps the
    16 levels for one of the compared formats, see :func:`codebook`;
    ``scale="e5m2"`` stores c2 as E5M2 with c1 = RN32(max / 57344);
    ``scale="e4m3_mean"`` centres each group on its mean first, see
    :data:`MEAN_CODECS`, and returns c1 as [c1_0, mu_0, c1_1, mu_1, ...]).

    Returns ``(codes, c2, c1)``:
      * ``codes`` uint8 ``[N*K/2]``: element 2j in the low nibble, 2j+1 in the
        high nibble, flat row-major order;
      * ``c2`` uint8 ``[N*K/64]``: E4M3 code of each block scale;
      * ``c1`` fp32 ``[ceil(N*K/16384)]``: one second-level scale per 256
        consecutive blocks.

    Steps (readings stated inline):
      1. c_b = absmax of the block (fp32, exact).
      2. x = RN32(w / c_b) by IEEE division; the code is the nearest level,
         ties to the lower code.  An all-zero block gives c_b = 0 and x = 0.
         The code is chosen against the unquantised c_b.
      3. c1_g = RN32(max_{b in g} c_b / 448).
      4. c2_b = E4M3(RN32(c_b / c1_g)), satfinite; c2_b = 0 when c1_g = 0.
    """
    W_bits = np.asarray(W_bits, dtype=np.uint16)
    N, K = W_bits.shape
    _check_shape(N, K)
    flat = W_bits.reshape(-1, BLOCK)
    nb = flat.shape[0]
    q = codebook(fmt)
    codes = np.empty((nb, BLOCK // 2), dtype=np.uint8)
    absmax = np.empty(nb, dtype=np.float32)
    for b0 in range(0, nb, chunk_blocks):
        w = bf16_bits_to_f32(flat[b0:b0 + chunk_blocks])
        if not np.all(np.isfinite(w)):
            raise ValueError("non-finite weight")
        c = np.abs(w).max(axis=1).astype(np.float32)
        absmax[b0:b0 + chunk_blocks] = c
        safe = np.where(c > 0, c, np.float32(1)).astype(np.float32)
        x = (w / safe[:, None]).astype(np.float32)      # IEEE fp32 division
        x = np.where(c[:, None] > 0, x, np.float32(0)).astype(np.float32)
        code = nearest_level(x, q)
        codes[b0:b0 + chunk_blocks] = code[:, 0::2] | (code[:, 1::2] << 4)
    G = (nb + DQ_BLOCK - 1) // DQ_BLOCK
    mean = scale in MEAN_CODECS
    c1 = np.empty(2 * G if mean else G, dtype=np.float32)
    c2 = np.empty(nb, dtype=np.uint8)
    smax, encode, _ = SCALE_CODECS[scale]
    for g in range(G):
        cg = absmax[g * DQ_BLOCK:(g + 1) * DQ_BLOCK]
        if mean:
            mu = np.float32(pairwise_sum_f32(cg) / np.float32(len(cg)))   # fp32 division
            d = (cg - mu).astype(np.float32)                                # fp32 subtraction
            c1g = np.float32(np.abs(d).max()) / np.float32(smax)
            c1[2 * g], c1[2 * g + 1] = c1g, mu
        else:
            d = cg
            c1g = np.float32(cg.max()) / np.float32(smax)       # fp32 division
            c1[g] = c1g
        if c1g > 0:
            c2[g * DQ_BLOCK:(g + 1) * DQ_BLOCK] = encode((d / c1g).astype(np.float32))
        else:
            c2[g * DQ_BLOCK:(g + 1) * DQ_BLOCK] = 0
    return codes.reshape(-1), c2, c1


def decoded_scales(c2: np.ndarray, c1: np.ndarray, scale: str = "e4m3") -> np.ndarray:
    """c^_b = RN32(dec(c2_b) * c1_g): the 32-bit scale used by the dequantiser
    (mean-centred codec: RN32(RN32(dec(c2_b) * c1_g) + mu_g), two fp32
    operations, no fused multiply-add)."""
    dec = SCALE_CODECS[scale][2](c2).astype(np.float32)  # every 8-bit float value is exact in fp32
    g = np.arange(len(c2)) // DQ_BLOCK
    if scale in MEAN_CODECS:
        prod = (dec * c1[2 * g]).astype(np.float32)
        return (prod + c1[2 * g + 1]).astype(np.float32)
    return (dec * c1[g]).astype(np.float32)             # fp32 multiply


def dequant(codes: np.ndarray, c2: np.ndarray, c1: np.ndarray, N: int, K: int, fmt: str = "nf4",
            scale: str = "e4m3") -> np.ndarray:
    """doubleDequant(c1, c2, W_NF4) -> bf16 bits ``[N, K]`` (``fmt``: the
    levels the codes index, see :func:`codebook`).

    ("The idea", notation paragraph; inferensys: dequantised to BFloat16.)
    w^ = RNbf16(RN32(q_code * c^_b)) with c^_b from :func:`decoded_scales`:
    two fp32 multiplies, no fused multiply-add, then round to bf16.
    """
    _check_shape(N, K)
    q = codebook(fmt)
    cb = np.asarray(codes, dtype=np.uint8).reshape(-1, BLOCK // 2)
    code = np.empty((cb.shape[0], BLOCK), dtype=np.uint8)
    code[:, 0::2] = cb & 0xF
    code[:, 1::2] = cb >> 4
    chat = decoded_scales(c2, c1, scale)
    w = (q[code] * chat[:, None]).astype(np.float32)    # fp32 multiply
    return f32_to_bf16_bits(w).reshape(N, K)


# ---------------------------------------------------------------------------
# Linear layer, forward and backward, fp64 ("The idea", notation paragraph:
# Y = X·doubleDequant(c1,c2,W_NF4) + X·L1·L2, only L1 and L2 get weight
# gradients; examadda "The Flow": no gradient reaches the 4-bit base).
# ---------------------------------------------------------------------------

def linear_fwd(X: np.ndarray, What: np.ndarray, L1: np.ndarray, L2: np.ndarray, s: float):
    """Y = X W^T + s (X L1) L2 and T = X L1, all fp64.

    ``X`` [M, K], ``What`` [N, K] (the dequantised weight), ``L1`` [K, r],
    ``L2`` [r, N].  ``s`` is the LoRA scale alpha/r (the pages' formula has
    none; s = 1 recovers it).
    """
    X = np.asarray(X, dtype=np.float64)
    T = X @ np.asarray(L1, dtype=np.float64)
    Y = X @ np.asarray(What, dtype=np.float64).T + s * (T @ np.asarray(L2, dtype=np.float64))
    return Y, T


def adapter_grads(dY, X, L1, L2, s, T=None):
    """The adapters' part of the backward, fp64: dT = dY L2^T,
    dL2 = s T^T dY, dL1 = s X^T dT.  Returns (dL1, dL2, dT, T)."""
    dY = np.asarray(dY, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    L1 = np.asarray(L1, dtype=np.float64)
    L2 = np.asarray(L2, dtype=np.float64)
    if T is None:
        T = X @ L1
    T = np.asarray(T, dtype=np.float64)
    dT = dY @ L2.T
    dL2 = s * (T.T @ dY)
    dL1 = s * (X.T @ dT)
    return dL1, dL2, dT, T


def linear_bwd(dY, X, What, L1, L2, s, T=None):
    """Gradients of <Y, dY> for the layer above, fp64.

    dT = dY L2^T; dX = dY W + s dT L1^T; dL2 = s T^T dY; dL1 = s X^T dT.
    There is no gradient for the frozen weight W.
    """
    dL1, dL2, dT, _ = adapter_grads(dY, X, L1, L2, s, T)
    dY = np.asarray(dY, dtype=np.float64)
    dX = dY @ np.asarray(What, dtype=np.float64) + s * (dT @ np.asarray(L1, dtype=np.float64).T)
    return dX, dL1, dL2, dT


# ---------------------------------------------------------------------------
# Storage accounting ("The idea", double-quantisation bullet: 0.5 bits per
# weight for 32-bit scales on blocks of 64, about 0.127 after quantising the
# scales to 8 bits).
# ---------------------------------------------------------------------------

def storage_bytes(N: int, K: int, double_quant: bool = True, scale: str = "e4m3") -> int:
    n = N * K
    nb = n // BLOCK
    if not double_quant:
        return n // 2 + 4 * nb
    per_group = 8 if scale in MEAN_CODECS else 4
    return n // 2 + nb + per_group * ((nb + DQ_BLOCK - 1) // DQ_BLOCK)


def bits_per_weight(N: int, K: int, double_quant: bool = True) -> float:
    return storage_bytes(N, K, double_quant) * 8.0 / (N * K)
