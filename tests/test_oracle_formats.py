"""Pins for the oracle's two compared 4-bit formats (nlp-lineage "QLoRA",
section "What it showed", third bullet: NF4 against "a standard 4-bit float"
and "4-bit integers").

The level tables are pinned against independent derivations: FP4 by decoding
all 16 E2M1 bit patterns from the format's bit layout, Int4 by the exact
rationals k/7, each rounded to fp32 by the exact-rational RN32 of
``test_oracle_quant``.  The quantiser and dequantiser for each format are
pinned against that file's brute-force rational implementations, given the
pinned levels.
"""

from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from test_oracle_quant import (_bf16, _halfgap, _tiny_inputs, bf16_value, brute_dequant, brute_quantize,
                               rn32)


def _e2m1_value(bits: int) -> Fraction:
    """OCP E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
    exponent 0 is subnormal (m * 1/2)."""
    s, e, m = (bits >> 3) & 1, (bits >> 1) & 3, bits & 1
    mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
    return -mag if s else mag


def _as_f32(fr: Fraction) -> np.float32:
    v = np.float32(float(fr))
    assert Fraction(float(v)) == fr, "value must be representable"
    return v


def test_fp4_levels_are_e2m1_over_6():
    vals = sorted({_e2m1_value(b) for b in range(16)})          # +0 and -0 collapse: 15 values
    assert len(vals) == 15 and max(vals) == 6 and min(vals) == -6
    want = [_as_f32(rn32(v / 6)) for v in vals]
    q = O.codebook("fp4")
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.array_equal(q[1:].view(np.uint32), np.array(want, np.float32).view(np.uint32))
    assert q[0] < -1 and (float(q[0]) + float(q[1])) / 2 < -1  # pad level never chosen
    assert q[8] == 0 and q[15] == 1 and q[1] == -1


def test_int4_levels_are_k_over_7():
    want = [_as_f32(rn32(Fraction(k, 7))) for k in range(-7, 8)]
    q = O.codebook("int4")
    assert np.array_equal(q[1:].view(np.uint32), np.array(want, np.float32).view(np.uint32))
    assert (float(q[0]) + float(q[1])) / 2 < -1
    gaps = np.diff(q[1:].astype(np.float64))
    assert np.all(np.abs(gaps - 1 / 7) < 2 ** -23)              # uniform spacing up to fp32 rounding


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_levels_strictly_increasing_with_zero(fmt):
    q = O.codebook(fmt).astype(np.float64)
    assert np.all(np.diff(q) > 0) and 0.0 in q and q[-1] == 1.0


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
@pytest.mark.parametrize("case", range(3))
def test_quantize_matches_bruteforce(fmt, case):
    W = _tiny_inputs()[case]
    a = O.quantize(W, fmt=fmt)
    b = brute_quantize(W, O.codebook(fmt))
    for x, y in zip(a, b):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
@pytest.mark.parametrize("case", range(3))
def test_dequant_matches_bruteforce(fmt, case):
    W = _tiny_inputs()[case]
    N, K = W.shape
    codes, c2, c1 = O.quantize(W, fmt=fmt)
    assert np.array_equal(O.dequant(codes, c2, c1, N, K, fmt=fmt),
                          brute_dequant(codes, c2, c1, N, K, O.codebook(fmt)))


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_special_blocks(fmt):
    blk = np.zeros(64, np.float32)
    blk[0], blk[1], blk[2] = 0.5, -0.5, 0.0
    codes, c2, c1 = O.quantize(_bf16(blk).reshape(1, 64), fmt=fmt)
    assert codes[0] & 15 == 15 and codes[0] >> 4 == 1 and codes[1] & 15 == 8   # +c, -c, 0
    codes, c2, c1 = O.quantize(np.zeros((2, 64), np.uint16), fmt=fmt)
    assert np.all(codes == 0x88) and np.all(O.dequant(codes, c2, c1, 2, 64, fmt=fmt) == 0)


def test_fp4_ties_go_to_lower_level():
    """x = 1/8 lies exactly between the FP4 levels 1/12 and 1/6 (in fp32:
    both levels and the midpoint are checked exactly) -> the lower one."""
    q = O.codebook("fp4").astype(np.float64)
    mid = (q[9] + q[10]) / 2
    if float(np.float32(mid)) == mid:
        assert O.nearest_level(np.array([np.float32(mid)]), O.codebook("fp4"))[0] == 9
    x = np.float32(0.125)   # w / c = 1/8 exactly
    code = O.nearest_level(np.array([x]), O.codebook("fp4"))[0]
    d9, d10 = abs(Fraction(float(x)) - Fraction(q[9])), abs(Fraction(float(x)) - Fraction(q[10]))
    assert code == (9 if d9 <= d10 else 10)


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_round_trip_error_bound(fmt):
    rng = np.random.default_rng(15)
    n = 64 * 1024
    a = rng.normal(0, 0.02, n // 2)
    t = rng.standard_t(3, n // 2) * 0.02
    t *= np.where(rng.random(n // 2) < 0.001, 50.0, 1.0)
    W = _bf16(np.concatenate([a, t])).reshape(64, -1)
    N, K = W.shape
    codes, c2, c1 = O.quantize(W, fmt=fmt)
    What = O.bf16_bits_to_f64(O.dequant(codes, c2, c1, N, K, fmt=fmt)).reshape(-1)
    w = O.bf16_bits_to_f64(W).reshape(-1)
    q = O.codebook(fmt)
    code = np.empty(n, np.uint8)
    code[0::2], code[1::2] = codes & 15, codes >> 4
    assert np.all(code >= 1)                                   # the pad level is never used
    c = np.repeat(O.block_absmax(W).astype(np.float64), 64)
    chat = np.repeat(O.decoded_scales(c2, c1).astype(np.float64), 64)
    hg = np.array([_halfgap(q, k) for k in range(16)])[code]
    qv = q.astype(np.float64)[code]
    bound = (c * (hg + 2.0 ** -24) + np.abs(qv) * np.abs(chat - c)
             + np.abs(qv * chat) * 2.0 ** -24 + np.abs(What) * 2.0 ** -8 + 1e-45)
    assert np.all(np.abs(w - What) <= bound * (1 + 1e-12))


def test_nf4_beats_the_compared_formats_on_normal_weights():
    """The pages' ranking (NF4 ahead of FP4 and Int4) holds for the
    quantisation error these readings give on normally distributed weights."""
    rng = np.random.default_rng(16)
    W = _bf16(rng.normal(0, 0.02, (64, 64 * 64)))
    N, K = W.shape
    w = O.bf16_bits_to_f64(W)
    err = {}
    for f in O.FORMATS:
        What = O.bf16_bits_to_f64(O.dequant(*O.quantize(W, fmt=f), N, K, fmt=f))
        err[f] = float(np.mean((w - What) ** 2))
    assert err["nf4"] < err["fp4"] and err["nf4"] < err["int4"]


# ------------------------------------------------ scale codec: E5M2 for c2
@pytest.mark.parametrize("fmt", ["nf4", "fp4"])
@pytest.mark.parametrize("case", range(3))
def test_e5m2_scales_match_bruteforce(fmt, case):
    W = _tiny_inputs()[case]
    N, K = W.shape
    a = O.quantize(W, fmt=fmt, scale="e5m2")
    b = brute_quantize(W, O.codebook(fmt), scale="e5m2")
    for x, y in zip(a, b):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))
    assert np.array_equal(O.dequant(*a, N, K, fmt=fmt, scale="e5m2"),
                          brute_dequant(*a, N, K, O.codebook(fmt), scale="e5m2"))


def test_e5m2_scale_bounds():
    """Two mantissa bits: relative scale error <= 2^-3 in E5M2's normal range;
    the codes do not depend on the scale codec."""
    rng = np.random.default_rng(17)
    W = _bf16(rng.standard_t(3, (256, 64 * 64)) * 0.02)
    codes, c2, c1 = O.quantize(W, scale="e5m2")
    assert np.array_equal(codes, O.quantize(W)[0])
    c = O.block_absmax(W).astype(np.float64)
    chat = O.decoded_scales(c2, c1, "e5m2").astype(np.float64)
    c1r = np.repeat(c1.astype(np.float64), 256)[: len(c)]
    assert np.all(O.e5m2_decode(c2) <= 57344.0)
    normal = c / c1r >= 2.0 ** -14
    assert (np.abs(chat - c)[normal] / c[normal]).max() <= 2.0 ** -3 + 1e-6


# ------------------------------------------ planted mistakes (CPU only)
def test_planted_e5m2_with_e4m3_range_is_caught():
    """E5M2 codes with the E4M3 divisor (448) for c1: the brute-force pin
    (57344) rejects it."""
    W = _tiny_inputs()[1]
    codes, _, _ = O.quantize(W, scale="e5m2")
    absmax = O.block_absmax(W)
    c1_bad = np.array([np.float32(absmax[g * 256:(g + 1) * 256].max()) / np.float32(448.0)
                       for g in range((len(absmax) + 255) // 256)], np.float32)
    ref = brute_quantize(W, O.codebook("nf4"), scale="e5m2")
    assert not np.array_equal(c1_bad.view(np.uint32), ref[2].view(np.uint32))


def test_planted_fp4_pad_at_the_top_is_caught():
    """The FP4 table with its pad level above +1 instead of below -1 fails
    the E2M1 level pin and changes the codes of the tiny cases."""
    good = O.codebook("fp4")
    bad = np.concatenate([good[1:], np.array([2.0], np.float32)])
    vals = sorted({_e2m1_value(b) for b in range(16)})
    want = np.array([_as_f32(rn32(v / 6)) for v in vals], np.float32)
    assert np.array_equal(good[1:], want) and not np.array_equal(bad[1:], want)
    W = _tiny_inputs()[0]
    assert not np.array_equal(brute_quantize(W, bad)[0], O.quantize(W, fmt="fp4")[0])


def test_planted_int4_over_8_is_caught():
    """Levels k/8 instead of k/7 (an asymmetric int4 reading) fail the pin."""
    bad = np.array([np.float32(k / 8) for k in range(-8, 8)], np.float32)
    assert not np.array_equal(bad, O.codebook("int4"))
