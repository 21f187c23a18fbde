"""Pins for the oracle's mean-centred double quantisation (scale codec
"e4m3_mean"): each group of 256 block scales is centred on its mean before
the 8-bit step, the signed residuals coded in E4M3 against
c1 = max |residual| / 448, and c^ = RN32(RN32(dec(c2) c1) + mean).

References written here and sharing nothing with the oracle: an exact
rational quantiser and dequantiser (own RN32, own pairwise tree of RN32
additions, nearest signed-E4M3 search), math.fsum, and closed forms.  Page:
inferensys glossary "QLoRA", double-quantisation paragraph (the scales are
quantised again to 8-bit floats); the centring is the variant's reading.
"""

import bisect
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from test_oracle_quant import _bf16, _three_groups, _tiny_inputs, bf16_value, e4m3_nearest, rn32


def _tree_rn32(vals):
    a = [Fraction(v) for v in vals] + [Fraction(0)] * (256 - len(vals))
    while len(a) > 1:
        a = [rn32(a[2 * i] + a[2 * i + 1]) for i in range(len(a) // 2)]
    return a[0]


def _e4m3_signed(x: Fraction) -> int:
    return (0x80 if x < 0 else 0) | e4m3_nearest(abs(x))


def _e4m3_value(code: int) -> Fraction:
    e, m = (code >> 3) & 15, code & 7
    v = (Fraction(m, 8) / 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if code & 0x80 else v


def brute_quantize_mean(W_bits):
    q = [Fraction(float(v)) for v in O.nf4_codebook()]
    mids = [(q[i] + q[i + 1]) / 2 for i in range(15)]
    flat = W_bits.reshape(-1).tolist()
    nb = len(flat) // 64
    codes = bytearray(len(flat) // 2)
    absmax = []
    for b in range(nb):
        ws = [bf16_value(v) for v in flat[64 * b:64 * b + 64]]
        c = max(abs(w) for w in ws)
        absmax.append(c)
        for j, w in enumerate(ws):
            x = Fraction(0) if c == 0 else rn32(w / c)
            idx = 64 * b + j
            codes[idx // 2] |= bisect.bisect_left(mids, x) << (4 * (idx & 1))
    c1, c2 = [], []
    for g in range((nb + 255) // 256):
        grp = absmax[256 * g:256 * g + 256]
        mu = rn32(_tree_rn32(grp) / len(grp))
        d = [rn32(c - mu) for c in grp]
        c1g = rn32(max(abs(x) for x in d) / 448)
        c1 += [c1g, mu]
        c2 += [0 if c1g == 0 else _e4m3_signed(rn32(x / c1g)) for x in d]
    return (np.frombuffer(bytes(codes), np.uint8), np.array(c2, np.uint8),
            np.array([float(v) for v in c1], np.float32))


def brute_chat_mean(c2, c1):
    out = []
    for b, code in enumerate(c2.tolist()):
        g = b // 256
        c1g, mu = Fraction(float(c1[2 * g])), Fraction(float(c1[2 * g + 1]))
        out.append(rn32(rn32(_e4m3_value(code) * c1g) + mu))
    return out


@pytest.mark.parametrize("case", range(3))
def test_quantize_mean_matches_bruteforce(case):
    W = _tiny_inputs()[case]
    got = O.quantize(W, scale="e4m3_mean")
    ref = brute_quantize_mean(W)
    for x, y in zip(got, ref):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))


def test_quantize_mean_across_groups_with_partial_last():
    W = _three_groups()
    N, K = W.shape
    got = O.quantize(W, scale="e4m3_mean")
    ref = brute_quantize_mean(W)
    assert got[2].shape == (6,)
    for x, y in zip(got, ref):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))
    chat = O.decoded_scales(got[1], got[2], "e4m3_mean")
    assert [Fraction(float(v)) for v in chat] == brute_chat_mean(ref[1], ref[2])
    # the dequantised weights follow: RNbf16(RN32(q c^)) with these scales
    deq = O.dequant(*got, N, K, scale="e4m3_mean")
    q = O.nf4_codebook()
    code = np.empty(N * K, np.uint8)
    code[0::2], code[1::2] = got[0] & 15, got[0] >> 4
    ref_w = O.f32_to_bf16_bits((q[code] * np.repeat(chat, 64)).astype(np.float32)).reshape(N, K)
    assert np.array_equal(deq, ref_w)


def test_pairwise_tree_sum():
    rng = np.random.default_rng(0)
    for n in (1, 7, 128, 200, 256):
        v = (rng.random(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
        exact = math.fsum(v.astype(np.float64))
        got = float(O.pairwise_sum_f32(v))
        assert abs(got - exact) <= 8 * 2.0 ** -24 * float(np.abs(v).astype(np.float64).sum())
        assert float(O.pairwise_sum_f32(np.ones(n, np.float32))) == n        # integers: exact
        assert O.pairwise_sum_f32(v) == np.float32(_tree_rn32([Fraction(float(x)) for x in v]))


def test_equal_scales_reconstruct_exactly():
    """A group whose block scales are all equal has zero residuals: c1 = 0,
    every c2 = 0, and c^ = mu = c exactly."""
    blk = np.zeros((256, 64), np.float32)
    blk[:, 0] = 0.0234375
    blk[:, 5] = -0.01
    W = _bf16(blk).reshape(64, 256 * 64 // 64)
    codes, c2, c1 = O.quantize(W, scale="e4m3_mean")
    assert c1[0] == 0 and np.all(c2 == 0) and c1[1] == np.float32(0.0234375)
    assert np.all(O.decoded_scales(c2, c1, "e4m3_mean") == np.float32(0.0234375))


def test_mean_centring_scale_error_bound_and_gain():
    """|c^ - c| <= 2^-4 |d| + 2^-10 c1 + 2^-23 (|c^| + |d|) per block (E4M3
    keeps 3 mantissa bits, its subnormals a 2^-9 quantum, then two fp32
    roundings); on normal weights the mean relative scale error is several
    times lower than without centring, the point of the variant."""
    rng = np.random.default_rng(1)
    W = _bf16(rng.normal(0, 0.02, (128, 64 * 256)))
    codes, c2, c1 = O.quantize(W, scale="e4m3_mean")
    c = O.block_absmax(W).astype(np.float64)
    chat = O.decoded_scales(c2, c1, "e4m3_mean").astype(np.float64)
    g = np.arange(len(c)) // 256
    mu, c1g = c1[2 * g + 1].astype(np.float64), c1[2 * g].astype(np.float64)
    d = np.abs(c - mu)
    assert np.all(np.abs(chat - c) <= 2.0 ** -4 * d + 2.0 ** -10 * c1g + 2.0 ** -23 * (np.abs(chat) + d) + 1e-30)
    _, c2p, c1p = O.quantize(W)
    plain = O.decoded_scales(c2p, c1p).astype(np.float64)
    assert np.mean(np.abs(chat - c) / c) * 4 < np.mean(np.abs(plain - c) / c)


def test_storage_of_the_mean_codec():
    assert O.bits_per_weight(4096, 4096) == 4 + 8 / 64 + 32 / 16384
    assert O.storage_bytes(4096, 4096, scale="e4m3_mean") * 8 / (4096 * 4096) == 4 + 8 / 64 + 64 / 16384


def test_planted_sequential_mean_is_caught():
    """Summing the scales left to right instead of as the pairwise tree gives
    a different fp32 mean on this group, and so different codes than the
    brute-force quantiser."""
    rng = np.random.default_rng(0)
    a = rng.normal(0, 0.02, 256 * 64) * np.repeat(np.exp2(rng.integers(-12, 12, 256)), 64)
    W = _bf16(a).reshape(16, 1024)
    cb = O.block_absmax(W)
    seq = np.float32(0)
    for v in cb:
        seq = np.float32(seq + v)
    assert np.float32(seq / np.float32(256)) != O.quantize(W, scale="e4m3_mean")[2][1]
    ref = brute_quantize_mean(W)
    assert np.array_equal(O.quantize(W, scale="e4m3_mean")[2].view(np.uint32), ref[2].view(np.uint32))
