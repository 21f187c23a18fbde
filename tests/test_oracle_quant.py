"""Pins for the oracle's NF4 double quantiser and dequantiser.

The reference used here is a brute-force quantiser written in exact rational
arithmetic in this file (its own RN32, nearest-level search by counting exact
midpoints, E4M3 by nearest-value search), so it shares nothing with the
vectorised oracle.  Pages: nlp-lineage 'QLoRA', section 'The idea' (blocks of
64, absmax scale, scales re-quantised to 8 bits, about 0.127 bits per weight);
inferensys glossary 'QLoRA' (scales become 8-bit floats).
"""

import bisect
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_numbers.json")


# ---------------------------------------------------------------- exact helpers
def _rn(x: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Round a rational to a binary float with ``mant_bits`` significand bits
    (hidden bit included) and minimum normal exponent ``emin``, ties to even."""
    if x == 0:
        return Fraction(0)
    s = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - (mant_bits - 1))
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return s * fl * quantum


def rn32(x):
    return _rn(Fraction(x), 24, -126)


def rnbf16(x):
    return _rn(Fraction(x), 8, -126)


_E4M3 = []
for _c in range(0x7F):
    _e, _m = _c >> 3, _c & 7
    _E4M3.append(((Fraction(_m, 8) / 64) if _e == 0 else (1 + Fraction(_m, 8)) * Fraction(2) ** (_e - 7), _c))


def e4m3_nearest(a: Fraction) -> int:
    """Non-negative rational -> E4M3 code: nearest value, ties to even code,
    anything at or above 448 saturates."""
    if a >= 448:
        return 0x7E
    best = min(_E4M3, key=lambda vc: (abs(a - vc[0]), vc[1] & 1))
    return best[1]


_E5M2 = []
for _c in range(0x7C):
    _e, _m = _c >> 2, _c & 3
    _E5M2.append(((Fraction(_m, 4) / 2 ** 14) if _e == 0 else (1 + Fraction(_m, 4)) * Fraction(2) ** (_e - 15), _c))


def e5m2_nearest(a: Fraction) -> int:
    """Non-negative rational -> E5M2 code: nearest value, ties to even code,
    anything at or above 57344 saturates."""
    if a >= 57344:
        return 0x7B
    best = min(_E5M2, key=lambda vc: (abs(a - vc[0]), vc[1] & 1))
    return best[1]


def bf16_value(bits: int) -> Fraction:
    return Fraction(float(O.bf16_bits_to_f32(np.array([bits], np.uint16))[0]))


def brute_quantize(W_bits: np.ndarray, levels=None, scale="e4m3"):
    q = [Fraction(float(v)) for v in (O.nf4_codebook() if levels is None else levels)]
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
            code = bisect.bisect_left(mids, x)        # number of midpoints strictly below x
            idx = 64 * b + j
            codes[idx // 2] |= code << (4 * (idx & 1))
    G = (nb + 255) // 256
    c1, c2 = [], []
    smax, nearest = (448, e4m3_nearest) if scale == "e4m3" else (57344, e5m2_nearest)
    for g in range(G):
        grp = absmax[256 * g:256 * g + 256]
        c1g = rn32(max(grp) / smax)
        c1.append(c1g)
        for c in grp:
            c2.append(0 if c1g == 0 else nearest(rn32(c / c1g)))
    return (np.frombuffer(bytes(codes), np.uint8), np.array(c2, np.uint8),
            np.array([float(v) for v in c1], np.float32))


def brute_dequant(codes, c2, c1, N, K, levels=None, scale="e4m3"):
    q = [Fraction(float(v)) for v in (O.nf4_codebook() if levels is None else levels)]
    out = np.empty(N * K, np.uint16)
    for idx in range(N * K):
        code = (int(codes[idx // 2]) >> (4 * (idx & 1))) & 15
        b = idx // 64
        dec = 0
        cc = int(c2[b])
        if scale == "e4m3":
            e, m = (cc >> 3) & 15, cc & 7
            dec = (Fraction(m, 8) / 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        else:
            e, m = (cc >> 2) & 31, cc & 3
            dec = (Fraction(m, 4) / 2 ** 14) if e == 0 else (1 + Fraction(m, 4)) * Fraction(2) ** (e - 15)
        chat = rn32(dec * Fraction(float(c1[b // 256])))
        v = rnbf16(rn32(q[code] * chat))
        out[idx] = O.f32_to_bf16_bits(np.array([float(v)], np.float32))[0]
    return out.reshape(N, K)


def _bf16(x):
    return np.atleast_1d(O.f32_to_bf16_bits(np.asarray(x, np.float32)))


def _tiny_inputs():
    rng = np.random.default_rng(7)
    cases = []
    cases.append(_bf16(rng.normal(0, 0.02, (3, 128))))
    t = rng.standard_t(3, (2, 192)) * 0.02
    t[0, 5] *= 50
    cases.append(_bf16(t))
    z = rng.normal(0, 1, (4, 64))
    z[1] = 0.0                                   # an all-zero block
    z[2, :] = np.where(np.arange(64) % 2 == 0, 1.0, -1.0)
    cases.append(_bf16(z))
    return cases


# -------------------------------------------------------------------- tests
@pytest.mark.parametrize("case", range(3))
def test_quantize_matches_bruteforce(case):
    W = _tiny_inputs()[case]
    a = O.quantize(W)
    b = brute_quantize(W)
    for x, y in zip(a, b):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))


@pytest.mark.parametrize("case", range(3))
def test_dequant_matches_bruteforce(case):
    W = _tiny_inputs()[case]
    N, K = W.shape
    codes, c2, c1 = O.quantize(W)
    assert np.array_equal(O.dequant(codes, c2, c1, N, K), brute_dequant(codes, c2, c1, N, K))


def _representable_midpoints():
    q = O.nf4_codebook().astype(np.float64)
    mids = (q[:-1] + q[1:]) / 2
    return [(i, np.float32(m)) for i, m in enumerate(mids) if float(np.float32(m)) == m]


def test_ties_on_midpoints_go_to_lower_code():
    """x exactly on a midpoint (only fp32-representable midpoints can be hit)
    takes the lower code; one ulp above takes the upper one."""
    reps = _representable_midpoints()
    assert any(i == 7 for i, _ in reps)          # (0 + q8)/2 = q8/2 is always exact
    for i, m in reps:
        assert O.nearest_level(np.array([m]))[0] == i
        assert O.nearest_level(np.array([np.nextafter(m, np.float32(2))]))[0] == i + 1
        assert O.nearest_level(np.array([np.nextafter(m, np.float32(-2))]))[0] == i


def test_bruteforce_codes_all_bf16_patterns():
    """Every bf16 pattern |w| <= c as a weight against several absmax values."""
    pats = np.arange(2 ** 16, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_bits_to_f32(pats)
    qf = [Fraction(float(v)) for v in O.nf4_codebook()]
    mids = [(qf[i] + qf[i + 1]) / 2 for i in range(15)]
    for c in [1.0, 1.5, 0.0234375, 3.0517578125e-05, 1.0e30]:
        cb = _bf16(c)[0]
        cv = float(O.bf16_bits_to_f32(np.array([cb]))[0])
        sel = pats[np.isfinite(vals) & (np.abs(vals) <= cv)]
        sel = sel[::37]                          # keep it quick: ~1000 per c
        pad = (-len(sel)) % 63
        sel = np.concatenate([sel, np.zeros(pad, np.uint16)])
        blocks = sel.reshape(-1, 63)
        W = np.concatenate([np.full((blocks.shape[0], 1), cb, np.uint16), blocks], axis=1)
        codes, _, _ = O.quantize(W.reshape(-1, 64))
        code = np.empty(codes.size * 2, np.uint8)
        code[0::2], code[1::2] = codes & 15, codes >> 4
        code = code.reshape(-1, 64)[:, 1:]
        for r in range(blocks.shape[0]):
            for j in range(63):
                x = rn32(bf16_value(int(blocks[r, j])) / Fraction(cv))
                assert code[r, j] == bisect.bisect_left(mids, x)


def test_special_values():
    blk = np.zeros(64, np.float32)
    blk[0], blk[1], blk[2] = 0.5, -0.5, 0.0
    codes, c2, c1 = O.quantize(_bf16(blk).reshape(1, 64))
    assert codes[0] & 15 == 15 and codes[0] >> 4 == 0 and codes[1] & 15 == 7
    z = np.zeros((2, 64), np.uint16)
    codes, c2, c1 = O.quantize(z)
    assert np.all(codes == 0x77) and np.all(c2 == 0) and np.all(c1 == 0)
    assert np.all(O.dequant(codes, c2, c1, 2, 64) == 0)


def test_nonfinite_rejected():
    w = np.zeros((1, 64), np.float32)
    w[0, 3] = np.inf
    with pytest.raises(ValueError):
        O.quantize(_bf16(w))


def test_partial_last_group():
    rng = np.random.default_rng(11)
    W = _bf16(rng.normal(0, 0.02, (5, 64 * 300)))   # 1500 blocks: 5 full groups + 220
    codes, c2, c1 = O.quantize(W)
    assert c1.shape == (6,) and c2.shape == (1500,)
    g5 = O.block_absmax(W)[1280:]
    assert c1[5] == np.float32(g5.max()) / np.float32(448)


def _halfgap(q, code):
    q = q.astype(np.float64)
    lo = (q[code] - q[max(code - 1, 0)]) / 2
    hi = (q[min(code + 1, 15)] - q[code]) / 2
    return max(lo, hi)


def test_round_trip_error_bound():
    """|w - w^| <= c (|x - q| + ulp32(x)/2) + |q| |c^ - c| + ulp32(q c^)/2
    + ulp_bf16(w^)/2, element by element, on normal and heavy-tailed data."""
    rng = np.random.default_rng(5)
    n = 64 * 4096
    a = rng.normal(0, 0.02, n // 2)
    t = rng.standard_t(3, n // 2) * 0.02
    t *= np.where(rng.random(n // 2) < 0.001, 50.0, 1.0)
    W = _bf16(np.concatenate([a, t])).reshape(64, -1)
    N, K = W.shape
    codes, c2, c1 = O.quantize(W)
    What = O.bf16_bits_to_f64(O.dequant(codes, c2, c1, N, K)).reshape(-1)
    w = O.bf16_bits_to_f64(W).reshape(-1)
    q = O.nf4_codebook()
    code = np.empty(n, np.uint8)
    code[0::2], code[1::2] = codes & 15, codes >> 4
    c = np.repeat(O.block_absmax(W).astype(np.float64), 64)
    chat = np.repeat(O.decoded_scales(c2, c1).astype(np.float64), 64)
    hg = np.array([_halfgap(q, k) for k in range(16)])[code]
    qv = q.astype(np.float64)[code]
    bound = (c * (hg + 2.0 ** -24) + np.abs(qv) * np.abs(chat - c)
             + np.abs(qv * chat) * 2.0 ** -24 + np.abs(What) * 2.0 ** -8 + 1e-45)
    assert np.all(np.abs(w - What) <= bound * (1 + 1e-12))


def test_scale_quantisation_bounds():
    rng = np.random.default_rng(6)
    W = _bf16(rng.standard_t(3, (256, 64 * 64)) * 0.02)
    codes, c2, c1 = O.quantize(W)
    c = O.block_absmax(W).astype(np.float64)
    chat = O.decoded_scales(c2, c1).astype(np.float64)
    c1r = np.repeat(c1.astype(np.float64), 256)[: len(c)]
    dec = O.e4m3_decode(c2)
    assert np.all(dec <= 448.0)
    normal = c / c1r >= 2.0 ** -6
    rel = np.abs(chat - c)[normal] / c[normal]
    assert rel.max() <= 2.0 ** -4 + 1e-6
    assert np.all(np.abs(chat - c)[~normal] <= 2.0 ** -10 * c1r[~normal] * (1 + 1e-6))


def test_storage_accounting_matches_pages():
    g = json.load(open(GOLDEN))
    for (N, K) in [(4096, 4096), (11008, 4096), (22016, 8192), (8192, 22016), (1, 2 ** 31 // 1)]:
        if N * K % 16384:
            continue
        bpw = O.bits_per_weight(N, K)
        assert bpw == 4 + 8 / 64 + 32 / 16384             # 4.126953125
        over = bpw - 4
        assert abs(over - g["overhead_double_quant_bits"]["value"]) <= 0.01 * 0.127
        assert O.bits_per_weight(N, K, double_quant=False) - 4 == g["overhead_single_quant_bits"]["value"]
        saving = O.bits_per_weight(N, K, False) - bpw
        assert abs(saving - g["saving_bits_per_param"]["value"]) <= 0.02 * 0.37
    saving_65b_gb = 65e9 * (O.bits_per_weight(1, 2 ** 20, False) - O.bits_per_weight(1, 2 ** 20)) / 8 / 1e9
    assert abs(saving_65b_gb - g["saving_65b_gb"]["value"]) <= 0.05 * 3.0
    assert 65e9 * O.bits_per_weight(1, 2 ** 20) / 8 / 1e9 < g["qlora_65b_max_gb"]["value"]
    assert abs(70e9 * 2 / 1e9 - g["fp16_70b_gb"]["value"]) < 1.5
    assert abs(7e9 * 2 / 1e9 - g["fp16_7b_gb"]["value"]) < 0.15
    assert 16 / 4 == g["base_compression"]["value"]
    assert len(O.nf4_codebook()) == g["nf4_levels"]["value"] and O.BLOCK == g["block_size"]["value"]


# ------------------------------------------------- planted mistakes (CPU only)
def _quantize_swapped_nibbles(W):
    codes, c2, c1 = O.quantize(W)
    return ((codes >> 4) | (codes << 4)).astype(np.uint8), c2, c1


def test_planted_nibble_swap_is_caught():
    W = _tiny_inputs()[0]
    ref = brute_quantize(W)
    got = _quantize_swapped_nibbles(W)
    assert not np.array_equal(got[0], ref[0])


def test_planted_tie_rule_is_caught():
    orig = O.nf4_oracle.nearest_level
    m = np.array([m for i, m in _representable_midpoints() if i == 7], np.float32)

    def up(x, q=None):
        q = O.nf4_codebook() if q is None else q
        x64 = np.asarray(x, np.float32).astype(np.float64)
        d = np.abs(x64[..., None] - q.astype(np.float64))
        return (15 - np.argmin(d[..., ::-1], axis=-1)).astype(np.uint8)

    assert orig(m)[0] == 7 and up(m)[0] == 8


def _three_groups():
    """600 blocks = two full c1 groups of 256 and a partial third of 88, each
    at its own magnitude (x1, x300, /500), so that a block or a scale read
    from the wrong group changes c1, c2 or the dequantised weights."""
    rng = np.random.default_rng(9)
    a = rng.normal(0, 0.02, 600 * 64)
    a[256 * 64:512 * 64] *= 300.0
    a[512 * 64:] /= 500.0
    return _bf16(a).reshape(25, 1536)


def test_bruteforce_spans_groups_with_partial_last():
    W = _three_groups()
    N, K = W.shape
    got = O.quantize(W)
    ref = brute_quantize(W)
    assert got[2].shape == (3,) and len(set(got[2].tolist())) == 3
    for x, y in zip(got, ref):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))
    assert np.array_equal(O.dequant(*got, N, K), brute_dequant(*ref, N, K))


def test_planted_group_index_slip_is_caught():
    """A dequantiser that takes c1 of block b from group b // 255 instead of
    b // 256 disagrees with the brute-force dequantiser on the three-group
    input."""
    W = _three_groups()
    N, K = W.shape
    codes, c2, c1 = O.quantize(W)
    dec = O.e4m3_decode(c2).astype(np.float32)
    g = np.minimum(np.arange(len(c2)) // 255, len(c1) - 1)
    chat = (dec * c1[g]).astype(np.float32)
    q = O.nf4_codebook()
    code = np.empty((len(c2), 64), np.uint8)
    cb = codes.reshape(-1, 32)
    code[:, 0::2], code[:, 1::2] = cb & 15, cb >> 4
    slipped = O.f32_to_bf16_bits((q[code] * chat[:, None]).astype(np.float32)).reshape(N, K)
    assert not np.array_equal(slipped, brute_dequant(codes, c2, c1, N, K))
