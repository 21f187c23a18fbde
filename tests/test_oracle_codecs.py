"""Pins for the oracle's bf16 and E4M3 codecs.

bf16 rounding is checked against torch's own conversion (an independent
library routine); the E4M3 decoder against the closed form of the OCP FP8
format and torch's float8_e4m3fn; the vectorised encoder against an exact
rational encoder on every tie and its neighbours.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O


def test_bf16_round_matches_torch_random():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    ours = O.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_round_ties_and_neighbours():
    hi = np.arange(0, 2 ** 16, 7, dtype=np.uint32) << 16
    cand = np.concatenate([hi | 0x8000, hi | 0x7FFF, hi | 0x8001, hi | 0x0001, hi | 0xFFFF])
    x = cand.view(np.float32)
    x = x[np.isfinite(x)]
    ours = O.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_widen_exact():
    b = np.arange(2 ** 16, dtype=np.uint32).astype(np.uint16)
    f = O.bf16_bits_to_f32(b)
    ref = torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    assert np.array_equal(f.view(np.uint32), ref.view(np.uint32))


def test_e4m3_decode_closed_form_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(codes)
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            assert math.isnan(v[c])
            continue
        mag = 2.0 ** (e - 7) * (1 + m / 8) if e else 2.0 ** -6 * (m / 8)
        assert v[c] == (-mag if s else mag)
    assert O.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert O.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    ours = O.e4m3_decode(codes)
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))


def _ties_and_neighbours():
    vals = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    vals = np.sort(vals)
    mids = (vals[:-1] + vals[1:]) / 2
    pts = [np.float32(v) for v in np.concatenate([vals, mids, [464.0, 480.0, 500.0, 1e6]])]
    out = []
    for p in pts:
        p = np.float32(p)
        out += [p, np.nextafter(p, np.float32(np.inf)), np.nextafter(p, np.float32(0))]
    return np.array(out, dtype=np.float32)


def test_e4m3_encode_matches_exact_on_ties():
    x = _ties_and_neighbours()
    x = np.concatenate([x, -x])
    fast = O.e4m3_encode(x)
    slow = np.array([O.e4m3_encode_exact(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(fast, slow)


def test_e4m3_encode_matches_exact_random():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.uniform(0, 470, 20000), np.exp2(rng.uniform(-14, 9, 20000))]).astype(np.float32)
    fast = O.e4m3_encode(x)
    slow = np.array([O.e4m3_encode_exact(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(fast, slow)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([_ties_and_neighbours(), rng.uniform(0, 448, 200000).astype(np.float32)])
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), ref)


def test_e4m3_encode_special():
    enc = lambda v: int(O.e4m3_encode(np.array([v], dtype=np.float32))[0])
    assert enc(0.0) == 0x00
    assert enc(448.0) == 0x7E
    assert enc(464.0) == 0x7E          # tie between 448 and the NaN slot: even code
    assert enc(470.0) == 0x7E          # satfinite
    assert enc(float("inf")) == 0x7E
    assert enc(float("nan")) == 0x7F
    assert enc(2.0 ** -10) == 0x00     # tie between 0 and 2^-9: even code 0
    assert enc(3 * 2.0 ** -10) == 0x02 # tie between 1 and 2 (x 2^-9): even
    assert enc(-1.0) == 0x80 | 0x38


# ------------------------------------------------------------------ E5M2
# The scale-codec variant of the double quantisation (c2 as E5M2).
def test_e5m2_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e5m2).double().numpy()
    ours = O.e5m2_decode(codes)
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))


def _e5m2_ties_and_neighbours():
    vals = np.sort(O.e5m2_decode(np.arange(0x7C, dtype=np.uint8)))
    mids = (vals[:-1] + vals[1:]) / 2
    pts = np.concatenate([vals, mids, [61440.0, 65536.0, 1e6]]).astype(np.float32)
    out = []
    for p in pts:
        out += [p, np.nextafter(p, np.float32(np.inf)), np.nextafter(p, np.float32(0))]
    return np.array(out, dtype=np.float32)


def test_e5m2_encode_matches_exact_on_ties():
    x = _e5m2_ties_and_neighbours()
    x = np.concatenate([x, -x])
    fast = O.e5m2_encode(x)
    slow = np.array([O.e5m2_encode_exact(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(fast, slow)


def test_e5m2_encode_matches_exact_random():
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.uniform(0, 60000, 10000), np.exp2(rng.uniform(-18, 16, 10000))]).astype(np.float32)
    fast = O.e5m2_encode(x)
    slow = np.array([O.e5m2_encode_exact(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(fast, slow)


def test_e5m2_encode_matches_torch_in_range():
    rng = np.random.default_rng(13)
    x = np.concatenate([_e5m2_ties_and_neighbours(), rng.uniform(0, 57344, 100000).astype(np.float32),
                        np.exp2(rng.uniform(-18, 15.8, 100000)).astype(np.float32)])
    x = x[np.abs(x) <= 57344]
    ref = torch.from_numpy(x.copy()).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(O.e5m2_encode(x), ref)


def test_e5m2_encode_special():
    enc = lambda v: int(O.e5m2_encode(np.array([v], dtype=np.float32))[0])
    assert enc(0.0) == 0x00
    assert enc(57344.0) == 0x7B
    assert enc(61440.0) == 0x7B        # beyond the largest finite value: satfinite
    assert enc(float("inf")) == 0x7B
    assert enc(float("nan")) == 0x7F
    assert enc(2.0 ** -17) == 0x00     # tie between 0 and 2^-16: even code 0
    assert enc(1.0) == 0x3C and enc(-1.0) == 0xBC
