"""Pins for the oracle's NF4 codebook (nlp-lineage 'QLoRA', section 'The idea',
NF4 bullet; inferensys glossary 'QLoRA', NF4 paragraphs).

The codebook is pinned to things outside the oracle: the standard library's
independent normal quantile, the defining equal-probability property, and
the structural facts the pages state (16 values, exact zero, denser near 0).
"""

import math
from statistics import NormalDist

import numpy as np
import pytest

import oracle as O

ND = NormalDist()


def _tol(y):
    # fp64 resolution of p near the tails times dx/dp = 1/phi(x), plus 4 ulp
    return 2.3e-16 / ND.pdf(y) + 4e-15 * max(1.0, abs(y))


@pytest.mark.parametrize("p", [1e-4, 0.01, 0.1, 0.3, 0.5, 0.5 + 1e-9, 0.7, 0.9,
                               O.nf4_delta(), 0.99, 1 - 1e-6])
def test_norm_ppf_matches_stdlib(p):
    # statistics.NormalDist.inv_cdf is an independent implementation (a
    # rational approximation), so agreement pins the bisection.
    x = O.norm_ppf(p)
    y = ND.inv_cdf(p)
    assert abs(x - y) <= _tol(y)


def test_norm_ppf_dense_grid():
    for p in np.linspace(0.501, 0.999, 997):
        assert abs(O.norm_ppf(float(p)) - ND.inv_cdf(float(p))) <= 4e-15 * 4


def test_codebook_structure():
    q = O.nf4_codebook()
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.all(np.diff(q.astype(np.float64)) > 0)      # strictly increasing
    assert q[7] == 0.0 and not np.signbit(q[7])            # exact zero
    assert q[0] == -1.0 and q[15] == 1.0                   # endpoints exactly +-1
    assert int(np.sum(q < 0)) == 7 and int(np.sum(q > 0)) == 8


def test_codebook_equal_probability_shares():
    """Each positive level sits at an equally spaced probability from 1/2 to
    delta, each negative level likewise on its own side: the 'equal share of
    the normal distribution' property."""
    lv = O.nf4_codebook_f64()
    top = ND.inv_cdf(O.nf4_delta())
    d = O.nf4_delta()
    pos = [ND.cdf(v * top) for v in lv[7:]]                   # 0 and 8 positive
    neg = [ND.cdf(-v * top) for v in reversed(lv[:8])]        # 0 and 7 negative
    assert np.allclose(np.diff(pos), (d - 0.5) / 8, rtol=0, atol=1e-13)
    assert np.allclose(np.diff(neg), (d - 0.5) / 7, rtol=0, atol=1e-13)


def test_codebook_denser_near_zero():
    q = O.nf4_codebook().astype(np.float64)
    gaps_pos = np.diff(q[7:])
    gaps_neg = np.diff(q[:8])[::-1]
    assert np.all(np.diff(gaps_pos) > 0) and np.all(np.diff(gaps_neg) > 0)


def test_codebook_fp32_rounding_is_robust():
    """No fp64 level lies near an fp32 rounding boundary, so a quantile
    error of 1e-14 cannot change the stored fp32 codebook."""
    for v in O.nf4_codebook_f64():
        if v in (0.0, -1.0, 1.0):
            continue
        f = np.float32(v)
        ulp = float(np.spacing(f))
        frac = abs(v - float(f)) / ulp          # in [0, 0.5]
        assert frac < 0.5 - 1e-6


def test_codebook_against_stdlib_derivation():
    """Rebuild the levels with the stdlib quantile; the fp32 tables agree."""
    d = O.nf4_delta()
    pos = [ND.inv_cdf(d + i * (0.5 - d) / 8) for i in range(8)]
    neg = [-ND.inv_cdf(d + i * (0.5 - d) / 7) for i in range(7)]
    lv = sorted(pos + [0.0] + neg)
    ref = np.array([v / max(lv) for v in lv], dtype=np.float32)
    assert np.array_equal(ref.view(np.uint32), O.nf4_codebook().view(np.uint32))


def test_midpoints_exact():
    q = O.nf4_codebook()
    m = O.nf4_midpoints(q)
    from fractions import Fraction
    for i in range(15):
        assert Fraction(float(m[i])) == (Fraction(float(q[i])) + Fraction(float(q[i + 1]))) / 2
