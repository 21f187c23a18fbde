"""Pins for the oracle's adapter merge and AdamW step (oracle/adapters.py).

Independent references: exact rational arithmetic written here (its own
round-to-bf16), torch.optim.AdamW (a library implementation of the same
update), closed forms of the first step, and special cases.  Pages: examadda
"QLoRA", "Practical Notes" (merging into a 4-bit base is lossy: dequantise
first); nlp-lineage "QLoRA", section "The idea", paged-optimizers bullet.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O


def _rn_bf16_exact(x: Fraction) -> Fraction:
    """Round a rational to bf16 (8 significant bits, min normal exponent
    -126, subnormal quantum 2^-133), ties to even."""
    if x == 0:
        return Fraction(0)
    sgn = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    q = Fraction(2) ** (e - 7)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sgn * fl * q


def _bits_of(v: Fraction) -> int:
    return int(O.f32_to_bf16_bits(np.array([float(v)], np.float32))[0])


def test_f64_to_bf16_single_rounding_matches_exact():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, 4000) * np.exp2(rng.integers(-140, 120, 4000))
    # ties and near-ties of the bf16 grid, where rounding twice would go wrong
    base = O.bf16_bits_to_f64(O.f32_to_bf16_bits(rng.normal(0, 1, 200).astype(np.float32)))
    ulp = np.exp2(np.floor(np.log2(np.abs(base))) - 7)
    x = np.concatenate([x, base + ulp / 2, base - ulp / 2, base + ulp / 2 + ulp * 2.0 ** -30,
                        base + ulp / 2 - ulp * 2.0 ** -30, [0.0, 1e-45, 2.0 ** -134, 3 * 2.0 ** -134]])
    got = O.f64_to_bf16_bits(x)
    for xi, gi in zip(x, got):
        ref = _bits_of(_rn_bf16_exact(Fraction(float(xi))))
        if ref == 0 and np.signbit(xi):      # a negative value that rounds to zero keeps its sign
            ref = 0x8000
        assert gi == ref, xi


def test_f64_to_bf16_differs_from_rounding_twice():
    """1 + 2^-8 + 2^-30 rounds up to 1 + 2^-7 in one step, but through fp32
    (1 + 2^-8, a tie) it would round down to 1: the helper must not do that."""
    x = np.array([1 + 2.0 ** -8 + 2.0 ** -30])
    assert O.f64_to_bf16_bits(x)[0] == 0x3F81
    assert O.f32_to_bf16_bits(x.astype(np.float32))[0] == 0x3F80


def _merge_case(N=6, K=128, r=8, seed=0):
    rng = np.random.default_rng(seed)
    W = O.f32_to_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    What = O.dequant(*O.quantize(W), N, K)
    L1 = O.f32_to_bf16_bits(rng.normal(0, 0.1, (K, r)).astype(np.float32))
    L2 = O.f32_to_bf16_bits(rng.normal(0, 0.1, (r, N)).astype(np.float32))
    return What, L1, L2


def _brute_merge(What, L1, L2, s):
    N, K = What.shape
    r = L1.shape[1]
    fw = lambda b: Fraction(float(O.bf16_bits_to_f64(np.array([b], np.uint16))[0]))
    out = np.empty((N, K), np.uint16)
    sf = Fraction(s)
    for n in range(N):
        for k in range(K):
            acc = sum(fw(L1[k, j]) * fw(L2[j, n]) for j in range(r))
            out[n, k] = _bits_of(_rn_bf16_exact(fw(What[n, k]) + sf * acc))
    return out


@pytest.mark.parametrize("s", [0.25, 2.0, 0.3])
def test_merge_matches_exact_rational_merge(s):
    What, L1, L2 = _merge_case(N=5, K=64, r=8, seed=int(s * 100))
    assert np.array_equal(O.adapter_merge(What, L1, L2, s), _brute_merge(What, L1, L2, s))


def test_merge_special_cases():
    What, L1, L2 = _merge_case()
    assert np.array_equal(O.adapter_merge(What, L1, np.zeros_like(L2), 0.5), What)   # L2 = 0
    assert np.array_equal(O.adapter_merge(What, L1, L2, 0.0), What)                  # s = 0
    # W^ = 0: the merge is the rounded adapter product itself
    got = O.adapter_merge(np.zeros_like(What), L1, L2, 1.0)
    ref = O.f64_to_bf16_bits((O.bf16_bits_to_f64(L1) @ O.bf16_bits_to_f64(L2)).T)
    assert np.array_equal(got, ref)


def test_merged_weight_reproduces_the_layer_forward():
    """X W_merged^T = X W^T + s X L1 L2 up to the bf16 rounding of the merged
    weight (half an ulp per element: relative 2^-9)."""
    What, L1, L2 = _merge_case(N=48, K=256, r=16, seed=4)
    s = 0.5
    rng = np.random.default_rng(9)
    X = rng.normal(0, 1, (7, 256))
    Y, _ = O.linear_fwd(X, O.bf16_bits_to_f64(What), O.bf16_bits_to_f64(L1), O.bf16_bits_to_f64(L2), s)
    Wm = O.bf16_bits_to_f64(O.adapter_merge(What, L1, L2, s))
    Ym = X @ Wm.T
    bound = np.abs(X) @ (np.abs(Wm) * 2.0 ** -8).T + 1e-12
    assert np.all(np.abs(Ym - Y) <= bound)


def test_planted_untransposed_merge_is_caught():
    """Adding L1 L2 (K x N) without the transpose, on a square weight where the
    shapes still agree, disagrees with the exact merge."""
    What, L1, L2 = _merge_case(N=64, K=64, r=8, seed=5)
    wrong = O.f64_to_bf16_bits(O.bf16_bits_to_f64(What) + 0.5 * (O.bf16_bits_to_f64(L1) @ O.bf16_bits_to_f64(L2)))
    assert not np.array_equal(wrong, O.adapter_merge(What, L1, L2, 0.5))


# ------------------------------------------------------------------ AdamW
def test_adamw_first_step_closed_form():
    """Step 1 with zero state and no decay: m^ = g and v^ = g^2 exactly, so
    p1 = p0 - lr g / (|g| + eps) up to the fp32 roundings of the update."""
    rng = np.random.default_rng(1)
    p = rng.normal(0, 1, 1000).astype(np.float32)
    g = (rng.normal(0, 1, 1000) * np.exp2(rng.integers(-10, 10, 1000))).astype(np.float32)
    c = O.adamw_scalars(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    p1, m, v, _ = O.adamw_step(p, g, np.zeros_like(p), np.zeros_like(p), c)
    ref = p.astype(np.float64) - 1e-3 * g / (np.abs(g) + 1e-8)
    assert np.allclose(p1, ref, rtol=0, atol=1e-9 + 4 * np.spacing(np.abs(p1)))
    assert np.allclose(m, 0.1 * g, rtol=2e-7) and np.allclose(v, 0.001 * g.astype(np.float64) ** 2, rtol=4e-7)


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_adamw_matches_torch_adamw_over_steps(wd):
    """torch.optim.AdamW (fp32, CPU) over 20 steps with varying gradients:
    the same update rule, a different operation order, so equal within a
    few fp32 ulps (wider with weight decay, which torch applies as
    p (1 - lr wd) with that factor rounded to fp32 first)."""
    rng = np.random.default_rng(2)
    p0 = rng.normal(0, 0.05, 4096).astype(np.float32)
    tp = torch.nn.Parameter(torch.tensor(p0))
    opt = torch.optim.AdamW([tp], lr=2e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t in range(1, 21):
        g = rng.normal(0, 1e-2, 4096).astype(np.float32)
        tp.grad = torch.tensor(g)
        opt.step()
        p, m, v, _ = O.adamw_step(p, g, m, v, O.adamw_scalars(2e-4, 0.9, 0.999, 1e-8, wd, t))
    assert np.allclose(p, tp.detach().numpy(), rtol=0, atol=5e-8 if wd == 0 else 5e-7)
    st = opt.state[tp]
    tm, tv = st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()
    # torch forms m by interpolation (m + (g - m)(1 - b1)): absolute differences
    # of a few ulps of the largest moment, relative ones only where m cancels
    assert np.allclose(m, tm, rtol=1e-5, atol=1e-6 * np.abs(tm).max())
    assert np.allclose(v, tv, rtol=1e-5, atol=1e-6 * np.abs(tv).max())


def test_planted_missing_bias_correction_is_caught():
    rng = np.random.default_rng(4)
    p = rng.normal(0, 0.05, 256).astype(np.float32)
    g = rng.normal(0, 1e-2, 256).astype(np.float32)
    c = O.adamw_scalars(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    good, _, _, _ = O.adamw_step(p, g, np.zeros_like(p), np.zeros_like(p), c)
    bad = dict(c, bc1=np.float32(1.0), bc2=np.float32(1.0))
    wrong, _, _, _ = O.adamw_step(p, g, np.zeros_like(p), np.zeros_like(p), bad)
    tp = torch.nn.Parameter(torch.tensor(p))
    opt = torch.optim.AdamW([tp], lr=1e-3, weight_decay=0.0)
    tp.grad = torch.tensor(g)
    opt.step()
    assert np.allclose(good, tp.detach().numpy(), atol=2e-7)
    assert not np.allclose(wrong, tp.detach().numpy(), atol=2e-7)


def test_adamw_bf16_copy_is_the_rounded_master():
    rng = np.random.default_rng(6)
    p = rng.normal(0, 0.05, 512).astype(np.float32)
    g = rng.normal(0, 1e-2, 512).astype(np.float32)
    p1, _, _, pb = O.adamw_step(p, g, np.zeros_like(p), np.zeros_like(p), O.adamw_scalars(1e-3, 0.9, 0.999, 1e-8,
                                                                                           0.01, 1))
    assert np.array_equal(pb, O.f64_to_bf16_bits(p1.astype(np.float64)))
