"""GPU parity of the adapter merge and of the paged AdamW step against the
oracle (oracle/adapters.py).

Merge: W_merged = RNbf16(W^ + s (L1 L2)^T).  The GPU accumulates the rank-r
product in fp32 on the tensor cores (order and internal alignment
unspecified) and the oracle in fp64; both round once to bf16.  The fp32
accumulation error is bounded relative to the size of the terms, not of the
result, which matters where W^ and the adapter term nearly cancel.  So each
element must lie within one bf16 ulp of the oracle's plus
2^-16 (|W^| + |s| sum_j |L1[k,j] L2[j,n]|) (256 times finer than a bf16 ulp
of the terms), and at most 1 in 1000 elements may differ at all.
Re-quantising the merged weight (the lossy step the pages warn about) must
give the oracle's codes and scales bit for bit, within the round-trip error
bound of the quantiser.

AdamW: every operation is an fp32 operation rounded in a fixed order on both
sides, so p, m, v and the bf16 copy of p must match bit for bit, with the
state in paged (managed) memory that is moved to the host and back between
steps, and in plain device memory.
"""

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import bits, from_bits
from bit_nf4_quantized_15_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _ulp_bf16(ref_bits):
    v = np.abs(O.bf16_bits_to_f64(ref_bits))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return np.exp2(np.maximum(e, -126) - 7)


def _check_merge(got_bits, ref_bits, name, What, L1, L2, s):
    g = O.bf16_bits_to_f64(got_bits)
    r = O.bf16_bits_to_f64(ref_bits)
    diff = np.abs(g - r)
    terms = np.abs(O.bf16_bits_to_f64(What)) + abs(s) * (np.abs(O.bf16_bits_to_f64(L1)) @
                                                        np.abs(O.bf16_bits_to_f64(L2))).T
    bound = _ulp_bf16(ref_bits) + 2.0 ** -16 * terms
    assert np.all(diff <= bound * (1 + 1e-9)), f"{name}: a merged weight is off by more than its bound"
    frac = np.count_nonzero(got_bits != ref_bits) / got_bits.size
    assert frac <= 1e-3, f"{name}: {frac:.2e} of the merged weights differ from the oracle"
    return frac


def _case(N, K, r, seed, l_std=0.05):
    rng = np.random.default_rng(seed)
    bf = lambda x: O.f32_to_bf16_bits(np.asarray(x, np.float32))
    W = bf(rng.normal(0, 0.02, (N, K)))
    L1 = bf(rng.normal(0, l_std, (K, r)))
    L2 = bf(rng.normal(0, l_std, (r, N)))
    return W, L1, L2


MERGE_SHAPES = [  # N, K, r: one tile, ragged tiles in both directions, every padded rank width
    (128, 128, 16), (200, 320, 8), (1000, 704, 24), (136, 4096, 64), (384, 192, 128), (8, 64, 32),
]


@pytest.mark.parametrize("N,K,r", MERGE_SHAPES)
@pytest.mark.parametrize("fmt,scale", [("nf4", "e4m3"), ("fp4", "e4m3"), ("nf4", "e5m2"), ("nf4", "e4m3_mean")])
def test_merge_parity(lib, N, K, r, fmt, scale):
    W, L1, L2 = _case(N, K, r, seed=N + K + r)
    s = 16.0 / r
    w = lib.quantize(from_bits(W), fmt=fmt, scale=scale)
    got = bits(lib.adapter_merge(w, from_bits(L1), from_bits(L2), s))
    torch.cuda.synchronize()
    assert lib.read_status() == 0
    What = O.dequant(*O.quantize(W, fmt=fmt, scale=scale), N, K, fmt=fmt, scale=scale)
    _check_merge(got, O.adapter_merge(What, L1, L2, s), f"{fmt}/{scale} {N}x{K} r={r}", What, L1, L2, s)


def test_merge_zero_adapter_is_the_dequantised_weight(lib):
    W, L1, L2 = _case(296, 512, 16, seed=3)
    w = lib.quantize(from_bits(W))
    got = bits(lib.adapter_merge(w, from_bits(L1), from_bits(np.zeros_like(L2)), 0.5))
    assert np.array_equal(got, bits(lib.dequant(w)))


@pytest.mark.parametrize("which", [4, 6])   # LLaMA-7B gate 11008x4096 and down 4096x11008, r = 64
def test_merge_full_size_and_requantise(lib, which):
    wl = WL.WORKLOADS["llama7b_block"]
    lin = wl.linears[which]
    t = WL.make_linear(wl, lin, seed=which, device="cpu")
    W, L1, L2 = (WL.bf16_bits(t[k]) for k in ("W", "L1", "L2"))
    L2 = (O.f32_to_bf16_bits(O.bf16_bits_to_f32(L2) * np.float32(5.0)))   # a trained-size adapter
    w = lib.quantize(from_bits(W))
    merged = lib.adapter_merge(w, from_bits(L1), from_bits(L2), wl.s)
    wq = lib.quantize(merged)                                               # the lossy re-quantisation
    torch.cuda.synchronize()
    assert lib.read_status() == 0
    got = bits(merged)
    What = O.dequant(*O.quantize(W), lin.N, lin.K)
    _check_merge(got, O.adapter_merge(What, L1, L2, wl.s), f"{lin.name} merge", What, L1, L2, wl.s)
    codes, c2, c1 = O.quantize(got)
    assert np.array_equal(wq.codes.cpu().numpy(), codes)
    assert np.array_equal(wq.c2.cpu().numpy(), c2)
    assert np.array_equal(wq.c1.cpu().numpy().view(np.uint32), c1.view(np.uint32))
    # what the re-quantisation loses, against the bound of the quantiser's own error
    m64 = O.bf16_bits_to_f64(got).reshape(-1)
    back = O.bf16_bits_to_f64(O.dequant(codes, c2, c1, lin.N, lin.K)).reshape(-1)
    c = np.repeat(O.block_absmax(got).astype(np.float64), 64)
    chat = np.repeat(O.decoded_scales(c2, c1).astype(np.float64), 64)
    q = O.nf4_codebook().astype(np.float64)
    halfgap = np.max(np.diff(q)) / 2
    bound = c * (halfgap + 2.0 ** -24) + np.abs(chat - c) + np.abs(back) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(m64 - back) <= bound)


# ------------------------------------------------------------------ AdamW
@pytest.mark.parametrize("n", [4096 + 3, 1 << 20])
@pytest.mark.parametrize("paged", [True, False])
def test_adamw_bit_exact(lib, n, paged):
    rng = np.random.default_rng(n)
    p0 = rng.normal(0, 0.05, n).astype(np.float32)
    dev = torch.device("cuda")
    p = torch.tensor(p0, device=dev)
    pb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    if paged:
        mb, vb = lib.paged_empty(n), lib.paged_empty(n)
        m, v = mb.tensor, vb.tensor
    else:
        m, v = torch.zeros(n, device=dev), torch.zeros(n, device=dev)
    rp, rm, rv = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t in range(1, 4):
        g = (rng.normal(0, 1e-2, n) * (1 + 0.5 * np.sin(t))).astype(np.float32)
        wd = 0.01 if t != 2 else 0.0
        lib.adamw_step(p, torch.tensor(g, device=dev), m, v, t, lr=3e-4, betas=(0.9, 0.999), eps=1e-8,
                       weight_decay=wd, p_bf16=pb)
        if paged:            # page the state out to the host and back between steps
            mb.prefetch(-1)
            vb.prefetch(-1)
            torch.cuda.synchronize()
            mb.prefetch(torch.cuda.current_device())
            vb.prefetch(torch.cuda.current_device())
        rp, rm, rv, rpb = O.adamw_step(rp, g, rm, rv, O.adamw_scalars(3e-4, 0.9, 0.999, 1e-8, wd, t))
        torch.cuda.synchronize()
        assert np.array_equal(p.cpu().numpy().view(np.uint32), rp.view(np.uint32)), f"p step {t}"
        assert np.array_equal(m.cpu().numpy().view(np.uint32), rm.view(np.uint32)), f"m step {t}"
        assert np.array_equal(v.cpu().numpy().view(np.uint32), rv.view(np.uint32)), f"v step {t}"
        assert np.array_equal(bits(pb), rpb), f"bf16 copy step {t}"
