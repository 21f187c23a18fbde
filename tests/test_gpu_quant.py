"""GPU parity of the NF4 double quantiser and dequantiser against the oracle:
bit-exact codes, E4M3 scale codes, fp32 second-level scales and bf16
dequantised weights (nlp-lineage 'QLoRA', section 'The idea')."""

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import bits, from_bits
from bit_nf4_quantized_15_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def gpu_quant(q, Wb, fmt="nf4", scale="e4m3"):
    W = from_bits(Wb)
    q.read_status()
    w = q.quantize(W, fmt=fmt, scale=scale)
    torch.cuda.synchronize()
    assert q.read_status() == 0
    return w


def assert_quant_equal(w, ref):
    codes, c2, c1 = ref
    assert np.array_equal(w.codes.cpu().numpy(), codes)
    assert np.array_equal(w.c2.cpu().numpy(), c2)
    assert np.array_equal(w.c1.cpu().numpy().view(np.uint32), c1.view(np.uint32))


def mixed_weights(N, K, seed):
    rng = np.random.default_rng(seed)
    a = rng.normal(0, 0.02, (N, K))
    t = rng.standard_t(3, (N, K)) * 0.02 * np.where(rng.random((N, K)) < 0.001, 50.0, 1.0)
    return O.f32_to_bf16_bits(np.where(rng.random((N, 1)) < 0.5, a, t).astype(np.float32))


@pytest.mark.parametrize("N,K,seed", [(1, 64, 0), (3, 128, 1), (24, 192, 2), (200, 320, 3), (37, 64 * 300, 4),
                                      (256, 4096, 5), (8, 16384 * 3, 6)])
def test_quantize_dequant_bitexact(lib, N, K, seed):
    Wb = mixed_weights(N, K, seed)
    ref = O.quantize(Wb)
    w = gpu_quant(lib, Wb)
    assert_quant_equal(w, ref)
    out = lib.dequant(w)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), O.dequant(*ref, N, K))


def mantissa_pair_matrix():
    """Blocks [c, w_1..w_63]: for every absmax c with a bf16 significand in
    [1, 2) every finite bf16 |w| <= c appears once; plus blocks with tiny
    and huge c (the IEEE-division path) and subnormal weights."""
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_bits_to_f32(pats)
    fin = np.isfinite(vals)
    rows = []
    cs = list(range(0x3F80, 0x4000)) + [0x0200, 0x1000, 0x1005, 0x0001, 0x007F, 0x127F, 0x1280, 0x717F,
                                         0x7180, 0x7F7F]
    for cb in cs:
        c = O.bf16_bits_to_f32(np.array([cb], np.uint16))[0]
        sel = pats[fin & (np.abs(vals) <= c)]
        if cb not in range(0x3F80, 0x4000):
            sel = sel[::5]
        pad = (-len(sel)) % 63
        sel = np.concatenate([sel, np.zeros(pad, np.uint16)])
        blk = sel.reshape(-1, 63)
        rows.append(np.concatenate([np.full((blk.shape[0], 1), cb, np.uint16), blk], axis=1))
    return np.concatenate(rows)


def test_quantize_every_significand_pair(lib):
    Wb = mantissa_pair_matrix()
    assert Wb.shape[0] > 60000
    ref = O.quantize(Wb)
    w = gpu_quant(lib, Wb)
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, *Wb.shape))


def test_special_blocks(lib):
    blocks = np.zeros((8, 64), np.float32)
    blocks[1, 3] = 0.5                       # single nonzero
    blocks[2, :] = -1.0                      # constant negative block
    blocks[3, ::2], blocks[3, 1::2] = 1e-3, -1e-3
    blocks[4, 0] = 3.0e38                    # huge absmax
    blocks[5, :] = np.linspace(-1e-38, 1e-38, 64)   # subnormal-scale block
    blocks[6, 5] = -448.0
    blocks[7, :] = 65504.0
    Wb = O.f32_to_bf16_bits(blocks)
    Wb[5, 7] = 0x0001                        # smallest subnormal
    ref = O.quantize(Wb)
    w = gpu_quant(lib, Wb)
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, 8, 64))


def test_nonfinite_weight_sets_status(lib):
    Wb = mixed_weights(4, 128, 9)
    Wb[2, 77] = 0x7F80                       # +inf
    W = from_bits(Wb)
    lib.read_status()
    lib.quantize(W)
    torch.cuda.synchronize()
    assert lib.read_status() == lib.QLORA_ERR_NONFINITE


def test_quantize_linear4096_full(lib):
    wl = WL.WORKLOADS["linear4096_m16"]
    W = WL.make_linear(wl, wl.linears[0])["W"]
    Wb = bits(W)
    ref = O.quantize(Wb)
    w = gpu_quant(lib, Wb)
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, 4096, 4096))


def test_roundtrip_2p31_sampled(lib):
    """The bulk 2^31-weight round trip in the launch configuration the bench
    times; 64 random 16384-weight groups plus the first and last are checked
    bit-exactly against the oracle."""
    n = WL.ROUNDTRIP_WEIGHTS
    W = WL.roundtrip_weights(n, seed=0, device="cuda")
    Wm = W.view(n // 64, 64)
    w = lib.quantize(Wm)
    out = lib.dequant(w)
    torch.cuda.synchronize()
    assert lib.read_status() == 0
    G = n // 16384
    rng = np.random.default_rng(0)
    groups = sorted(set([0, G - 1, G // 2, G // 2 - 1] + rng.integers(0, G, 60).tolist()))
    for g in groups:
        sl = slice(g * 16384, (g + 1) * 16384)
        Wb = bits(W[sl]).reshape(256, 64)
        codes, c2, c1 = O.quantize(Wb)
        assert np.array_equal(w.codes[g * 8192:(g + 1) * 8192].cpu().numpy(), codes)
        assert np.array_equal(w.c2[g * 256:(g + 1) * 256].cpu().numpy(), c2)
        assert w.c1[g].cpu().numpy().view(np.uint32) == c1.view(np.uint32)[0]
        assert np.array_equal(bits(out.view(-1)[sl]), O.dequant(codes, c2, c1, 256, 64).reshape(-1))
    del W, out, w
    torch.cuda.empty_cache()


# ------------------------------------------- the compared formats (FP4, Int4)
# nlp-lineage 'QLoRA', section 'What it showed', third bullet: NF4 against a
# standard 4-bit float and 4-bit integers.  Same blocks and double
# quantisation, other levels; the quantiser takes its threshold-search path.
@pytest.mark.parametrize("fmt", ["fp4", "int4"])
@pytest.mark.parametrize("N,K,seed", [(1, 64, 10), (24, 192, 11), (37, 64 * 300, 12), (256, 4096, 13)])
def test_formats_quantize_dequant_bitexact(lib, fmt, N, K, seed):
    Wb = mixed_weights(N, K, seed)
    ref = O.quantize(Wb, fmt=fmt)
    w = gpu_quant(lib, Wb, fmt)
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, N, K, fmt=fmt))


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_formats_every_significand_pair(lib, fmt):
    Wb = mantissa_pair_matrix()
    ref = O.quantize(Wb, fmt=fmt)
    w = gpu_quant(lib, Wb, fmt)
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, *Wb.shape, fmt=fmt))


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_formats_special_blocks(lib, fmt):
    blocks = np.zeros((6, 64), np.float32)
    blocks[1, 3] = 0.5
    blocks[2, :] = -1.0
    blocks[3, 0], blocks[3, 1], blocks[3, 2] = 1.0, 0.125, -0.125   # FP4 ties at 1/8
    blocks[4, 0] = 3.0e38
    blocks[5, :] = np.linspace(-1e-38, 1e-38, 64)
    Wb = O.f32_to_bf16_bits(blocks)
    ref = O.quantize(Wb, fmt=fmt)
    w = gpu_quant(lib, Wb, fmt)
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, 6, 64, fmt=fmt))


# ------------------------------------ scale codec variant: c2 stored as E5M2
@pytest.mark.parametrize("fmt", ["nf4", "fp4"])
@pytest.mark.parametrize("N,K,seed", [(3, 128, 20), (37, 64 * 300, 21), (256, 4096, 22)])
def test_e5m2_scales_quantize_dequant_bitexact(lib, fmt, N, K, seed):
    Wb = mixed_weights(N, K, seed)
    ref = O.quantize(Wb, fmt=fmt, scale="e5m2")
    w = gpu_quant(lib, Wb, fmt, "e5m2")
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, N, K, fmt=fmt, scale="e5m2"))


def test_e5m2_scales_every_significand_pair(lib):
    Wb = mantissa_pair_matrix()
    ref = O.quantize(Wb, scale="e5m2")
    w = gpu_quant(lib, Wb, "nf4", "e5m2")
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, *Wb.shape, scale="e5m2"))


# --------------- scale codec variant: E4M3 residuals from each group's mean
@pytest.mark.parametrize("fmt", ["nf4", "int4"])
@pytest.mark.parametrize("N,K,seed", [(1, 64, 30), (3, 128, 31), (37, 64 * 300, 32), (256, 4096, 33),
                                      (8, 16384 * 3, 34)])
def test_mean_scales_quantize_dequant_bitexact(lib, fmt, N, K, seed):
    """Group mean (fp32 pairwise tree), signed E4M3 residual codes, [c1, mean]
    pairs and the dequantised weights, bit for bit; partial last groups and
    one-block groups included."""
    Wb = mixed_weights(N, K, seed)
    ref = O.quantize(Wb, fmt=fmt, scale="e4m3_mean")
    w = gpu_quant(lib, Wb, fmt, "e4m3_mean")
    assert w.c1.numel() == 2 * ((N * K // 64 + 255) // 256)
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, N, K, fmt=fmt, scale="e4m3_mean"))


def test_mean_scales_every_significand_pair(lib):
    """The significand-pair matrix (group sums stay finite: absmax values up
    to about 1e30 only), where scales of very different size share groups
    and the residuals take both signs."""
    Wb = mantissa_pair_matrix()
    cmax = O.bf16_bits_to_f32(Wb[:, 0])
    Wb = Wb[cmax < 1e30]
    Wb = Wb[: (Wb.shape[0] // 4) * 4]
    ref = O.quantize(Wb, scale="e4m3_mean")
    assert np.any(ref[1] & 0x80) and np.any((ref[1] & 0x80) == 0)      # residuals of both signs
    w = gpu_quant(lib, Wb, "nf4", "e4m3_mean")
    assert_quant_equal(w, ref)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, *Wb.shape, scale="e4m3_mean"))


def test_mean_scales_equal_blocks_reconstruct(lib):
    """A group of 256 blocks with the same absmax: c1 = 0, all c2 = 0 and the
    decoded scale is the mean, i.e. exactly the absmax."""
    blk = np.zeros((256, 64), np.float32)
    blk[:, 0] = 0.0234375
    blk[:, 9] = -0.01
    Wb = O.f32_to_bf16_bits(blk).reshape(64, 256)
    ref = O.quantize(Wb, scale="e4m3_mean")
    w = gpu_quant(lib, Wb, "nf4", "e4m3_mean")
    assert_quant_equal(w, ref)
    assert ref[2][0] == 0 and np.all(ref[1] == 0)
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*ref, 64, 256, scale="e4m3_mean"))


def test_quantize_sharded_single_rank_equals_quantize(lib):
    """The sharded quantiser's per-rank step (the library quantiser on a flat
    [1, len] view of a run of whole 16384-weight groups) without a process
    group: the whole weight as one share, bit-exact against the oracle."""
    from bit_nf4_quantized_15_b200.sharded import quantize_sharded
    Wb = mixed_weights(37, 64 * 300, 23)
    w = quantize_sharded(from_bits(Wb))
    torch.cuda.synchronize()
    assert (w.N, w.K) == (37, 64 * 300)
    assert_quant_equal(w, O.quantize(Wb))
    assert np.array_equal(bits(lib.dequant(w)), O.dequant(*O.quantize(Wb), 37, 64 * 300))
