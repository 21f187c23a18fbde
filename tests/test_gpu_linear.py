"""GPU parity of the quantized linear forward and backward against the fp64
oracle evaluated on the oracle's own dequantised weights (which the
quantiser tests show are bit-identical to the GPU's).  Tolerance: relative
L2 error <= 5e-3 and max abs error <= 1e-2 * max|ref| per output.

nlp-lineage 'QLoRA', section 'The idea', notation paragraph: Y = X.W^ +
X.L1.L2 (here with the scale s), gradients only for L1 and L2.
"""

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close, bits, from_bits, to_f64
from bit_nf4_quantized_15_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def bf(x):
    return O.f32_to_bf16_bits(np.asarray(x, np.float32))


def make_case(M, N, K, r, seed, regime="config", zero_W=False, zero_L2=False):
    rng = np.random.default_rng(seed)
    X = bf(rng.normal(0, 1, (M, K)))
    W = bf(rng.normal(0, 0.02, (N, K)) * (0 if zero_W else 1))
    if regime == "config":                       # adapters as in the workloads
        L1 = bf(rng.normal(0, 1.0 / K, (K, r)))
        L2 = bf(rng.normal(0, 0.01, (r, N)))
    else:                                        # LoRA term comparable to X.W^T
        L1 = bf(rng.normal(0, 1.0 / np.sqrt(K), (K, r)))
        L2 = bf(rng.normal(0, 0.3 / np.sqrt(r), (r, N)))
    if zero_L2:
        L2 = np.zeros_like(L2)
    dY = bf(rng.normal(0, 1, (M, N)))
    return X, W, L1, L2, dY


def run_gpu(q, X, W, L1, L2, dY, s, backward=True, fmt="nf4", scale="e4m3"):
    tX, tW, tL1, tL2 = (from_bits(a) for a in (X, W, L1, L2))
    q.read_status()
    w = q.quantize(tW, fmt=fmt, scale=scale)
    Y, T = q.linear_fwd(tX, w, tL1, tL2, s)
    out = {"Y": Y, "T": T}
    if backward:
        dX, dL1, dL2 = q.linear_bwd(from_bits(dY), tX, T, w, tL1, tL2, s)
        out.update(dX=dX, dL1=dL1, dL2=dL2)
    torch.cuda.synchronize()
    assert q.read_status() == 0
    return {k: to_f64(v) for k, v in out.items()}


def oracle_ref(X, W, L1, L2, dY, s, backward=True, fmt="nf4", scale="e4m3"):
    N, K = W.shape
    What = O.bf16_bits_to_f64(O.dequant(*O.quantize(W, fmt=fmt, scale=scale), N, K, fmt=fmt, scale=scale))
    X64, L164, L264 = (O.bf16_bits_to_f64(a) for a in (X, L1, L2))
    Y, T = O.linear_fwd(X64, What, L164, L264, s)
    ref = {"Y": Y, "T": T}
    if backward:
        dX, dL1, dL2, _ = O.linear_bwd(O.bf16_bits_to_f64(dY), X64, What, L164, L264, s, T)
        ref.update(dX=dX, dL1=dL1, dL2=dL2)
    return ref


SHAPES = [  # M, N, K, r: single tiles, ragged tails, split reductions, every token-tile width
    (1, 64, 64, 16), (5, 200, 320, 16), (16, 512, 1024, 64), (37, 136, 256, 32), (64, 128, 128, 48),
    (100, 264, 704, 64), (200, 384, 512, 128), (300, 256, 192, 16), (513, 1000, 640, 64), (1024, 1024, 2048, 64),
    # several tiles per persistent CTA, each ending with a LoRA extension stage
    (2048, 4096, 512, 32), (1536, 2560, 1024, 64),
]


@pytest.mark.parametrize("M,N,K,r", SHAPES)
@pytest.mark.parametrize("regime", ["config", "lora_heavy"])
def test_fwd_bwd_parity(lib, M, N, K, r, regime):
    s = 16.0 / r if regime == "config" else 0.75
    case = make_case(M, N, K, r, seed=M * 7 + N + K + r, regime=regime)
    got = run_gpu(lib, *case, s)
    ref = oracle_ref(*case, s)
    for k in ("T", "Y", "dX", "dL1", "dL2"):
        assert_close(got[k], ref[k], f"{k} M={M} N={N} K={K} r={r} {regime}")


# Forward on CTA pairs (256 x 256 output tile per pair of SMs): grids with at
# least one tile per SM and 256-token tiles.  The last pair's odd CTA entirely
# beyond N (4736 = 18.5 x 256), ragged tokens inside the odd CTA's half
# (1000) or the even one's (1800), two LoRA extension blocks (r = 128) and
# fewer k-blocks than dequant groups (K = 192), r = 16 zero-filled to 64.
# The pair path is opt-in (QLORA_NF4_PAIR=1); each case also runs on the
# default single-CTA engine.
PAIR_SHAPES = [(1000, 4736, 256, 64), (1800, 4000, 192, 128), (600, 9000, 128, 16), (2048, 4096, 512, 32)]


@pytest.mark.parametrize("M,N,K,r", PAIR_SHAPES)
@pytest.mark.parametrize("pair", ["1", "0"])
def test_pair_forward_parity(lib, monkeypatch, M, N, K, r, pair):
    monkeypatch.setenv("QLORA_NF4_PAIR", pair)
    s = 0.75
    case = make_case(M, N, K, r, seed=M * 11 + N + K + r, regime="lora_heavy")
    got = run_gpu(lib, *case, s, backward=False)
    ref = oracle_ref(*case, s, backward=False)
    for k in got:
        assert_close(got[k], ref[k], f"{k} M={M} N={N} K={K} r={r} pair={pair}")


# The compared 4-bit formats and the E5M2 and mean-centred scale codecs
# through every kernel that dequantises on chip:
# the forward and dX engines (with a split reduction and without), the
# few-token GEMV path and the opt-in CTA-pair forward.
FORMAT_SHAPES = [(300, 256, 192, 16, "0"), (2048, 4096, 512, 32, "1"), (7, 1000, 704, 32, "0")]


@pytest.mark.parametrize("fmt,scale", [("fp4", "e4m3"), ("int4", "e4m3"), ("nf4", "e5m2"), ("int4", "e5m2"),
                                       ("nf4", "e4m3_mean"), ("fp4", "e4m3_mean")])
@pytest.mark.parametrize("M,N,K,r,pair", FORMAT_SHAPES)
def test_formats_linear_parity(lib, monkeypatch, fmt, scale, M, N, K, r, pair):
    monkeypatch.setenv("QLORA_NF4_PAIR", pair)
    s = 0.75
    case = make_case(M, N, K, r, seed=M * 17 + N + K + r, regime="lora_heavy")
    backward = pair == "0"
    got = run_gpu(lib, *case, s, backward=backward, fmt=fmt, scale=scale)
    ref = oracle_ref(*case, s, backward=backward, fmt=fmt, scale=scale)
    for k in got:
        assert_close(got[k], ref[k], f"{k} {fmt}/{scale} M={M} N={N} K={K} r={r} pair={pair}")


# Few-token forward (M <= 16, the weight-streaming stream-K GEMV path): one
# unit, ragged row tiles, a row tile spread over every CTA, CTAs with three
# segments (K = 64), every T-slice thread layout (r = 48, 80, 128).
GEMV_SHAPES = [
    (1, 8, 64, 16), (7, 1000, 704, 32), (16, 2056, 1536, 48), (2, 128, 22016, 64),
    (3, 40000, 64, 16), (16, 4096, 128, 128), (9, 384, 8192, 80), (12, 22016, 512, 64),
]


@pytest.mark.parametrize("M,N,K,r", GEMV_SHAPES)
@pytest.mark.parametrize("regime", ["config", "lora_heavy"])
def test_gemv_forward_parity(lib, M, N, K, r, regime):
    s = 16.0 / r if regime == "config" else 0.75
    case = make_case(M, N, K, r, seed=M * 13 + N + K + r, regime=regime)
    got = run_gpu(lib, *case, s, backward=(regime == "config"))
    ref = oracle_ref(*case, s, backward=(regime == "config"))
    for k in got:
        assert_close(got[k], ref[k], f"{k} M={M} N={N} K={K} r={r} {regime}")


def test_gemv_forward_is_deterministic(lib):
    X, W, L1, L2, _ = make_case(5, 2056, 2048, 64, seed=21)
    tX, tW, tL1, tL2 = (from_bits(a) for a in (X, W, L1, L2))
    w = lib.quantize(tW)
    Y0, T0 = lib.linear_fwd(tX, w, tL1, tL2, 0.25)
    Y1, T1 = lib.linear_fwd(tX, w, tL1, tL2, 0.25)
    torch.cuda.synchronize()
    assert np.array_equal(bits(Y0), bits(Y1)) and torch.equal(T0, T1)


def test_zero_weight_is_pure_lora(lib):
    """W = 0: Y = s.X.L1.L2 and dX = s.dT.L1^T, so the LoRA extension is
    checked on its own."""
    case = make_case(48, 256, 384, 32, seed=11, regime="lora_heavy", zero_W=True)
    got = run_gpu(lib, *case, 0.5)
    ref = oracle_ref(*case, 0.5)
    assert np.abs(ref["Y"]).max() > 0
    for k in ("Y", "dX", "dL1", "dL2"):
        assert_close(got[k], ref[k], k)


def test_zero_L2_is_base_only(lib):
    case = make_case(40, 192, 256, 16, seed=12, zero_L2=True)
    got = run_gpu(lib, *case, 2.0)
    ref = oracle_ref(*case, 2.0)
    assert_close(got["Y"], ref["Y"], "Y")
    assert_close(got["dX"], ref["dX"], "dX")
    assert np.all(got["dL1"] == 0.0)


def test_backward_optional_outputs(lib):
    X, W, L1, L2, dY = make_case(20, 128, 192, 16, seed=13)
    tX, tW, tL1, tL2, tdY = (from_bits(a) for a in (X, W, L1, L2, dY))
    w = lib.quantize(tW)
    Y, T = lib.linear_fwd(tX, w, tL1, tL2, 1.0)
    ref = oracle_ref(X, W, L1, L2, dY, 1.0)
    dX, dL1, dL2 = lib.linear_bwd(tdY, tX, T, w, tL1, tL2, 1.0, need_dX=False, need_dL2=False)
    assert dX is None and dL2 is None
    assert_close(to_f64(dL1), ref["dL1"], "dL1")
    dX, dL1, dL2 = lib.linear_bwd(tdY, tX, T, w, tL1, tL2, 1.0, need_dL1=False)
    assert_close(to_f64(dX), ref["dX"], "dX")
    assert_close(to_f64(dL2), ref["dL2"], "dL2")


def test_workspace_too_small_is_rejected(lib):
    X, W, L1, L2, dY = make_case(16, 128, 128, 16, seed=14)
    tX, tW, tL1, tL2 = (from_bits(a) for a in (X, W, L1, L2))
    w = lib.quantize(tW)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.QLoRAError):
        lib.linear_fwd(tX, w, tL1, tL2, 1.0, ws=ws)


def test_repeatable(lib):
    """Deterministic: the split reductions sum in a fixed order."""
    case = make_case(16, 512, 2048, 64, seed=15)
    a = run_gpu(lib, *case, 0.25)
    b = run_gpu(lib, *case, 0.25)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_engine_repeatable_long_reduction(lib):
    """The large-M engine, run three times on a long reduction (dX: 172
    64-wide stages per tile through the four A buffers and the eight-stage
    code ring), gives the same bits every time: a stage reused before its
    readers are done would show up as a difference."""
    case = make_case(1024, 11008, 2048, 64, seed=21)
    runs = [run_gpu(lib, *case, 0.25) for _ in range(3)]
    for k in runs[0]:
        for other in runs[1:]:
            assert np.array_equal(runs[0][k], other[k]), k


# ------------------------------------------------------------- full sizes
def _full_linear(q, wl, lin, M=None, sample_rows=64, seed=0):
    t = WL.make_linear(wl, lin, seed=seed, device="cpu", M=M)
    X, W, L1, L2 = (bits(t[k]) for k in ("X", "W", "L1", "L2"))
    dY = bits(t["dY"]) if "dY" in t else None
    backward = dY is not None
    got = run_gpu(q, X, W, L1, L2, dY, wl.s, backward=backward)
    Mtot = X.shape[0]
    rng = np.random.default_rng(seed)
    rows = np.arange(Mtot) if Mtot <= sample_rows else np.sort(rng.choice(Mtot, sample_rows, replace=False))
    N, K = W.shape
    What = O.bf16_bits_to_f64(O.dequant(*O.quantize(W), N, K))
    X64, L164, L264 = (O.bf16_bits_to_f64(a) for a in (X, L1, L2))
    Ys, Ts = O.linear_fwd(X64[rows], What, L164, L264, wl.s)
    assert_close(got["Y"][rows], Ys, f"{wl.name}/{lin.name} Y")
    assert_close(got["T"][rows], Ts, f"{wl.name}/{lin.name} T")
    if backward:
        dY64 = O.bf16_bits_to_f64(dY)
        dL1, dL2, _, T = O.adapter_grads(dY64, X64, L164, L264, wl.s)
        dXs, _, _, _ = O.linear_bwd(dY64[rows], X64[rows], What, L164, L264, wl.s, T[rows])
        assert_close(got["dX"][rows], dXs, f"{wl.name}/{lin.name} dX")
        assert_close(got["dL1"], dL1, f"{wl.name}/{lin.name} dL1")
        assert_close(got["dL2"], dL2, f"{wl.name}/{lin.name} dL2")


def test_full_linear4096_m16(lib):
    wl = WL.WORKLOADS["linear4096_m16"]
    _full_linear(lib, wl, wl.linears[0])


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("which", [0, 1])
def test_full_llama65b_ffn_gemv(lib, M, which):
    wl = WL.WORKLOADS["llama65b_ffn_gemv"]
    _full_linear(lib, wl, wl.linears[which], M=M)


@pytest.mark.parametrize("which", [0, 4, 6])   # q (4096x4096), gate (11008x4096), down (4096x11008)
def test_full_llama7b_block_linear(lib, which):
    wl = WL.WORKLOADS["llama7b_block"]
    _full_linear(lib, wl, wl.linears[which], seed=which)


@pytest.mark.parametrize("which", [0, 4, 6])   # q (8192x8192), gate (22016x8192), down (8192x22016)
def test_full_llama65b_block_linear(lib, which):
    """The LLaMA-65B block at its full size: 8192 tokens, r = 64, alpha = 16,
    W ~ N(0, 0.015), dY ~ N(0, 1e-2), in the launch configuration the bench
    times (64 sampled rows of Y, T and dX against the fp64 oracle; dL1 and dL2
    in full)."""
    wl = WL.WORKLOADS["llama65b_block"]
    _full_linear(lib, wl, wl.linears[which], seed=which)


# Ranks that are multiples of 8 but not of 16 (r = 8, 24): the adapters are
# narrower than one 16-wide MMA step and the TMA zero-fills the rest of the
# 64-wide operand tiles; the few-token path's T slices and finish kernel see
# odd per-warp column counts.  Engine (with and without split reductions),
# few-token GEMV and the opt-in CTA-pair forward.
RANK8_SHAPES = [(37, 136, 256, 8, "0"), (300, 1000, 640, 24, "0"), (1024, 1024, 2048, 8, "0"),
                (5, 2056, 1536, 8, "0"), (16, 4096, 512, 24, "0"), (1000, 4736, 256, 8, "1")]


@pytest.mark.parametrize("M,N,K,r,pair", RANK8_SHAPES)
@pytest.mark.parametrize("regime", ["config", "lora_heavy"])
def test_rank_multiple_of_8(lib, monkeypatch, M, N, K, r, pair, regime):
    monkeypatch.setenv("QLORA_NF4_PAIR", pair)
    s = 16.0 / r if regime == "config" else 0.75
    case = make_case(M, N, K, r, seed=M * 19 + N + K + r, regime=regime)
    backward = pair == "0"
    got = run_gpu(lib, *case, s, backward=backward)
    ref = oracle_ref(*case, s, backward=backward)
    for k in got:
        assert_close(got[k], ref[k], f"{k} M={M} N={N} K={K} r={r} pair={pair} {regime}")
