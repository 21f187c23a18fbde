"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every symbol the header declares, derives the same NF4 codebook as the
oracle on its own, and rejects bad arguments before touching a device."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_15_b200 as q
    from bit_nf4_quantized_15_b200 import build
    build.build()
    return q


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(qlora_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    syms = declared_symbols()
    for name in ("qlora_nf4_quantize", "qlora_nf4_dequant", "qlora_linear_fwd", "qlora_linear_bwd"):
        assert name in syms


def test_library_exports_every_declared_symbol(q):
    h = ctypes.CDLL(q.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(h, name), name


def test_codebook_matches_oracle_bitwise(q):
    ours = np.array(q.codebook(), dtype=np.float32)
    ref = O.nf4_codebook()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_storage_bytes(q):
    nc, n2, n1 = q.storage_bytes(4096, 4096)
    assert (nc, n2, n1) == (4096 * 4096 // 2, 4096 * 4096 // 64, 4 * (4096 * 4096 // 16384))
    assert (nc + n2 + n1) * 8 / (4096 * 4096) == O.bits_per_weight(4096, 4096)
    assert (nc + n2 + n1) == O.storage_bytes(4096, 4096)
    nc, n2, n1 = q.storage_bytes(5, 64 * 300)            # partial last c1 group
    assert n1 == 4 * 6
    with pytest.raises(q.QLoRAError):
        q.storage_bytes(4, 100)


def test_status_strings(q):
    for code in range(-11, 1):
        assert q.status_string(code)
    assert "unknown" in q.status_string(-99)


def test_workspace_bytes_host(q):
    L = q.lib()
    assert L.qlora_workspace_bytes(16, 4096, 4096, 16) > 0
    assert L.qlora_workspace_bytes(16, 4096, 4096, 17) == 0      # bad rank
    assert L.qlora_workspace_bytes(16, 4096, 4096, 8) > 0        # r % 8 == 0 in [8, 128]
    assert L.qlora_workspace_bytes(1000, 4096, 4096, 24) > 0
    for bad in (0, 4, 12, 136, 256):
        assert L.qlora_workspace_bytes(16, 4096, 4096, bad) == 0
    assert L.qlora_workspace_bytes(16, 4096, 100, 16) == 0       # K % 64
    assert L.qlora_workspace_bytes(16, 4100, 4096, 16) == 0      # N % 8


def test_argument_checks_before_any_launch(q):
    """Bad arguments are rejected on the host: these fake, never dereferenced
    pointers would fault if any kernel were launched."""
    L = q.lib()
    P = ctypes.c_void_p
    w = q.qlora_nf4_weight(0x1000, 0x2000, 0x3000, 64, 128)
    fake = P(0x10000)
    # NULL input
    assert L.qlora_linear_fwd(None, 4, ctypes.byref(w), fake, fake, 16, 1.0, fake, fake, fake, 1 << 20, None, None) == -1
    # rank
    assert L.qlora_linear_fwd(fake, 4, ctypes.byref(w), fake, fake, 17, 1.0, fake, fake, fake, 1 << 20, None, None) == -4
    # shape: K % 64
    w_bad = q.qlora_nf4_weight(0x1000, 0x2000, 0x3000, 64, 100)
    assert L.qlora_linear_fwd(fake, 4, ctypes.byref(w_bad), fake, fake, 16, 1.0, fake, fake, fake, 1 << 20, None, None) == -3
    # alignment
    assert L.qlora_linear_fwd(P(0x10008), 4, ctypes.byref(w), fake, fake, 16, 1.0, fake, fake, fake, 1 << 20, None, None) == -2
    assert L.qlora_linear_bwd(fake, fake, 4, fake, ctypes.byref(w), fake, fake, 16, 1.0, P(0x10004), None, None,
                              fake, 1 << 20, None, None) == -2
    # quantize
    assert L.qlora_nf4_quantize(fake, 64, 100, ctypes.byref(w), None, None) == -3
    assert L.qlora_nf4_quantize(None, 64, 128, ctypes.byref(w), None, None) == -1
    assert L.qlora_nf4_dequant(ctypes.byref(w_bad), fake, None, None) == -3


def test_compared_format_levels_match_oracle_bitwise(q):
    """FP4 (E2M1 / 6) and Int4 (k / 7) levels: the library's own host
    derivation against the oracle's, bit for bit."""
    for fmt in ("fp4", "int4"):
        ours = np.array(q.codebook(fmt), dtype=np.float32)
        ref = O.codebook(fmt)
        assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32)), fmt
    assert np.array_equal(np.array(q.codebook("nf4"), np.float32).view(np.uint32), O.nf4_codebook().view(np.uint32))


def test_format_checks_before_any_launch(q):
    """An unknown format or scale codec is rejected on the host
    (the fake pointers would fault if a kernel were launched)."""
    L = q.lib()
    P = ctypes.c_void_p
    fake = P(0x10000)
    arr = (ctypes.c_float * 16)()
    assert L.qlora_code_levels(3, arr) == -11 and L.qlora_code_levels(-1, arr) == -11
    for fmt, res in ((3, 0), (0, 3), (0, -1)):
        w = q.qlora_nf4_weight(0x1000, 0x2000, 0x3000, 64, 128, fmt, res)
        assert L.qlora_nf4_quantize(fake, 64, 128, ctypes.byref(w), None, None) == -11
        assert L.qlora_nf4_dequant(ctypes.byref(w), fake, None, None) == -11
        assert L.qlora_linear_fwd(fake, 4, ctypes.byref(w), fake, fake, 16, 1.0, fake, fake, fake, 1 << 20,
                                  None, None) == -11
        assert L.qlora_linear_bwd(fake, fake, 4, fake, ctypes.byref(w), fake, fake, 16, 1.0, fake, None, None,
                                  fake, 1 << 20, None, None) == -11
    assert "format" in q.status_string(-11)


def test_adapter_entry_points_check_arguments_before_any_launch(q):
    """Merge and AdamW reject bad arguments on the host (fake pointers that
    would fault if a kernel ran); the paged helpers reject NULL."""
    L = q.lib()
    P = ctypes.c_void_p
    fake = P(0x10000)
    w = q.qlora_nf4_weight(0x1000, 0x2000, 0x3000, 64, 128)
    assert L.qlora_adapter_merge(ctypes.byref(w), None, fake, 16, 1.0, fake, None, None) == -1
    assert L.qlora_adapter_merge(ctypes.byref(w), fake, fake, 12, 1.0, fake, None, None) == -4
    assert L.qlora_adapter_merge(ctypes.byref(w), fake, fake, 16, 1.0, P(0x10002), None, None) == -2
    w_bad = q.qlora_nf4_weight(0x1000, 0x2000, 0x3000, 64, 96)
    assert L.qlora_adapter_merge(ctypes.byref(w_bad), fake, fake, 16, 1.0, fake, None, None) == -3
    cfg = q.qlora_adamw_config(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    pc = ctypes.cast(ctypes.byref(cfg), ctypes.c_void_p)
    assert L.qlora_adamw_step(fake, None, fake, fake, P(0x10004), 100, pc, None) == -2
    assert L.qlora_adamw_step(fake, P(0x20002), fake, fake, fake, 100, pc, None) == -2
    assert L.qlora_adamw_step(fake, None, None, fake, fake, 100, pc, None) == -1
    cfg0 = q.qlora_adamw_config(1e-3, 0.9, 0.999, 1e-8, 0.0, 0)
    assert L.qlora_adamw_step(fake, None, fake, fake, fake, 100, ctypes.cast(ctypes.byref(cfg0), ctypes.c_void_p),
                              None) == -3
    assert L.qlora_adamw_step(fake, None, fake, fake, fake, 0, pc, None) == 0      # nothing to do
    assert L.qlora_paged_alloc(16, None) == -1 and L.qlora_paged_prefetch(None, 16, 0, None) == -1
    assert L.qlora_paged_free(None) == 0


def test_storage_bytes_per_scale_codec(q):
    """The mean-centred codec stores [c1, mean] per group of 256 blocks."""
    assert q.storage_bytes(4096, 4096, "e4m3") == (4096 * 4096 // 2, 4096 * 4096 // 64, 4096 * 4096 // 16384 * 4)
    assert q.storage_bytes(4096, 4096, "e5m2") == q.storage_bytes(4096, 4096)
    assert q.storage_bytes(4096, 4096, "e4m3_mean")[2] == 2 * q.storage_bytes(4096, 4096)[2]
    assert q.storage_bytes(3, 128, "e4m3_mean")[2] == 8                      # one partial group
    L = q.lib()
    a = ctypes.c_size_t()
    assert L.qlora_weight_storage_bytes(64, 128, 3, ctypes.byref(a), None, None) == -11
    P = ctypes.c_void_p
    w = q.qlora_nf4_weight(0x1000, 0x2000, 0x3004, 64, 128, 0, 2)          # [c1, mean] pairs need 8 bytes
    assert L.qlora_nf4_dequant(ctypes.byref(w), P(0x10000), None, None) == -2
