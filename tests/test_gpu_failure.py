"""Failure detection on the GPU without a fault: every internal wait of the
fused dequant-GEMM is bounded, and an expired wait ends the kernel with
QLORA_ERR_TIMEOUT in the caller's status word instead of hanging.

The test makes a wait expire on purpose, with nothing in flight: the
library's hook (qlora_debug_stall_next_gemm) has the next fused launch's
producer issue no loads at all and bounds its waits by a few milliseconds.
Afterwards the same context must still compute correct results."""

import numpy as np
import pytest
import torch

from gpu_util import assert_close, from_bits, to_f64
from test_gpu_linear import make_case, oracle_ref

pytestmark = pytest.mark.gpu

QLORA_ERR_TIMEOUT = -8


@pytest.mark.parametrize("direction", ["fwd", "bwd"])
def test_expired_wait_reports_timeout_and_context_stays_usable(lib, direction):
    M, N, K, r, s = 200, 384, 512, 64, 0.25
    X, W, L1, L2, dY = make_case(M, N, K, r, seed=41)
    tX, tW, tL1, tL2, tdY = (from_bits(a) for a in (X, W, L1, L2, dY))
    lib.read_status()
    w = lib.quantize(tW)
    Y, T = lib.linear_fwd(tX, w, tL1, tL2, s)
    torch.cuda.synchronize()
    assert lib.read_status() == 0
    lib.debug_stall_next_gemm(5_000_000)          # 5 ms
    if direction == "fwd":
        lib.linear_fwd(tX, w, tL1, tL2, s)
    else:
        lib.linear_bwd(tdY, tX, T, w, tL1, tL2, s)
    torch.cuda.synchronize()                       # returns: the kernel ended by itself
    assert lib.read_status() == QLORA_ERR_TIMEOUT
    # the hook is one-shot and the context is intact: the next calls are correct
    Y, T = lib.linear_fwd(tX, w, tL1, tL2, s)
    dX, dL1, dL2 = lib.linear_bwd(tdY, tX, T, w, tL1, tL2, s)
    torch.cuda.synchronize()
    assert lib.read_status() == 0
    ref = oracle_ref(X, W, L1, L2, dY, s)
    for k, v in (("Y", Y), ("T", T), ("dX", dX), ("dL1", dL1), ("dL2", dL2)):
        assert_close(to_f64(v), ref[k], k)


def test_cancelled_stall_request_has_no_effect(lib):
    X, W, L1, L2, _ = make_case(64, 128, 256, 16, seed=42)
    tX, tW, tL1, tL2 = (from_bits(a) for a in (X, W, L1, L2))
    w = lib.quantize(tW)
    lib.read_status()
    lib.debug_stall_next_gemm(5_000_000)
    lib.debug_stall_next_gemm(0)
    Y, T = lib.linear_fwd(tX, w, tL1, tL2, 1.0)
    torch.cuda.synchronize()
    assert lib.read_status() == 0
    ref = oracle_ref(X, W, L1, L2, None, 1.0, backward=False)
    assert_close(to_f64(Y), ref["Y"], "Y")
