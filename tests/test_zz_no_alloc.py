"""The forward entry point that allocates nothing (qlora_linear_fwd_noalloc).

It exists for callers that cannot allocate device memory themselves, such as
operators run inside a host framework that owns the device memory pool and
forbids allocation while it executes them, or serving loops that must not
call cudaMalloc after start-up.  Instead of a caller workspace it uses a
static 8 MiB device array inside the library.  Checked here through the C ABI
against the regular forward (with a caller workspace), bit for bit, on two
calls in a row, each right after a call on another problem (the array keeps
the previous call's contents), and for its size limit.  This file sorts last so a run that stops
at the first failure has run everything else before it.
"""

import ctypes

import numpy as np
import pytest
import torch

from gpu_util import assert_close, from_bits, to_f64

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = -10


def _bf(rng, shape, std):
    x = torch.from_numpy(rng.normal(0, std, shape).astype(np.float32))
    return x.to(torch.bfloat16).cuda()


def _noalloc(q, X, w, L1, L2, s, Y, T, status):
    d = w.descriptor()
    M, r = X.shape[0], L1.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return q.lib().qlora_linear_fwd_noalloc(ctypes.c_void_p(X.data_ptr()), M, ctypes.byref(d),
                                            ctypes.c_void_p(L1.data_ptr()), ctypes.c_void_p(L2.data_ptr()), r,
                                            float(s), ctypes.c_void_p(Y.data_ptr()), ctypes.c_void_p(T.data_ptr()),
                                            ctypes.c_void_p(status.data_ptr()), stream)


def _problem(lib, rng, M, N, K, r):
    X, W = _bf(rng, (M, K), 1.0), _bf(rng, (N, K), 0.02)
    L1, L2 = _bf(rng, (K, r), K ** -0.5), _bf(rng, (r, N), 0.05)
    return X, lib.quantize(W), L1, L2, 16.0 / r


@pytest.mark.parametrize("M,N,K,r", [(16, 4096, 4096, 16), (200, 384, 512, 64), (37, 136, 256, 32),
                                     (5, 2056, 1536, 8)])
def test_noalloc_forward_matches_regular_forward(lib, M, N, K, r):
    """Bit for bit the regular forward's result (the same kernels and launch
    plan), on two calls in a row, each after the array was left holding
    another problem's workspace: a different token regime (few-token GEMV
    path against the tcgen05 engine), rank and data."""
    rng = np.random.default_rng(M + N + K + r)
    X, w, L1, L2, s = _problem(lib, rng, M, N, K, r)
    assert lib.workspace_bytes(M, N, K, r) <= 8 << 20
    Y_ref, T_ref = lib.linear_fwd(X, w, L1, L2, s)
    # the other problem: few tokens if this one has many, and the reverse
    pM, pr = (300, 48) if M <= 16 else (9, 128)
    pX, pw, pL1, pL2, ps = _problem(lib, np.random.default_rng(7), pM, 1024, 512, pr)
    pY = torch.empty((pM, 1024), dtype=torch.bfloat16, device="cuda")
    pT = torch.empty((pM, pr), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        assert _noalloc(lib, pX, pw, pL1, pL2, ps, pY, pT, status) == 0
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        T = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(lib, X, w, L1, L2, s, Y, T, status) == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16)), "Y differs from the regular forward"
        assert torch.equal(T.view(torch.int32), T_ref.view(torch.int32)), "T differs from the regular forward"
        assert_close(to_f64(Y), to_f64(Y_ref), "Y")


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    M, N, K, r = 65536, 8, 64, 128          # s.T alone is 16 MiB of workspace
    assert lib.workspace_bytes(M, N, K, r) > 8 << 20
    rng = np.random.default_rng(1)
    X, W = _bf(rng, (M, K), 1.0), _bf(rng, (N, K), 0.02)
    L1, L2 = _bf(rng, (K, r), 0.1), _bf(rng, (r, N), 0.1)
    w = lib.quantize(W)
    Y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    T = torch.zeros((M, r), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _noalloc(lib, X, w, L1, L2, 1.0, Y, T, status) == SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0 and torch.count_nonzero(T).item() == 0
    assert "8 MiB" in lib.status_string(SCRATCH_LIMIT)
