"""QLoRA NF4 quantized linear layer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libqlora_nf4.so`` (declared in
``include/qlora_nf4.h``).  It only marshals arguments: every step of the
computation runs in the library's CUDA kernels.  PyTorch is used for device
memory and the current stream.  There is no CPU fallback: if the library
is missing or the device is not sm_100, calls raise.

    w = quantize(W)                       # NF4 double quantisation (fmt="fp4"/"int4": compared formats)
    What = dequant(w)                     # doubleDequant -> bf16
    Y, T = linear_fwd(X, w, L1, L2, s)    # Y = X.W^T + s.X.L1.L2
    dX, dL1, dL2 = linear_bwd(dY, X, T, w, L1, L2, s)
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "lib", "NF4Weight", "quantize", "quantize_into", "dequant", "workspace_bytes", "linear_fwd", "linear_bwd",
    "codebook", "FORMATS", "SCALES", "status_string", "kernel_launches", "set_gemm_events",
    "debug_stall_next_gemm", "read_status", "storage_bytes", "LIB_PATH", "QLoRAError",
    "adapter_merge", "adamw_step", "PagedBuffer", "paged_empty",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlora_nf4.so")

QLORA_OK = 0
QLORA_ERR_NONFINITE = -7
QLORA_ERR_TIMEOUT = -8

# Code formats (QLORA_FMT_*): NF4, and the two 4-bit formats the method is
# compared with (FP4 = E2M1/6, Int4 = k/7).
FORMATS = {"nf4": 0, "fp4": 1, "int4": 2}
# Codec of the 8-bit block scales c2 (QLORA_SCALE_*): E4M3, E5M2 as the
# compared alternative, or E4M3 of the residuals from each group's mean
# (mean-centred; c1 then holds [c1, mean] per group).
SCALES = {"e4m3": 0, "e5m2": 1, "e4m3_mean": 2}


class QLoRAError(RuntimeError):
    pass


class qlora_nf4_weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("c2", ctypes.c_void_p), ("c1", ctypes.c_void_p),
                ("n_rows", ctypes.c_int64), ("n_cols", ctypes.c_int64),
                ("format", ctypes.c_int32), ("scale_codec", ctypes.c_int32)]


class qlora_adamw_config(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double), ("step", ctypes.c_int64)]


_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "qlora_nf4_storage_bytes": (ctypes.c_int, [_I64, _I64, ctypes.POINTER(ctypes.c_size_t),
                                               ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "qlora_weight_storage_bytes": (ctypes.c_int, [_I64, _I64, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t),
                                                  ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "qlora_nf4_codebook": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float)]),
    "qlora_code_levels": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_float)]),
    "qlora_nf4_quantize": (ctypes.c_int, [_P, _I64, _I64, ctypes.POINTER(qlora_nf4_weight), _P, _P]),
    "qlora_nf4_dequant": (ctypes.c_int, [ctypes.POINTER(qlora_nf4_weight), _P, _P, _P]),
    "qlora_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, ctypes.c_int]),
    "qlora_linear_fwd": (ctypes.c_int, [_P, _I64, ctypes.POINTER(qlora_nf4_weight), _P, _P, ctypes.c_int,
                                        ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "qlora_linear_bwd": (ctypes.c_int, [_P, _P, _I64, _P, ctypes.POINTER(qlora_nf4_weight), _P, _P, ctypes.c_int,
                                        ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_kernel_launches": (ctypes.c_uint64, []),
    "qlora_set_gemm_events": (ctypes.c_int, [_P, _P]),
    "qlora_debug_stall_next_gemm": (ctypes.c_int, [ctypes.c_uint64]),
    "qlora_adapter_merge": (ctypes.c_int, [ctypes.POINTER(qlora_nf4_weight), _P, _P, ctypes.c_int, ctypes.c_float,
                                           _P, _P, _P]),
    "qlora_adamw_step": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, ctypes.c_void_p, _P]),
    "qlora_paged_alloc": (ctypes.c_int, [ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p)]),
    "qlora_paged_free": (ctypes.c_int, [_P]),
    "qlora_paged_prefetch": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.c_int, _P]),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [_P, _I64, ctypes.POINTER(qlora_nf4_weight), _P, _P, ctypes.c_int,
                                                ctypes.c_float, _P, _P, _P, _P]),
}


def lib():
    """The loaded C-ABI library (ctypes handle with typed entry points)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise QLoRAError(f"{LIB_PATH} is missing: build it with `python -m bit_nf4_quantized_15_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def kernel_launches() -> int:
    """Kernels launched through the library so far in this process."""
    return int(lib().qlora_kernel_launches())


def set_gemm_events(ev_start, ev_end):
    """Record two torch.cuda.Event objects around the next call's fused
    dequant-GEMM (diagnostic timing).  Both events must have been recorded
    once already so that they exist."""
    h0 = None if ev_start is None else ctypes.c_void_p(ev_start.cuda_event)
    h1 = None if ev_end is None else ctypes.c_void_p(ev_end.cuda_event)
    _check(lib().qlora_set_gemm_events(h0, h1))


def debug_stall_next_gemm(wait_ns: int):
    """Failure-detection test hook: the next fused dequant-GEMM launch issues
    no loads and bounds its waits by `wait_ns`, so they expire and the device
    status word reads QLORA_ERR_TIMEOUT (see qlora_debug_stall_next_gemm)."""
    _check(lib().qlora_debug_stall_next_gemm(int(wait_ns)))


def status_string(code: int) -> str:
    return lib().qlora_status_string(int(code)).decode()


def _check(rc: int):
    if rc != QLORA_OK:
        raise QLoRAError(f"{status_string(rc)} (code {rc})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


_status_bufs = {}


def _status(device) -> torch.Tensor:
    idx = torch.device(device).index
    if idx is None:
        idx = torch.cuda.current_device()
    buf = _status_bufs.get(idx)
    if buf is None:
        buf = torch.zeros(1, dtype=torch.int32, device=f"cuda:{idx}")
        _status_bufs[idx] = buf
    return buf


def read_status(device="cuda") -> int:
    """Synchronise, return and clear the device status word of `device`
    (QLORA_OK or a QLORA_ERR_* the kernels reported)."""
    buf = _status(device)
    v = int(buf.item())
    buf.zero_()
    return v


def _bf16_cuda(t, name):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise QLoRAError(f"{name} must be a contiguous bf16 CUDA tensor")
    return t


def storage_bytes(N: int, K: int, scale: str = "e4m3"):
    """(codes, c2, c1) bytes of an N x K weight with the given scale codec."""
    if scale not in SCALES:
        raise QLoRAError(f"unknown scale codec {scale!r}")
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().qlora_weight_storage_bytes(N, K, SCALES[scale], ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


@dataclass
class NF4Weight:
    """Quantized weight: codes uint8[N*K/2], c2 uint8[N*K/64] (E4M3), c1 float32[ceil(N*K/16384)]
    (two per group for the mean-centred codec);
    ``fmt`` names the 16 levels the codes index (see FORMATS), ``scale`` the
    8-bit float of c2 (see SCALES)."""
    codes: torch.Tensor
    c2: torch.Tensor
    c1: torch.Tensor
    N: int
    K: int
    fmt: str = "nf4"
    scale: str = "e4m3"

    def descriptor(self) -> qlora_nf4_weight:
        if self.fmt not in FORMATS or self.scale not in SCALES:
            raise QLoRAError(f"unknown format {self.fmt!r} or scale codec {self.scale!r}")
        return qlora_nf4_weight(self.codes.data_ptr(), self.c2.data_ptr(), self.c1.data_ptr(), self.N, self.K,
                                FORMATS[self.fmt], SCALES[self.scale])

    @property
    def device(self):
        return self.codes.device

    @staticmethod
    def empty(N: int, K: int, device="cuda", fmt: str = "nf4", scale: str = "e4m3") -> "NF4Weight":
        nc, n2, n1 = storage_bytes(N, K, scale)
        return NF4Weight(torch.empty(nc, dtype=torch.uint8, device=device),
                         torch.empty(n2, dtype=torch.uint8, device=device),
                         torch.empty(n1 // 4, dtype=torch.float32, device=device), N, K, fmt, scale)


def codebook(fmt: str = "nf4"):
    """The 16 ascending levels the kernels use for a format."""
    if fmt not in FORMATS:
        raise QLoRAError(f"unknown format {fmt!r}")
    arr = (ctypes.c_float * 16)()
    _check(lib().qlora_code_levels(FORMATS[fmt], arr))
    return [float(v) for v in arr]


def quantize_into(W: torch.Tensor, out: NF4Weight, status=None):
    _bf16_cuda(W, "W")
    N, K = W.shape
    d = out.descriptor()
    _check(lib().qlora_nf4_quantize(_ptr(W), N, K, ctypes.byref(d), _ptr(status if status is not None else _status(W.device)),
                                    _stream(W.device)))
    return out


def quantize(W: torch.Tensor, status=None, fmt: str = "nf4", scale: str = "e4m3") -> NF4Weight:
    """NF4 double quantisation of a bf16 CUDA weight [N, K] (K % 64 == 0);
    fmt="fp4" or "int4" quantises to one of the compared formats instead,
    scale="e5m2" stores the block scales as E5M2."""
    _bf16_cuda(W, "W")
    N, K = W.shape
    return quantize_into(W, NF4Weight.empty(N, K, W.device, fmt, scale), status)


def dequant(w: NF4Weight, out: torch.Tensor | None = None, status=None) -> torch.Tensor:
    """doubleDequant(c1, c2, W_NF4) -> bf16 [N, K]."""
    if out is None:
        out = torch.empty((w.N, w.K), dtype=torch.bfloat16, device=w.device)
    d = w.descriptor()
    _check(lib().qlora_nf4_dequant(ctypes.byref(d), _ptr(out), _ptr(status if status is not None else _status(w.device)),
                                   _stream(w.device)))
    return out


def workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    n = lib().qlora_workspace_bytes(M, N, K, r)
    if n == 0:
        raise QLoRAError("invalid shape or rank for qlora_workspace_bytes")
    return n


def _workspace(ws, M, N, K, r, device):
    need = workspace_bytes(M, N, K, r)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws


def linear_fwd(X, w: NF4Weight, L1, L2, s: float, ws=None, Y=None, T=None, status=None):
    """Y = X.W^T + s.(X.L1).L2 and T = X.L1 (fp32, for the backward)."""
    _bf16_cuda(X, "X"), _bf16_cuda(L1, "L1"), _bf16_cuda(L2, "L2")
    M, K = X.shape
    r = L1.shape[1]
    dev = X.device
    Y = torch.empty((M, w.N), dtype=torch.bfloat16, device=dev) if Y is None else Y
    T = torch.empty((M, r), dtype=torch.float32, device=dev) if T is None else T
    ws = _workspace(ws, M, w.N, w.K, r, dev)
    d = w.descriptor()
    _check(lib().qlora_linear_fwd(_ptr(X), M, ctypes.byref(d), _ptr(L1), _ptr(L2), r, float(s), _ptr(Y), _ptr(T),
                                  _ptr(ws), ws.numel(), _ptr(status if status is not None else _status(dev)),
                                  _stream(dev)))
    return Y, T


def linear_bwd(dY, X, T, w: NF4Weight, L1, L2, s: float, ws=None, need_dX=True, need_dL1=True, need_dL2=True,
               status=None, dX=None, dL1=None, dL2=None):
    """dX = dY.W^ + s.dT.L1^T, dL1 = s.X^T.dT, dL2 = s.T^T.dY (dT = dY.L2^T)."""
    _bf16_cuda(dY, "dY"), _bf16_cuda(X, "X")
    M, K = X.shape
    r = L1.shape[1]
    dev = X.device
    if dX is None and need_dX:
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    if dL1 is None and need_dL1:
        dL1 = torch.empty((K, r), dtype=torch.float32, device=dev)
    if dL2 is None and need_dL2:
        dL2 = torch.empty((r, w.N), dtype=torch.float32, device=dev)
    ws = _workspace(ws, M, w.N, w.K, r, dev)
    d = w.descriptor()
    _check(lib().qlora_linear_bwd(_ptr(dY), _ptr(X), M, _ptr(T), ctypes.byref(d), _ptr(L1), _ptr(L2), r, float(s),
                                  _ptr(dX), _ptr(dL1), _ptr(dL2), _ptr(ws), ws.numel(),
                                  _ptr(status if status is not None else _status(dev)), _stream(dev)))
    return dX, dL1, dL2


def adapter_merge(w: NF4Weight, L1, L2, s: float, out=None, status=None) -> torch.Tensor:
    """W_merged = RNbf16(W^ + s (L1 L2)^T) as a bf16 [N, K] tensor (the adapter
    folded into the dequantised weight; quantize() it again for a 4-bit copy)."""
    _bf16_cuda(L1, "L1"), _bf16_cuda(L2, "L2")
    r = L1.shape[1]
    dev = w.device
    if out is None:
        out = torch.empty((w.N, w.K), dtype=torch.bfloat16, device=dev)
    d = w.descriptor()
    _check(lib().qlora_adapter_merge(ctypes.byref(d), _ptr(L1), _ptr(L2), r, float(s), _ptr(out),
                                     _ptr(status if status is not None else _status(dev)), _stream(dev)))
    return out


def adamw_step(p, g, m, v, step: int, lr: float, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
               p_bf16=None):
    """One AdamW step in place on fp32 p, m, v (device or paged memory) for
    the gradient g; writes RNbf16(p) into p_bf16 when given."""
    for t, name in ((p, "p"), (g, "g"), (m, "m"), (v, "v")):
        if t.dtype != torch.float32 or not t.is_contiguous() or t.numel() != p.numel():
            raise QLoRAError(f"{name} must be a contiguous float32 tensor of p's size")
    if p_bf16 is not None and (p_bf16.dtype != torch.bfloat16 or p_bf16.numel() != p.numel()):
        raise QLoRAError("p_bf16 must be a bf16 tensor of p's size")
    cfg = qlora_adamw_config(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay), int(step))
    _check(lib().qlora_adamw_step(_ptr(p), _ptr(p_bf16), _ptr(g), _ptr(m), _ptr(v), p.numel(),
                                  ctypes.cast(ctypes.byref(cfg), ctypes.c_void_p), _stream(p.device)))


class PagedBuffer:
    """fp32 optimizer state in paged (CUDA managed) memory from
    qlora_paged_alloc; ``tensor`` views it as a CUDA tensor without a copy.
    ``prefetch(device)`` moves it ahead of use (-1: host memory)."""

    def __init__(self, n: int, device="cuda"):
        self.n = int(n)
        self.device = torch.device(device)
        ptr = ctypes.c_void_p()
        _check(lib().qlora_paged_alloc(max(self.n, 1) * 4, ctypes.byref(ptr)))
        self.ptr = ptr.value
        self.__cuda_array_interface__ = {"shape": (self.n,), "typestr": "<f4", "data": (self.ptr, False),
                                         "version": 3, "strides": None}
        self.tensor = torch.as_tensor(self, device=self.device)

    def prefetch(self, device: int, stream=None):
        st = ctypes.c_void_p(torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream)
        _check(lib().qlora_paged_prefetch(ctypes.c_void_p(self.ptr), self.n * 4, int(device), st))

    def __del__(self):
        try:
            if getattr(self, "ptr", None) and _lib is not None:
                _lib.qlora_paged_free(ctypes.c_void_p(self.ptr))
                self.ptr = None
        except Exception:
            pass


def paged_empty(n: int, device="cuda") -> "PagedBuffer":
    """A zeroed fp32 paged buffer of n elements (optimizer state: m or v)."""
    b = PagedBuffer(n, device)
    b.tensor.zero_()
    return b
