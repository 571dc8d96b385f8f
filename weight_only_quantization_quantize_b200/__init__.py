"""AWQ W4A16 group-quantized linear layer for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libawq_b200.so`` (C ABI in ``include/awq_b200.h``).
This module only marshals arguments: PyTorch provides device memory and the
current CUDA stream; every step of the computation runs in the library's
kernels.  There is no fallback: if the shared library is missing or the device
is not sm_100, the calls raise.

Functions (names follow the C ABI):
  act_stats(xcal)                  -> m float32 [K]
  compute_scales(m)                -> s float16 [K]
  quantize_pack(W, s)              -> (Q int32 [K/8,N], scales float16 [K/128,N], zeros int32 [K/128,N/8])
  quantize_pack(W, s, zero_point=False) -> (Q, scales, None)   symmetric grid, zero point 8
  fold_inverse_scale(a, s)         -> fp16(a / s), a [K] or [rows,K] (1/s folded upstream)
  w4a16_gemv(X, s, Q, scales, zeros)   X [1,K] -> Y [1,N]   (zeros None: symmetric weights;
                                                             s None: X already holds X/s)
  w4a16_gemm(X, s, Q, scales, zeros)   X [M,K] -> Y [M,N]
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libawq_b200.so")

GROUP_SIZE = 128
W_BIT = 4
MAX_CALIB_ROWS = 8192

STATUS = {
    0: "AWQ_OK", 1: "AWQ_ERR_NULL", 2: "AWQ_ERR_SHAPE", 3: "AWQ_ERR_ALIGN",
    4: "AWQ_ERR_NONFINITE", 5: "AWQ_ERR_ARCH", 6: "AWQ_ERR_CUDA",
    7: "AWQ_ERR_DEVICE_TIMEOUT", 8: "AWQ_ERR_WORKSPACE",
}
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_NONFINITE, ERR_ARCH, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(9)

# exported symbols, in declaration order of include/awq_b200.h
SYMBOLS = (
    "awq_status_string", "awq_abi_version", "awq_act_stats", "awq_compute_scales",
    "awq_quantize_pack", "awq_quantize_pack_symmetric", "awq_fold_inverse_scale",
    "awq_w4a16_gemv_workspace_size",
    "awq_w4a16_gemv",
    "awq_w4a16_gemm_workspace_size", "awq_w4a16_gemm", "awq_w4a16_gemm_noalloc",
)
NOALLOC_SCRATCH_BYTES = 4 << 20


class AwqError(RuntimeError):
    def __init__(self, code: int, where: str):
        name = STATUS.get(code, f"status {code}")
        super().__init__(f"{where}: {name}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libawq_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m weight_only_quantization_quantize_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        L.awq_status_string.argtypes = [ctypes.c_int]
        L.awq_status_string.restype = ctypes.c_char_p
        L.awq_abi_version.argtypes = []
        L.awq_abi_version.restype = ctypes.c_int
        L.awq_act_stats.argtypes = [P, I64, I64, P, P, P]
        L.awq_compute_scales.argtypes = [P, I64, P, P, P]
        L.awq_quantize_pack.argtypes = [P, P, I64, I64, P, P, P, P, P]
        L.awq_quantize_pack_symmetric.argtypes = [P, P, I64, I64, P, P, P, P]
        L.awq_fold_inverse_scale.argtypes = [P, I64, I64, P, P, P, P]
        L.awq_w4a16_gemv_workspace_size.argtypes = [I64, I64]
        L.awq_w4a16_gemv_workspace_size.restype = SZ
        L.awq_w4a16_gemv.argtypes = [P, P, P, P, P, I64, I64, P, P, SZ, P, P]
        L.awq_w4a16_gemm_workspace_size.argtypes = [I64, I64, I64]
        L.awq_w4a16_gemm_workspace_size.restype = SZ
        L.awq_w4a16_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, SZ, P, P]
        L.awq_w4a16_gemm_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, P]
        for name in ("awq_act_stats", "awq_compute_scales", "awq_quantize_pack",
                     "awq_quantize_pack_symmetric", "awq_fold_inverse_scale", "awq_w4a16_gemv",
                     "awq_w4a16_gemm",
                     "awq_w4a16_gemm_noalloc"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().awq_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(t: torch.Tensor):
    return torch.cuda.current_stream(t.device).cuda_stream


def _on(dev: torch.device):
    """The device context for a call: a no-op when `dev` is already current."""
    if dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _need(t: torch.Tensor, dtype, ndim, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check(code: int, where: str):
    if code != OK:
        raise AwqError(code, where)


def new_status(device) -> torch.Tensor:
    """A zeroed device status word for the calls' dev_status argument."""
    return torch.zeros(1, dtype=torch.int32, device=device)


def raise_on_status(status: torch.Tensor, where: str = "device"):
    """Synchronize on the status word and raise if a kernel recorded an error."""
    code = int(status.item())
    if code != OK:
        raise AwqError(code, where)


def act_stats(xcal: torch.Tensor, status: torch.Tensor | None = None) -> torch.Tensor:
    """m[k] = mean_r |xcal[r,k]| (exact), float32 [K]."""
    _need(xcal, torch.float16, 2, "xcal")
    R, K = xcal.shape
    m = torch.empty(K, dtype=torch.float32, device=xcal.device)
    with torch.cuda.device(xcal.device):
        _check(lib().awq_act_stats(_ptr(xcal), R, K, _ptr(m), _ptr(status), _stream(xcal)),
               "awq_act_stats")
    return m


def compute_scales(m: torch.Tensor, status: torch.Tensor | None = None) -> torch.Tensor:
    """s = sqrt(max(m, 1e-8)) / sqrt(max t * min t), float16 [K]."""
    _need(m, torch.float32, 1, "m")
    s = torch.empty(m.shape[0], dtype=torch.float16, device=m.device)
    with torch.cuda.device(m.device):
        _check(lib().awq_compute_scales(_ptr(m), m.shape[0], _ptr(s), _ptr(status), _stream(m)),
               "awq_compute_scales")
    return s


def quantize_pack(W: torch.Tensor, s: torch.Tensor, status: torch.Tensor | None = None, out=None,
                  zero_point: bool = True):
    """Fold s into W, 4-bit group-128 quantization, packed int32.

    zero_point=True: asymmetric grid with a per-group zero point (Q, scales, zeros).
    zero_point=False: symmetric grid, zero point 8, no zeros tensor (Q, scales, None).
    """
    _need(W, torch.float16, 2, "W")
    _need(s, torch.float16, 1, "s")
    K, N = W.shape
    dev = W.device
    if out is None:
        Q = torch.empty(K // 8, N, dtype=torch.int32, device=dev)
        sc = torch.empty(max(K // GROUP_SIZE, 1), N, dtype=torch.float16, device=dev)
        z = (torch.empty(max(K // GROUP_SIZE, 1), max(N // 8, 1), dtype=torch.int32, device=dev)
             if zero_point else None)
    else:
        Q, sc, z = out
    with torch.cuda.device(dev):
        if zero_point:
            _check(lib().awq_quantize_pack(_ptr(W), _ptr(s), K, N, _ptr(Q), _ptr(sc), _ptr(z),
                                           _ptr(status), _stream(W)), "awq_quantize_pack")
        else:
            _check(lib().awq_quantize_pack_symmetric(_ptr(W), _ptr(s), K, N, _ptr(Q), _ptr(sc),
                                                     _ptr(status), _stream(W)),
                   "awq_quantize_pack_symmetric")
    return Q, sc, z


def fold_inverse_scale(a: torch.Tensor, s: torch.Tensor, status: torch.Tensor | None = None,
                       out=None) -> torch.Tensor:
    """out = fp16(a / s) per input channel; a is [K] (a norm weight) or [rows, K]."""
    if a.dim() not in (1, 2):
        raise ValueError("a must be [K] or [rows, K]")
    a2 = a.view(1, -1) if a.dim() == 1 else a
    _need(a2, torch.float16, 2, "a")
    _need(s, torch.float16, 1, "s")
    rows, K = a2.shape
    o = torch.empty_like(a) if out is None else out
    with torch.cuda.device(a.device):
        _check(lib().awq_fold_inverse_scale(_ptr(a2), rows, K, _ptr(s), _ptr(o), _ptr(status),
                                            _stream(a)), "awq_fold_inverse_scale")
    return o


def gemm_workspace_size(M: int, K: int, N: int) -> int:
    return int(lib().awq_w4a16_gemm_workspace_size(M, K, N))


def w4a16_gemm(X, s, Q, scales, zeros, status=None, out=None, workspace=None) -> torch.Tensor:
    """Y = (X / s) . dequant(Q), float16 [M, N]."""
    _need(X, torch.float16, 2, "X")
    M, K = X.shape
    N = Q.shape[1]
    dev = X.device
    Y = torch.empty(M, N, dtype=torch.float16, device=dev) if out is None else out
    wsz = gemm_workspace_size(M, K, N)
    if wsz and workspace is None:
        workspace = torch.empty(wsz, dtype=torch.uint8, device=dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _on(dev):
        _check(lib().awq_w4a16_gemm(_ptr(X), _ptr(s), _ptr(Q), _ptr(scales), _ptr(zeros), M, K, N,
                                    _ptr(Y), _ptr(workspace), wbytes, _ptr(status), _stream(X)),
               "awq_w4a16_gemm")
    return Y


def w4a16_gemv(X, s, Q, scales, zeros, status=None, out=None) -> torch.Tensor:
    """Single-token decode: X [1, K] (or [K]) -> Y [1, N]."""
    if X.dim() == 1:
        X = X.view(1, -1)
    _need(X, torch.float16, 2, "X")
    if X.shape[0] != 1:
        raise ValueError("w4a16_gemv takes exactly one token; use w4a16_gemm")
    K = X.shape[1]
    N = Q.shape[1]
    dev = X.device
    Y = torch.empty(1, N, dtype=torch.float16, device=dev) if out is None else out
    with _on(dev):
        _check(lib().awq_w4a16_gemv(_ptr(X), _ptr(s), _ptr(Q), _ptr(scales), _ptr(zeros), K, N,
                                    _ptr(Y), None, 0, _ptr(status), _stream(X)), "awq_w4a16_gemv")
    return Y
