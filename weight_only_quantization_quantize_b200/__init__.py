"""AWQ W4A16 group-quantized linear layer for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libawq_b200.so`` (C ABI in ``include/awq_b200.h``).
This module only marshals arguments: PyTorch provides device memory and the
current CUDA stream; every step of the computation runs in the library's
kernels.  There is no fallback: if the shared library is missing or the device
is not sm_100, the calls raise.

Every tensor argument is checked here (type, dtype, shape, device,
contiguity) before the C ABI is called: the library sees raw device pointers
and cannot tell a mis-shaped tensor from a correct one.

Functions (names follow the C ABI):
  act_stats(xcal)                  -> m float32 [K]
  compute_scales(m)                -> s float16 [K]
  quantize_pack(W, s)              -> (Q int32 [K/8,N], scales float16 [K/128,N], zeros int32 [K/128,N/8])
  quantize_pack(W, s, zero_point=False) -> (Q, scales, None)   symmetric grid, zero point 8
  quantize_pack_clip(W, s, xcal)   -> (Q, scales, zeros, ratio_index): with weight clipping
  fold_inverse_scale(a, s)         -> fp16(a / s), a [K] or [rows,K] (1/s folded upstream)
  w4a16_gemv(X, s, Q, scales, zeros)   X [1,K] -> Y [1,N]   (zeros None: symmetric weights;
                                                             s None: X already holds X/s)
  w4a16_gemm(X, s, Q, scales, zeros)   X [M,K] -> Y [M,N]
  scales_alpha(m, j)               -> s float16 [K] of grid point alpha = j/8
  scale_search(xcal, W)            -> (s_best float16 [K], j_best, losses float64 [9]): the scale
                                      s = m^(j/8) (normalised) whose quantized layer has the
                                      smallest output error on the calibration rows
  QuantLinear(Q, scales, zeros, s)     a quantized layer ("WQLinear"): weights checked once,
                                       layer(X) -> Y with only X and Y checked per call
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
ABI_VERSION = 5

STATUS = {
    0: "AWQ_OK", 1: "AWQ_ERR_NULL", 2: "AWQ_ERR_SHAPE", 3: "AWQ_ERR_ALIGN",
    4: "AWQ_ERR_NONFINITE", 5: "AWQ_ERR_ARCH", 6: "AWQ_ERR_CUDA",
    7: "AWQ_ERR_DEVICE_TIMEOUT", 8: "AWQ_ERR_WORKSPACE",
}
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_NONFINITE, ERR_ARCH, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(9)

# exported symbols, in declaration order of include/awq_b200.h
SYMBOLS = (
    "awq_status_string", "awq_abi_version", "awq_act_stats", "awq_compute_scales",
    "awq_quantize_pack", "awq_quantize_pack_symmetric", "awq_quantize_pack_clip",
    "awq_fold_inverse_scale",
    "awq_w4a16_gemv_workspace_size",
    "awq_w4a16_gemv",
    "awq_w4a16_gemm_workspace_size", "awq_w4a16_gemm",
    "awq_scales_alpha", "awq_scale_search_workspace_size", "awq_scale_search",
    "awq_w4a16_gemm_noalloc",
)
NOALLOC_SCRATCH_BYTES = 24 << 20


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
        L.awq_quantize_pack_clip.argtypes = [P, P, P, I64, I64, I64, ctypes.c_int32, P, P, P, P, P, P]
        L.awq_w4a16_gemv_workspace_size.argtypes = [I64, I64]
        L.awq_w4a16_gemv_workspace_size.restype = SZ
        L.awq_w4a16_gemv.argtypes = [P, P, P, P, P, I64, I64, P, P, SZ, P, P]
        L.awq_w4a16_gemm_workspace_size.argtypes = [I64, I64, I64]
        L.awq_w4a16_gemm_workspace_size.restype = SZ
        L.awq_w4a16_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, SZ, P, P]
        L.awq_w4a16_gemm_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, P]
        L.awq_scales_alpha.argtypes = [P, I64, ctypes.c_int32, P, P, P]
        L.awq_scale_search_workspace_size.argtypes = [I64, I64, I64]
        L.awq_scale_search_workspace_size.restype = SZ
        L.awq_scale_search.argtypes = [P, I64, I64, P, I64, P, P, P, P, SZ, P, P]
        for name in ("awq_act_stats", "awq_compute_scales", "awq_quantize_pack",
                     "awq_quantize_pack_symmetric", "awq_quantize_pack_clip", "awq_fold_inverse_scale",
                     "awq_w4a16_gemv",
                     "awq_w4a16_gemm", "awq_scales_alpha", "awq_scale_search",
                     "awq_w4a16_gemm_noalloc"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().awq_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else t.data_ptr()


def _raw_stream(dev: torch.device) -> int:
    """The current CUDA stream of `dev` as a raw cudaStream_t value."""
    return torch._C._cuda_getCurrentRawStream(dev.index if dev.index is not None
                                              else torch.cuda.current_device())


def _stream(t: torch.Tensor):
    return _raw_stream(t.device)


def _on(dev: torch.device):
    """The device context for a call: a no-op when `dev` is already current."""
    if dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _need(t, dtype, shape, name, device=None):
    """Check a tensor argument: CUDA, dtype, exact shape (None = any extent),
    contiguous, and on `device` when given."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if isinstance(shape, int):
        if t.dim() != shape:
            raise ValueError(f"{name} must have {shape} dims, got {tuple(t.shape)}")
    else:
        if t.dim() != len(shape) or any(e is not None and e != d for e, d in zip(shape, t.shape)):
            want = tuple("*" if e is None else e for e in shape)
            raise ValueError(f"{name} must have shape {want}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


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


def _need_status(status, device):
    if status is not None:
        _need(status, torch.int32, (None,), "status", device)
        if status.numel() < 1:
            raise ValueError("status must hold at least one int32")


def act_stats(xcal: torch.Tensor, status: torch.Tensor | None = None) -> torch.Tensor:
    """m[k] = mean_r |xcal[r,k]| (exact), float32 [K]."""
    _need(xcal, torch.float16, 2, "xcal")
    _need_status(status, xcal.device)
    R, K = xcal.shape
    m = torch.empty(K, dtype=torch.float32, device=xcal.device)
    with torch.cuda.device(xcal.device):
        _check(lib().awq_act_stats(_ptr(xcal), R, K, _ptr(m), _ptr(status), _stream(xcal)),
               "awq_act_stats")
    return m


def compute_scales(m: torch.Tensor, status: torch.Tensor | None = None) -> torch.Tensor:
    """s = sqrt(max(m, 1e-8)) / sqrt(max t * min t), float16 [K]."""
    _need(m, torch.float32, 1, "m")
    _need_status(status, m.device)
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
    K, N = W.shape
    dev = W.device
    _need(s, torch.float16, (K,), "s", dev)
    _need_status(status, dev)
    G = max(K // GROUP_SIZE, 1)
    if out is None:
        Q = torch.empty(K // 8, N, dtype=torch.int32, device=dev)
        sc = torch.empty(G, N, dtype=torch.float16, device=dev)
        z = (torch.empty(G, max(N // 8, 1), dtype=torch.int32, device=dev)
             if zero_point else None)
    else:
        Q, sc, z = out
        _need(Q, torch.int32, (K // 8, N), "Q", dev)
        _need(sc, torch.float16, (G, N), "scales", dev)
        if zero_point:
            _need(z, torch.int32, (G, N // 8), "zeros", dev)
    with torch.cuda.device(dev):
        if zero_point:
            _check(lib().awq_quantize_pack(_ptr(W), _ptr(s), K, N, _ptr(Q), _ptr(sc), _ptr(z),
                                           _ptr(status), _stream(W)), "awq_quantize_pack")
        else:
            _check(lib().awq_quantize_pack_symmetric(_ptr(W), _ptr(s), K, N, _ptr(Q), _ptr(sc),
                                                     _ptr(status), _stream(W)),
                   "awq_quantize_pack_symmetric")
    return Q, sc, z


def quantize_pack_clip(W: torch.Tensor, s: torch.Tensor, xcal: torch.Tensor, n_cand: int = 11,
                       status: torch.Tensor | None = None):
    """Fold s into W and quantize with weight clipping: per group and column the
    range shrink c = 1 - i/20 (i < n_cand) with the smallest output error on
    the calibration rows.  Returns (Q, scales, zeros, ratio_index int32 [K/128, N])."""
    _need(W, torch.float16, 2, "W")
    K, N = W.shape
    dev = W.device
    _need(s, torch.float16, (K,), "s", dev)
    _need(xcal, torch.float16, (None, K), "xcal", dev)
    _need_status(status, dev)
    G = max(K // GROUP_SIZE, 1)
    Q = torch.empty(K // 8, N, dtype=torch.int32, device=dev)
    sc = torch.empty(G, N, dtype=torch.float16, device=dev)
    z = torch.empty(G, max(N // 8, 1), dtype=torch.int32, device=dev)
    ri = torch.empty(G, N, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().awq_quantize_pack_clip(_ptr(W), _ptr(s), _ptr(xcal), xcal.shape[0], K, N, int(n_cand),
                                            _ptr(Q), _ptr(sc), _ptr(z), _ptr(ri), _ptr(status), _stream(W)),
               "awq_quantize_pack_clip")
    return Q, sc, z, ri


def fold_inverse_scale(a: torch.Tensor, s: torch.Tensor, status: torch.Tensor | None = None,
                       out=None) -> torch.Tensor:
    """out = fp16(a / s) per input channel; a is [K] (a norm weight) or [rows, K]."""
    if not isinstance(a, torch.Tensor) or a.dim() not in (1, 2):
        raise ValueError("a must be a [K] or [rows, K] tensor")
    a2 = a.view(1, -1) if a.dim() == 1 else a
    _need(a2, torch.float16, 2, "a")
    rows, K = a2.shape
    _need(s, torch.float16, (K,), "s", a.device)
    _need_status(status, a.device)
    if out is None:
        o = torch.empty_like(a)
    else:
        _need(out, torch.float16, tuple(a.shape), "out", a.device)
        o = out
    with torch.cuda.device(a.device):
        _check(lib().awq_fold_inverse_scale(_ptr(a2), rows, K, _ptr(s), _ptr(o), _ptr(status),
                                            _stream(a)), "awq_fold_inverse_scale")
    return o


def gemm_workspace_size(M: int, K: int, N: int) -> int:
    return int(lib().awq_w4a16_gemm_workspace_size(M, K, N))


# Zero-filled workspaces, one per (device, stream): the matmul keeps arrival
# counters in its workspace that must read zero when a call starts, and every
# call leaves them at zero again.  Calls on one stream are ordered, so they can
# share one workspace; calls on different streams get different ones.
_workspaces: dict = {}


def workspace_for(device: torch.device, nbytes: int) -> torch.Tensor:
    """The zero-filled workspace this binding uses on `device`'s current stream,
    grown (as a new zero-filled buffer) when a call needs more."""
    key = (device.index, _raw_stream(device))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def scales_alpha(m: torch.Tensor, j: int, status: torch.Tensor | None = None) -> torch.Tensor:
    """Scales of grid point alpha = j/8: s = m^(j/8) normalised, float16 [K]."""
    _need(m, torch.float32, 1, "m")
    _need_status(status, m.device)
    if not 0 <= int(j) <= 8:
        raise ValueError("j must be in 0..8")
    s = torch.empty(m.shape[0], dtype=torch.float16, device=m.device)
    with torch.cuda.device(m.device):
        _check(lib().awq_scales_alpha(_ptr(m), m.shape[0], int(j), _ptr(s), _ptr(status), _stream(m)),
               "awq_scales_alpha")
    return s


def scale_search(xcal: torch.Tensor, W: torch.Tensor, status: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None):
    """Search alpha = j/8 (j = 0..8) for s = m^alpha (normalised) minimizing the
    quantized layer's output error on the calibration rows.

    Returns (s_best float16 [K], j_best int32 [1], losses float64 [9]), all on
    the device.  workspace: zero-filled uint8 of at least
    scale_search_workspace_size(R, K, N) bytes (default: a fresh one)."""
    _need(xcal, torch.float16, 2, "xcal")
    R, K = xcal.shape
    dev = xcal.device
    _need(W, torch.float16, (K, None), "W", dev)
    N = W.shape[1]
    _need_status(status, dev)
    need = scale_search_workspace_size(R, K, N)
    if need == 0:
        raise ValueError(f"unsupported shape R={R}, K={K}, N={N}")
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    else:
        _check_workspace(workspace, need, dev)
    losses = torch.empty(9, dtype=torch.float64, device=dev)
    s_best = torch.empty(K, dtype=torch.float16, device=dev)
    j_best = torch.empty(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().awq_scale_search(_ptr(xcal), R, K, _ptr(W), N, _ptr(losses), _ptr(s_best), _ptr(j_best),
                                      _ptr(workspace), workspace.numel(), _ptr(status), _stream(xcal)),
               "awq_scale_search")
    return s_best, j_best, losses


def scale_search_workspace_size(R: int, K: int, N: int) -> int:
    return int(lib().awq_scale_search_workspace_size(R, K, N))


def _check_weights(K, N, s, Q, scales, zeros, dev):
    if K % GROUP_SIZE or K < GROUP_SIZE:
        raise ValueError(f"K = {K} must be a positive multiple of {GROUP_SIZE}")
    if N % 8 or N < 8:
        raise ValueError(f"N = {N} must be a positive multiple of 8")
    G = K // GROUP_SIZE
    if s is not None:
        _need(s, torch.float16, (K,), "s", dev)
    _need(Q, torch.int32, (K // 8, N), "Q", dev)
    _need(scales, torch.float16, (G, N), "scales", dev)
    if zeros is not None:
        _need(zeros, torch.int32, (G, N // 8), "zeros", dev)


def _check_out(out, M, N, dev):
    _need(out, torch.float16, (M, N), "out", dev)


def _check_workspace(ws, need, dev):
    _need(ws, torch.uint8, 1, "workspace", dev)
    if ws.numel() < need:
        raise ValueError(f"workspace holds {ws.numel()} bytes, the call needs {need}")


def w4a16_gemm(X, s, Q, scales, zeros, status=None, out=None, workspace=None) -> torch.Tensor:
    """Y = (X / s) . dequant(Q), float16 [M, N].

    workspace: a uint8 CUDA tensor of at least gemm_workspace_size(M, K, N)
    bytes, zero-filled before its first use (the calls keep it that way); by
    default a cached zero-filled workspace of the current stream is used."""
    _need(X, torch.float16, 2, "X")
    M, K = X.shape
    dev = X.device
    if not isinstance(Q, torch.Tensor) or Q.dim() != 2:
        raise ValueError("Q must be an int32 [K/8, N] tensor")
    N = Q.shape[1]
    _check_weights(K, N, s, Q, scales, zeros, dev)
    _need_status(status, dev)
    if out is None:
        Y = torch.empty(M, N, dtype=torch.float16, device=dev)
    else:
        _check_out(out, M, N, dev)
        Y = out
    with _on(dev):
        wsz = gemm_workspace_size(M, K, N)
        if workspace is None:
            workspace = workspace_for(dev, wsz)
        else:
            _check_workspace(workspace, wsz, dev)
        _check(lib().awq_w4a16_gemm(_ptr(X), _ptr(s), _ptr(Q), _ptr(scales), _ptr(zeros), M, K, N,
                                    _ptr(Y), _ptr(workspace), workspace.numel(), _ptr(status),
                                    _stream(X)),
               "awq_w4a16_gemm")
    return Y


def w4a16_gemv(X, s, Q, scales, zeros, status=None, out=None, workspace=None) -> torch.Tensor:
    """Single-token decode: X [1, K] (or [K]) -> Y [1, N]."""
    if isinstance(X, torch.Tensor) and X.dim() == 1:
        X = X.view(1, -1)
    _need(X, torch.float16, 2, "X")
    if X.shape[0] != 1:
        raise ValueError("w4a16_gemv takes exactly one token; use w4a16_gemm")
    K = X.shape[1]
    dev = X.device
    if not isinstance(Q, torch.Tensor) or Q.dim() != 2:
        raise ValueError("Q must be an int32 [K/8, N] tensor")
    N = Q.shape[1]
    _check_weights(K, N, s, Q, scales, zeros, dev)
    _need_status(status, dev)
    if out is None:
        Y = torch.empty(1, N, dtype=torch.float16, device=dev)
    else:
        _check_out(out, 1, N, dev)
        Y = out
    with _on(dev):
        wsz = int(lib().awq_w4a16_gemv_workspace_size(K, N))
        if workspace is None:
            workspace = workspace_for(dev, wsz)
        else:
            _check_workspace(workspace, wsz, dev)
        _check(lib().awq_w4a16_gemv(_ptr(X), _ptr(s), _ptr(Q), _ptr(scales), _ptr(zeros), K, N,
                                    _ptr(Y), _ptr(workspace), workspace.numel(), _ptr(status),
                                    _stream(X)), "awq_w4a16_gemv")
    return Y


class QuantLinear:
    """A quantized linear layer ("Awq Quantization", "WQLinear Kernel
    Variants": one module whose forward runs the fused-dequantization kernel).

    The weights (Q, scales, zeros, s) are checked once here; a call checks
    only X and the output, and passes prepared pointers to the C ABI."""

    def __init__(self, Q, scales, zeros=None, s=None):
        if not isinstance(Q, torch.Tensor) or Q.dim() != 2:
            raise ValueError("Q must be an int32 [K/8, N] tensor")
        self.K, self.N = Q.shape[0] * 8, Q.shape[1]
        self.device = Q.device
        _check_weights(self.K, self.N, s, Q, scales, zeros, self.device)
        self.Q, self.scales, self.zeros, self.s = Q, scales, zeros, s
        self._wptrs = (_ptr(s), _ptr(Q), _ptr(scales), _ptr(zeros))
        self._dev_index = self.device.index if self.device.index is not None else torch.cuda.current_device()
        self._lib = lib()

    def __call__(self, X, out=None, status=None, workspace=None) -> torch.Tensor:
        if not isinstance(X, torch.Tensor) or X.dtype != torch.float16 or X.dim() != 2 \
                or X.shape[1] != self.K or X.device != self.device or not X.is_contiguous():
            raise ValueError(f"X must be a contiguous float16 [M, {self.K}] tensor on {self.device}")
        M = X.shape[0]
        if out is None:
            out = torch.empty(M, self.N, dtype=torch.float16, device=self.device)
        elif out.dtype != torch.float16 or tuple(out.shape) != (M, self.N) or out.device != self.device \
                or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous float16 [{M}, {self.N}] tensor on {self.device}")
        if status is not None:
            _need_status(status, self.device)
        stream = torch._C._cuda_getCurrentRawStream(self._dev_index)
        wsz = self._lib.awq_w4a16_gemm_workspace_size(M, self.K, self.N)
        if workspace is None:
            workspace = workspace_for(self.device, wsz)
        else:
            _check_workspace(workspace, wsz, self.device)
        s, q, sc, z = self._wptrs
        with _on(self.device):
            _check(self._lib.awq_w4a16_gemm(X.data_ptr(), s, q, sc, z, M, self.K, self.N, out.data_ptr(),
                                            workspace.data_ptr(), workspace.numel(), _ptr(status), stream),
                   "awq_w4a16_gemm")
        return out
