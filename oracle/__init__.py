"""CPU oracle for the AWQ W4A16 linear layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
the oracle never imports the product: the two share nothing but the seeded
input generators in ``synth``.

The arithmetic lives in ``awq_oracle.c`` (plain scalar C, compiled with
``-ffp-contract=off -fno-fast-math``); this module only compiles it on first
use and marshals numpy arrays through ctypes.  Each function states the page
and section it restates; the C file holds the step-by-step readings.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "awq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_awq.so")
# A pre-built oracle library to load instead (used by the tests that check the
# pins catch deliberately broken copies of the oracle).
_LIB_OVERRIDE = os.environ.get("AWQ_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

OK, ERR_NULL, ERR_SHAPE, ERR_NONFINITE = 0, 1, 2, 4
GROUP = 128


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with status {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile awq_oracle.c into liboracle_awq.so next to it (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-pthread", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def configure(lib):
    """Declare the C signatures on a loaded oracle library (marshalling only)."""
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.awq_oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.awq_oracle_half_to_double.restype = ctypes.c_double
    lib.awq_oracle_double_to_half.argtypes = [ctypes.c_double]
    lib.awq_oracle_double_to_half.restype = ctypes.c_uint16
    lib.awq_oracle_act_stats.argtypes = [P, I64, I64, P]
    lib.awq_oracle_compute_scales.argtypes = [P, I64, P]
    lib.awq_oracle_quantize_pack.argtypes = [P, P, I64, I64, P, P, P]
    lib.awq_oracle_quantize_pack_symmetric.argtypes = [P, P, I64, I64, P, P]
    lib.awq_oracle_dequant.argtypes = [P, P, P, I64, I64, P]
    lib.awq_oracle_fold_inverse_scale.argtypes = [P, I64, I64, P, P]
    lib.awq_oracle_scales_alpha.argtypes = [P, I64, I, P]
    lib.awq_oracle_quantize_pack_clip.argtypes = [P, P, P, I64, I64, I64, I, P, P, P, P]
    lib.awq_oracle_scale_search.argtypes = [P, I64, I64, P, I64, P, P, P, I]
    lib.awq_oracle_matmul.argtypes = [P, P, P, P, P, I64, I64, I64, P, I64, P, I, I]
    for f in (lib.awq_oracle_act_stats, lib.awq_oracle_compute_scales,
              lib.awq_oracle_quantize_pack, lib.awq_oracle_quantize_pack_symmetric,
              lib.awq_oracle_dequant, lib.awq_oracle_matmul, lib.awq_oracle_fold_inverse_scale,
              lib.awq_oracle_scales_alpha, lib.awq_oracle_scale_search,
              lib.awq_oracle_quantize_pack_clip):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                _lib = configure(ctypes.CDLL(_LIB_OVERRIDE))
            else:
                build()
                _lib = configure(ctypes.CDLL(_LIB))
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _h(a) -> np.ndarray:
    """binary16 data as a C-contiguous uint16 view (accepts float16 or uint16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16/uint16 bits, got {a.dtype}")
    return a


def _check(code: int, what: str):
    if code != OK:
        raise OracleError(code, what)


def half_to_double(bits: int) -> float:
    """Exact value of one binary16 bit pattern (IEEE 754 binary16 definition)."""
    return _load().awq_oracle_half_to_double(int(bits) & 0xFFFF)


def double_to_half(x: float) -> int:
    """Bit pattern of the binary16 nearest to x, ties to even (one rounding)."""
    return int(_load().awq_oracle_double_to_half(float(x)))


def act_stats(xcal) -> np.ndarray:
    """m[k] = mean_r |xcal[r, k]| (exact double sum, one division, float result).

    Lansai AWQ explainer, "AWQ 的四步链路", row "采集激活": calibration forward,
    per-channel input magnitude.  xcal: binary16 [R, K] -> float32 [K].
    """
    x = _h(xcal)
    R, K = x.shape
    m = np.empty(K, dtype=np.float32)
    _check(_load().awq_oracle_act_stats(_p(x), R, K, _p(m)), "act_stats")
    return m


def compute_scales(m) -> np.ndarray:
    """s = sqrt(max(m, 1e-8)) / sqrt(max t * min t), rounded once to binary16.

    Lansai AWQ explainer, "AWQ 的四步链路" (Y = (X/s)(sW), s > 0 per input
    channel); "Awq Quantization", "How AWQ Works" (objective L(s)).
    m: float32 [K] -> float16 [K].
    """
    m = np.ascontiguousarray(m, dtype=np.float32)
    s = np.empty(m.shape[0], dtype=np.uint16)
    _check(_load().awq_oracle_compute_scales(_p(m), m.shape[0], _p(s)), "compute_scales")
    return s.view(np.float16)


def quantize_pack(W, s, zero_point: bool = True):
    """Fold s into W, 4-bit group-128 quantization, pack.

    "Awq Quantization", "Group Size Configuration" / "Zero-Point
    Quantization"; lansai explainer, four-step chain ("真实量化/打包").
    W: binary16 [K, N] (Y = X W), s: binary16 [K].
    zero_point=True: asymmetric grid with a per-group zero point.
    zero_point=False: symmetric grid (step from the largest magnitude, codes
    stored with an implicit zero point of 8); zeros is then None.
    Returns (Q int32 [K/8, N], scales float16 [K/128, N], zeros int32 [K/128, N/8] or None).
    """
    w = _h(W)
    sv = _h(s)
    K, N = w.shape
    if sv.shape != (K,):
        raise ValueError("s must have shape [K]")
    Q = np.zeros((max(K // 8, 1), N), dtype=np.int32)
    sc = np.zeros((max(K // GROUP, 1), N), dtype=np.uint16)
    if not zero_point:
        _check(_load().awq_oracle_quantize_pack_symmetric(_p(w), _p(sv), K, N, _p(Q), _p(sc)),
               "quantize_pack_symmetric")
        return Q, sc.view(np.float16), None
    z = np.zeros((max(K // GROUP, 1), max(N // 8, 1)), dtype=np.int32)
    _check(_load().awq_oracle_quantize_pack(_p(w), _p(sv), K, N, _p(Q), _p(sc), _p(z)),
           "quantize_pack")
    return Q, sc.view(np.float16), z


def quantize_pack_clip(W, s, xcal, n_cand: int = 11):
    """quantize_pack with a searched clipping ratio per (group, column).

    "Awq Quantization", calibration parameters (apply_clip).  Candidates
    c = 1 - i/20 (i < n_cand); the loss is the group's output error on the
    calibration rows.  Returns (Q, scales, zeros, ratio_index int32 [K/128, N]).
    """
    w = _h(W)
    sv = _h(s)
    x = _h(xcal)
    K, N = w.shape
    R = x.shape[0]
    if sv.shape != (K,) or x.shape[1] != K:
        raise ValueError("s must be [K] and xcal [R, K]")
    G = max(K // GROUP, 1)
    Q = np.zeros((max(K // 8, 1), N), dtype=np.int32)
    sc = np.zeros((G, N), dtype=np.uint16)
    z = np.zeros((G, max(N // 8, 1)), dtype=np.int32)
    ri = np.zeros((G, N), dtype=np.int32)
    _check(_load().awq_oracle_quantize_pack_clip(_p(w), _p(sv), _p(x), R, K, N, int(n_cand), _p(Q),
                                                 _p(sc), _p(z), _p(ri)), "quantize_pack_clip")
    return Q, sc.view(np.float16), z, ri


def scales_alpha(m, j: int) -> np.ndarray:
    """s = normalised m^(j/8), j = 0..8, by the fixed sqrt/product chain (float16 [K]).

    "Awq Quantization", "How AWQ Works" (the search over s); j = 4 is compute_scales.
    """
    m = np.ascontiguousarray(m, dtype=np.float32)
    s = np.empty(m.shape[0], dtype=np.uint16)
    _check(_load().awq_oracle_scales_alpha(_p(m), m.shape[0], int(j), _p(s)), "scales_alpha")
    return s.view(np.float16)


def scale_search(xcal, W, nthreads: int = 1):
    """Grid search of alpha = j/8 minimising L(s) = ||Q(W s)(X/s) - X W||^2 on the calibration rows.

    "Awq Quantization", "How AWQ Works"; lansai four-step chain, row "搜索缩放".
    Returns (j_best, s_best float16 [K], losses float64 [9]).
    """
    x = _h(xcal)
    w = _h(W)
    R, K = x.shape
    if w.shape[0] != K:
        raise ValueError("W must be [K, N]")
    N = w.shape[1]
    losses = np.empty(9, dtype=np.float64)
    s = np.empty(K, dtype=np.uint16)
    jb = ctypes.c_int(-1)
    _check(_load().awq_oracle_scale_search(_p(x), R, K, _p(w), N, _p(losses), _p(s),
                                           ctypes.byref(jb), int(nthreads)), "scale_search")
    return jb.value, s.view(np.float16), losses


def fold_inverse_scale(a, s) -> np.ndarray:
    """out = fp16(a / s) per input channel (1/s folded into the preceding operator).

    Lansai explainer, four-step chain: (X/s)(sW); a is [K] (a normalisation
    weight) or [rows, K] (activations).  Returns float16 of a's shape.
    """
    av = _h(a)
    shape = av.shape
    a2 = av.reshape(1, -1) if av.ndim == 1 else av
    sv = _h(s)
    rows, K = a2.shape
    if sv.shape != (K,):
        raise ValueError("s must have shape [K]")
    out = np.empty((rows, K), dtype=np.uint16)
    _check(_load().awq_oracle_fold_inverse_scale(_p(np.ascontiguousarray(a2)), rows, K, _p(sv), _p(out)),
           "fold_inverse_scale")
    return out.reshape(shape).view(np.float16)


def _zeros_ptr(zeros):
    """(array, pointer) for a zeros tensor; None (symmetric weights) is NULL."""
    if zeros is None:
        return None, None
    z = np.ascontiguousarray(zeros, dtype=np.int32)
    return z, _p(z)


def dequant(Q, scales, zeros) -> np.ndarray:
    """w_hat = (q - z) * scale (the fake-quantized weights), float64 [K, N].

    zeros=None: symmetric weights, z = 8 everywhere."""
    Q = np.ascontiguousarray(Q, dtype=np.int32)
    sc = _h(scales)
    z, zp = _zeros_ptr(zeros)
    K, N = Q.shape[0] * 8, Q.shape[1]
    out = np.empty((K, N), dtype=np.float64)
    _check(_load().awq_oracle_dequant(_p(Q), _p(sc), zp, K, N, _p(out)), "dequant")
    return out


def matmul(X, s, Q, scales, zeros, cols=None, precision: int = 64, nthreads: int = 1) -> np.ndarray:
    """Y = (X / s) . dequant(Q) by the plain definition, for the output columns ``cols``.

    Lansai explainer, four-step chain: Y = (X/s)(sW).  precision=64 computes
    everything in double; precision=32 is the dequantise-then-float-matmul
    (IEEE float division for X/s, float accumulation, k ascending, no FMA).
    zeros=None: symmetric weights (z = 8).  s=None: X already holds X/s.
    X: binary16 [M, K].  Returns float64 [M, len(cols)].
    """
    x = _h(X)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    sv = None if s is None else _h(s)
    Q = np.ascontiguousarray(Q, dtype=np.int32)
    sc = _h(scales)
    z, zp = _zeros_ptr(zeros)
    M, K = x.shape
    N = Q.shape[1]
    if cols is None:
        cols = np.arange(N, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    Y = np.empty((M, cols.shape[0]), dtype=np.float64)
    _check(_load().awq_oracle_matmul(_p(x), None if sv is None else _p(sv), _p(Q), _p(sc), zp, M, K, N, _p(cols),
                                     cols.shape[0], _p(Y), int(precision), int(nthreads)),
           "matmul")
    return Y
