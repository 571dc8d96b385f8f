"""Host-side tests of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the device.

Every call here fails validation on the host (null pointer, shape, alignment
or workspace), so no kernel is launched and no GPU is needed.  The fake device
addresses are never dereferenced.
"""
import ctypes
import os
import re
import subprocess

import pytest

import weight_only_quantization_quantize_b200 as awq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq_b200.h")

A = 0x7F0000000000           # a 16-byte aligned fake device address
MIS = A + 2                  # misaligned
P = ctypes.c_void_p


@pytest.fixture(scope="module")
def L():
    from weight_only_quantization_quantize_b200 import _build
    _build.build()
    return awq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(awq_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_functions() == sorted(awq.SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", awq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (awq_\w+)", out))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(L, f)
    # nothing but the ABI is exported with the awq_ prefix
    assert exported == set(declared_functions())


def test_abi_version_and_status_strings(L):
    assert L.awq_abi_version() == 5 == awq.ABI_VERSION
    for code, name in awq.STATUS.items():
        assert awq.status_string(code).startswith(name)
    assert awq.status_string(99) == "AWQ_ERR_UNKNOWN"


def test_workspace_sizes(L):
    # every matmul takes a workspace: 32 KB of counters first, then X / s
    # (2 M K bytes, rounded up to 256), then for M >= 64 the prefill kernel's
    # fp32 partial tiles: one 128-column slot per CTA, its tokens 128 (M <= 128)
    # or 256, as many CTAs as the k stages allow at 16 per CTA, at most 20 MB
    counters = 32 * 1024

    def xp(M, K):
        return (2 * M * K + 255) // 256 * 256

    def partials(M, K, N):
        bt = 128 if M <= 128 else 256
        units = -(-N // 128) * -(-M // bt) * (K // 64)
        ctas = min(max(units // 16, 1), (160 if bt == 256 else 320))
        return ctas * 128 * bt * 4

    g1 = L.awq_w4a16_gemv_workspace_size(4096, 4096)
    assert g1 == L.awq_w4a16_gemm_workspace_size(1, 4096, 4096) == counters + xp(1, 4096)
    assert L.awq_w4a16_gemm_workspace_size(2, 4096, 4096) > g1
    assert L.awq_w4a16_gemm_workspace_size(48, 5120, 5120) == counters + xp(48, 5120)
    for M, K, N in [(64, 1024, 512), (100, 8192, 264), (128, 128, 8), (129, 4096, 4096), (520, 1152, 1032),
                    (4096, 14336, 4096), (4096, 4096, 28672)]:
        assert L.awq_w4a16_gemm_workspace_size(M, K, N) == counters + xp(M, K) + partials(M, K, N), (M, K, N)
    assert partials(64, 1024, 512) == 4 * 128 * 128 * 4                 # one CTA per tile
    assert partials(4096, 14336, 4096) == 20 << 20                      # the cap
    assert L.awq_w4a16_gemm_workspace_size(4, 100, 4096) == 0          # invalid shape
    assert L.awq_w4a16_gemv_workspace_size(4096, 4097) == 0            # invalid shape


def gemm(L, X=A, s=A, Q=A, sc=A, z=A, M=64, K=4096, N=4096, Y=A, ws=A, wsb=1 << 40, st=None):
    return L.awq_w4a16_gemm(P(X), P(s), P(Q), P(sc), P(z), M, K, N, P(Y), P(ws), wsb, P(st), None)


def test_matmul_validation(L):
    assert gemm(L, X=0) == awq.ERR_NULL
    # zeros = NULL is legal (symmetric weights); the other checks still apply
    assert gemm(L, z=0, K=100) == awq.ERR_SHAPE
    assert gemm(L, z=0, Y=0) == awq.ERR_NULL
    assert gemm(L, z=MIS) == awq.ERR_ALIGN
    # s = NULL is legal too (X already holds X/s)
    assert gemm(L, s=0, N=12) == awq.ERR_SHAPE
    assert gemm(L, s=MIS) == awq.ERR_ALIGN
    assert gemm(L, Y=0) == awq.ERR_NULL
    assert gemm(L, K=100) == awq.ERR_SHAPE            # K % 128
    assert gemm(L, K=0) == awq.ERR_SHAPE
    assert gemm(L, N=12) == awq.ERR_SHAPE             # N % 8
    assert gemm(L, M=0) == awq.ERR_SHAPE
    assert gemm(L, M=-3) == awq.ERR_SHAPE
    assert gemm(L, K=1 << 20) == awq.ERR_SHAPE        # above AWQ_MAX_K
    assert gemm(L, X=MIS) == awq.ERR_ALIGN
    assert gemm(L, Q=A + 4) == awq.ERR_ALIGN
    assert gemm(L, st=A + 1) == awq.ERR_ALIGN         # status word alignment
    assert gemm(L, ws=0) == awq.ERR_WORKSPACE
    assert gemm(L, wsb=100) == awq.ERR_WORKSPACE
    r = L.awq_w4a16_gemv(P(A), P(A), P(A), P(A), P(A), 4096, 4097, P(A), None, 0, None, None)
    assert r == awq.ERR_SHAPE
    r = L.awq_w4a16_gemv(P(0), P(A), P(A), P(A), P(A), 4096, 4096, P(A), None, 0, None, None)
    assert r == awq.ERR_NULL


def test_quantize_and_stats_validation(L):
    q = L.awq_quantize_pack
    assert q(P(0), P(A), 128, 8, P(A), P(A), P(A), None, None) == awq.ERR_NULL
    assert q(P(A), P(A), 192, 8, P(A), P(A), P(A), None, None) == awq.ERR_SHAPE
    assert q(P(A), P(A), 128, 4, P(A), P(A), P(A), None, None) == awq.ERR_SHAPE
    assert q(P(A), P(MIS), 128, 8, P(A), P(A), P(A), None, None) == awq.ERR_ALIGN
    assert q(P(A), P(A), 128, 8, P(A), P(A), P(0), None, None) == awq.ERR_NULL   # zeros required
    qs = L.awq_quantize_pack_symmetric
    assert qs(P(0), P(A), 128, 8, P(A), P(A), None, None) == awq.ERR_NULL
    assert qs(P(A), P(A), 128, 8, P(A), P(0), None, None) == awq.ERR_NULL
    assert qs(P(A), P(A), 192, 8, P(A), P(A), None, None) == awq.ERR_SHAPE
    assert qs(P(A), P(A), 128, 12, P(A), P(A), None, None) == awq.ERR_SHAPE
    assert qs(P(A), P(A), 128, 8, P(MIS), P(A), None, None) == awq.ERR_ALIGN
    assert qs(P(A), P(A), 128, 8, P(A), P(A), P(A + 1), None) == awq.ERR_ALIGN
    st = L.awq_act_stats
    assert st(P(A), 0, 1024, P(A), None, None) == awq.ERR_SHAPE       # empty calibration
    assert st(P(A), 8193, 1024, P(A), None, None) == awq.ERR_SHAPE    # exactness limit
    assert st(P(A), 16, 1020, P(A), None, None) == awq.ERR_SHAPE
    assert st(P(0), 16, 1024, P(A), None, None) == awq.ERR_NULL
    assert st(P(A), 16, 1024, P(MIS), None, None) == awq.ERR_ALIGN
    fo = L.awq_fold_inverse_scale
    assert fo(P(0), 1, 4096, P(A), P(A), None, None) == awq.ERR_NULL
    assert fo(P(A), 1, 4096, P(0), P(A), None, None) == awq.ERR_NULL
    assert fo(P(A), 1, 4096, P(A), P(0), None, None) == awq.ERR_NULL
    assert fo(P(A), 0, 4096, P(A), P(A), None, None) == awq.ERR_SHAPE
    assert fo(P(A), 1, 4100, P(A), P(A), None, None) == awq.ERR_SHAPE
    assert fo(P(A), 1, 4096, P(A), P(MIS), None, None) == awq.ERR_ALIGN
    cs = L.awq_compute_scales
    assert cs(P(A), 0, P(A), None, None) == awq.ERR_SHAPE
    assert cs(P(A), 16, P(0), None, None) == awq.ERR_NULL


def test_scale_search_validation(L):
    ss = L.awq_scale_search
    ws = L.awq_scale_search_workspace_size(256, 4096, 4096)
    assert ws > 2 * 4096 * 4096 + 4 * 256 * 4096             # holds W transposed and X W in float
    assert L.awq_scale_search_workspace_size(0, 4096, 4096) == 0     # empty calibration
    assert L.awq_scale_search_workspace_size(9000, 4096, 4096) == 0  # above the exact-sum limit
    assert L.awq_scale_search_workspace_size(256, 100, 4096) == 0

    def call(x=A, R=256, K=4096, w=A, N=4096, lo=A, sb=A, jb=A, wsp=A, wsb=ws, st=None):
        return ss(P(x), R, K, P(w), N, P(lo), P(sb), P(jb), P(wsp), wsb, P(st), None)
    assert call(x=0) == awq.ERR_NULL
    assert call(jb=0) == awq.ERR_NULL
    assert call(R=0) == awq.ERR_SHAPE
    assert call(K=200) == awq.ERR_SHAPE
    assert call(N=20) == awq.ERR_SHAPE
    assert call(sb=MIS) == awq.ERR_ALIGN
    assert call(jb=A + 2) == awq.ERR_ALIGN
    assert call(wsp=0) == awq.ERR_WORKSPACE
    assert call(wsb=ws - 1) == awq.ERR_WORKSPACE
    sa = L.awq_scales_alpha
    assert sa(P(0), 16, 4, P(A), None, None) == awq.ERR_NULL
    assert sa(P(A), 16, 9, P(A), None, None) == awq.ERR_SHAPE
    assert sa(P(A), 16, -1, P(A), None, None) == awq.ERR_SHAPE
    assert sa(P(A), 0, 4, P(A), None, None) == awq.ERR_SHAPE
    assert sa(P(A), 16, 4, P(MIS), None, None) == awq.ERR_ALIGN
