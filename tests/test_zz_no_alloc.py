"""awq_w4a16_gemm_noalloc: the matmul for callers that cannot allocate device memory.

Some callers may not allocate device memory at the moment they run a layer --
an inference-engine plugin that may only touch memory the engine planned in
advance, a fixed-budget or real-time deployment that allocates everything at
start-up, a C caller without a device allocator.  For them the library offers
an entry point that needs no workspace: it stages X / s in a fixed scratch
array inside the library's device image instead.

These tests call it through the C ABI (ctypes, no Python wrapper) and compare
its output with the workspace-taking awq_w4a16_gemm on the same inputs, bit for
bit (both run the same kernels), for several calls in a row (the scratch array
is shared by every call and keeps the previous call's contents).  The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import synth
import weight_only_quantization_quantize_b200 as awq

P = ctypes.c_void_p


def _p(t):
    return P(t.data_ptr())


def test_noalloc_refuses_problems_larger_than_its_scratch():
    # the call's workspace (counters + 2 * M * K bytes of X / s staging) must fit
    # the fixed array; refused before any device work, so this runs without a
    # GPU (the pointers are never used).
    L = awq.lib()
    A = P(0x7F0000000000)
    M, K = 4096, 4096
    assert 2 * M * K > awq.NOALLOC_SCRATCH_BYTES
    assert L.awq_w4a16_gemm_noalloc(A, A, A, A, A, M, K, 4096, A, None, None) == awq.ERR_WORKSPACE
    assert L.awq_w4a16_gemm_noalloc(A, A, A, A, A, 8, 100, 4096, A, None, None) == awq.ERR_SHAPE


def _layer(M, K, N, seed):
    Lr = synth.make_layer(14, seed, M=M, K=K, N=N, R=64, device="cuda")
    s = awq.compute_scales(awq.act_stats(Lr.Xcal))
    Q, sc, z = awq.quantize_pack(Lr.W, s)
    return Lr.X, s, Q, sc, z


@pytest.mark.gpu
def test_noalloc_matches_gemm_on_consecutive_calls():
    assert torch.cuda.is_available()
    L = awq.lib()
    stream = P(torch.cuda.current_stream().cuda_stream)
    # consecutive calls with different problems (decode, small-batch and tcgen05
    # tile paths), then earlier problems again: stale scratch contents must not leak
    cases = [(16, 4096, 4096, 1), (200, 2048, 1032, 2), (1, 4096, 6144, 4), (48, 14336, 1024, 3),
             (2, 14336, 1032, 5), (1, 4096, 6144, 4), (16, 4096, 4096, 1)]
    layers = {}
    for M, K, N, seed in cases:
        if seed not in layers:
            layers[seed] = _layer(M, K, N, seed)
        X, s, Q, sc, z = layers[seed]
        ref = awq.w4a16_gemm(X, s, Q, sc, z)
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = L.awq_w4a16_gemm_noalloc(_p(X), _p(s), _p(Q), _p(sc), _p(z), M, K, N, _p(Y),
                                      _p(st), stream)
        assert rc == awq.OK, awq.status_string(rc)
        torch.cuda.synchronize()
        assert int(st.item()) == awq.OK
        assert torch.isfinite(Y).all()
        # same kernels on the same inputs: the result is the same bits
        assert torch.equal(Y, ref), f"M={M} K={K} N={N}"
