"""The bounded-wait path of the kernels, run for real on the GPU.

Every wait inside a kernel (ring barriers, the arrival of pushed partial sums)
gives up after a time limit, records AWQ_ERR_DEVICE_TIMEOUT in the status word
and lets the kernel finish without faulting: the copies it had issued still
land before it exits, so the CUDA context stays usable.  Nothing here makes a
wait hang: a test build of the library sets the limit to zero and reads the
timer on every poll, so any wait that does not complete at its first poll runs
out at once (its polls use the non-blocking barrier test, which never
suspends the thread).  The test then checks the status word, and that the regular
library still computes a correct result on the same context afterwards.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_quantization_quantize_b200 as awq
from weight_only_quantization_quantize_b200 import _build

pytestmark = pytest.mark.gpu

TEST_LIB = os.path.join(os.path.dirname(awq.LIB_PATH), "libawq_b200_waittest.so")
P, I64, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t


@pytest.fixture(scope="module")
def waitlib():
    if not os.path.exists(TEST_LIB) or os.path.getmtime(TEST_LIB) < os.path.getmtime(awq.LIB_PATH):
        _build.build(force=True, extra_flags=("-DAWQ_WAIT_LIMIT_NS=0ull", "-DAWQ_WAIT_POLL_MASK=0u",
                                                 "-DAWQ_WAIT_NONBLOCKING_POLL"), out=TEST_LIB)
    L = ctypes.CDLL(TEST_LIB)
    L.awq_w4a16_gemv.argtypes = [P, P, P, P, P, I64, I64, P, P, SZ, P, P]
    L.awq_w4a16_gemv.restype = ctypes.c_int
    return L


def test_gemv_wait_runs_out_and_the_context_survives(waitlib):
    # the 7B down-projection shape: 14 groups per CTA against an 8-deep ring,
    # so ring slots are refilled and waits cannot all find their data ready
    K, N = 14336, 4096
    L = synth.make_layer(17, 0, M=1, K=K, N=N, R=64)
    s = awq.compute_scales(awq.act_stats(L.Xcal.cuda()))
    Q, sc, z = awq.quantize_pack(L.W.cuda(), s)
    X = L.X.cuda()
    ws = torch.zeros(awq.gemm_workspace_size(1, K, N), dtype=torch.uint8, device="cuda")
    Y = torch.zeros(1, N, dtype=torch.float16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    rc = waitlib.awq_w4a16_gemv(X.data_ptr(), s.data_ptr(), Q.data_ptr(), sc.data_ptr(), z.data_ptr(), K, N,
                                Y.data_ptr(), ws.data_ptr(), ws.numel(), st.data_ptr(), stream)
    assert rc == awq.OK
    torch.cuda.synchronize()              # the kernel finished: no hang, no fault
    assert int(st.item()) == awq.ERR_TIMEOUT
    # the same context, the regular library: a correct decode token
    st2 = awq.new_status("cuda")
    Y2 = awq.w4a16_gemv(X, s, Q, sc, z, status=st2)
    awq.raise_on_status(st2, "gemv after a timed-out call")
    sr = s.cpu().numpy()
    Qr, scr, zr = oracle.quantize_pack(L.W.numpy(), sr)
    Yr = oracle.matmul(L.X.numpy(), sr, Qr, scr, zr, precision=64, nthreads=16)
    y = Y2.cpu().numpy().astype(np.float64)
    assert np.abs(y - Yr).max() <= 1e-2 * np.abs(Yr).max()
    assert np.linalg.norm(y - Yr) <= 5e-3 * np.linalg.norm(Yr)


def test_prefill_wait_runs_out_and_the_context_survives(waitlib):
    # the tcgen05 path with the weights in tensor memory: 16 stages of 64 k per
    # tile against a 5-deep load ring, so the producer has to wait for a slot
    M, K, N = 256, 1024, 512
    waitlib.awq_w4a16_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, SZ, P, P]
    waitlib.awq_w4a16_gemm.restype = ctypes.c_int
    L = synth.make_layer(19, 0, M=M, K=K, N=N, R=64)
    s = awq.compute_scales(awq.act_stats(L.Xcal.cuda()))
    Q, sc, z = awq.quantize_pack(L.W.cuda(), s)
    X = L.X.cuda()
    ws = torch.zeros(awq.gemm_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    Y = torch.zeros(M, N, dtype=torch.float16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    rc = waitlib.awq_w4a16_gemm(X.data_ptr(), s.data_ptr(), Q.data_ptr(), sc.data_ptr(), z.data_ptr(), M, K, N,
                                Y.data_ptr(), ws.data_ptr(), ws.numel(), st.data_ptr(), stream)
    assert rc == awq.OK
    torch.cuda.synchronize()              # the kernel finished: no hang, no fault
    assert int(st.item()) == awq.ERR_TIMEOUT
    st2 = awq.new_status("cuda")
    Y2 = awq.w4a16_gemm(X, s, Q, sc, z, status=st2)
    awq.raise_on_status(st2, "prefill matmul after a timed-out call")
    sr = s.cpu().numpy()
    Qr, scr, zr = oracle.quantize_pack(L.W.numpy(), sr)
    Yr = oracle.matmul(L.X.numpy(), sr, Qr, scr, zr, precision=64, nthreads=16)
    y = Y2.cpu().numpy().astype(np.float64)
    assert np.abs(y - Yr).max() <= 1e-2 * np.abs(Yr).max()
    assert np.linalg.norm(y - Yr) <= 5e-3 * np.linalg.norm(Yr)
