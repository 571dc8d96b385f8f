"""GPU parity of 1/s folded upstream (lansai explainer, "AWQ 的四步链路":
Y = XW = (X/s)(sW)) against the CPU oracle, through the C ABI.

Bit-exact: awq_fold_inverse_scale, and a matmul on folded activations with
s = NULL against the same matmul on X and s, on every tile path.  Within the
matmul tolerance: those results against the oracle's plain definition.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_quantization_quantize_b200 as awq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    awq.lib()          # raises if the extension is missing: no fallback exists


@pytest.mark.parametrize("rows,K", [(1, 4096), (1, 8), (3, 1032), (48, 5120), (1, 28672)])
def test_fold_inverse_scale_bit_exact(rows, K):
    rng = np.random.default_rng(rows * 7 + K)
    a = (rng.standard_normal((rows, K)) * rng.uniform(0.01, 30.0, K)).astype(np.float16)
    s = rng.uniform(0.05, 20.0, K).astype(np.float16)
    st = awq.new_status("cuda")
    at = torch.from_numpy(a).cuda()
    got = awq.fold_inverse_scale(at[0] if rows == 1 else at, torch.from_numpy(s).cuda(), status=st)
    awq.raise_on_status(st, "fold_inverse_scale")
    ref = oracle.fold_inverse_scale(a[0] if rows == 1 else a, s)
    assert np.array_equal(got.cpu().numpy().view(np.uint16), ref.view(np.uint16))


def test_fold_inverse_scale_reports_bad_scales():
    K = 1024
    s = torch.ones(K, dtype=torch.float16, device="cuda")
    s[100] = 0.0
    st = awq.new_status("cuda")
    awq.fold_inverse_scale(torch.ones(K, dtype=torch.float16, device="cuda"), s, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == awq.ERR_NONFINITE


# every tile path and both sides of each routing boundary
@pytest.mark.parametrize("M", [1, 2, 3, 39, 40, 63, 64, 128])
def test_prescaled_activations_match_the_s_path_bit_for_bit(M):
    K, N = 1152, 1032
    L = synth.make_layer(23, M, M=M, K=K, N=N, R=64)
    s = awq.compute_scales(awq.act_stats(L.Xcal.cuda()))
    Q, sc, z = awq.quantize_pack(L.W.cuda(), s)
    X = L.X.cuda()
    Xp = awq.fold_inverse_scale(X, s)
    st = awq.new_status("cuda")
    y_s = awq.w4a16_gemm(X, s, Q, sc, z, status=st)
    y_f = awq.w4a16_gemm(Xp, None, Q, sc, z, status=st)
    awq.raise_on_status(st, "matmul")
    assert torch.equal(y_s, y_f)
    if M == 1:
        assert torch.equal(awq.w4a16_gemv(Xp, None, Q, sc, z), y_s)
    # and against the oracle's definition on the folded activations
    Yref = oracle.matmul(Xp.cpu().numpy(), None, Q.cpu().numpy(), sc.cpu().numpy(), z.cpu().numpy(),
                         precision=64, nthreads=8)
    y = y_f.cpu().numpy().astype(np.float64)
    assert np.abs(y - Yref).max() <= 1e-2 * np.abs(Yref).max()
    assert np.linalg.norm(y - Yref) <= 5e-3 * np.linalg.norm(Yref)


def test_prescaled_symmetric_decode_full_size():
    # both next-row features together on a Mistral-7B-shaped QKV projection
    wl = synth.WORKLOADS[2]
    K, N, _ = wl.shapes[0]
    L = synth.make_layer(2, 0, M=1, K=K, N=N, R=wl.R, device="cuda", shape_id=0)
    s = awq.compute_scales(awq.act_stats(L.Xcal))
    Q, sc, _ = awq.quantize_pack(L.W, s, zero_point=False)
    Xp = awq.fold_inverse_scale(L.X, s)
    assert torch.equal(awq.w4a16_gemv(Xp, None, Q, sc, None), awq.w4a16_gemv(L.X, s, Q, sc, None))
