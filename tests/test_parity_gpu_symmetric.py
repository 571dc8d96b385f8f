"""GPU parity of the symmetric variant ("Awq Quantization", "Zero-Point
Quantization": zero_point False) against the CPU oracle, through the C ABI.

Bit-exact: packed codes and steps of awq_quantize_pack_symmetric.  Within
max|dY| <= 1e-2 max|Y_ref| and ||dY||_F <= 5e-3 ||Y_ref||_F: the matmul with
zeros = NULL on every tile path (decode GEMV, register-fed small batch,
tcgen05 small batch, tcgen05 prefill).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_quantization_quantize_b200 as awq

pytestmark = pytest.mark.gpu

MAX_REL = 1e-2
FRO_REL = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    awq.lib()          # raises if the extension is missing: no fallback exists


def h(t):
    return t.detach().cpu().numpy()


def assert_y_close(y_gpu, y_ref, what=""):
    y = y_gpu.astype(np.float64)
    err = np.abs(y - y_ref)
    scale = np.abs(y_ref).max()
    assert err.max() <= MAX_REL * scale, f"{what}: max|dY| {err.max():.3e} > {MAX_REL} * {scale:.3e}"
    fro = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert fro <= FRO_REL, f"{what}: relative Frobenius error {fro:.3e}"


def quantize_sym_both(W, s):
    """GPU and oracle symmetric quantize_pack on the same bits; assert bit-exact."""
    st = awq.new_status("cuda")
    Q, sc, z = awq.quantize_pack(W.to("cuda"), s.to("cuda"), status=st, zero_point=False)
    awq.raise_on_status(st, "quantize_pack_symmetric")
    assert z is None
    Qr, scr, zr = oracle.quantize_pack(h(W), h(s), zero_point=False)
    assert zr is None
    assert np.array_equal(Q.cpu().numpy(), Qr), "packed codes differ"
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), scr.view(np.uint16)), "steps differ"
    return (Q, sc), (Qr, scr)


def scales_of(Xcal):
    s = awq.compute_scales(awq.act_stats(Xcal.to("cuda")))
    return s


def matmul_gpu(X, s, Q, sc):
    st = awq.new_status("cuda")
    if X.shape[0] == 1:
        Y = awq.w4a16_gemv(X, s, Q, sc, None, status=st)
    else:
        Y = awq.w4a16_gemm(X, s, Q, sc, None, status=st)
    awq.raise_on_status(st, "matmul (symmetric)")
    return Y


def _hex32(v):
    return np.int64(int(v, 16)).astype(np.uint32).astype(np.int32)


def test_symmetric_hand_worked_group_on_gpu(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "hand_group_symmetric_k128_n8.json")))
    K, N = fx["K"], fx["N"]
    W = np.zeros((K, N), dtype=np.float64)
    for c in range(N):
        spec = fx["W"][f"col{c}"]
        if "other_rows" in spec:
            W[:, c] = spec["other_rows"]
            for r, v in spec["rows"].items():
                W[int(r), c] = v
        else:
            (key, vals), = spec.items()
            W[:, c] = np.array(vals, dtype=np.float64)[np.arange(K) % 16] * 2.0 ** int(key.split("2^")[1])
    Wt = torch.from_numpy(W).half()
    (Q, sc), _ = quantize_sym_both(Wt, torch.ones(K, dtype=torch.float16))
    exp = fx["expected"]
    assert [f"{v:#06x}" for v in sc.cpu().numpy().view(np.uint16)[0]] == [e.lower() for e in exp["scales_bits"]]
    Qh = Q.cpu().numpy()
    assert Qh[0, 0] == _hex32(exp["Q_hex_by_column"]["col0"]["row0"])
    assert Qh[0, 7] == _hex32(exp["Q_hex_by_column"]["col7"]["even_rows"])
    assert Qh[1, 7] == _hex32(exp["Q_hex_by_column"]["col7"]["odd_rows"])


@pytest.mark.parametrize("K,N", [(128, 8), (1024, 1024), (384, 1032), (1152, 520)])
def test_symmetric_quantize_bit_exact_small_and_ragged(K, N):
    L = synth.make_layer(20, K + N, M=1, K=K, N=N, R=64)
    quantize_sym_both(L.W, scales_of(L.Xcal).cpu())


def test_symmetric_quantize_exact_ties():
    # Columns spanning [-0.875, 0.875] in multiples of 1/16 (times a power-of-two
    # channel scale): the step is exactly 1/8 and half of the quotients are exact
    # half-integers, which must round to even.
    rng = np.random.default_rng(9)
    K, N = 512, 1040
    W = rng.integers(-14, 15, size=(K, N)).astype(np.float32) / 16
    W[0::128, :] = -0.875
    s = np.ones(K, dtype=np.float32)
    s[256:384] = 2.0
    s[384:] = 0.5
    W = W / s[:, None]
    assert np.mean(np.abs(W * s[:, None] * 8 - np.round(W * s[:, None] * 8)) == 0.5) > 0.3
    quantize_sym_both(torch.from_numpy(W).half(), torch.from_numpy(s).half())


# every tile path and both sides of each routing boundary
@pytest.mark.parametrize("M", [1, 2, 3, 39, 40, 63, 64, 128])
def test_symmetric_matmul_parity_all_paths(M):
    K, N = 1152, 1032
    L = synth.make_layer(21, M, M=M, K=K, N=N, R=64)
    s = scales_of(L.Xcal)
    (Q, sc), (Qr, scr) = quantize_sym_both(L.W, s.cpu())
    Y = matmul_gpu(L.X.to("cuda"), s, Q, sc).cpu().numpy()
    sr = s.cpu().numpy()
    Yref = oracle.matmul(h(L.X), sr, Qr, scr, None, precision=64, nthreads=8)
    assert_y_close(Y, Yref, f"symmetric M={M}")


@pytest.mark.parametrize("M", [1, 8, 48, 256])
def test_null_zeros_equal_explicit_zero_points_of_eight(M):
    # zeros = NULL must mean exactly a zeros tensor of 0x88888888 words
    K, N = 2048, 1024
    L = synth.make_layer(22, M, M=M, K=K, N=N, R=64)
    s = scales_of(L.Xcal)
    Q, sc, _ = awq.quantize_pack(L.W.to("cuda"), s, zero_point=False)
    word = 0x88888888 - (1 << 32)          # eight nibbles of 8, as an int32
    eights = torch.full((K // 128, N // 8), word, dtype=torch.int32, device="cuda")
    X = L.X.to("cuda")
    a = awq.w4a16_gemm(X, s, Q, sc, None)
    b = awq.w4a16_gemm(X, s, Q, sc, eights)
    assert torch.equal(a, b)


def test_symmetric_full_size_7b_gate_up_decode():
    # Mistral-7B-shaped gate+up projection, M = 1: every code bit-exact, Y on
    # sampled columns against the oracle
    W5 = synth.WORKLOADS[2]
    K, N, _ = W5.shapes[2]
    L = synth.make_layer(2, 0, M=1, K=K, N=N, R=W5.R, device="cuda", shape_id=2)
    s = awq.compute_scales(awq.act_stats(L.Xcal))
    (Q, sc), (Qr, scr) = quantize_sym_both(L.W.cpu(), s.cpu())
    Y = matmul_gpu(L.X, s, Q, sc).cpu().numpy()
    rng = np.random.default_rng(77)
    cols = np.sort(rng.choice(N, size=512, replace=False))
    cols[0], cols[-1] = 0, N - 1
    Yref = oracle.matmul(h(L.X), s.cpu().numpy(), Qr, scr, None, cols=cols, precision=64, nthreads=16)
    assert_y_close(Y[:, cols], Yref, "symmetric 7B gate+up M=1")
