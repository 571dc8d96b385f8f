"""GPU parity: the CUDA library (called through its C ABI) against the CPU oracle.

Bit-exact: activation statistics, scales, packed codes, step sizes, zero
points.  Within the tolerance max|dY| <= 1e-2 max|Y_ref| and
||dY||_F <= 5e-3 ||Y_ref||_F: the fused-dequantization matmul (float
accumulation, X / s rounded to binary16 for the tensor cores).

Inputs are the seeded synthetic workloads (synth) with the shapes of the five
workloads: the small cases run the oracle on every output, the full-size layer
shapes (in the launch configuration the benchmark uses) on sampled columns.
"""
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


def dev(t):
    return t.to("cuda")


def h(t):
    """float16 tensor -> numpy float16 (host)."""
    return t.detach().cpu().numpy()


def assert_y_close(y_gpu, y_ref, what=""):
    y = y_gpu.astype(np.float64)
    err = np.abs(y - y_ref)
    scale = np.abs(y_ref).max()
    assert err.max() <= MAX_REL * scale, f"{what}: max|dY| {err.max():.3e} > {MAX_REL} * {scale:.3e}"
    fro = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert fro <= FRO_REL, f"{what}: relative Frobenius error {fro:.3e}"
    return fro


def quantize_both(W, s):
    """GPU and oracle quantize_pack on the same bits; assert bit-exact."""
    st = awq.new_status("cuda")
    Q, sc, z = awq.quantize_pack(dev(W), dev(s), status=st)
    awq.raise_on_status(st, "quantize_pack")
    Qr, scr, zr = oracle.quantize_pack(h(W), h(s))
    assert np.array_equal(Q.cpu().numpy(), Qr), "packed codes differ"
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), scr.view(np.uint16)), "steps differ"
    assert np.array_equal(z.cpu().numpy(), zr), "zero points differ"
    return (Q, sc, z), (Qr, scr, zr)


def stats_and_scales_both(Xcal):
    st = awq.new_status("cuda")
    m = awq.act_stats(dev(Xcal), status=st)
    s = awq.compute_scales(m, status=st)
    awq.raise_on_status(st, "stats/scales")
    mr = oracle.act_stats(h(Xcal))
    sr = oracle.compute_scales(mr)
    assert np.array_equal(m.cpu().numpy(), mr), "activation statistics differ"
    assert np.array_equal(s.cpu().numpy().view(np.uint16), sr.view(np.uint16)), "scales differ"
    return s, sr


def gemm_gpu(X, s, Q, sc, z):
    st = awq.new_status("cuda")
    if X.shape[0] == 1:
        Y = awq.w4a16_gemv(X, s, Q, sc, z, status=st)
    else:
        Y = awq.w4a16_gemm(X, s, Q, sc, z, status=st)
    awq.raise_on_status(st, "matmul")
    return Y.cpu().numpy()


# ------------------------------------------------------------------ statistics and scales
@pytest.mark.parametrize("R,K", [(128, 1024), (256, 4096), (7, 136), (1, 8), (8192, 64), (3, 28672)])
def test_act_stats_and_scales_bit_exact(R, K):
    L = synth.make_layer(9, R + K, M=1, K=K, N=8, R=R)
    stats_and_scales_both(L.Xcal)


def test_scales_edge_cases():
    # zero channels hit the 1e-8 floor; a single channel gives s = 1
    m = torch.tensor([0.0, 1.0, 4.0, 0.0, 1e-3, 65504.0], dtype=torch.float32)
    s = awq.compute_scales(dev(m)).cpu().numpy()
    assert np.array_equal(s.view(np.uint16), oracle.compute_scales(m.numpy()).view(np.uint16))
    s1 = awq.compute_scales(dev(torch.tensor([3.5], dtype=torch.float32))).cpu().numpy()
    assert s1.view(np.uint16)[0] == 0x3C00


def test_nonfinite_inputs_are_reported_on_device():
    x = torch.randn(16, 256).half()
    x[3, 7] = float("nan")
    st = awq.new_status("cuda")
    awq.act_stats(dev(x), status=st)
    assert int(st.item()) == awq.ERR_NONFINITE
    st = awq.new_status("cuda")
    m = torch.ones(256)
    m[9] = float("inf")
    awq.compute_scales(dev(m), status=st)
    assert int(st.item()) == awq.ERR_NONFINITE
    W = torch.randn(256, 64).half() * 0.02
    W[130, 5] = float("nan")
    st = awq.new_status("cuda")
    awq.quantize_pack(dev(W), dev(torch.ones(256).half()), status=st)
    assert int(st.item()) == awq.ERR_NONFINITE


# ------------------------------------------------------------------ quantize_pack
def test_quantize_hand_worked_group_on_gpu(golden_dir):
    import json
    import os
    from tests.test_oracle_pins import _golden_W, _hex32
    fx = json.load(open(os.path.join(golden_dir, "hand_group_k128_n8.json")))
    W = torch.from_numpy(_golden_W(fx))
    Q, sc, z = awq.quantize_pack(dev(W), dev(torch.ones(128).half()))
    Q = Q.cpu().numpy()
    assert [f"{v:#06x}" for v in sc.cpu().numpy().view(np.uint16)[0]] == \
        [e.lower() for e in fx["expected"]["scales_bits"]]
    assert z.cpu().numpy()[0, 0] == _hex32(fx["expected"]["zeros_word_hex"])
    assert Q[0, 0] == _hex32(fx["expected"]["Q_hex_by_column"]["col0"]["row0"])
    assert Q[1, 4] == _hex32("0xFEDCBA98") and Q[0, 5] == _hex32("0x89ABCDEF")


@pytest.mark.parametrize("K,N", [(128, 8), (1024, 1024), (384, 1032), (1152, 520), (256, 4104)])
def test_quantize_pack_bit_exact_small_and_ragged(K, N):
    L = synth.make_layer(10, K + N, M=1, K=K, N=N, R=64)
    s, _ = stats_and_scales_both(L.Xcal)
    quantize_both(L.W, s.cpu())


def test_quantize_pack_exact_ties_and_clamping():
    # Every group column spans [-1, 0.875] in multiples of 1/16 (times a
    # power-of-two scale), so the step is exactly 1/8 of the scale and half of
    # the quotients w'/step are exact half-integers: the code decision must
    # break those ties to even exactly as the definition does.  One block of
    # groups is shifted positive, so its zero point clamps to 0 and its codes
    # clamp at 15.
    rng = np.random.default_rng(5)
    K, N = 512, 1040
    W = rng.integers(-16, 15, size=(K, N)).astype(np.float32) / 16
    W[0::128, :] = -1.0
    W[1::128, :] = 0.875
    W[128:256, :64] = np.abs(W[128:256, :64]) + 0.5
    s = np.ones(K, dtype=np.float32)
    s[256:384] = 2.0
    s[384:] = 0.5
    Wh = torch.from_numpy(W).half()
    sh = torch.from_numpy(s).half()
    wp = W.astype(np.float64) * s[:, None]
    assert np.mean(np.abs(wp * 8 / s[:, None] - np.round(wp * 8 / s[:, None]) ) == 0.5) > 0.3  # many exact ties
    quantize_both(Wh, sh)


# ------------------------------------------------------------------ matmul (all tile paths)
# every tile path and both sides of each routing boundary: decode GEMV (1, 2),
# register-fed small batch (3 .. 23), tcgen05 small batch (24 .. 63), tcgen05
# prefill (64 ..)
@pytest.mark.parametrize("M", [1, 2, 3, 7, 8, 9, 16, 23, 24, 33, 39, 40, 48, 63, 64, 65, 127, 128, 200, 256, 300, 520])
@pytest.mark.parametrize("K,N", [(1024, 1024), (1152, 1032), (128, 8), (2048, 264)])
def test_matmul_parity_small_shapes(M, K, N):
    L = synth.make_layer(11, M * 7 + K + N, M=M, K=K, N=N, R=64)
    s, sr = stats_and_scales_both(L.Xcal)
    (Q, sc, z), (Qr, scr, zr) = quantize_both(L.W, s.cpu())
    Y = gemm_gpu(dev(L.X), s, Q, sc, z)
    Yref = oracle.matmul(h(L.X), sr, Qr, scr, zr, precision=64, nthreads=8)
    assert_y_close(Y, Yref, f"M={M} K={K} N={N}")
    Y32 = oracle.matmul(h(L.X), sr, Qr, scr, zr, precision=32, nthreads=8)
    assert_y_close(Y, Y32, f"M={M} K={K} N={N} (float oracle)")


@pytest.mark.parametrize("M", [1, 8, 20, 40])
def test_matmul_parity_long_k(M):
    # k ranges longer than the per-CTA staging of steps and zero words (the
    # register-fed small-batch kernel then reads them from global memory)
    K, N = 131072, 64
    L = synth.make_layer(12, K + M, M=M, K=K, N=N, R=16)
    s, sr = stats_and_scales_both(L.Xcal)
    (Q, sc, z), (Qr, scr, zr) = quantize_both(L.W, s.cpu())
    Y = gemm_gpu(dev(L.X), s, Q, sc, z)
    Yref = oracle.matmul(h(L.X), sr, Qr, scr, zr, precision=64, nthreads=8)
    assert_y_close(Y, Yref, f"M={M} K={K} N={N}")


def test_matmul_is_deterministic():
    L = synth.make_layer(12, 0, M=1, K=4096, N=4096, R=64)
    s = awq.compute_scales(awq.act_stats(dev(L.Xcal)))
    Q, sc, z = awq.quantize_pack(dev(L.W), s)
    X = dev(L.X)
    a = awq.w4a16_gemv(X, s, Q, sc, z)
    b = awq.w4a16_gemv(X, s, Q, sc, z)
    assert torch.equal(a, b)
    X2 = dev(synth.activations(48, 4096, 5, L.outliers))
    assert torch.equal(awq.w4a16_gemm(X2, s, Q, sc, z), awq.w4a16_gemm(X2, s, Q, sc, z))


def test_gemv_matches_gemm_at_one_token():
    L = synth.make_layer(13, 0, M=1, K=2048, N=1024, R=64)
    s = awq.compute_scales(awq.act_stats(dev(L.Xcal)))
    Q, sc, z = awq.quantize_pack(dev(L.W), s)
    X = dev(L.X)
    assert torch.equal(awq.w4a16_gemv(X, s, Q, sc, z), awq.w4a16_gemm(X, s, Q, sc, z))


# ------------------------------------------------------------------ full-size workloads
def _full_layer(wid, shape_id, M):
    W = synth.WORKLOADS[wid]
    K, N, _ = W.shapes[shape_id]
    return synth.make_layer(wid, 0, M=M, K=K, N=N, R=W.R, device="cuda", shape_id=shape_id)


def _check_full(wid, shape_id, M, ncols, seed):
    L = _full_layer(wid, shape_id, M)
    s, sr = stats_and_scales_both(L.Xcal.cpu())
    W_host = L.W.cpu()
    (Q, sc, z), (Qr, scr, zr) = quantize_both(W_host, s.cpu())
    Y = gemm_gpu(L.X, s, Q, sc, z)
    rng = np.random.default_rng(seed)
    cols = np.sort(rng.choice(L.N, size=min(ncols, L.N), replace=False))
    cols[0], cols[-1] = 0, L.N - 1
    Yref = oracle.matmul(h(L.X), sr, Qr, scr, zr, cols=cols, precision=64, nthreads=16)
    return assert_y_close(Y[:, cols], Yref, f"workload {wid} shape {shape_id} M={M}")


@pytest.mark.parametrize("shape_id", [0, 1, 2, 3])
def test_full_size_decode_7b_shapes(shape_id):
    # Mistral-7B-shaped decode set, M = 1 (every column checked)
    L = _full_layer(2, shape_id, 1)
    _check_full(2, shape_id, 1, L.N, 100 + shape_id)


def test_full_size_single_layer_1024():
    _check_full(1, 0, 1, 1024, 7)


@pytest.mark.parametrize("shape_id,M", [(0, 8), (1, 16), (2, 32), (3, 48)])
def test_full_size_13b_small_batch(shape_id, M):
    _check_full(3, shape_id, M, 384, 200 + shape_id)


@pytest.mark.parametrize("shape_id,M", [(1, 512), (0, 2048), (3, 4096), (2, 4096)])
def test_full_size_7b_prefill(shape_id, M):
    _check_full(4, shape_id, M, 48, 300 + shape_id)


@pytest.mark.parametrize("shape_id", [0, 1, 2, 3])
def test_full_size_70b_layer(shape_id):
    # every (projection, token count) pair of the 70B-shaped layer: the packed
    # weights bit-exact once per projection, then M = 1, 32, 256 on sampled columns
    wl = synth.WORKLOADS[5]
    K, N, _ = wl.shapes[shape_id]
    L = synth.make_layer(5, 0, M=256, K=K, N=N, R=wl.R, device="cuda", shape_id=shape_id)
    s, sr = stats_and_scales_both(L.Xcal.cpu())
    (Q, sc, z), (Qr, scr, zr) = quantize_both(L.W.cpu(), s.cpu())
    del L.W
    rng = np.random.default_rng(400 + shape_id)
    cols = np.sort(rng.choice(N, size=96, replace=False))
    cols[0], cols[-1] = 0, N - 1
    for M in wl.Ms:
        X = L.X[:M].contiguous()
        Y = gemm_gpu(X, s, Q, sc, z)
        Yref = oracle.matmul(h(X), sr, Qr, scr, zr, cols=cols, precision=64, nthreads=16)
        assert_y_close(Y[:, cols], Yref, f"70B projection {shape_id} M={M}")


# ------------------------------------------------------------------ stream ordering and workspace state
def test_quantize_then_matmul_on_one_stream_without_sync():
    # The matmul fetches its packed weights before it waits on the previous
    # kernel of the stream (programmatic dependent launch).  The quantizer
    # triggers its dependents only when it completes, so a matmul issued right
    # behind it on the same stream, with no synchronization in between, must
    # read the freshly written weights.
    L = synth.make_layer(15, 0, M=1, K=4096, N=6144, R=64)
    sr = oracle.compute_scales(oracle.act_stats(h(L.Xcal)))
    Qr, scr, zr = oracle.quantize_pack(h(L.W), sr)
    Yref = oracle.matmul(h(L.X), sr, Qr, scr, zr, precision=64, nthreads=16)
    Wd, sd, Xd = dev(L.W), dev(torch.from_numpy(sr)), dev(L.X)
    Q = torch.zeros(4096 // 8, 6144, dtype=torch.int32, device="cuda")
    sc = torch.zeros(32, 6144, dtype=torch.float16, device="cuda")
    z = torch.zeros(32, 768, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    for M in (1, 2, 16, 48, 128):
        X = dev(synth.activations(M, 4096, 17 + M, L.outliers))
        Q.zero_()
        awq.quantize_pack(Wd, sd, out=(Q, sc, z))            # no sync after this
        Y = awq.w4a16_gemm(X, sd, Q, sc, z)
        Yr = oracle.matmul(h(X), sr, Qr, scr, zr, precision=64, nthreads=16)
        assert_y_close(Y.cpu().numpy(), Yr, f"M={M} right after quantize_pack")
    Q.zero_()
    awq.quantize_pack(Wd, sd, out=(Q, sc, z))
    assert_y_close(awq.w4a16_gemv(Xd, sd, Q, sc, z).cpu().numpy(), Yref, "gemv right after quantize_pack")


def test_workspace_counters_return_to_zero():
    # The prefill kernel raises flags for split tiles in the first 32 KB of the
    # workspace; every call must leave that block at zero for the next one.
    cases = [(4096, 6144, 1), (14336, 4096, 2), (1152, 1032, 1), (128, 8, 2), (4096, 28672, 1),
             (4096, 6144, 512), (16384, 136, 130), (8192, 264, 100), (1152, 1032, 520)]
    ws = torch.zeros(max(awq.gemm_workspace_size(M, K, N) for K, N, M in cases), dtype=torch.uint8, device="cuda")
    for (K, N, M) in cases:
        L = synth.make_layer(16, K + N, M=M, K=K, N=N, R=64, device="cuda")
        s = awq.compute_scales(awq.act_stats(L.Xcal))
        Q, sc, z = awq.quantize_pack(L.W, s)
        Y1 = awq.w4a16_gemm(L.X, s, Q, sc, z, workspace=ws)
        Y2 = awq.w4a16_gemm(L.X, s, Q, sc, z, workspace=ws)
        torch.cuda.synchronize()
        assert int(ws[:32 * 1024].view(torch.int32).abs().sum().item()) == 0, (K, N, M)
        assert torch.equal(Y1, Y2)


def test_chained_calls_are_bit_identical():
    # Calls chained on one stream overlap under programmatic dependent launch;
    # every repetition of the same product must give the same bits (a race in
    # a kernel's rings or reductions shows up here as a few differing columns).
    cases = [(4096, 28672, 1, 24), (4096, 6144, 1, 8), (14336, 4096, 2, 8), (1152, 1032, 1, 8),
             (4096, 6144, 512, 6), (16384, 136, 130, 6)]
    ws = torch.zeros(max(awq.gemm_workspace_size(M, K, N) for K, N, M, _ in cases), dtype=torch.uint8,
                     device="cuda")
    for (K, N, M, reps) in cases:
        L = synth.make_layer(18, K + N, M=M, K=K, N=N, R=64, device="cuda")
        s = awq.compute_scales(awq.act_stats(L.Xcal))
        Q, sc, z = awq.quantize_pack(L.W, s)
        Ys = [awq.w4a16_gemm(L.X, s, Q, sc, z, workspace=ws) for _ in range(reps)]
        torch.cuda.synchronize()
        for i, Y in enumerate(Ys[1:], 1):
            assert torch.equal(Y, Ys[0]), (K, N, M, i, torch.nonzero(Y != Ys[0])[:4].tolist())


@pytest.mark.parametrize("M,K,N", [(130, 16384, 136), (100, 8192, 264), (64, 4096, 8), (257, 8192, 1032),
                                   (1000, 4096, 1040)])
def test_prefill_split_tiles(M, K, N):
    # Shapes whose one-tile-per-CTA grid would leave most SMs idle run the
    # stream-K prefill kernel: every CTA takes an equal range of the tiles'
    # 64-k stages, so a tile's k range is shared by up to 16 CTAs here (long K,
    # few tiles), with ragged tokens and columns; the CTA holding the tile's
    # first stages adds the others' partial tiles and writes Y.
    L = synth.make_layer(21, M + K + N, M=M, K=K, N=N, R=64)
    s, sr = stats_and_scales_both(L.Xcal)
    (Q, sc, z), (Qr, scr, zr) = quantize_both(L.W, s.cpu())
    Y = gemm_gpu(dev(L.X), s, Q, sc, z)
    Yref = oracle.matmul(h(L.X), sr, Qr, scr, zr, precision=64, nthreads=16)
    assert_y_close(Y, Yref, f"M={M} K={K} N={N}")
