"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these compares the oracle with itself.  The pins are
  * the IEEE binary16 codec against numpy's float16 (a library routine that
    the oracle does not use);
  * closed forms for the statistics and the scales;
  * a hand-worked group fixture (tests/golden) for quantization and packing;
  * a textbook min-max round-to-nearest quantizer written independently here
    in vectorised numpy, for s = 1 (the RTN special case the lansai explainer
    lists as the plain baseline in its method comparison table);
  * per-group round-trip bounds, equivariances, and exact reconstruction when
    the weights already sit on a 4-bit grid (the pipeline is then lossless and
    Y must equal X W, the pages' equivalence Y = XW = (X/s)(sW));
  * the expected direction of the objective in "How AWQ Works".
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# --------------------------------------------------------------------------
# binary16 codec
# --------------------------------------------------------------------------
def test_half_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zero keeps its sign
    assert math.copysign(1.0, oracle.half_to_double(0x8000)) == -1.0


def _half_grid_points():
    """Finite halves, the midpoints between neighbours (ties) and points just off them."""
    h = np.arange(0, 0x7BFF, dtype=np.uint16)            # +0 .. next-to-max finite
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2.0                                  # exact in double
    pts = np.concatenate([lo, mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)])
    return np.concatenate([pts, -pts])


def test_half_encode_matches_numpy_rne():
    rng = np.random.default_rng(7)
    rand = np.concatenate([
        rng.standard_normal(4000),
        np.exp(rng.uniform(np.log(1e-9), np.log(7e4), 4000)) * rng.choice([-1, 1], 4000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -25,
                  2.0 ** -25 * 1.0000001, 2.0 ** -24, 3 * 2.0 ** -25, 2.0 ** -14,
                  2.0 ** -14 - 2.0 ** -25]),
    ])
    pts = np.concatenate([rand, _half_grid_points()[::7]])
    ref = pts.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(float(x)) for x in pts], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"first mismatch at {pts[bad[0]]!r}: {got[bad[0]]:#06x} vs {ref[bad[0]]:#06x}"
    assert oracle.double_to_half(float("inf")) == 0x7C00
    assert oracle.double_to_half(float("-inf")) == 0xFC00
    assert (oracle.double_to_half(float("nan")) & 0x7C00) == 0x7C00


# --------------------------------------------------------------------------
# act_stats: closed forms and exactness invariants
# --------------------------------------------------------------------------
def test_act_stats_hand_example():
    x = np.array([[1.0, -2.0, 0.0], [3.0, 0.5, -0.0]], dtype=np.float16)
    assert oracle.act_stats(x).tolist() == [2.0, 1.25, 0.0]


def test_act_stats_constant_rows_and_two_levels():
    R, K = 64, 256
    x = np.full((R, K), -1.5, dtype=np.float16)
    assert np.all(oracle.act_stats(x) == 1.5)
    x = np.empty((R, K), dtype=np.float16)
    x[:, ::2] = 4.0
    x[:, 1::2] = 1.0
    x[::2, 1::2] *= -1
    m = oracle.act_stats(x)
    assert np.all(m[::2] == 4.0) and np.all(m[1::2] == 1.0)


def test_act_stats_exact_sum_is_order_free_and_scales_exactly():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((300, 512)) * rng.choice([1, 20], 512)).astype(np.float16)
    m = oracle.act_stats(x)
    perm = rng.permutation(300)
    assert np.array_equal(m, oracle.act_stats(x[perm]))          # exact => order free
    assert np.array_equal(2 * m, oracle.act_stats(x * np.float16(2)))
    # the value is the double-precision mean rounded once to float
    exact = np.abs(x.astype(np.float64)).sum(axis=0)              # exact: multiples of 2^-24
    assert np.array_equal(m, (exact / 300).astype(np.float32))


def test_act_stats_rejects_empty_calibration():
    # "Calibration samples are empty" (Awq Quantization, Troubleshooting Guide)
    with pytest.raises(oracle.OracleError) as e:
        oracle.act_stats(np.zeros((0, 128), dtype=np.float16))
    assert e.value.code == oracle.ERR_SHAPE


# --------------------------------------------------------------------------
# compute_scales: closed forms
# --------------------------------------------------------------------------
def test_scales_constant_statistics_give_unit_scale():
    for c in (1.0, 0.37, 123.0):
        s = oracle.compute_scales(np.full(384, c, dtype=np.float32))
        assert np.all(s.view(np.uint16) == 0x3C00)


def test_scales_two_levels_hand_values():
    # t in {2, 1}, centre sqrt(2*1) = sqrt2, s in {sqrt2, 1/sqrt2} rounded to half:
    # sqrt2 = 1448.15 * 2^-10 -> 0x3DA8 (1.4140625); 1/sqrt2 = 1448.15 * 2^-11 -> 0x39A8
    m = np.array([4.0, 1.0] * 64, dtype=np.float32)
    s = oracle.compute_scales(m).view(np.uint16)
    assert np.all(s[::2] == 0x3DA8) and np.all(s[1::2] == 0x39A8)


def test_scales_floor_and_invariances():
    rng = np.random.default_rng(11)
    m = rng.uniform(0.5, 20.0, 1024).astype(np.float32)
    m[5] = 0.0                                                    # floored at 1e-8
    s = oracle.compute_scales(m)
    sf = s.astype(np.float64)
    assert np.all(sf > 0)
    # scaling m by 4 scales t and the centre by exactly 2: s unchanged, bit for bit
    # (on channels above the floor, which does not scale)
    mp = np.delete(m, 5)
    sp = oracle.compute_scales(mp)
    assert np.array_equal(sp.view(np.uint16), oracle.compute_scales(mp * 4).view(np.uint16))
    # monotone in m
    order = np.argsort(m, kind="stable")
    assert np.all(np.diff(sf[order]) >= 0)
    # geometric centring: max s * min s = 1 up to the two half roundings
    assert abs(sf.max() * sf.min() - 1.0) < 2 * 2.0 ** -10
    spf = sp.astype(np.float64)
    assert abs(spf.max() * spf.min() - 1.0) < 2 * 2.0 ** -10
    # the floored channel: t = 1e-4
    tmax = math.sqrt(float(m.max()))
    assert s[5] == np.float16(1e-4 / math.sqrt(tmax * 1e-4))


def test_scales_reject_nonfinite():
    m = np.ones(256, dtype=np.float32)
    m[17] = np.nan
    with pytest.raises(oracle.OracleError) as e:
        oracle.compute_scales(m)
    assert e.value.code == oracle.ERR_NONFINITE


# --------------------------------------------------------------------------
# quantize_pack: hand-worked fixture
# --------------------------------------------------------------------------
def _golden_W(fx):
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
            e = int(key.split("2^")[1])
            W[:, c] = np.array(vals, dtype=np.float64)[np.arange(K) % 16] * 2.0 ** e
    Wh = W.astype(np.float16)
    assert np.array_equal(Wh.astype(np.float64), W)        # every value exact in half
    return Wh


def _hex32(s):
    return np.int64(int(s, 16)).astype(np.uint32).astype(np.int32)


def test_quantize_hand_worked_group(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "hand_group_k128_n8.json")))
    W = _golden_W(fx)
    s = np.ones(fx["K"], dtype=np.float16)
    Q, sc, z = oracle.quantize_pack(W, s)
    exp = fx["expected"]
    assert [f"{v:#06x}" for v in sc.view(np.uint16)[0]] == [e.lower() for e in exp["scales_bits"]]
    assert [(int(z[0, 0]) >> (4 * j)) & 15 for j in range(8)] == exp["zeros"]
    assert z[0, 0] == _hex32(exp["zeros_word_hex"])
    codes0 = [(int(Q[0, 0]) >> (4 * j)) & 15 for j in range(8)]
    assert codes0 == exp["codes_col0_rows0to7"]
    qh = exp["Q_hex_by_column"]
    for c in range(8):
        spec = qh[f"col{c}"]
        for r in range(16):
            if "all" in spec:
                want = spec["all"]
            elif "row0" in spec:
                want = spec["row0"] if r == 0 else spec["rows1to15"]
            else:
                want = spec["even_rows"] if r % 2 == 0 else spec["odd_rows"]
            assert Q[r, c] == _hex32(want), (c, r)
    wh = oracle.dequant(Q, sc, z)
    assert wh[:9, 0].tolist() == exp["dequant_col0_rows0to8"]


def test_quantize_folds_s_into_w(golden_dir):
    # W = grid / s with power-of-two s: the folded weights s*W are the golden grid,
    # so the codes must be the golden ones (dividing instead of multiplying fails).
    fx = json.load(open(os.path.join(golden_dir, "hand_group_k128_n8.json")))
    Wg = _golden_W(fx).astype(np.float64)
    s = np.where(np.arange(128) % 2 == 0, 2.0, 0.5)
    W = (Wg / s[:, None]).astype(np.float16)
    assert np.array_equal(W.astype(np.float64) * s[:, None], Wg)
    Q, sc, z = oracle.quantize_pack(W, s.astype(np.float16))
    Q0, sc0, z0 = oracle.quantize_pack(Wg.astype(np.float16), np.ones(128, np.float16))
    # column 7's grid step 2^-20 / 2 underflows nothing; all columns must agree
    assert np.array_equal(Q, Q0) and np.array_equal(sc.view(np.uint16), sc0.view(np.uint16))
    assert np.array_equal(z, z0)


# --------------------------------------------------------------------------
# quantize_pack: textbook RTN special case (s = 1), independent numpy restatement
# --------------------------------------------------------------------------
def _textbook_minmax_rtn(W16):
    """Plain asymmetric min-max round-to-nearest, 4 bits, groups of 128 rows.

    Vectorised numpy float32, written independently of the oracle's loops.
    Returns codes [K, N], scales (float16) [G, N], zeros [G, N].
    """
    K, N = W16.shape
    w = W16.astype(np.float32).reshape(K // 128, 128, N)
    hi = w.max(axis=1)
    lo = w.min(axis=1)
    rng_ = np.maximum(hi - lo, np.float32(1e-5))
    scale = (rng_ / np.float32(15)).astype(np.float16)
    scale[scale == 0] = np.float16(2.0 ** -24)
    sf = scale.astype(np.float32)
    zero = np.clip(np.rint(-lo / sf), 0, 15)
    q = np.clip(np.rint(w / sf[:, None, :]) + zero[:, None, :], 0, 15)
    return q.reshape(K, N).astype(np.int64), scale, zero.astype(np.int64)


def _unpack(Q, zeros, K, N):
    j = np.arange(8)
    codes = ((Q.astype(np.int64)[:, None, :] & 0xFFFFFFFF) >> (4 * j)[None, :, None]) & 15
    codes = codes.reshape(K, N)
    zz = ((zeros.astype(np.int64)[:, :, None] & 0xFFFFFFFF) >> (4 * j)[None, None, :]) & 15
    return codes, zz.reshape(zeros.shape[0], N)


@pytest.mark.parametrize("K,N,sigma", [(128, 8, 0.02), (512, 264, 0.02), (384, 40, 3.0)])
def test_quantize_equals_textbook_rtn_when_s_is_one(K, N, sigma):
    rng = np.random.default_rng(K + N)
    W = (rng.standard_normal((K, N)) * sigma).astype(np.float16)
    Q, sc, z = oracle.quantize_pack(W, np.ones(K, np.float16))
    codes, zz = _unpack(Q, z, K, N)
    q_ref, s_ref, z_ref = _textbook_minmax_rtn(W)
    assert np.array_equal(sc.view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(zz, z_ref)
    assert np.array_equal(codes, q_ref)


# --------------------------------------------------------------------------
# quantize_pack: per-group round-trip bounds and equivariances
# --------------------------------------------------------------------------
def test_quantize_round_trip_bounds_on_workload_data():
    L = synth.make_layer(1, 0, M=1, K=1024, N=1024, R=128)
    m = oracle.act_stats(L.Xcal.numpy())
    s = oracle.compute_scales(m)
    W = L.W.numpy()
    Q, sc, z = oracle.quantize_pack(W, s)
    K, N = W.shape
    codes, zz = _unpack(Q, z, K, N)
    assert codes.min() >= 0 and codes.max() <= 15
    wf = W.astype(np.float32) * s.astype(np.float32)[:, None]          # exact fold
    wg = wf.reshape(K // 128, 128, N).astype(np.float64)
    cg = codes.reshape(K // 128, 128, N)
    sfg = sc.astype(np.float64)[:, None, :]
    wh = (cg - zz[:, None, :]) * sfg
    lo, hi = wg.min(axis=1), wg.max(axis=1)
    straddle = (lo <= 0) & (hi >= 0)
    assert straddle.mean() > 0.999
    # the group minimum encodes to 0 when the range straddles zero
    argmin = wg.argmin(axis=1)
    cmin = np.take_along_axis(cg, argmin[:, None, :], axis=1)[:, 0, :]
    assert np.all(cmin[straddle] == 0)
    err = np.abs(wg - wh)
    clamped = (np.rint(wg / sfg) + zz[:, None, :] > 15) | (np.rint(wg / sfg) + zz[:, None, :] < 0)
    bound = 0.5 * sfg * (1 + 2.0 ** -9)
    ok = straddle[:, None, :]
    assert np.all((err <= bound)[~clamped & ok])
    assert np.all((err <= 2 * bound)[clamped & ok])
    assert clamped.mean() < 1e-3


def test_quantize_column_permutation_and_power_of_two_scaling():
    rng = np.random.default_rng(5)
    K, N = 256, 64
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    s = (rng.uniform(0.3, 3.0, K)).astype(np.float16)
    Q, sc, z = oracle.quantize_pack(W, s)
    codes, zz = _unpack(Q, z, K, N)
    perm = rng.permutation(N)
    Qp, scp, zp = oracle.quantize_pack(np.ascontiguousarray(W[:, perm]), s)
    cp, zzp = _unpack(Qp, zp, K, N)
    assert np.array_equal(cp, codes[:, perm]) and np.array_equal(zzp, zz[:, perm])
    assert np.array_equal(scp.view(np.uint16), sc.view(np.uint16)[:, perm])
    Q2, sc2, z2 = oracle.quantize_pack((W.astype(np.float32) * 2).astype(np.float16), s)
    assert np.array_equal(Q2, Q) and np.array_equal(z2, z)
    assert np.array_equal(sc2.astype(np.float64), 2 * sc.astype(np.float64))


def test_quantize_rejects_nan_and_bad_shapes():
    W = np.zeros((128, 8), np.float16)
    W[3, 4] = np.nan                    # "NaN detected in weights" (Troubleshooting Guide)
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize_pack(W, np.ones(128, np.float16))
    assert e.value.code == oracle.ERR_NONFINITE
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize_pack(np.zeros((192, 8), np.float16), np.ones(192, np.float16))
    assert e.value.code == oracle.ERR_SHAPE
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize_pack(np.zeros((128, 12), np.float16), np.ones(128, np.float16))
    assert e.value.code == oracle.ERR_SHAPE


# --------------------------------------------------------------------------
# matmul: lossless grid => Y = X W exactly (the pages' equivalence)
# --------------------------------------------------------------------------
def _grid_layer(rng, K, N, pow2_s):
    """Weights whose folded values sit on each group's 4-bit grid (codes cover 0 and 15)."""
    G = K // 128
    step = 2.0 ** rng.integers(-9, -4, (G, N))
    zero = rng.integers(1, 15, (G, N))
    codes = rng.integers(0, 16, (K, N))
    codes[0::128, :] = 0
    codes[1::128, :] = 15
    wfold = (codes - np.repeat(zero, 128, axis=0)) * np.repeat(step, 128, axis=0)
    s = 2.0 ** rng.integers(-2, 3, K) if pow2_s else np.ones(K)
    W = wfold / s[:, None]
    Wh = W.astype(np.float16)
    assert np.array_equal(Wh.astype(np.float64), W)
    return Wh, s.astype(np.float16), codes


@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (3, 384, 72), (5, 1024, 40)])
def test_matmul_lossless_grid_equals_plain_xw(M, K, N):
    rng = np.random.default_rng(M * K + N)
    W, s, codes = _grid_layer(rng, K, N, pow2_s=True)
    Q, sc, z = oracle.quantize_pack(W, s)
    got_codes, _ = _unpack(Q, z, K, N)
    assert np.array_equal(got_codes, codes)
    X = rng.standard_normal((M, K)).astype(np.float16)
    Y = oracle.matmul(X, s, Q, sc, z, precision=64)
    ref = X.astype(np.float64) @ W.astype(np.float64)
    assert np.max(np.abs(Y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    Y32 = oracle.matmul(X, s, Q, sc, z, precision=32)
    assert np.max(np.abs(Y32 - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref)))


def test_matmul_column_subset_and_thread_count_do_not_change_values():
    L = synth.make_layer(1, 0, M=3, K=512, N=96, R=32)
    m = oracle.act_stats(L.Xcal.numpy())
    s = oracle.compute_scales(m)
    Q, sc, z = oracle.quantize_pack(L.W.numpy(), s)
    full = oracle.matmul(L.X.numpy(), s, Q, sc, z, precision=64, nthreads=1)
    cols = np.array([95, 0, 17, 17, 64])
    sub = oracle.matmul(L.X.numpy(), s, Q, sc, z, cols=cols, precision=64, nthreads=3)
    assert np.array_equal(sub, full[:, cols])
    f32a = oracle.matmul(L.X.numpy(), s, Q, sc, z, precision=32, nthreads=1)
    f32b = oracle.matmul(L.X.numpy(), s, Q, sc, z, precision=32, nthreads=4)
    assert np.array_equal(f32a, f32b)
    rel = np.linalg.norm(f32a - full) / np.linalg.norm(full)
    assert rel < 1e-5


def test_scaling_equivalence_before_quantization():
    # lansai explainer, four-step chain: Y = XW = (X/s)(sW) before quantization.
    rng = np.random.default_rng(2)
    X = rng.standard_normal((7, 256))
    W = rng.standard_normal((256, 33)) * 0.02
    s = rng.uniform(0.1, 10.0, 256)
    lhs = X @ W
    rhs = (X / s) @ (s[:, None] * W)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(lhs))


# --------------------------------------------------------------------------
# expected direction of the objective ("How AWQ Works": L(s))
# --------------------------------------------------------------------------
def test_activation_aware_scaling_beats_plain_rtn_on_outlier_data():
    L = synth.make_layer(1, 0, M=64, K=1024, N=256, R=128)
    X = L.X.numpy()
    W = L.W.numpy()
    ref = X.astype(np.float64) @ W.astype(np.float64)
    s = oracle.compute_scales(oracle.act_stats(L.Xcal.numpy()))
    Qa, sa, za = oracle.quantize_pack(W, s)
    ya = oracle.matmul(X, s, Qa, sa, za, precision=64)
    one = np.ones(1024, np.float16)
    Qr, sr, zr = oracle.quantize_pack(W, one)
    yr = oracle.matmul(X, one, Qr, sr, zr, precision=64)
    ea = np.linalg.norm(ya - ref)
    er = np.linalg.norm(yr - ref)
    assert ea < er, (ea, er)


# --------------------------------------------------------------------------
# symmetric variant ("Zero-Point Quantization": zero_point False)
# --------------------------------------------------------------------------
def test_symmetric_hand_worked_group(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "hand_group_symmetric_k128_n8.json")))
    W = _golden_W(fx)
    s = np.ones(fx["K"], dtype=np.float16)
    Q, sc, z = oracle.quantize_pack(W, s, zero_point=False)
    assert z is None
    exp = fx["expected"]
    assert [f"{v:#06x}" for v in sc.view(np.uint16)[0]] == [e.lower() for e in exp["scales_bits"]]
    assert [(int(Q[0, 0]) >> (4 * j)) & 15 for j in range(8)] == exp["codes_col0_rows0to7"]
    qh = exp["Q_hex_by_column"]
    for c in range(8):
        spec = qh[f"col{c}"]
        for r in range(16):
            if "all" in spec:
                want = spec["all"]
            elif "row0" in spec:
                want = spec["row0"] if r == 0 else spec["rows1to15"]
            else:
                want = spec["even_rows"] if r % 2 == 0 else spec["odd_rows"]
            assert Q[r, c] == _hex32(want), (c, r)
    wh = oracle.dequant(Q, sc, None)
    assert wh[:9, 0].tolist() == exp["dequant_col0_rows0to8"]


def _textbook_symmetric_rtn(W16):
    """Plain symmetric round-to-nearest, 4 bits (levels -8..7), groups of 128 rows.

    Vectorised numpy float32, written independently of the oracle's loops.
    Returns codes (level + 8) [K, N] and scales (float16) [G, N].
    """
    K, N = W16.shape
    w = W16.astype(np.float32).reshape(K // 128, 128, N)
    a = np.maximum(np.abs(w).max(axis=1), np.float32(1e-5))
    scale = (a / np.float32(7)).astype(np.float16)
    scale[scale == 0] = np.float16(2.0 ** -24)
    level = np.clip(np.rint(w / scale.astype(np.float32)[:, None, :]), -8, 7)
    return (level + 8).reshape(K, N).astype(np.int64), scale


@pytest.mark.parametrize("K,N,sigma", [(128, 8, 0.02), (512, 264, 0.02), (384, 40, 3.0)])
def test_symmetric_equals_textbook_rtn_when_s_is_one(K, N, sigma):
    rng = np.random.default_rng(K * 3 + N)
    W = (rng.standard_normal((K, N)) * sigma).astype(np.float16)
    Q, sc, _ = oracle.quantize_pack(W, np.ones(K, np.float16), zero_point=False)
    codes, _ = _unpack(Q, np.zeros((K // 128, N // 8), np.int32), K, N)
    q_ref, s_ref = _textbook_symmetric_rtn(W)
    assert np.array_equal(sc.view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(codes, q_ref)


def test_symmetric_negation_bounds_and_implicit_zero_point():
    L = synth.make_layer(1, 0, M=1, K=1024, N=512, R=128)
    s = oracle.compute_scales(oracle.act_stats(L.Xcal.numpy()))
    W = L.W.numpy()
    K, N = W.shape
    Q, sc, _ = oracle.quantize_pack(W, s, zero_point=False)
    codes, _ = _unpack(Q, np.zeros((K // 128, N // 8), np.int32), K, N)
    # every |w'| <= max |w'| = 7 steps (up to the step's binary16 rounding): no
    # level -8, nothing clamps, and rint is odd-symmetric under half-to-even
    assert codes.min() >= 1 and codes.max() <= 15
    Qn, scn, _ = oracle.quantize_pack(-W, s, zero_point=False)
    cn, _ = _unpack(Qn, np.zeros((K // 128, N // 8), np.int32), K, N)
    assert np.array_equal(scn.view(np.uint16), sc.view(np.uint16))
    assert np.array_equal(cn, 16 - codes)
    # round trip within half a step; the largest magnitude of a group lands on +-7
    wf = (W.astype(np.float32) * s.astype(np.float32)[:, None]).astype(np.float64)
    wg = wf.reshape(K // 128, 128, N)
    sfg = sc.astype(np.float64)[:, None, :]
    wh = (codes.reshape(K // 128, 128, N) - 8) * sfg
    assert np.all(np.abs(wg - wh) <= 0.5 * sfg * (1 + 2.0 ** -9))
    am = np.abs(wg).argmax(axis=1)
    lv = np.take_along_axis(codes.reshape(K // 128, 128, N), am[:, None, :], axis=1)[:, 0, :] - 8
    assert np.all(np.abs(lv) == 7)
    # no zeros tensor means a zero point of 8 everywhere
    eights = np.full((K // 128, N // 8), np.int32(np.int64(0x88888888).astype(np.uint32).astype(np.int32)))
    assert np.array_equal(oracle.dequant(Q, sc, None), oracle.dequant(Q, sc, eights))


@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (4, 512, 40)])
def test_symmetric_matmul_lossless_grid_equals_plain_xw(M, K, N):
    # folded weights on each group's symmetric grid (levels -7..7, both ends
    # present): quantization is lossless and Y must equal X W exactly
    rng = np.random.default_rng(M + K + N)
    G = K // 128
    step = 2.0 ** rng.integers(-9, -4, (G, N))
    level = rng.integers(-7, 8, (K, N))
    level[0::128, :] = -7
    level[1::128, :] = 7
    s = 2.0 ** rng.integers(-2, 3, K)
    W = (level * np.repeat(step, 128, axis=0)) / s[:, None]
    Wh = W.astype(np.float16)
    assert np.array_equal(Wh.astype(np.float64), W)
    Q, sc, z = oracle.quantize_pack(Wh, s.astype(np.float16), zero_point=False)
    codes, _ = _unpack(Q, np.zeros((G, N // 8), np.int32), K, N)
    assert np.array_equal(codes, level + 8)
    X = rng.standard_normal((M, K)).astype(np.float16)
    Y = oracle.matmul(X, s.astype(np.float16), Q, sc, None, precision=64)
    ref = X.astype(np.float64) @ W
    assert np.max(np.abs(Y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


# --------------------------------------------------------------------------
# 1/s folded into the preceding operator (lansai four-step chain: (X/s)(sW))
# --------------------------------------------------------------------------
def test_fold_inverse_scale_equals_numpy_float_division():
    rng = np.random.default_rng(31)
    K = 4096
    a = (rng.standard_normal((3, K)) * rng.uniform(0.01, 30, K)).astype(np.float16)
    s = rng.uniform(0.05, 20.0, K).astype(np.float16)
    got = oracle.fold_inverse_scale(a, s)
    ref = (a.astype(np.float32) / s.astype(np.float32)).astype(np.float16)   # IEEE float, one RNE
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))
    g1 = oracle.fold_inverse_scale(a[0], s)                                # a norm weight [K]
    assert g1.shape == (K,) and np.array_equal(g1.view(np.uint16), got[0].view(np.uint16))


def test_fold_inverse_scale_closed_forms_and_errors():
    rng = np.random.default_rng(32)
    K = 256
    a = rng.standard_normal((2, K)).astype(np.float16)
    assert np.array_equal(oracle.fold_inverse_scale(a, np.ones(K, np.float16)).view(np.uint16),
                          a.view(np.uint16))
    p2 = 2.0 ** rng.integers(-3, 4, K)
    out = oracle.fold_inverse_scale(a, p2.astype(np.float16)).astype(np.float64)
    assert np.array_equal(out, a.astype(np.float64) / p2)                  # exact, no underflow here
    bad = np.ones(K, np.float16)
    bad[7] = 0
    with pytest.raises(oracle.OracleError) as e:
        oracle.fold_inverse_scale(a, bad)
    assert e.value.code == oracle.ERR_NONFINITE


def test_matmul_without_s_reads_prescaled_activations():
    L = synth.make_layer(1, 0, M=4, K=512, N=64, R=32)
    s = oracle.compute_scales(oracle.act_stats(L.Xcal.numpy()))
    Q, sc, z = oracle.quantize_pack(L.W.numpy(), s)
    X = L.X.numpy()
    # no s is the same as s = 1 (division by one is exact)
    ones = np.ones(512, np.float16)
    for prec in (64, 32):
        assert np.array_equal(oracle.matmul(X, None, Q, sc, z, precision=prec),
                              oracle.matmul(X, ones, Q, sc, z, precision=prec))
    # power-of-two s: X/s is exact in binary16, so folding it upstream changes nothing
    rng = np.random.default_rng(33)
    p2 = (2.0 ** rng.integers(-2, 3, 512)).astype(np.float16)
    Xp = oracle.fold_inverse_scale(X, p2)
    assert np.array_equal(oracle.matmul(Xp, None, Q, sc, z, precision=64),
                          oracle.matmul(X, p2, Q, sc, z, precision=64))


# --------------------------------------------------------------------------
# scale search over alpha ("How AWQ Works": L(s); lansai chain row "搜索缩放")
# --------------------------------------------------------------------------
def test_alpha_scales_closed_forms():
    rng = np.random.default_rng(41)
    m = rng.uniform(0.01, 9.0, 512).astype(np.float32)
    # j = 4 (alpha = 1/2) is the pinned single-point scale
    assert np.array_equal(oracle.scales_alpha(m, 4).view(np.uint16), oracle.compute_scales(m).view(np.uint16))
    # j = 0: every t is 1, so s is exactly 1
    assert np.all(oracle.scales_alpha(m, 0) == 1.0)
    # two levels 16 and 1: s = 16^(j/8) / 16^(j/16) = 2^(j/4) or its inverse;
    # the double chain is within a few ulps of it, far from any binary16
    # rounding boundary, so the stored value is 2^(+-j/4) rounded once
    two = np.where(np.arange(64) % 2 == 0, 16.0, 1.0).astype(np.float32)
    for j in range(9):
        s = oracle.scales_alpha(two, j).astype(np.float64)
        hi, lo = 2.0 ** (j / 4), 2.0 ** (-j / 4)
        assert np.array_equal(s[0::2], np.full(32, float(np.float16(hi))))
        assert np.array_equal(s[1::2], np.full(32, float(np.float16(lo))))
    with pytest.raises(oracle.OracleError):
        oracle.scales_alpha(m, 9)


def _plain_rtn_loss(X16, W16):
    """Output error of plain min-max RTN (s = 1), by the independent numpy quantizer."""
    q, step, zero = _textbook_minmax_rtn(W16)
    K, N = W16.shape
    wh = (q - np.repeat(zero, 128, axis=0)) * np.repeat(step.astype(np.float64), 128, axis=0)
    X = X16.astype(np.float64)
    return float(np.sum((X @ wh - X @ W16.astype(np.float64)) ** 2))


def test_scale_search_loss_grid_and_choice():
    L = synth.make_layer(1, 0, M=1, K=256, N=64, R=32)
    X, W = L.Xcal.numpy(), L.W.numpy()
    j, s, losses = oracle.scale_search(X, W, nthreads=4)
    # alpha = 0 is plain RTN: the loss equals the independent restatement's
    ref0 = _plain_rtn_loss(X, W)
    assert abs(losses[0] - ref0) <= 1e-9 * ref0
    # the choice is the first minimiser, and its scales are that grid point's
    assert j == int(np.argmin(losses)) and losses[j] == losses.min()
    m = oracle.act_stats(X)
    assert np.array_equal(s.view(np.uint16), oracle.scales_alpha(m, j).view(np.uint16))
    # on data with outlier channels the activation-aware point beats plain RTN
    assert j > 0 and losses[j] < losses[0]


def test_scale_search_power_of_two_invariance():
    # X * 256: m * 256, so r1, r2, r3 scale by 16, 4, 2 exactly and the normalised
    # scales are unchanged; Y and Yq scale by 256 and every loss by 2^16 exactly
    L = synth.make_layer(1, 1, M=1, K=256, N=32, R=16)
    X = (L.Xcal.numpy().astype(np.float32) / 4).astype(np.float16)
    X2 = (X.astype(np.float32) * 256).astype(np.float16)
    assert np.array_equal(X2.astype(np.float64), X.astype(np.float64) * 256)
    W = L.W.numpy()
    j1, s1, l1 = oracle.scale_search(X, W)
    j2, s2, l2 = oracle.scale_search(X2, W)
    assert j1 == j2 and np.array_equal(s1.view(np.uint16), s2.view(np.uint16))
    assert np.array_equal(l2, l1 * 65536.0)


# --------------------------------------------------------------------------
# weight clipping ("Awq Quantization", calibration parameters: apply_clip)
# --------------------------------------------------------------------------
def _group_losses(X16, s, W16, Q, sc, z):
    """Per (group, column) output error on the calibration rows, from packed outputs (numpy)."""
    K, N = W16.shape
    codes, zz = _unpack(Q, z, K, N)
    wf = W16.astype(np.float32) * s.astype(np.float32)[:, None]
    wh = (codes - np.repeat(zz, 128, axis=0)) * np.repeat(sc.astype(np.float64), 128, axis=0)
    e = (wh - wf.astype(np.float64)).reshape(K // 128, 128, N)
    xp = (X16.astype(np.float64) / s.astype(np.float64)).reshape(X16.shape[0], K // 128, 128)
    y = np.einsum("rgk,gkn->rgn", xp, e)
    return (y ** 2).sum(axis=0)                                    # [G, N]


def test_clip_without_candidates_is_plain_quantization():
    L = synth.make_layer(1, 2, M=1, K=384, N=40, R=16)
    s = oracle.compute_scales(oracle.act_stats(L.Xcal.numpy()))
    Q, sc, z, ri = oracle.quantize_pack_clip(L.W.numpy(), s, L.Xcal.numpy(), n_cand=1)
    Qp, scp, zp = oracle.quantize_pack(L.W.numpy(), s)
    assert np.all(ri == 0)
    assert np.array_equal(Q, Qp) and np.array_equal(z, zp)
    assert np.array_equal(sc.view(np.uint16), scp.view(np.uint16))


def test_clip_never_raises_a_groups_output_error():
    L = synth.make_layer(1, 3, M=1, K=512, N=64, R=32)
    X, W = L.Xcal.numpy(), L.W.numpy()
    s = oracle.compute_scales(oracle.act_stats(X))
    Q, sc, z, ri = oracle.quantize_pack_clip(W, s, X)
    Qp, scp, zp = oracle.quantize_pack(W, s)
    lc = _group_losses(X, s, W, Q, sc, z)
    lp = _group_losses(X, s, W, Qp, scp, zp)
    assert np.all(lc <= lp * (1 + 1e-9))
    assert np.all((ri == 0) | (lc < lp))          # a clipped group strictly gains
    assert (ri > 0).any() and (ri == 0).any()


def test_clip_drops_an_outlier_that_no_activation_sees():
    # Every column: weights k/16 (k = 0..15, so the minimum is 0 at any ratio)
    # plus one weight 1.875 on a channel whose calibration activations are all
    # zero.  At c = 1/2 the range is [0, 0.9375], the step exactly 1/16, and
    # every seen weight is represented exactly: loss 0.  At c = 1 (step 1/8)
    # the odd sixteenths sit on ties and err by 1/16; the ratios in between give
    # steps on which the sixteenths are not exact.  So c = 1/2 is the only
    # zero-loss choice and the search must take it.  Columns 8..15 are the
    # mirror image (maximum 0, outlier -1.875), where only a shrunk lower end
    # reaches zero loss.
    rng = np.random.default_rng(44)
    K, N, R = 128, 16, 8
    W = (rng.integers(0, 16, (K, N)) / 16.0).astype(np.float16)
    W[0, :] = 0
    W[5, :] = np.float16(1.875)
    W[:, 8:] = -W[:, 8:]
    X = rng.standard_normal((R, K)).astype(np.float16)
    X[:, 5] = 0
    s = np.ones(K, np.float16)
    Q, sc, z, ri = oracle.quantize_pack_clip(W, s, X)
    assert np.all(ri == 10)
    _, zz = _unpack(Q, z, K, N)
    assert np.all(sc.astype(np.float64) == 1 / 16)
    assert np.all(zz[:, :8] == 0) and np.all(zz[:, 8:] == 15)
    assert np.all(_group_losses(X, s, W, Q, sc, z) == 0)
    Qp, scp, zp = oracle.quantize_pack(W, s)
    assert np.all(_group_losses(X, s, W, Qp, scp, zp) > 0)


def test_clip_keeps_a_lossless_grid_and_rejects_bad_counts():
    rng = np.random.default_rng(45)
    W, s, codes = _grid_layer(rng, 256, 24, pow2_s=True)
    X = rng.standard_normal((8, 256)).astype(np.float16)
    Q, sc, z, ri = oracle.quantize_pack_clip(W, s, X)
    assert np.all(ri == 0)                         # loss 0 at c = 1, the first minimiser
    got, _ = _unpack(Q, z, 256, 24)
    assert np.array_equal(got, codes)
    for bad in (0, 12):
        with pytest.raises(oracle.OracleError) as e:
            oracle.quantize_pack_clip(W, s, X, n_cand=bad)
        assert e.value.code == oracle.ERR_SHAPE
