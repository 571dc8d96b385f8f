"""GPU parity of weight clipping ("Awq Quantization", calibration parameters,
apply_clip): per group and column the range shrink c = 1 - i/20 whose codes
give the smallest output error on the calibration rows.

Checked against the oracle's quantize_pack_clip:
  * n_cand = 1 (no clipping) equals the plain quantizer bit for bit;
  * the chosen index agrees with the oracle's, except where the two
    candidates' losses (recomputed here in double from each side's choice)
    agree to float precision -- the GPU scores in float, the oracle in double;
  * steps, zero points and packed codes are bit-exact wherever the index agrees.
The full-size case runs the GPU on the whole 7B O projection and the oracle
on a seeded sample of its columns (the choice is made per column).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_quantization_quantize_b200 as awq

pytestmark = pytest.mark.gpu
NEAR_TIE = 1e-5   # relative loss difference treated as a tie (float scoring)


def _unpack_codes(Q):
    Q = Q.astype(np.uint32)
    return np.stack([(Q >> (4 * j)) & 15 for j in range(8)], axis=1).reshape(-1, Q.shape[1])


def _unpack_zeros(z):
    z = z.astype(np.uint32)
    return np.stack([(z >> (4 * j)) & 15 for j in range(8)], axis=2).reshape(z.shape[0], -1)


def _loss(xp, wp, i):
    """Double output error of one group column for candidate i (the reading
    of apply_clip, float parameters as in the quantizer)."""
    f = np.float32
    c = f(1) - f(i) / f(20)
    lo, hi = c * wp.min(), c * wp.max()
    r = max(f(hi - lo), f(1e-5))
    sh = np.float16(f(r) / f(15))
    if sh == 0:
        sh = np.float16(2.0 ** -24)
    z = int(np.clip(np.rint(f(-lo) / f(sh)), 0, 15))
    q = np.clip(np.rint(wp / f(sh)).astype(np.int64) + z, 0, 15)
    e = (q - z).astype(np.float64) * float(sh) - wp.astype(np.float64)
    return float(np.sum((xp @ e) ** 2))


def _check(W, s, xcal, cols=None, n_cand=11):
    Q, sc, z, ri = awq.quantize_pack_clip(W.cuda(), s.cuda(), xcal.cuda(), n_cand)
    Q, sc, z, ri = Q.cpu().numpy(), sc.cpu().numpy(), z.cpu().numpy(), ri.cpu().numpy()
    Wn, sn, xn = W.numpy(), s.numpy(), xcal.numpy()
    if cols is None:
        cols = np.arange(Wn.shape[1])
    Qr, scr, zr, rir = oracle.quantize_pack_clip(np.ascontiguousarray(Wn[:, cols]), sn, xn, n_cand)
    ri_g = ri[:, cols]
    agree = ri_g == rir
    G = Wn.shape[0] // 128
    wp_all = Wn.astype(np.float32) * sn.astype(np.float32)[:, None]
    xp_all = xn.astype(np.float64) / sn.astype(np.float64)[None, :]
    for g, j in zip(*np.nonzero(~agree)):
        n = cols[j]
        wp = wp_all[128 * g:128 * g + 128, n]
        xp = xp_all[:, 128 * g:128 * g + 128]
        lg = _loss(xp, wp, int(ri_g[g, j]))
        lr = _loss(xp, wp, int(rir[g, j]))
        assert abs(lg - lr) <= NEAR_TIE * max(lg, lr), (g, n, ri_g[g, j], rir[g, j], lg, lr)
    assert agree.mean() >= 0.99
    # bit-exact wherever the choice agrees
    assert np.array_equal(sc[:, cols].view(np.uint16)[agree], scr.view(np.uint16)[agree])
    zg, zo = _unpack_zeros(z)[:, cols], _unpack_zeros(zr)
    assert np.array_equal(zg[agree], zo[agree])
    cg, co = _unpack_codes(Q)[:, cols], _unpack_codes(Qr)
    rows_agree = np.repeat(agree, 128, axis=0)
    assert np.array_equal(cg[rows_agree], co[rows_agree])
    return ri, rir


def test_one_candidate_is_the_plain_quantizer():
    L = synth.make_layer(22, 0, M=1, K=512, N=264, R=64)
    s = awq.compute_scales(awq.act_stats(L.Xcal.cuda()))
    Q0, sc0, z0 = awq.quantize_pack(L.W.cuda(), s)
    Q1, sc1, z1, ri = awq.quantize_pack_clip(L.W.cuda(), s, L.Xcal.cuda(), 1)
    assert torch.equal(Q0, Q1) and torch.equal(sc0, sc1) and torch.equal(z0, z1)
    assert int(ri.abs().sum().item()) == 0


@pytest.mark.parametrize("R,K,N", [(64, 256, 64), (256, 1024, 1032), (100, 1152, 520), (1, 128, 8),
                                   (65, 384, 40)])
def test_clip_small(R, K, N):
    L = synth.make_layer(23, R + K + N, M=1, K=K, N=N, R=R)
    s = torch.from_numpy(oracle.compute_scales(oracle.act_stats(L.Xcal.numpy())))
    ri, _ = _check(L.W, s, L.Xcal)
    assert (ri > 0).any() or N * K < 2048     # clipping is chosen somewhere on real-sized groups


@pytest.mark.parametrize("n_cand", [2, 6])
def test_clip_fewer_candidates(n_cand):
    L = synth.make_layer(24, n_cand, M=1, K=512, N=128, R=128)
    s = torch.from_numpy(oracle.compute_scales(oracle.act_stats(L.Xcal.numpy())))
    ri, _ = _check(L.W, s, L.Xcal, n_cand=n_cand)
    assert ri.max() < n_cand


def test_clip_nonfinite_reported():
    W = torch.randn(256, 64).half() * 0.02
    W[3, 9] = float("nan")
    st = awq.new_status("cuda")
    awq.quantize_pack_clip(W.cuda(), torch.ones(256).half().cuda(), torch.randn(16, 256).half().cuda(), status=st)
    assert int(st.item()) == awq.ERR_NONFINITE


def test_clip_full_size_7b_o_projection():
    wl = synth.WORKLOADS[2]
    K, N, _ = wl.shapes[1]
    L = synth.make_layer(2, 0, M=1, K=K, N=N, R=wl.R, shape_id=1)
    s = torch.from_numpy(oracle.compute_scales(oracle.act_stats(L.Xcal.numpy())))
    rng = np.random.default_rng(31)
    cols = np.sort(rng.choice(N, size=96, replace=False))
    _check(L.W, s, L.Xcal, cols=cols)
