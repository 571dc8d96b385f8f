"""The seeded input generators draw what the input recipe states.

The recipe (stand-ins for checkpoints and calibration text): X and X_cal are
float16 N(0, 1) with a seeded 1% of the input channels, shared by both,
multiplied by 20; W is float16 N(0, 0.02^2); every tensor is reproducible from
its (workload, layer, tensor) seed on its own; the workload table lists the
layer shapes and token counts of the single-layer, 7B decode, 13B small-batch,
7B prefill and 70B-stack workloads.
"""
import math

import torch

import synth


def test_outlier_channels_are_one_percent_shared_and_scaled_by_20():
    K = 4096
    L = synth.make_layer(2, 0, M=512, K=K, N=64, R=512)
    n = math.ceil(0.01 * K)
    assert L.outliers.numel() == n and torch.unique(L.outliers).numel() == n
    assert bool((L.outliers[1:] > L.outliers[:-1]).all()) and 0 <= int(L.outliers[0]) and int(L.outliers[-1]) < K
    mask = torch.zeros(K, dtype=torch.bool)
    mask[L.outliers] = True
    for A in (L.X, L.Xcal):
        assert A.dtype == torch.float16 and A.shape == (512, K)
        a = A.float()
        std_out = a[:, mask].std().item()
        std_in = a[:, ~mask].std().item()
        mean_in = a[:, ~mask].mean().item()
        assert abs(std_in - 1.0) < 0.01 and abs(mean_in) < 0.01
        assert abs(std_out / std_in - 20.0) < 0.5
    # the largest per-channel magnitudes of the calibration rows are exactly the outliers
    top = torch.topk(L.Xcal.float().abs().mean(0), n).indices
    assert set(top.tolist()) == set(L.outliers.tolist())


def test_weights_are_normal_with_sigma_0_02():
    L = synth.make_layer(4, 0, M=1, K=2048, N=1024, R=1)
    w = L.W.float()
    assert L.W.dtype == torch.float16 and L.W.shape == (2048, 1024)
    assert abs(w.std().item() - 0.02) < 2e-4 and abs(w.mean().item()) < 2e-4
    # about 4.55% of a normal sample lies beyond two standard deviations
    tail = (w.abs() > 0.04).float().mean().item()
    assert abs(tail - 0.0455) < 0.003


def test_tensors_are_reproducible_and_independent():
    a = synth.make_layer(3, 5, M=8, K=512, N=64, R=16, shape_id=2)
    b = synth.make_layer(3, 5, M=8, K=512, N=64, R=16, shape_id=2)
    for x, y in ((a.X, b.X), (a.Xcal, b.Xcal), (a.W, b.W), (a.outliers, b.outliers)):
        assert torch.equal(x, y)
    # another layer, projection or workload draws other bits
    for other in (synth.make_layer(3, 6, M=8, K=512, N=64, R=16, shape_id=2),
                  synth.make_layer(3, 5, M=8, K=512, N=64, R=16, shape_id=1),
                  synth.make_layer(2, 5, M=8, K=512, N=64, R=16, shape_id=2)):
        assert not torch.equal(other.W, a.W) and not torch.equal(other.X, a.X)
    # X and X_cal of one layer are different draws over the same outlier channels
    assert not torch.equal(a.X[:8], a.Xcal[:8])
    seeds = {synth.seed_for(w, l, t) for w in range(1, 6) for l in range(80 * 16) for t in range(1, 5)}
    assert len(seeds) == 5 * 80 * 16 * 4


def test_workload_table_matches_the_configured_shapes():
    W = synth.WORKLOADS
    assert [s[:2] for s in W[1].shapes] == [(1024, 1024)] and W[1].Ms == (1,) and W[1].R == 128
    assert [s[:2] for s in W[2].shapes] == [(4096, 6144), (4096, 4096), (4096, 28672), (14336, 4096)]
    assert W[2].Ms == (1,) and W[2].R == 256
    assert [s[:2] for s in W[3].shapes] == [(5120, 15360), (5120, 5120), (5120, 27648), (13824, 5120)]
    assert W[3].Ms == (8, 16, 32, 48)
    assert [s[:2] for s in W[4].shapes] == [s[:2] for s in W[2].shapes] and W[4].Ms == (512, 2048, 4096)
    assert [s[:2] for s in W[5].shapes] == [(8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192)]
    assert W[5].Ms == (1, 32, 256) and W[5].layers == 80
    # every shape is a valid matmul problem: K a whole number of 128-row groups, N of 8-column words
    for w in W.values():
        for K, N, _ in w.shapes:
            assert K % 128 == 0 and N % 8 == 0
    # the 70B stack's packed weights: 0.5195 B per weight over 80 layers, about 35.6 GB
    per_layer = sum(K * N for K, N, _ in W[5].shapes)
    assert abs(per_layer * 80 * (0.5 + 2 / 128 + 0.5 / 128) / 1e9 - 35.6) < 0.1
