"""Seeded synthetic inputs for the AWQ W4A16 linear layer.

This module is shared by the tests, the benchmark and the smoke check so that
the CUDA library and the CPU oracle see identical input bits.  It holds none of
the method's arithmetic: it only draws random tensors and lists the layer
shapes.  Inputs are drawn with torch's seeded generators (on the CPU, or on a
CUDA device for the large layer stacks); whoever needs the same bits on the
other side copies the tensor.

Distributions (stand-ins for real checkpoints and calibration text, neither of
which is available here):
  * activations X and calibration rows X_cal: float16 ~ N(0, 1), with a seeded
    1% of the input channels (ceil(0.01 K), shared by X and X_cal) multiplied
    by 20 -- the "about 1% salient channels" the AWQ pages describe;
  * weights W: float16 ~ N(0, 0.02^2), drawn in float32 and rounded to nearest.
Seeds are derived from (workload, layer, tensor) so every tensor of every layer
is reproducible on its own.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

OUTLIER_FRACTION = 0.01
OUTLIER_GAIN = 20.0
W_SIGMA = 0.02

# tensor ids used in seed derivation
_T_X, _T_XCAL, _T_W, _T_OUTLIERS = 1, 2, 3, 4


def seed_for(workload: int, layer: int, tensor: int, base: int = 0x5EED) -> int:
    """Deterministic 63-bit seed for one tensor of one layer of one workload."""
    h = (base * 1_000_003 + workload) * 1_000_033 + layer
    h = (h * 1_000_037 + tensor) & ((1 << 63) - 1)
    # mix the bits (splitmix64 finaliser) so neighbouring ids decorrelate
    h = (h ^ (h >> 30)) * 0xBF58476D1CE4E5B9 & ((1 << 64) - 1)
    h = (h ^ (h >> 27)) * 0x94D049BB133111EB & ((1 << 64) - 1)
    return (h ^ (h >> 31)) & ((1 << 63) - 1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_channels(K: int, seed: int) -> torch.Tensor:
    """Sorted int64 indices of the ceil(0.01 K) salient input channels (CPU)."""
    n = max(1, math.ceil(OUTLIER_FRACTION * K))
    perm = torch.randperm(K, generator=_gen(seed, "cpu"))
    return torch.sort(perm[:n]).values


def activations(M: int, K: int, seed: int, outliers: torch.Tensor, device="cpu") -> torch.Tensor:
    """float16 [M, K] ~ N(0,1) with the outlier channels scaled by 20."""
    x = torch.randn(M, K, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if outliers.numel():
        x[:, outliers.to(device)] *= OUTLIER_GAIN
    return x.to(torch.float16)


def weights(K: int, N: int, seed: int, device="cpu") -> torch.Tensor:
    """float16 [K, N] ~ N(0, 0.02^2) (Y = X W, K = input channels)."""
    w = torch.randn(K, N, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return (w * W_SIGMA).to(torch.float16)


@dataclass
class Layer:
    """One synthetic linear layer's inputs (all float16)."""
    K: int
    N: int
    M: int
    R: int
    X: torch.Tensor
    Xcal: torch.Tensor
    W: torch.Tensor
    outliers: torch.Tensor = field(repr=False)


def make_layer(workload: int, layer: int, M: int, K: int, N: int, R: int, device="cpu",
               shape_id: int = 0) -> Layer:
    """Seeded X [M,K], X_cal [R,K], W [K,N] for one layer shape of one workload."""
    tag = layer * 16 + shape_id
    outl = outlier_channels(K, seed_for(workload, tag, _T_OUTLIERS))
    X = activations(M, K, seed_for(workload, tag, _T_X), outl, device)
    Xcal = activations(R, K, seed_for(workload, tag, _T_XCAL), outl, device)
    W = weights(K, N, seed_for(workload, tag, _T_W), device)
    return Layer(K, N, M, R, X, Xcal, W, outl)


# --------------------------------------------------------------------------
# The five workloads: shapes are (K, N) of y = x W per linear projection.
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    shapes: tuple          # ((K, N, label), ...)
    Ms: tuple              # token counts
    R: int                 # calibration rows
    layers: int = 1


WORKLOADS = {
    1: Workload(1, "single linear layer 1024x1024, M=1",
                ((1024, 1024, "linear"),), (1,), 128),
    2: Workload(2, "Mistral-7B-shaped decode GEMV set, M=1",
                ((4096, 6144, "qkv"), (4096, 4096, "o"), (4096, 28672, "gate_up"),
                 (14336, 4096, "down")), (1,), 256),
    3: Workload(3, "13B-shaped small-batch GEMM, M in {8,16,32,48}",
                ((5120, 15360, "qkv"), (5120, 5120, "o"), (5120, 27648, "gate_up"),
                 (13824, 5120, "down")), (8, 16, 32, 48), 256),
    4: Workload(4, "7B-shaped prefill GEMM, M in {512,2048,4096}",
                ((4096, 6144, "qkv"), (4096, 4096, "o"), (4096, 28672, "gate_up"),
                 (14336, 4096, "down")), (512, 2048, 4096), 256),
    5: Workload(5, "70B-shaped 80-layer stack, M in {1,32,256}",
                ((8192, 10240, "qkv"), (8192, 8192, "o"), (8192, 57344, "gate_up"),
                 (28672, 8192, "down")), (1, 32, 256), 256, layers=80),
}
