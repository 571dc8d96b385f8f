"""Argument checks of the Python binding.

The C ABI sees only raw device pointers, so a mis-shaped scales or out tensor
would make a kernel read or write outside its buffer.  The binding therefore
checks every tensor argument (type, dtype, shape, device, contiguity) and
raises before anything reaches the library.  The GPU cases check that the
error comes before any launch: the output buffer keeps its sentinel bits.
"""
import pytest
import torch

import weight_only_quantization_quantize_b200 as awq


def test_host_tensors_are_refused_without_a_gpu():
    X = torch.zeros(1, 256, dtype=torch.float16)
    with pytest.raises(TypeError, match="CUDA"):
        awq.w4a16_gemm(X, None, None, None, None)
    with pytest.raises(TypeError, match="CUDA"):
        awq.w4a16_gemv(X, None, None, None, None)
    with pytest.raises(TypeError, match="CUDA"):
        awq.act_stats(X)
    with pytest.raises(TypeError, match="CUDA"):
        awq.quantize_pack(torch.zeros(256, 8, dtype=torch.float16), torch.ones(256, dtype=torch.float16))


def _layer(K=256, N=64, M=2):
    d = "cuda"
    X = torch.randn(M, K, device=d).half()
    s = torch.ones(K, dtype=torch.float16, device=d)
    Q = torch.zeros(K // 8, N, dtype=torch.int32, device=d)
    sc = torch.ones(K // 128, N, dtype=torch.float16, device=d)
    z = torch.zeros(K // 128, N // 8, dtype=torch.int32, device=d)
    return X, s, Q, sc, z


BAD_CASES = [
    ("s", lambda t: t[:-8], ValueError),                          # [K-8]
    ("s", lambda t: t.float(), TypeError),
    ("Q", lambda t: t[:, :-8].contiguous(), None),                # changes N: scales no longer match
    ("Q", lambda t: t.view(torch.float32), TypeError),
    ("sc", lambda t: t[:1], ValueError),                          # too few groups
    ("sc", lambda t: t.t().contiguous().t(), ValueError),         # not contiguous
    ("sc", lambda t: t.float(), TypeError),
    ("z", lambda t: t[:, :4].contiguous(), ValueError),           # [G, 4] instead of [G, N/8]
    ("z", lambda t: t.to(torch.int64), TypeError),
]


@pytest.mark.gpu
@pytest.mark.parametrize("which,bad,exc", BAD_CASES)
def test_mis_shaped_weights_raise_before_launch(which, bad, exc):
    X, s, Q, sc, z = _layer()
    args = dict(s=s, Q=Q, sc=sc, z=z)
    args[which] = bad(args[which])
    out = torch.full((2, Q.shape[1]), 7.0, dtype=torch.float16, device="cuda")
    with pytest.raises((ValueError, TypeError) if exc is None else exc):
        awq.w4a16_gemm(X, args["s"], args["Q"], args["sc"], args["z"], out=out)
    with pytest.raises((ValueError, TypeError) if exc is None else exc):
        awq.w4a16_gemv(X[:1].contiguous(), args["s"], args["Q"], args["sc"], args["z"], out=out[:1])
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()), "nothing may be launched"


@pytest.mark.gpu
def test_mis_shaped_outputs_and_workspace_raise_before_launch():
    X, s, Q, sc, z = _layer()
    with pytest.raises(ValueError, match="out"):
        awq.w4a16_gemm(X, s, Q, sc, z, out=torch.empty(2, 56, dtype=torch.float16, device="cuda"))
    with pytest.raises(TypeError, match="out"):
        awq.w4a16_gemm(X, s, Q, sc, z, out=torch.empty(2, 64, dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError, match="out"):
        awq.w4a16_gemm(X, s, Q, sc, z, out=torch.empty(64, 2, dtype=torch.float16, device="cuda").t())
    need = awq.gemm_workspace_size(2, 256, 64)
    with pytest.raises(ValueError, match="workspace"):
        awq.w4a16_gemm(X, s, Q, sc, z, workspace=torch.zeros(need - 16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(TypeError, match="workspace"):
        awq.w4a16_gemm(X, s, Q, sc, z, workspace=torch.zeros(need, dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError, match="status"):
        awq.w4a16_gemm(X, s, Q, sc, z, status=torch.zeros(2, 2, dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError, match="X"):
        awq.w4a16_gemm(X[:, :128], s, Q, sc, z)                     # X not contiguous
    W = torch.zeros(256, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError, match="s"):
        awq.quantize_pack(W, s[:128])
    with pytest.raises(ValueError, match="scales"):
        awq.quantize_pack(W, s, out=(Q, sc[:, :8].contiguous(), z))
    with pytest.raises(ValueError, match="out"):
        awq.fold_inverse_scale(X, s, out=torch.empty(2, 128, dtype=torch.float16, device="cuda"))


@pytest.mark.gpu
def test_quant_linear_checks_weights_once_and_inputs_every_call():
    X, s, Q, sc, z = _layer()
    with pytest.raises(ValueError):
        awq.QuantLinear(Q, sc[:1], z, s)
    lin = awq.QuantLinear(Q, sc, z, s)
    with pytest.raises(ValueError, match="X"):
        lin(torch.zeros(2, 128, dtype=torch.float16, device="cuda"))
    with pytest.raises(ValueError, match="out"):
        lin(X, out=torch.empty(2, 8, dtype=torch.float16, device="cuda"))
    # the prepared layer runs the same call as the functional entry point
    Q.random_(-2**31, 2**31 - 1)
    z.random_(-2**31, 2**31 - 1)
    assert torch.equal(lin(X), awq.w4a16_gemm(X, s, Q, sc, z))
    assert torch.equal(lin(X[:1].contiguous()), awq.w4a16_gemv(X[:1].contiguous(), s, Q, sc, z))
