// fold.cu -- 1/s folded into the operator that precedes the matmul.
//
// Source: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路":
// Y = XW = (X/s)(sW).  The X/s side can be carried upstream (by a
// normalisation weight, or by activations divided once and reused by several
// projections), after which the matmul calls take s = NULL.
//
//   out[r, k] = binary16_RNE(float(a[r, k]) / float(s_k))   (IEEE division)
//
// the same operations the matmul kernels apply to X when they get s, so a
// matmul on folded activations equals, bit for bit, the one on X and s.  One
// HBM pass: 16-byte loads of a and s, 16-byte stores, grid-stride over
// 8-channel chunks.
#include "awq_kernels.cuh"

namespace awq {

namespace {

__global__ void __launch_bounds__(256) fold_inverse_scale_kernel(const __half *__restrict__ a,
                                                                 const __half *__restrict__ s,
                                                                 int64_t chunks, int kchunks,
                                                                 __half *__restrict__ out,
                                                                 int32_t *status)
{
    bool bad = false;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < chunks; i += stride) {
        const int kc = static_cast<int>(i % kchunks);
        const uint4 av = __ldg(reinterpret_cast<const uint4 *>(a) + i);
        const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(s) + kc);
        const __half *ah = reinterpret_cast<const __half *>(&av);
        const __half *sh = reinterpret_cast<const __half *>(&sv);
        uint4 r;
        uint16_t *o = reinterpret_cast<uint16_t *>(&r);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float sj = __half2float(sh[j]);
            bad |= !(sj > 0.0f) || !isfinite(sj);
            o[j] = __half_as_ushort(__float2half_rn(__fdiv_rn(__half2float(ah[j]), sj)));
        }
        reinterpret_cast<uint4 *>(out)[i] = r;
    }
    if (bad) report(status, AWQ_ERR_NONFINITE);
}

}  // namespace

cudaError_t launch_fold_inverse_scale(const __half *a, int64_t rows, int K, const __half *s,
                                      __half *out, int32_t *status, int num_sms, cudaStream_t st)
{
    const int kchunks = K / 8;
    const int64_t chunks = rows * kchunks;
    int64_t blocks = (chunks + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    fold_inverse_scale_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(a, s, chunks, kchunks, out,
                                                                            status);
    return cudaGetLastError();
}

}  // namespace awq
