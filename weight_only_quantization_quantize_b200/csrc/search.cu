// search.cu -- the scale search over alpha on the GPU: the per-channel scale
// chosen by the output error of the quantized layer on calibration rows.
//
// Sources: "Awq Quantization" (skillselion.com), "How AWQ Works": s is chosen
// to make L(s) = ||Q(W*s)(s^-1*X) - W*X|| small; lansai AWQ explainer
// (ai.lansai.wang/107648), "AWQ 的四步链路", row "搜索缩放" (evaluate the effect
// of different channel scalings on the reconstruction error).  The pages give
// neither the family nor the grid; this library reads them as
//   family   s(alpha) = m^alpha, normalised by the geometric centre of its
//            extremes (alpha = 1/2 is awq_compute_scales)
//   grid     alpha = j/8, j = 0..8, with m^alpha formed by one fixed chain of
//            IEEE double operations: u = max(m, 1e-8), r1 = sqrt(u),
//            r2 = sqrt(r1), r3 = sqrt(r2); t = u for j = 8, otherwise the
//            product of r1, r2, r3 chosen by the bits 4, 2, 1 of j, in that
//            order; s = binary16_RNE(t / sqrt(max t * min t))
//   loss     L(j) = sum over calibration rows and outputs of (Yq - Y)^2 in
//            double, Yq the quantized layer's output (the library's own
//            quantizer and matmul) and Y = X W
//   choice   the smallest j with the minimum loss.
//
// Kernels here: the scales of one grid point (bit-exact, one rounding), a
// transpose of W (so that the unquantized product can take both operands
// K-major), that product on the tcgen05 tensor cores with a float result, and
// the two-pass fixed-order loss reduction.  The quantizer and the W4A16 matmul
// are the library's own kernels.
#include "awq_kernels.cuh"

namespace awq {

namespace {

// m^(j/8) by the fixed chain (each operation correctly rounded, so the value is
// reproducible bit for bit, and monotone non-decreasing in m).
__device__ __forceinline__ double alpha_t(float mk, int j)
{
    const double u = fmax(static_cast<double>(mk), 1e-8);
    if (j == 8) return u;
    const double r1 = __dsqrt_rn(u);
    const double r2 = __dsqrt_rn(r1);
    const double r3 = __dsqrt_rn(r2);
    double v = 1.0;
    if (j & 4) v = __dmul_rn(v, r1);
    if (j & 2) v = __dmul_rn(v, r2);
    if (j & 1) v = __dmul_rn(v, r3);
    return v;
}

// s(j) for all K channels.  Every block finds max m and min m itself (t is
// monotone in m, so the extreme t are those of the extreme m, bit for bit) and
// rounds its own 1024 channels.  j comes from jptr when it is not NULL.
__global__ void __launch_bounds__(1024) scales_alpha_kernel(const float *__restrict__ m, int K, int j,
                                                           const int32_t *jptr, uint16_t *__restrict__ s,
                                                           int32_t *status)
{
    __shared__ float smax[32], smin[32];
    __shared__ int sbad;
    if (threadIdx.x == 0) sbad = 0;
    __syncthreads();
    const int jj = jptr ? *jptr : j;
    float mx = 0.0f, mn = INFINITY;
    bool bad = false;
    for (int k0 = threadIdx.x; k0 < K; k0 += 8 * blockDim.x) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int k = k0 + u * blockDim.x;
            v[u] = k < K ? m[k] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (k0 + u * blockDim.x >= K) continue;
            if (!isfinite(v[u]) || v[u] < 0.0f) {
                bad = true;
                continue;
            }
            mx = fmaxf(mx, v[u]);
            mn = fminf(mn, v[u]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        smax[warp] = mx;
        smin[warp] = mn;
    }
    if (bad) atomicOr(&sbad, 1);
    __syncthreads();
    if (warp == 0) {
        const int nw = (blockDim.x + 31) >> 5;
        mx = lane < nw ? smax[lane] : 0.0f;
        mn = lane < nw ? smin[lane] : INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        if (lane == 0) {
            smax[0] = mx;
            smin[0] = mn;
        }
    }
    __syncthreads();
    if (sbad || jj < 0 || jj > 8) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report(status, AWQ_ERR_NONFINITE);
        return;
    }
    const double c = __dsqrt_rn(__dmul_rn(alpha_t(smax[0], jj), alpha_t(smin[0], jj)));
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k < K) s[k] = double_to_half_rn(__ddiv_rn(alpha_t(m[k], jj), c));
}

// WT[n, k] = W[k, n] (binary16 bits), 32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256) transpose_kernel(const uint16_t *__restrict__ W, int K, int N,
                                                       uint16_t *__restrict__ WT)
{
    __shared__ uint16_t tile[32][33];
    const int n0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
    for (int r = threadIdx.y; r < 32; r += 8) {
        const int k = k0 + r, n = n0 + threadIdx.x;
        if (k < K && n < N) tile[r][threadIdx.x] = W[static_cast<size_t>(k) * N + n];
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += 8) {
        const int n = n0 + r, k = k0 + threadIdx.x;
        if (k < K && n < N) WT[static_cast<size_t>(n) * K + k] = tile[threadIdx.x][r];
    }
}

// ------------------------------------------------------------------ Y = X W (float out)
// One CTA computes a 128 x 256 tile of Y on the tcgen05 tensor cores; both
// operands arrive K-major through TMA (X [R, K] and WT [N, K], 128-byte
// swizzle), the accumulator lives in 256 TMEM columns.
//   warp 0      TMA producer, 4-stage ring (16 KB of X + 32 KB of WT per stage)
//   warp 1      TMEM allocation; one lane issues tcgen05.mma (128 x 256 x 16)
//               x 4 per stage and commits each stage back to the ring
//   warps 2..5  read the accumulator (tcgen05.ld) and write float Y
constexpr int kDBM = 128, kDBN = 256, kDBK = 64, kDStages = 4;
constexpr int kDABytes = kDBM * kDBK * 2;
constexpr int kDBBytes = kDBN * kDBK * 2;
constexpr int kDStageBytes = kDABytes + kDBBytes;
constexpr int kDThreads = 192;
constexpr uint32_t kDIdesc = tc_idesc_f16(kDBM, kDBN);
constexpr size_t kDSmem = 1024 + static_cast<size_t>(kDStages) * kDStageBytes + 256;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__global__ void __launch_bounds__(kDThreads, 1)
    dense_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWT,
                      float *__restrict__ Y, int R, int K, int N, int32_t *status)
{
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kDStages * kDStageBytes);
    uint64_t *empty = full + kDStages;
    uint64_t *tmem_full = empty + kDStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tmem_full + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kDBN, m0 = blockIdx.y * kDBM;
    const int KB = K / kDBK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(tmem_full, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kDBN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmWT);
            for (int kb = 0; kb < KB; ++kb) {
                const int st = kb % kDStages;
                if (kb >= kDStages && !mbar_wait(&empty[st], ((kb / kDStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                uint8_t *stg = smem + st * kDStageBytes;
                mbar_arrive_expect_tx(&full[st], kDStageBytes);
                tma_load_2d(stg, &tmX, &full[st], kb * kDBK, m0);
                tma_load_2d(stg + kDABytes, &tmWT, &full[st], kb * kDBK, n0);
            }
            if (!ok) report(status, AWQ_ERR_DEVICE_TIMEOUT);
        }
    } else if (warp == 1) {
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kDStages;
            if (!mbar_wait(&full[st], (kb / kDStages) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a0 = smem_u32(smem + st * kDStageBytes);
                const uint32_t b0 = a0 + kDABytes;
#pragma unroll
                for (int k = 0; k < kDBK / 16; ++k)
                    tc_mma(tmem_base, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), kDIdesc,
                           (kb > 0 || k > 0) ? 1u : 0u);
                tc_commit(&empty[st]);
            }
            __syncwarp();
        }
        if (lane == 0) {
            if (ok)
                tc_commit(tmem_full);
            else
                report(status, AWQ_ERR_DEVICE_TIMEOUT);
        }
        __syncwarp();
    } else {
        if (mbar_wait(tmem_full, 0)) {
            tc_fence_after();
            const int quarter = warp & 3;
            const int m = m0 + quarter * 32 + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < kDBN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + c0, v);
                if (m < R) {
                    float *dst = Y + static_cast<size_t>(m) * N + n0 + c0;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (n0 + c0 + 4 * i < N)
                            *reinterpret_cast<float4 *>(dst + 4 * i) =
                                make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                            __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
                }
            }
        } else if (lane == 0) {
            report(status, AWQ_ERR_DEVICE_TIMEOUT);
        }
    }
    // a producer that gave up may have copies in flight: let them land
    if (warp == 0 && lane == 0 && !ok)
        for (int st = 0; st < kDStages; ++st) mbar_wait(&full[st], 0);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kDBN)
                     : "memory");
    }
}

// ------------------------------------------------------------------ loss
// sum (Yq - Y)^2 in double: block b adds its contiguous share in a fixed order
// (strided per thread, then a fixed tree), the final pass adds the blocks'
// partial sums in block order, so the loss has the same bits on every run.
constexpr int kLossBlocks = 256;

__global__ void __launch_bounds__(256) sq_err_partial_kernel(const __half *__restrict__ Yq,
                                                            const float *__restrict__ Yr, int64_t n,
                                                            double *__restrict__ partial)
{
    __shared__ double sm[256];
    const int64_t lo = static_cast<int64_t>(blockIdx.x) * n / kLossBlocks;
    const int64_t hi = static_cast<int64_t>(blockIdx.x + 1) * n / kLossBlocks;
    double acc = 0.0;
    for (int64_t i = lo + threadIdx.x; i < hi; i += 256) {
        const double d = static_cast<double>(__half2float(Yq[i])) - static_cast<double>(Yr[i]);
        acc = fma(d, d, acc);
    }
    sm[threadIdx.x] = acc;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if (threadIdx.x < s) sm[threadIdx.x] += sm[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) partial[blockIdx.x] = sm[0];
}

__global__ void __launch_bounds__(32) sq_err_final_kernel(const double *__restrict__ partial,
                                                         double *__restrict__ loss)
{
    if (threadIdx.x == 0) {
        double acc = 0.0;
        for (int b = 0; b < kLossBlocks; ++b) acc += partial[b];
        *loss = acc;
    }
}

// j_best = the smallest j whose loss is the minimum.
__global__ void __launch_bounds__(32) pick_best_kernel(const double *__restrict__ losses, int32_t *j_best)
{
    if (threadIdx.x == 0) {
        double best = INFINITY;
        int jb = 0;
        for (int j = 0; j <= 8; ++j)
            if (losses[j] < best) {
                best = losses[j];
                jb = j;
            }
        *j_best = jb;
    }
}

}  // namespace

size_t loss_partial_bytes() { return kLossBlocks * sizeof(double); }

cudaError_t configure_search()
{
    return cudaFuncSetAttribute(dense_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kDSmem));
}

cudaError_t launch_scales_alpha(const float *m, int K, int j, const int32_t *jptr, uint16_t *s, int32_t *status,
                                cudaStream_t st)
{
    scales_alpha_kernel<<<(K + 1023) / 1024, 1024, 0, st>>>(m, K, j, jptr, s, status);
    return cudaGetLastError();
}

cudaError_t launch_transpose(const uint16_t *W, int K, int N, uint16_t *WT, cudaStream_t st)
{
    transpose_kernel<<<dim3((N + 31) / 32, (K + 31) / 32), dim3(32, 8), 0, st>>>(W, K, N, WT);
    return cudaGetLastError();
}

cudaError_t launch_dense_gemm(const CUtensorMap &tmX, const CUtensorMap &tmWT, float *Y, int R, int K, int N,
                              int32_t *status, cudaStream_t st)
{
    dim3 grid((N + kDBN - 1) / kDBN, (R + kDBM - 1) / kDBM);
    dense_gemm_kernel<<<grid, kDThreads, kDSmem, st>>>(tmX, tmWT, Y, R, K, N, status);
    return cudaGetLastError();
}

cudaError_t launch_sq_err(const __half *Yq, const float *Yr, int64_t n, double *partial, double *loss,
                          cudaStream_t st)
{
    sq_err_partial_kernel<<<kLossBlocks, 256, 0, st>>>(Yq, Yr, n, partial);
    sq_err_final_kernel<<<1, 32, 0, st>>>(partial, loss);
    return cudaGetLastError();
}

cudaError_t launch_pick_best(const double *losses, int32_t *j_best, cudaStream_t st)
{
    pick_best_kernel<<<1, 32, 0, st>>>(losses, j_best);
    return cudaGetLastError();
}

}  // namespace awq
