// quantize.cu -- activation statistics, per-channel scales, and the fused
// fold + asymmetric 4-bit group quantization + packing (sm_100a).
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (collect input magnitudes, Y = (X/s)(sW), quantize and pack by bits/group/
// zero point); "Awq Quantization" (skillselion.com), "Group Size
// Configuration" and "Zero-Point Quantization".
//
// All three kernels are HBM-streaming passes; every floating-point decision
// that selects a stored bit (a code, a zero point, a binary16 rounding) is
// made with correctly rounded IEEE operations (__fdiv_rn, __fsub_rn,
// __dsqrt_rn, ...), so the outputs are bit-exact functions of the inputs.
#include "awq_kernels.cuh"

namespace awq {

// ------------------------------------------------------------------ act_stats
// Block: 16 column chunks (8 channels each, one 16-byte load) x 16 row slices.
// |x| is accumulated in double: every binary16 is a multiple of 2^-24 below
// 2^16, so with R <= 8192 rows each partial and total sum is an exact double
// and the order of the reduction cannot change the result.
__global__ void __launch_bounds__(256) act_stats_kernel(const __half *__restrict__ xcal, int R,
                                                       int K, float *__restrict__ m,
                                                       int32_t *status)
{
    __shared__ double part[16][129];
    const int cc = threadIdx.x & 15;
    const int rs = threadIdx.x >> 4;
    const int k0 = blockIdx.x * 128 + cc * 8;
    double acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0;
    bool bad = false;
    if (k0 < K) {
        for (int r = rs; r < R; r += 16) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xcal + (size_t)r * K + k0));
            const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(h[j]);
                bad |= !isfinite(f.x) || !isfinite(f.y);
                acc[2 * j] += fabs(static_cast<double>(f.x));
                acc[2 * j + 1] += fabs(static_cast<double>(f.y));
            }
        }
    }
    if (bad) report(status, AWQ_ERR_NONFINITE);
#pragma unroll
    for (int j = 0; j < 8; ++j) part[rs][cc * 8 + j] = acc[j];
    __syncthreads();
    if (threadIdx.x < 128) {
        const int k = blockIdx.x * 128 + threadIdx.x;
        if (k < K) {
            double s = 0.0;
#pragma unroll
            for (int i = 0; i < 16; ++i) s += part[i][threadIdx.x];
            m[k] = __double2float_rn(__ddiv_rn(s, static_cast<double>(R)));
        }
    }
}

// ------------------------------------------------------------------ compute_scales
// Round a positive finite double to the nearest binary16, ties to even, in a
// single rounding (IEEE 754 binary16: quantum 2^(e-10) in the binade
// [2^e, 2^(e+1)), never finer than the subnormal quantum 2^-24).
__device__ uint16_t double_to_half_rn(double x)
{
    if (!(x < 65520.0)) return 0x7C00;  // rounds to +inf (x >= 65520)
    if (x == 0.0) return 0;
    const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
    int e = static_cast<int>((b >> 52) & 0x7FF) - 1023;  // x normal in double here
    int q = e - 10;
    if (q < -24) q = -24;
    const double inv_quantum = __longlong_as_double(static_cast<long long>(1023 - q) << 52);
    const double n = rint(__dmul_rn(x, inv_quantum));  // exact scaling, then RNE
    return static_cast<uint16_t>(((q + 24) << 10) + static_cast<int>(n));
}

__device__ __forceinline__ double scale_t(float mk)
{
    return __dsqrt_rn(fmax(static_cast<double>(mk), 1e-8));
}

// One block of 1024 threads: a min/max pass, then the rounding pass.
__global__ void __launch_bounds__(1024) compute_scales_kernel(const float *__restrict__ m, int K,
                                                             uint16_t *__restrict__ s,
                                                             int32_t *status)
{
    __shared__ double smax[32], smin[32];
    __shared__ int sbad;
    if (threadIdx.x == 0) sbad = 0;
    __syncthreads();
    double tmax = 0.0, tmin = INFINITY;
    bool bad = false;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float mk = m[k];
        if (!isfinite(mk) || mk < 0.0f) {
            bad = true;
            continue;
        }
        const double t = scale_t(mk);
        tmax = fmax(tmax, t);
        tmin = fmin(tmin, t);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tmax = fmax(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        tmin = fmin(tmin, __shfl_xor_sync(0xffffffffu, tmin, o));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        smax[warp] = tmax;
        smin[warp] = tmin;
    }
    if (bad) atomicOr(&sbad, 1);
    __syncthreads();
    if (warp == 0) {
        const int nw = (blockDim.x + 31) >> 5;
        tmax = lane < nw ? smax[lane] : 0.0;
        tmin = lane < nw ? smin[lane] : INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            tmax = fmax(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
            tmin = fmin(tmin, __shfl_xor_sync(0xffffffffu, tmin, o));
        }
        if (lane == 0) {
            smax[0] = tmax;
            smin[0] = tmin;
        }
    }
    __syncthreads();
    if (sbad) {
        if (threadIdx.x == 0) report(status, AWQ_ERR_NONFINITE);
        return;
    }
    const double c = __dsqrt_rn(__dmul_rn(smax[0], smin[0]));
    for (int k = threadIdx.x; k < K; k += blockDim.x)
        s[k] = double_to_half_rn(__ddiv_rn(scale_t(m[k]), c));
}

// ------------------------------------------------------------------ quantize_pack
// rint(fl(w / sf)), the code decision, without a division per weight.
// y = fl(w * fl(1/sf)) differs from the IEEE quotient by at most
// |w/sf| * (2^-23 + 2^-24 + 2^-47) < |y| * 2^-21.  Both values round to the same
// integer whenever y lies farther than that from the nearest tie point k + 1/2;
// otherwise (rarely) the correctly rounded quotient decides.
__device__ __forceinline__ int rint_quotient(float w, float sf, float rsf)
{
    const float y = __fmul_rn(w, rsf);
    const float tie = floorf(y) + 0.5f;
    if (fabsf(y - tie) > fmaf(fabsf(y), 0x1p-21f, 0x1p-60f)) return __float2int_rn(y);
    return __float2int_rn(__fdiv_rn(w, sf));
}

// Block = one 128-row group x 256 columns.  Warp w owns rows 16w..16w+15 of
// the group; lane l owns columns 8l..8l+7, so every row is read as one
// 512-byte coalesced warp load.  The per-column min/max is reduced across the
// 8 warps in shared memory, every thread derives (scale, zero) for its 8
// columns, encodes its 16 x 8 codes and writes two packed rows of 8 words.
__global__ void __launch_bounds__(256) quantize_pack_kernel(const __half *__restrict__ W,
                                                           const __half *__restrict__ s, int K,
                                                           int N, int32_t *__restrict__ Q,
                                                           __half *__restrict__ scales,
                                                           int32_t *__restrict__ zeros,
                                                           int32_t *status)
{
    __shared__ float red_max[8][256];
    __shared__ float red_min[8][256];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = blockIdx.y;
    const int n = blockIdx.x * 256 + lane * 8;
    const int k0 = g * kGroup + warp * 16;
    const bool active = n < N;

    // per-row channel scale (same for every lane: broadcast loads)
    float sk[16];
    bool bad = false;
    {
        const uint4 s0 = __ldg(reinterpret_cast<const uint4 *>(s + k0));
        const uint4 s1 = __ldg(reinterpret_cast<const uint4 *>(s + k0 + 8));
        const __half *h0 = reinterpret_cast<const __half *>(&s0);
        const __half *h1 = reinterpret_cast<const __half *>(&s1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            sk[j] = __half2float(h0[j]);
            sk[8 + j] = __half2float(h1[j]);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) bad |= !isfinite(sk[j]) || !(sk[j] > 0.0f);
    }

    // The raw binary16 rows stay in registers; the folded value w' = w * s_k
    // (exact in float: 11 x 11 significant bits) is recomputed where needed.
    uint4 raw[16];
    float mx[8], mn[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        mx[c] = -INFINITY;
        mn[c] = INFINITY;
    }
    if (active) {
#pragma unroll
        for (int r = 0; r < 16; ++r)
            raw[r] = __ldg(reinterpret_cast<const uint4 *>(W + (size_t)(k0 + r) * N + n));
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const __half *h = reinterpret_cast<const __half *>(&raw[r]);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float v = __fmul_rn(__half2float(h[c]), sk[r]);
                bad |= !isfinite(v);
                mx[c] = fmaxf(mx[c], v);
                mn[c] = fminf(mn[c], v);
            }
        }
    }
    if (bad && active) report(status, AWQ_ERR_NONFINITE);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        red_max[warp][lane * 8 + c] = mx[c];
        red_min[warp][lane * 8 + c] = mn[c];
    }
    __syncthreads();
    if (!active) return;

    float sf[8], rsf[8];
    int zc[8];
    uint16_t sh[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float a = red_max[0][lane * 8 + c], b = red_min[0][lane * 8 + c];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            a = fmaxf(a, red_max[i][lane * 8 + c]);
            b = fminf(b, red_min[i][lane * 8 + c]);
        }
        float r = __fsub_rn(a, b);
        if (r < 1e-5f) r = 1e-5f;
        uint16_t bits = __half_as_ushort(__float2half_rn(__fdiv_rn(r, 15.0f)));
        if ((bits & 0x7FFF) == 0) bits = 1;  // never a zero step
        sh[c] = bits;
        sf[c] = __half2float(__ushort_as_half(bits));
        rsf[c] = __frcp_rn(sf[c]);
        float zf = rintf(__fdiv_rn(-b, sf[c]));
        zf = fminf(fmaxf(zf, 0.0f), 15.0f);
        zc[c] = static_cast<int>(zf);
    }

    uint32_t word[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t acc = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const __half *hr = reinterpret_cast<const __half *>(&raw[h * 8 + j]);
                const float v = __fmul_rn(__half2float(hr[c]), sk[h * 8 + j]);
                int q = rint_quotient(v, sf[c], rsf[c]) + zc[c];
                q = min(max(q, 0), 15);
                acc |= static_cast<uint32_t>(q) << (4 * j);
            }
            word[h][c] = acc;
        }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        int32_t *dst = Q + (size_t)(k0 / 8 + h) * N + n;
        reinterpret_cast<uint4 *>(dst)[0] = make_uint4(word[h][0], word[h][1], word[h][2], word[h][3]);
        reinterpret_cast<uint4 *>(dst)[1] = make_uint4(word[h][4], word[h][5], word[h][6], word[h][7]);
    }
    if (warp == 0) {
        uint4 sv;
        sv.x = sh[0] | (static_cast<uint32_t>(sh[1]) << 16);
        sv.y = sh[2] | (static_cast<uint32_t>(sh[3]) << 16);
        sv.z = sh[4] | (static_cast<uint32_t>(sh[5]) << 16);
        sv.w = sh[6] | (static_cast<uint32_t>(sh[7]) << 16);
        *reinterpret_cast<uint4 *>(scales + (size_t)g * N + n) = sv;
        uint32_t zw = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) zw |= static_cast<uint32_t>(zc[c]) << (4 * c);
        zeros[(size_t)g * (N / 8) + n / 8] = static_cast<int32_t>(zw);
    }
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_act_stats(const __half *xcal, int R, int K, float *m, int32_t *status,
                             cudaStream_t st)
{
    act_stats_kernel<<<(K + 127) / 128, 256, 0, st>>>(xcal, R, K, m, status);
    return cudaGetLastError();
}

cudaError_t launch_compute_scales(const float *m, int K, uint16_t *s, int32_t *status,
                                  cudaStream_t st)
{
    compute_scales_kernel<<<1, 1024, 0, st>>>(m, K, s, status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_pack(const __half *W, const __half *s, int K, int N, int32_t *Q,
                                 __half *scales, int32_t *zeros, int32_t *status, cudaStream_t st)
{
    dim3 grid((N + 255) / 256, K / kGroup);
    quantize_pack_kernel<<<grid, 256, 0, st>>>(W, s, K, N, Q, scales, zeros, status);
    return cudaGetLastError();
}

}  // namespace awq
