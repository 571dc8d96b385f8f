// clip.cu -- weight clipping: per group and column, the shrink of the
// quantization range that minimizes the group's output error on calibration
// rows, then the codes of that choice.
//
// Source: "Awq Quantization" (skillselion.com), calibration parameters:
// apply_clip ("Apply weight clipping"); the page names only the flag.  This
// library reads it as (per group g of 128 rows and column n, w' = w * s_k):
//   candidates  c_i = 1 - i/20, i < n_cand (n_cand <= 11, down to c = 1/2;
//               c_0 = 1 is no clipping)
//   clipped     the range [c min w', c max w'] gives the step and zero point
//               exactly as awq_quantize_pack does for [min w', max w']; every
//               weight of the group is coded on that grid (clamping)
//   loss        sum over calibration rows r of (sum_{k in g} x'_rk e_k)^2,
//               x' = x / s_k, e = (q - z) step - w' (the group's share of the
//               output error)
//   choice      the first candidate (largest c) with the minimum loss.
//
// One CTA = one group x 32 columns:
//   1. per column the range of w' (exact), per candidate the step and zero
//      point (the quantizer's IEEE float operations, bit for bit), and the
//      error vectors e (float) of all 11 x 32 candidate columns in shared memory;
//   2. calibration rows in chunks of 64: X' = x / s (float) staged in shared
//      memory; each thread owns one row and runs eight candidate columns at a
//      time (float FMA over the 128 k), squares, and the rows' squares are
//      added per warp (fixed butterfly) and per chunk in a fixed order;
//   3. the first minimum per column; steps, zero points, codes and the chosen
//      index are written.
// The loss is float (the oracle's is double), so a choice can differ only
// where two candidates' losses agree to float rounding.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kCTN = 32;        // columns per CTA
constexpr int kCRows = 64;      // calibration rows per chunk
constexpr int kCMaxCand = 11;
constexpr int kCThreads = 256;
constexpr int kXpStride = 132;  // floats per staged row (padding: conflict-free row-wise loads)
constexpr int kPairs = kCMaxCand * kCTN;

struct ClipSmem {
    float e[kCMaxCand * kCTN * kGroup];  // [candidate][column][k]
    float xp[kCRows * kXpStride];        // [row][k]
    float part[2][kPairs];               // per warp half of the 64 rows
    float loss[kPairs];
    float mx[8][kCTN], mn[8][kCTN];
    uint16_t sh[kPairs];
    uint8_t zz[kPairs];
    int best[kCTN];
    int bad;
};

struct ClipParams {
    const __half *W;
    const __half *s;
    const __half *xcal;
    int32_t *Q;
    __half *scales;
    int32_t *zeros;
    int32_t *ratio;
    int32_t *status;
    int R, K, N, n_cand;
};

__device__ __forceinline__ float h2f_bits(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// step and zero point of the range [lo, hi] (the quantizer's float operations)
__device__ __forceinline__ void group_params(float lo, float hi, uint16_t &sh, int &z)
{
    float r = __fsub_rn(hi, lo);
    if (r < 1e-5f) r = 1e-5f;
    sh = __half_as_ushort(__float2half_rn(__fdiv_rn(r, 15.0f)));
    if ((sh & 0x7FFF) == 0) sh = 1;
    float zf = rintf(__fdiv_rn(-lo, h2f_bits(sh)));
    zf = fminf(fmaxf(zf, 0.0f), 15.0f);
    z = static_cast<int>(zf);
}

__device__ __forceinline__ int code_of(float w, uint16_t sh, int z)
{
    int q = static_cast<int>(rintf(__fdiv_rn(w, h2f_bits(sh)))) + z;
    return q < 0 ? 0 : (q > 15 ? 15 : q);
}

__global__ void __launch_bounds__(kCThreads, 1) clip_kernel(const ClipParams p)
{
    extern __shared__ uint8_t smem_raw[];
    ClipSmem &sm = *reinterpret_cast<ClipSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.y;
    const int n0 = blockIdx.x * kCTN;
    const int nc = p.n_cand;
    const int k0 = g * kGroup;
    if (tid == 0) sm.bad = 0;

    // ---------------------------------------------------------------- 1. ranges, parameters, errors
    // thread: column n = tid % 32, rows 16 * (tid / 32) .. +15
    {
        const int n = tid & 31, part = tid >> 5;
        float mx = -INFINITY, mn = INFINITY;
        bool bad = false;
        if (n0 + n < p.N) {
            for (int kk = part * 16; kk < part * 16 + 16; ++kk) {
                const float w = __half2float(p.W[static_cast<size_t>(k0 + kk) * p.N + n0 + n]);
                const float sk = __half2float(p.s[k0 + kk]);
                bad |= !isfinite(w) || !isfinite(sk) || !(sk > 0.0f);
                const float wp = __fmul_rn(w, sk);
                mx = fmaxf(mx, wp);
                mn = fminf(mn, wp);
            }
        }
        sm.mx[part][n] = mx;
        sm.mn[part][n] = mn;
        if (bad) atomicOr(&sm.bad, 1);
    }
    __syncthreads();
    for (int pr = tid; pr < nc * kCTN; pr += kCThreads) {
        const int i = pr / kCTN, n = pr - i * kCTN;
        float mx = sm.mx[0][n], mn = sm.mn[0][n];
        for (int q = 1; q < 8; ++q) {
            mx = fmaxf(mx, sm.mx[q][n]);
            mn = fminf(mn, sm.mn[q][n]);
        }
        const float c = __fsub_rn(1.0f, __fdiv_rn(static_cast<float>(i), 20.0f));
        uint16_t sh = 1;
        int z = 0;
        if (n0 + n < p.N) group_params(__fmul_rn(c, mn), __fmul_rn(c, mx), sh, z);
        sm.sh[pr] = sh;
        sm.zz[pr] = static_cast<uint8_t>(z);
    }
    __syncthreads();
    for (int idx = tid; idx < nc * kCTN * kGroup; idx += kCThreads) {
        const int kk = idx & (kGroup - 1);
        const int pr = idx >> 7;
        const int n = pr % kCTN;
        float e = 0.0f;
        if (n0 + n < p.N) {
            const float w = __half2float(p.W[static_cast<size_t>(k0 + kk) * p.N + n0 + n]);
            const float wp = __fmul_rn(w, __half2float(p.s[k0 + kk]));
            const uint16_t sh = sm.sh[pr];
            const int z = sm.zz[pr];
            const float what = __fmul_rn(static_cast<float>(code_of(wp, sh, z) - z), h2f_bits(sh));
            e = __fsub_rn(what, wp);
        }
        sm.e[idx] = e;
    }
    for (int pr = tid; pr < nc * kCTN; pr += kCThreads) sm.loss[pr] = 0.0f;
    __syncthreads();
    if (sm.bad) {
        if (tid == 0) report(p.status, AWQ_ERR_NONFINITE);
        return;
    }

    // ---------------------------------------------------------------- 2. losses over the calibration rows
    const int rr = lane + 32 * (warp & 1);  // this thread's row within the chunk
    const int pg = warp >> 1;               // pair group: pairs pg, pg + 4, pg + 8, ...
    const int npairs = nc * kCTN;
    bool xbad = false;
    for (int r0 = 0; r0 < p.R; r0 += kCRows) {
        // stage X' = x / s for rows r0 .. r0 + 63 (zeros past R)
        for (int idx = tid; idx < kCRows * 16; idx += kCThreads) {
            const int row = idx >> 4, c8 = idx & 15;
            const int r = r0 + row;
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (r < p.R) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(p.xcal + static_cast<size_t>(r) * p.K + k0 + c8 * 8));
                const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(p.s + k0 + c8 * 8));
                const __half *xh = reinterpret_cast<const __half *>(&xv);
                const __half *shh = reinterpret_cast<const __half *>(&sv);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    v[j] = __fdiv_rn(__half2float(xh[j]), __half2float(shh[j]));
                    xbad |= !isfinite(v[j]);
                }
            }
            float4 *dst = reinterpret_cast<float4 *>(&sm.xp[row * kXpStride + c8 * 8]);
            dst[0] = make_float4(v[0], v[1], v[2], v[3]);
            dst[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
        __syncthreads();
        const float *xrow = &sm.xp[rr * kXpStride];
        for (int b = pg; b < npairs; b += 32) {
            // eight candidate columns b, b + 4, ..., b + 28 (those below npairs)
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const float *ep[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int pr = b + 4 * j;
                ep[j] = &sm.e[(pr < npairs ? pr : 0) * kGroup];
            }
#pragma unroll 2
            for (int kk = 0; kk < kGroup; kk += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(xrow + kk);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 e = *reinterpret_cast<const float4 *>(ep[j] + kk);
                    acc[j] = fmaf(x.x, e.x, acc[j]);
                    acc[j] = fmaf(x.y, e.y, acc[j]);
                    acc[j] = fmaf(x.z, e.z, acc[j]);
                    acc[j] = fmaf(x.w, e.w, acc[j]);
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float y2 = acc[j] * acc[j];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) y2 += __shfl_xor_sync(0xffffffffu, y2, o);
                const int pr = b + 4 * j;
                if (lane == 0 && pr < npairs) sm.part[warp & 1][pr] = y2;
            }
        }
        __syncthreads();
        for (int pr = tid; pr < npairs; pr += kCThreads) sm.loss[pr] += sm.part[0][pr] + sm.part[1][pr];
        __syncthreads();
    }
    if (xbad) atomicOr(&sm.bad, 1);
    __syncthreads();
    if (sm.bad) {
        if (tid == 0) report(p.status, AWQ_ERR_NONFINITE);
        return;
    }

    // ---------------------------------------------------------------- 3. choice and outputs
    if (tid < kCTN) {
        int bi = 0;
        float best = sm.loss[tid];
        for (int i = 1; i < nc; ++i) {
            const float l = sm.loss[i * kCTN + tid];
            if (l < best) {
                best = l;
                bi = i;
            }
        }
        sm.best[tid] = bi;
        const int n = n0 + tid;
        if (n < p.N) {
            p.scales[static_cast<size_t>(g) * p.N + n] = __ushort_as_half(sm.sh[bi * kCTN + tid]);
            if (p.ratio) p.ratio[static_cast<size_t>(g) * p.N + n] = bi;
        }
    }
    __syncthreads();
    if (tid < kCTN / 8) {
        const int n = n0 + 8 * tid;
        if (n < p.N) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = 8 * tid + j;
                word |= static_cast<uint32_t>(sm.zz[sm.best[c] * kCTN + c]) << (4 * j);
            }
            p.zeros[static_cast<size_t>(g) * (p.N / 8) + n / 8] = static_cast<int32_t>(word);
        }
    }
    // codes: 16 packed rows x 32 columns, consecutive threads on consecutive columns
    for (int idx = tid; idx < 16 * kCTN; idx += kCThreads) {
        const int w = idx / kCTN, c = idx - w * kCTN;
        const int n = n0 + c;
        if (n >= p.N) continue;
        const int pr = sm.best[c] * kCTN + c;
        const uint16_t sh = sm.sh[pr];
        const int z = sm.zz[pr];
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = k0 + 8 * w + j;
            const float wp = __fmul_rn(__half2float(p.W[static_cast<size_t>(k) * p.N + n]), __half2float(p.s[k]));
            word |= static_cast<uint32_t>(code_of(wp, sh, z)) << (4 * j);
        }
        p.Q[static_cast<size_t>(g * 16 + w) * p.N + n] = static_cast<int32_t>(word);
    }
}

}  // namespace

cudaError_t configure_clip()
{
    return cudaFuncSetAttribute(clip_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(ClipSmem)));
}

cudaError_t launch_clip(const __half *W, const __half *s, const __half *xcal, int R, int K, int N, int n_cand,
                        int32_t *Q, __half *scales, int32_t *zeros, int32_t *ratio, int32_t *status,
                        cudaStream_t st)
{
    ClipParams prm{W, s, xcal, Q, scales, zeros, ratio, status, R, K, N, n_cand};
    dim3 grid((N + kCTN - 1) / kCTN, K / kGroup);
    clip_kernel<<<grid, kCThreads, sizeof(ClipSmem), st>>>(prm);
    return cudaGetLastError();
}

}  // namespace awq
