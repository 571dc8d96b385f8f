// quantize.cu -- activation statistics, per-channel scales, and the fused
// fold + 4-bit group quantization + packing (sm_100a): asymmetric with a
// per-group zero point, or symmetric ("Zero-Point Quantization" with
// zero_point False: step = fp16(max(max|w'|, 1e-5) / 7), zero point 8, no
// zeros tensor written).
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
// Block: 16 column chunks (8 channels each, one 16-byte load) x 64 row slices.
// |x| is accumulated in double: every binary16 is a multiple of 2^-24 below
// 2^16, so with R <= 8192 rows each partial and total sum is an exact double
// and the order of the reduction cannot change the result.  Each thread keeps
// four rows' loads in flight.
__global__ void __launch_bounds__(1024) act_stats_kernel(const __half *__restrict__ xcal, int R,
                                                        int K, float *__restrict__ m,
                                                        int32_t *status)
{
    constexpr int kSlices = 64;
    __shared__ double part[kSlices / 2][129];
    const int cc = threadIdx.x & 15;
    const int rs = threadIdx.x >> 4;
    const int k0 = blockIdx.x * 128 + cc * 8;
    double acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0;
    bool bad = false;
    if (k0 < K) {
        for (int r0 = rs; r0 < R; r0 += 4 * kSlices) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = r0 + u * kSlices;
                v[u] = r < R ? __ldg(reinterpret_cast<const uint4 *>(xcal + (size_t)r * K + k0))
                             : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const __half2 *h = reinterpret_cast<const __half2 *>(&v[u]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __half22float2(h[j]);
                    bad |= !isfinite(f.x) || !isfinite(f.y);
                    acc[2 * j] += fabs(static_cast<double>(f.x));
                    acc[2 * j + 1] += fabs(static_cast<double>(f.y));
                }
            }
        }
    }
    if (bad) report(status, AWQ_ERR_NONFINITE);
    // lanes l and l + 16 hold the same channels for two row slices
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += __shfl_down_sync(0xffffffffu, acc[j], 16);
    if ((threadIdx.x & 16) == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j) part[rs >> 1][cc * 8 + j] = acc[j];
    }
    __syncthreads();
    if (threadIdx.x < 128) {
        const int k = blockIdx.x * 128 + threadIdx.x;
        if (k < K) {
            double s = 0.0;
            for (int i = 0; i < kSlices / 2; ++i) s += part[i][threadIdx.x];
            m[k] = __double2float_rn(__ddiv_rn(s, static_cast<double>(R)));
        }
    }
}

// ------------------------------------------------------------------ compute_scales
__device__ __forceinline__ double scale_t(float mk)
{
    return __dsqrt_rn(fmax(static_cast<double>(mk), 1e-8));
}

// Every block first finds max m and min m over all K channels (plain float
// compares: t = sqrt(max(m, 1e-8)) is monotone, so the largest and smallest t
// are the square roots of the largest and smallest m, bit for bit), then
// rounds its own 1024 channels.  No block depends on another.
__global__ void __launch_bounds__(1024) compute_scales_kernel(const float *__restrict__ m, int K,
                                                             uint16_t *__restrict__ s,
                                                             int32_t *status)
{
    __shared__ float smax[32], smin[32];
    __shared__ int sbad;
    if (threadIdx.x == 0) sbad = 0;
    __syncthreads();
    float mx = 0.0f, mn = INFINITY;
    bool bad = false;
    // eight loads in flight per thread: the scan is bound by L2 latency otherwise
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
            const float mk = v[u];
            if (!isfinite(mk) || mk < 0.0f) {
                bad = true;
                continue;
            }
            mx = fmaxf(mx, mk);
            mn = fminf(mn, mk);
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
    if (sbad) {
        if (threadIdx.x == 0 && blockIdx.x == 0) report(status, AWQ_ERR_NONFINITE);
        return;
    }
    const double c = __dsqrt_rn(__dmul_rn(scale_t(smax[0]), scale_t(smin[0])));
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k < K) s[k] = double_to_half_rn(__ddiv_rn(scale_t(m[k]), c));
}

// ------------------------------------------------------------------ quantize_pack
// Persistent CTAs (one per SM) of two independent halves of 8 warps.  Each half
// walks its own tiles of one 128-row group x 128 columns, fed by its own TMA
// double buffer of 32 KB tiles and synchronised by its own named barrier, so
// one half's per-column phase overlaps the other half's streaming work.  In a
// half, warp w owns rows 16w..16w+15 (packed rows 2w, 2w+1 of the group) and
// lane l owns columns 4l..4l+3: every thread reads 16 x 8 bytes of the tile and
// writes two 16-byte runs of packed words.
//   pass 1  w' = w * s_k (exact: an fma of two binary16 into float), column
//           max / min over the thread's 16 rows (NaN-propagating), then across
//           the half's 8 warps in shared memory by one thread per column, which
//           also derives the column's step, zero point and reciprocal step.
//   pass 2  the code decision rint(fl(w' / step)) without a division per
//           weight: y = w' * fl(1 / step) lies within |y| * 2^-23 of the
//           exact quotient, and adding 1.5 * 2^23 + z rounds y to an integer
//           in the low mantissa bits (q = those bits, packed by one shift-add
//           per code).  A code whose y lies within 2^-18 of a half-integer is
//           redone with the IEEE division, as is every code of a column whose
//           extreme codes fall outside 0..15 (clamping).
// Pairs of columns go through the packed float32x2 multiply / add.
namespace {

constexpr int kQTileN = 128;                       // columns per tile
constexpr int kQTileBytes = kGroup * kQTileN * 2;  // 32 KB of binary16
constexpr int kQHalfWarps = 8;
constexpr int kQThreads = 2 * kQHalfWarps * 32;    // two halves of 8 warps
constexpr float kMagic = 12582912.0f;              // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;
// sum_j kMagicBits * 16^j (mod 2^32): removed once from a word built with
// one shift-add per code from the raw bits of magic + code
constexpr uint32_t kMagicWord = kMagicBits * 0x11111111u;
constexpr float kTieMargin = 0.5f - 0x1p-18f;

struct QuantParams {
    const __half *s;
    int32_t *Q;
    __half *scales;
    int32_t *zeros;
    int32_t *status;
    int K, N, G, n_ctiles;
    int tiles;
};

struct alignas(128) QuantHalf {
    uint8_t stage[2][kQTileBytes];
    float red_max[kQHalfWarps][kQTileN];
    float red_min[kQHalfWarps][kQTileN];
    float rsf[kQTileN];   // fl(1 / step)
    float cmag[kQTileN];  // 1.5 * 2^23 + z
    float step[kQTileN];  // step as float (exact fallback)
    int zc[kQTileN];      // zero point | 0x100 when the column needs clamping
    uint64_t full[2];
};

__device__ __forceinline__ float fold(uint16_t w, uint16_t sk)
{
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(w), "h"(sk), "f"(-0.0f));
    return d;  // w * s_k, exact in float (11 x 11 significant bits)
}
__device__ __forceinline__ float fmax_nan(float a, float b)
{
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ float fmin_nan(float a, float b)
{
    float d;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ unsigned long long pk(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk(unsigned long long v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// y - r for pairs, as fma(r, -1, y): exact when r = rint(y)
__device__ __forceinline__ unsigned long long fms2(unsigned long long r, unsigned long long y)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(r), "l"(0xBF800000BF800000ull), "l"(y));
    return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// rint(fl(v / sf)) from y = v * fl(1 / sf), which lies within |y| * 2^-23 of
// the exact quotient (|y| < 2^22 here: v and sf are finite, sf >= 2^-24);
// only when y is within |y| * 2^-21 of a half-integer is the IEEE division
// needed to decide.
__device__ __forceinline__ float rint_quotient(float v, float sf, float rsf)
{
    const float y = __fmul_rn(v, rsf);
    const float q = rintf(y);
    if (fabsf(y - q) < 0.5f - fabsf(y) * 0x1p-21f) return q;
    return rintf(__fdiv_rn(v, sf));
}

// The code decision with the correctly rounded quotient (the definition).
__device__ __forceinline__ uint32_t code_exact(float wp, float step, int z)
{
    int q = static_cast<int>(rintf(__fdiv_rn(wp, step))) + z;
    return static_cast<uint32_t>(min(max(q, 0), 15));
}

}  // namespace

__global__ void __launch_bounds__(kQThreads, 1) quantize_pack_kernel(const __grid_constant__ CUtensorMap tmW,
                                                                    const QuantParams p)
{
    extern __shared__ uint8_t qsmem_raw[];
    QuantHalf *halves = reinterpret_cast<QuantHalf *>(qsmem_raw + ((128u - (smem_u32(qsmem_raw) & 127u)) & 127u));
    const int half = threadIdx.x >> 8;
    const int tid = threadIdx.x & 255;  // thread index within the half
    const int warp = tid >> 5;
    const int lane = tid & 31;
    QuantHalf &sm = halves[half];
    const uint32_t bar_id = 1 + half;

    if (tid == 0) {
        prefetch_tmap(&tmW);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        fence_barrier_init();
    }
    __syncthreads();
    // this half's tiles: first, then every (2 * gridDim.x)-th
    const int t_first = 2 * blockIdx.x + half;
    const int t_step = 2 * gridDim.x;
    auto issue = [&](int t, int st) {
        const int g = t / p.n_ctiles;
        const int ct = t - g * p.n_ctiles;
        mbar_arrive_expect_tx(&sm.full[st], kQTileBytes);
        tma_load_2d(sm.stage[st], &tmW, &sm.full[st], ct * kQTileN, g * kGroup);
    };
    if (tid == 0) {
        if (t_first < p.tiles) issue(t_first, 0);
        if (t_first + t_step < p.tiles) issue(t_first + t_step, 1);
    }

    bool ok = true, bad = false;
    int it = 0;
    for (int t = t_first; t < p.tiles; t += t_step, ++it) {
        const int st = it & 1;
        const int g = t / p.n_ctiles;
        const int n0 = (t - g * p.n_ctiles) * kQTileN;
        const int k0 = g * kGroup + 16 * warp;
        // per-row channel scales: the same for the whole warp (broadcast loads)
        const uint4 sv0 = __ldg(reinterpret_cast<const uint4 *>(p.s + k0));
        const uint4 sv1 = __ldg(reinterpret_cast<const uint4 *>(p.s + k0 + 8));
        uint16_t sk[16];
        *reinterpret_cast<uint4 *>(&sk[0]) = sv0;
        *reinterpret_cast<uint4 *>(&sk[8]) = sv1;
        if (ok && !mbar_wait(&sm.full[st], static_cast<uint32_t>(it >> 1) & 1u)) ok = false;

        uint2 raw[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            raw[j] = *reinterpret_cast<const uint2 *>(sm.stage[st] + ((16 * warp + j) * kQTileN + 4 * lane) * 2);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float sj = __half2float(__ushort_as_half(sk[j]));
            bad |= !(sj > 0.0f) || !isfinite(sj);
        }

        // ---- pass 1: column max / min of w' over this thread's 16 rows
        float mx[4], mn[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            mx[c] = -INFINITY;
            mn[c] = INFINITY;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint16_t *w = reinterpret_cast<const uint16_t *>(&raw[j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = fold(w[c], sk[j]);
                mx[c] = fmax_nan(mx[c], v);
                mn[c] = fmin_nan(mn[c], v);
            }
        }
        *reinterpret_cast<float4 *>(&sm.red_max[warp][4 * lane]) = make_float4(mx[0], mx[1], mx[2], mx[3]);
        *reinterpret_cast<float4 *>(&sm.red_min[warp][4 * lane]) = make_float4(mn[0], mn[1], mn[2], mn[3]);
        named_bar_sync(bar_id, 256);  // the stage is read, the partial extremes are written

        // the stage is free: bring this half's tile two steps ahead
        if (tid == 0 && t + 2 * t_step < p.tiles) issue(t + 2 * t_step, st);

        // ---- one thread per column: step, zero point, reciprocal, clamp flag
        if (tid < kQTileN) {
            float a = sm.red_max[0][tid], b = sm.red_min[0][tid];
#pragma unroll
            for (int i = 1; i < kQHalfWarps; ++i) {
                a = fmax_nan(a, sm.red_max[i][tid]);
                b = fmin_nan(b, sm.red_min[i][tid]);
            }
            const bool col_in = n0 + tid < p.N;
            const bool fin = isfinite(a) && isfinite(b);
            bad |= col_in && !fin;
            if (!fin) {
                a = 0.0f;
                b = 0.0f;
            }
            // asymmetric: step from the range, zero point from the minimum;
            // symmetric (no zeros tensor): step from the largest magnitude over
            // 7 levels, zero point 8, i.e. codes clamp(rint(w'/step), -8, 7) + 8
            const bool symmetric = p.zeros == nullptr;
            float r = symmetric ? fmaxf(fabsf(a), fabsf(b)) : __fsub_rn(a, b);
            if (r < 1e-5f) r = 1e-5f;
            uint16_t bits = __half_as_ushort(__float2half_rn(__fdiv_rn(r, symmetric ? 7.0f : 15.0f)));
            if ((bits & 0x7FFF) == 0) bits = 1;  // never a zero step
            const float sf = __half2float(__ushort_as_half(bits));
            const float rsf = __frcp_rn(sf);
            float zf = symmetric ? 8.0f : rint_quotient(-b, sf, rsf);
            zf = fminf(fmaxf(zf, 0.0f), 15.0f);
            const int z = static_cast<int>(zf);
            // codes are monotone in w', so the extremes decide whether any clamps
            const int qa = static_cast<int>(rint_quotient(a, sf, rsf)) + z;
            const int qb = static_cast<int>(rint_quotient(b, sf, rsf)) + z;
            sm.rsf[tid] = rsf;
            sm.cmag[tid] = kMagic + zf;
            sm.step[tid] = sf;
            sm.zc[tid] = z | ((qa > 15 || qb < 0) ? 0x100 : 0);
            if (col_in) p.scales[static_cast<size_t>(g) * p.N + n0 + tid] = __ushort_as_half(bits);
        }
        named_bar_sync(bar_id, 256);  // column parameters ready

        if (p.zeros != nullptr && tid < kQTileN / 8 && n0 + 8 * tid < p.N) {
            uint32_t zw = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) zw |= static_cast<uint32_t>(sm.zc[8 * tid + c] & 15) << (4 * c);
            p.zeros[static_cast<size_t>(g) * (p.N / 8) + n0 / 8 + tid] = static_cast<int32_t>(zw);
        }

        // ---- pass 2: codes, packed 8 to a word: words[h][c] for packed row 2w + h
        const int cb = 4 * lane;
        int clamp_any = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) clamp_any |= sm.zc[cb + c] & 0x100;
        uint32_t word[2][4];
        if (!clamp_any) {
#pragma unroll
            for (int cp = 0; cp < 2; ++cp) {
                const int c0 = 2 * cp;
                const unsigned long long rs2 = pk(sm.rsf[cb + c0], sm.rsf[cb + c0 + 1]);
                const float m0 = sm.cmag[cb + c0], m1 = sm.cmag[cb + c0 + 1];
                const unsigned long long cm2 = pk(m0, m1), ncm2 = pk(-m0, -m1);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t acc0 = 0u - kMagicWord, acc1 = 0u - kMagicWord;
                    float dmax0 = 0.0f, dmax1 = 0.0f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int row = 8 * h + j;
                        const uint16_t *w = reinterpret_cast<const uint16_t *>(&raw[row]);
                        const unsigned long long y2 =
                            mul2(pk(fold(w[c0], sk[row]), fold(w[c0 + 1], sk[row])), rs2);
                        const unsigned long long t2 = add2(y2, cm2);   // magic + z + rint(y)
                        const unsigned long long r2 = add2(t2, ncm2);  // rint(y), exact
                        const unsigned long long d2 = fms2(r2, y2);    // y - rint(y), exact
                        float t0, t1, d0, d1;
                        upk(t2, t0, t1);
                        upk(d2, d0, d1);
                        dmax0 = fmaxf(dmax0, fabsf(d0));
                        dmax1 = fmaxf(dmax1, fabsf(d1));
                        acc0 += __float_as_uint(t0) << (4 * j);
                        acc1 += __float_as_uint(t1) << (4 * j);
                    }
                    word[h][c0] = acc0;
                    word[h][c0 + 1] = acc1;
                    // a code near a tie: redo that word with the IEEE quotient
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if ((e ? dmax1 : dmax0) >= kTieMargin) {
                            const int c = c0 + e;
                            const float sf = sm.step[cb + c];
                            const int z = sm.zc[cb + c] & 15;
                            uint32_t acc = 0;
                            for (int j = 0; j < 8; ++j) {
                                const uint16_t *w = reinterpret_cast<const uint16_t *>(&raw[8 * h + j]);
                                acc |= code_exact(fold(w[c], sk[8 * h + j]), sf, z) << (4 * j);
                            }
                            word[h][c] = acc;
                        }
                    }
                }
            }
        } else {
            // some column of this thread clamps: every code with the IEEE quotient
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float sf = sm.step[cb + c];
                const int z = sm.zc[cb + c] & 15;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t acc = 0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint16_t *w = reinterpret_cast<const uint16_t *>(&raw[8 * h + j]);
                        acc |= code_exact(fold(w[c], sk[8 * h + j]), sf, z) << (4 * j);
                    }
                    word[h][c] = acc;
                }
            }
        }
        if (n0 + cb < p.N) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                int32_t *dst = p.Q + static_cast<size_t>(g * 16 + 2 * warp + h) * p.N + n0 + cb;
                *reinterpret_cast<uint4 *>(dst) = make_uint4(word[h][0], word[h][1], word[h][2], word[h][3]);
            }
        }
    }
    if (bad) report(p.status, AWQ_ERR_NONFINITE);
    if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_act_stats(const __half *xcal, int R, int K, float *m, int32_t *status,
                             cudaStream_t st)
{
    act_stats_kernel<<<(K + 127) / 128, 1024, 0, st>>>(xcal, R, K, m, status);
    return cudaGetLastError();
}

cudaError_t launch_compute_scales(const float *m, int K, uint16_t *s, int32_t *status,
                                  cudaStream_t st)
{
    compute_scales_kernel<<<(K + 1023) / 1024, 1024, 0, st>>>(m, K, s, status);
    return cudaGetLastError();
}

size_t quantize_smem_bytes() { return 2 * sizeof(QuantHalf) + 128; }

cudaError_t configure_quantize()
{
    return cudaFuncSetAttribute(quantize_pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(quantize_smem_bytes()));
}

cudaError_t launch_quantize_pack(const CUtensorMap &tmW, const __half *s, int K, int N, int32_t *Q,
                                 __half *scales, int32_t *zeros, int32_t *status, int num_sms,
                                 cudaStream_t st)
{
    QuantParams prm{};
    prm.s = s;
    prm.Q = Q;
    prm.scales = scales;
    prm.zeros = zeros;
    prm.status = status;
    prm.K = K;
    prm.N = N;
    prm.G = K / kGroup;
    prm.n_ctiles = (N + kQTileN - 1) / kQTileN;
    prm.tiles = prm.G * prm.n_ctiles;
    const int pairs = (prm.tiles + 1) / 2;  // a CTA's two halves take two tiles at a time
    const int grid = pairs < num_sms ? pairs : num_sms;
    quantize_pack_kernel<<<grid, kQThreads, quantize_smem_bytes(), st>>>(tmW, prm);
    return cudaGetLastError();
}

}  // namespace awq
