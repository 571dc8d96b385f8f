// matmul_tc.cu -- Y = (X / s) . dequant(Q) for M >= 64 tokens (batched and
// prefill), the tensor-bound regime of the W4A16 linear layer, on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (GEMM kernel for batch sizes > 1), "Group Size Configuration",
// "Zero-Point Quantization".
//
// One CTA computes a 128 (tokens) x 256 (output columns) tile of Y:
//   warp 0      TMA producer (6-stage ring): X' tile [128 x 64] (128-byte
//               swizzled, the canonical K-major operand layout) and the
//               packed-word tile [8 x 256]; cp.async for the group's scales
//               and zero points.
//   warp 1      allocates 256 TMEM columns; one lane issues
//               tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256, K=16) x 4
//               per 64-k stage and commits each stage back to both rings.
//   warps 2..9  dequantize (32 columns each): word -> 8 binary16
//               (q - z) * step values, stored as one 16-byte chunk of the
//               K-major, 128-byte-swizzled B operand (2-slot ring); after the
//               last stage they drain TMEM (tcgen05.ld) to binary16 Y.
// Within each 8-channel chunk the contraction runs in the pair order
// (0,4),(1,5),(2,6),(3,7) on both operands (X' is stored that way by the
// pre-pass), which leaves the sum unchanged.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kLoadStages = 6;   // X' tile + packed words + steps/zeros
constexpr int kBStages = 2;      // dequantized B operand
constexpr int kDequantWarps = 8;
constexpr int kThreads = 64 + 32 * kDequantWarps;
constexpr int kABytes = kBM * kBK * 2;        // 16 KB
constexpr int kBBytes = kBN * kBK * 2;        // 32 KB
constexpr int kQBytes = (kBK / 8) * kBN * 4;  // 8 KB
constexpr int kMetaBytes = 1024;              // 512 B steps + 128 B zero words, padded
constexpr int kLoadBytes = kABytes + kQBytes + kMetaBytes;  // 25 KB, a multiple of 1 KB
constexpr int kTmemCols = 256;

struct Params {
    const __half *scales;
    const int32_t *zeros;
    __half *Y;
    int32_t *status;
    int M, K, N;
    UnpackConsts uk;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// Instruction descriptor: kind::f16, A = B = f16, D = f32, both K-major,
// N = 256, M = 128.
constexpr uint32_t kIdesc = tc_idesc_f16(kBM, kBN);

__device__ __forceinline__ uint32_t pack_half2(float a, float b)
{
    return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(a))) |
           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(b))) << 16);
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
              const Params p)
{
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    uint8_t *bring = smem + kLoadStages * kLoadBytes;  // 1 KB aligned
    uint64_t *full_load = reinterpret_cast<uint64_t *>(bring + kBStages * kBBytes);
    uint64_t *empty_load = full_load + kLoadStages;
    uint64_t *full_b = empty_load + kLoadStages;
    uint64_t *empty_b = full_b + kBStages;
    uint64_t *tmem_full = empty_b + kBStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tmem_full + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kBN;
    const int m0 = blockIdx.y * kBM;
    const int KB = p.K / kBK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kLoadStages; ++i) {
            mbar_init(&full_load[i], 1 + 32);  // expect_tx + 32 cp.async arrivals
            mbar_init(&empty_load[i], 1);      // MMA commit
        }
        for (int i = 0; i < kBStages; ++i) {
            mbar_init(&full_b[i], kDequantWarps);
            mbar_init(&empty_b[i], 1);         // MMA commit
        }
        mbar_init(tmem_full, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmQ);
        }
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kLoadStages;
            if (kb >= kLoadStages && !mbar_wait(&empty_load[st], ((kb / kLoadStages) - 1) & 1)) {
                ok = false;
                break;
            }
            uint8_t *stg = smem + st * kLoadBytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full_load[st], kABytes + kQBytes);
                tma_load_2d(stg, &tmA, &full_load[st], kb * kBK, m0);
                tma_load_2d(stg + kABytes, &tmQ, &full_load[st], n0, kb * (kBK / 8));
            }
            uint8_t *meta = stg + kABytes + kQBytes;
            const int g = (kb * kBK) / kGroup;
            const int n = n0 + 8 * lane;
            const bool in_s = n < p.N;
            cp_async_16(meta + 16 * lane, p.scales + static_cast<size_t>(g) * p.N + (in_s ? n : 0),
                        in_s ? 16u : 0u);
            const int wi = n0 / 8 + lane;
            const bool in_z = wi < p.N / 8;
            cp_async_4(meta + 512 + 4 * lane,
                       zero_word_src(p.zeros, g, p.N / 8, in_z ? wi : 0, lane), in_z ? 4u : 0u);
            cp_async_arrive_noinc(&full_load[st]);
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kLoadStages;
            const int bs = kb % kBStages;
            if (!mbar_wait(&full_load[st], (kb / kLoadStages) & 1) ||
                !mbar_wait(&full_b[bs], (kb / kBStages) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a0 = smem_u32(smem + st * kLoadBytes);
                const uint32_t b0 = smem_u32(bring + bs * kBBytes);
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    tc_mma(tmem_base, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), kIdesc,
                           (kb > 0 || k > 0) ? 1u : 0u);
                tc_commit(&empty_load[st]);
                tc_commit(&empty_b[bs]);
            }
            __syncwarp();
        }
        if (lane == 0) {
            if (ok)
                tc_commit(tmem_full);
            else
                report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dequant
        // dequant warp d handles columns d*32 .. d*32+31 of the 256-column tile
        const int dw = warp - 2;
        const int n = dw * 32 + lane;
        const UnpackConsts uk = p.uk;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kLoadStages;
            const int bs = kb % kBStages;
            if (!mbar_wait(&full_load[st], (kb / kLoadStages) & 1) ||
                (kb >= kBStages && !mbar_wait(&empty_b[bs], ((kb / kBStages) - 1) & 1))) {
                ok = false;
                break;
            }
            const uint8_t *stg = smem + st * kLoadBytes;
            const uint8_t *q = stg + kABytes;
            const uint8_t *meta = q + kQBytes;
            const uint32_t bbase = smem_u32(bring + bs * kBBytes);
            const uint16_t sbits = reinterpret_cast<const uint16_t *>(meta)[n];
            const uint32_t sc2 = static_cast<uint32_t>(sbits) | (static_cast<uint32_t>(sbits) << 16);
            const uint32_t zw = reinterpret_cast<const uint32_t *>(meta + 512)[n >> 3];
            uint32_t za, zb;
            zero_constants((zw >> (4 * (n & 7))) & 15u, za, zb);
            uint32_t w[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) w[r] = reinterpret_cast<const uint32_t *>(q + r * (kBN * 4))[n];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                uint32_t d[4];
                unpack_minus_zero(w[r], za, zb, d, uk);
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[i]) : "r"(d[i]), "r"(sc2));
                const uint32_t dst = bbase + n * 128 + ((r ^ (n & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o[0]), "r"(o[1]),
                             "r"(o[2]), "r"(o[3])
                             : "memory");
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_b[bs]);
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);

        // ------------------------------------------------------------ epilogue
        // warp d reads TMEM lanes 32*(warp % 4).. and columns (dw / 4)*128 ..+127
        if (ok && mbar_wait(tmem_full, 0)) {
            tc_fence_after();
            const int quarter = warp & 3;
            const int row = quarter * 32 + lane;
            const int m = m0 + row;
            const int cbase = (dw >> 2) * 128;
#pragma unroll 1
            for (int c0 = cbase; c0 < cbase + 128; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + c0, v);
                if (m < p.M) {
                    __half *dst = p.Y + static_cast<size_t>(m) * p.N + n0 + c0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (n0 + c0 + 8 * i < p.N) {
                            uint4 o;
                            o.x = pack_half2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
                            o.y = pack_half2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
                            o.z = pack_half2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
                            o.w = pack_half2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
                            *reinterpret_cast<uint4 *>(dst + 8 * i) = o;
                        }
                    }
                }
            }
        } else if (lane == 0) {
            report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

TcPlan plan_tc(int M, int K, int N, int num_sms)
{
    (void)K;
    (void)num_sms;
    TcPlan pl{};
    pl.m_tiles = (M + kBM - 1) / kBM;
    pl.n_tiles = (N + kBN - 1) / kBN;
    pl.smem = 1024 + static_cast<size_t>(kLoadStages) * kLoadBytes + static_cast<size_t>(kBStages) * kBBytes +
              256;
    return pl;
}

cudaError_t configure_tc()
{
    return cudaFuncSetAttribute(tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(plan_tc(128, 128, 256, 1).smem));
}

cudaError_t launch_tc(const TcPlan &plan, const CUtensorMap &tmA, const CUtensorMap &tmQ,
                      const __half *scales, const int32_t *zeros, __half *Y, int M, int K, int N,
                      int32_t *status, cudaStream_t st)
{
    Params prm{scales, zeros, Y, status, M, K, N, unpack_consts()};
    dim3 grid(plan.n_tiles, plan.m_tiles);
    tc_kernel<<<grid, kThreads, plan.smem, st>>>(tmA, tmQ, prm);
    return cudaGetLastError();
}

}  // namespace awq
