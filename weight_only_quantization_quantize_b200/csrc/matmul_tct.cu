// matmul_tct.cu -- Y = (X / s) . dequant(Q) for M >= 64 tokens (batched and
// prefill) on the 5th-generation tensor cores, with the dequantized weights
// held in tensor memory instead of shared memory.
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (GEMM kernel for batch sizes > 1), "Group Size Configuration",
// "Zero-Point Quantization".
//
// The kernel computes the transposed tile Y^T = dequant(W)^T . X'^T: the MMA's
// A operand (M = 128 output columns in the TMEM lanes, K along the columns) is
// the dequantized weight tile, written by the dequantization warps straight
// into tensor memory (tcgen05.st); B is the X' tile (BT tokens x 64 k, K-major,
// 128-byte swizzle) that TMA writes into shared memory; the accumulator
// (128 output columns x BT tokens) is in TMEM.  Shared memory then carries only
// the TMA loads and the MMA's reads of X', not a dequantized copy of the
// weights.
//
// One CTA = 128 output columns x BT tokens (BT = 128 or 256):
//   warp 0      TMA ring (5 stages): X' tile [BT x 64], packed words [8 x 128]
//               (4 KB), cp.async of the group's steps and zero words.
//   warp 1      allocates TMEM (accumulator + a 4-slot ring of 32-column A
//               tiles); one lane issues tcgen05.mma.cta_group::1.kind::f16
//               (M = 128, N = BT, K = 16, A from TMEM) x 4 per stage.
//   warps 2..9  dequantize: warp w owns TMEM lanes 32 (w % 4) .. +31 (one output
//               column per lane) and half of a stage's packed rows; it writes
//               16 columns of (q - z) * step binary16 pairs per stage; at the
//               end the same warps read the accumulator and write Y.
// Within each 8-channel chunk the contraction runs in the pair order
// (0,4),(1,5),(2,6),(3,7) on both operands (X' is stored that way by the
// pre-pass, the unpack produces the weights that way), which leaves the sum
// unchanged.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kCols = 128;            // output columns per CTA (MMA M, TMEM lanes)
constexpr int kBK = 64;               // k per stage
constexpr int kLoadStages = 5;
constexpr int kASlots = 4;            // TMEM slots of dequantized weights
constexpr int kASlotCols = kBK / 2;   // 32 TMEM columns: 64 binary16 per lane
constexpr int kDequantWarps = 8;
constexpr int kThreads = 64 + 32 * kDequantWarps;
constexpr int kQBytes = (kBK / 8) * kCols * 4;  // 4 KB of packed words
constexpr int kMetaBytes = 1024;                // 256 B steps + 64 B zero words, padded

template <int BT>
struct TctCfg {
    static constexpr int kXBytes = BT * kBK * 2;                    // 16 or 32 KB
    static constexpr int kStageBytes = kXBytes + kQBytes + kMetaBytes;  // a multiple of 1 KB
    static constexpr int kACol = BT;                                // A slots after the accumulator
    static constexpr int kTmemCols = BT == 256 ? 512 : 256;
    static constexpr size_t kSmem = 1024 + static_cast<size_t>(kLoadStages) * kStageBytes + 256;
};

struct TctParams {
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

template <int BT>
__global__ void __launch_bounds__(kThreads, 1)
    tct_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
               const TctParams p)
{
    using C = TctCfg<BT>;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    uint64_t *full_load = reinterpret_cast<uint64_t *>(smem + kLoadStages * C::kStageBytes);
    uint64_t *empty_load = full_load + kLoadStages;
    uint64_t *full_a = empty_load + kLoadStages;
    uint64_t *empty_a = full_a + kASlots;
    uint64_t *tmem_full = empty_a + kASlots;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tmem_full + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kCols;
    const int m0 = blockIdx.y * BT;
    const int KB = p.K / kBK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kLoadStages; ++i) {
            mbar_init(&full_load[i], 1 + 32);  // expect_tx + 32 cp.async arrivals
            mbar_init(&empty_load[i], 1);      // MMA commit
        }
        for (int i = 0; i < kASlots; ++i) {
            mbar_init(&full_a[i], kDequantWarps);
            mbar_init(&empty_a[i], 1);         // MMA commit
        }
        mbar_init(tmem_full, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // Waits inside a warp that issues .sync.aligned tensor-memory instructions
    // must end the same way on every lane: each wait's outcome is voted.
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmQ);
        }
        bool ok = true;
        int issued = 0;
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kLoadStages;
            const bool w = kb < kLoadStages || mbar_wait(&empty_load[st], ((kb / kLoadStages) - 1) & 1);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            uint8_t *stg = smem + st * C::kStageBytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full_load[st], C::kXBytes + kQBytes);
                tma_load_2d(stg, &tmX, &full_load[st], kb * kBK, m0);
                tma_load_2d(stg + C::kXBytes, &tmQ, &full_load[st], n0, kb * (kBK / 8));
            }
            // lanes 0..15: 8 steps (16 B) each; lanes 16..31: one zero word each
            uint8_t *meta = stg + C::kXBytes + kQBytes;
            const int g = (kb * kBK) / kGroup;
            if (lane < 16) {
                const int n = n0 + 8 * lane;
                const bool in = n < p.N;
                cp_async_16(meta + 16 * lane, p.scales + static_cast<size_t>(g) * p.N + (in ? n : 0),
                            in ? 16u : 0u);
            } else {
                const int wi = n0 / 8 + (lane - 16);
                const bool in = wi < p.N / 8;
                cp_async_4(meta + 256 + 4 * (lane - 16),
                           zero_word_src(p.zeros, g, p.N / 8, in ? wi : 0, lane - 16), in ? 4u : 0u);
            }
            cp_async_arrive_noinc(&full_load[st]);
            ++issued;
        }
        if (!ok) {
            // let the copies already issued land before the CTA exits
            asm volatile("cp.async.wait_all;" ::: "memory");
            if (lane == 0) {
                report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
                const int first = issued > kLoadStages ? issued - kLoadStages : 0;
                for (int it = first; it < issued; ++it)
                    mbar_wait_for(&full_load[it % kLoadStages], (it / kLoadStages) & 1, kDrainLimitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = tc_idesc_f16(kCols, BT);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kLoadStages;
            const int as = kb % kASlots;
            bool w = mbar_wait(&full_load[st], (kb / kLoadStages) & 1);
            if (w) w = mbar_wait(&full_a[as], (kb / kASlots) & 1);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t x0 = smem_u32(smem + st * C::kStageBytes);
                const uint32_t a0 = tmem_base + C::kACol + as * kASlotCols;
#pragma unroll
                for (int s = 0; s < kBK / 16; ++s)
                    tc_mma_ta(tmem_base, a0 + 8 * s, sw128_desc(x0 + 32 * s), idesc,
                              (kb > 0 || s > 0) ? 1u : 0u);
                tc_commit(&empty_load[st]);
                tc_commit(&empty_a[as]);
            }
            __syncwarp();
        }
        if (lane == 0) {
            // tmem_full completes when every MMA issued has completed; on a
            // timeout this lane waits for that itself before TMEM is freed
            tc_commit(tmem_full);
            if (!ok) {
                report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
                mbar_wait_for(tmem_full, 0, kDrainLimitNs);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dequant
        // warp w: TMEM lanes 32 (w % 4) .. +31 = output columns; packed rows
        // 4 h .. 4 h + 3 of each stage (h = 0 for warps 2..5, 1 for 6..9)
        const int quarter = warp & 3;
        const int h = (warp - 2) >> 2;
        const int col = quarter * 32 + lane;  // column within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const UnpackConsts uk = p.uk;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int st = kb % kLoadStages;
            const int as = kb % kASlots;
            bool w = mbar_wait(&full_load[st], (kb / kLoadStages) & 1);
            if (w && kb >= kASlots) w = mbar_wait(&empty_a[as], ((kb / kASlots) - 1) & 1);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint8_t *q = smem + st * C::kStageBytes + C::kXBytes;
            const uint8_t *meta = q + kQBytes;
            const uint16_t sbits = reinterpret_cast<const uint16_t *>(meta)[col];
            const uint32_t sc2 = static_cast<uint32_t>(sbits) | (static_cast<uint32_t>(sbits) << 16);
            const uint32_t zw = reinterpret_cast<const uint32_t *>(meta + 256)[col >> 3];
            uint32_t za, zb;
            zero_constants((zw >> (4 * (col & 7))) & 15u, za, zb);
            uint32_t wv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
                wv[r] = reinterpret_cast<const uint32_t *>(q + (4 * h + r) * (kCols * 4))[col];
            uint32_t o[16];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                uint32_t d[4];
                unpack_minus_zero(wv[r], za, zb, d, uk);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[4 * r + i]) : "r"(d[i]), "r"(sc2));
            }
            tmem_st16(tmem_base + lane_addr + C::kACol + as * kASlotCols + 16 * h, o);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_a[as]);
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);

        // ------------------------------------------------------------ epilogue
        // lane = output column n0 + col, TMEM column c = token m0 + c; warp
        // half h writes tokens h BT/2 .. (h + 1) BT/2 - 1 of the tile
        const bool ready = ok && mbar_wait(tmem_full, 0);
        if (__all_sync(0xffffffffu, ready)) {
            tc_fence_after();
            const int n = n0 + col;
            const bool n_in = n < p.N;
#pragma unroll 1
            for (int c0 = h * (BT / 2); c0 < (h + 1) * (BT / 2); c0 += 32) {
                const int mrem = p.M - (m0 + c0);  // the same on every lane
                if (mrem <= 0) break;
                uint32_t v[32];
                tmem_ld32(tmem_base + lane_addr + c0, v);
                if (n_in) {
                    __half *dst = p.Y + static_cast<size_t>(m0 + c0) * p.N + n;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < mrem) dst[static_cast<size_t>(i) * p.N] = __float2half_rn(__uint_as_float(v[i]));
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::kTmemCols)
                     : "memory");
    }
}

// Relative cost of a token tile per weight tile: a 128-token tile does half
// the MMA work of a 256-token one with the same dequantization.
constexpr int kCost128 = 6, kCost256 = 10;

}  // namespace

TctPlan plan_tct(int M, int K, int N, int num_sms)
{
    (void)K;
    TctPlan pl{};
    pl.n_tiles = (N + kCols - 1) / kCols;
    const int sms = num_sms > 0 ? num_sms : 148;
    const int t128 = (M + 127) / 128, t256 = (M + 255) / 256;
    const long long w128 = (static_cast<long long>(t128) * pl.n_tiles + sms - 1) / sms;
    const long long w256 = (static_cast<long long>(t256) * pl.n_tiles + sms - 1) / sms;
    pl.bt = (w256 * kCost256 <= w128 * kCost128) ? 256 : 128;
    pl.m_tiles = pl.bt == 256 ? t256 : t128;
    pl.smem = pl.bt == 256 ? TctCfg<256>::kSmem : TctCfg<128>::kSmem;
    return pl;
}

cudaError_t configure_tct()
{
    cudaError_t e = cudaFuncSetAttribute(tct_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(TctCfg<256>::kSmem));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(tct_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(TctCfg<128>::kSmem));
}

cudaError_t launch_tct(const TctPlan &plan, const CUtensorMap &tmX, const CUtensorMap &tmQ, const __half *scales,
                       const int32_t *zeros, __half *Y, int M, int K, int N, int32_t *status, cudaStream_t st)
{
    TctParams prm{scales, zeros, Y, status, M, K, N, unpack_consts()};
    dim3 grid(plan.n_tiles, plan.m_tiles);
    if (plan.bt == 256)
        tct_kernel<256><<<grid, kThreads, plan.smem, st>>>(tmX, tmQ, prm);
    else
        tct_kernel<128><<<grid, kThreads, plan.smem, st>>>(tmX, tmQ, prm);
    return cudaGetLastError();
}

}  // namespace awq
