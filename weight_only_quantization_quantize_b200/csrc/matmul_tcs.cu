// matmul_tcs.cu -- Y = (X / s) . dequant(Q) for small batches (24 <= M < 64
// tokens) on the 5th-generation tensor cores, with the roles of the operands
// swapped: the dequantized weights are the 128-row A operand and the tokens
// (padded to a multiple of 16) are the N dimension.
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (GEMM kernel for batch sizes > 1), "Group Size Configuration",
// "Zero-Point Quantization".
//
// At a few dozen tokens the layer does 2 M flops per weight: at HBM speed
// that is more than the register-fed mma.sync path can issue on sm_100, while
// tcgen05 has twice the rate and needs no register accumulators.
//
// One CTA = 128 output columns x one k range; the k ranges of a column tile are
// the CTAs of a thread-block cluster (split-K, up to 8):
//   warp 0      TMA ring (4 stages): X' tile [Nt tokens x 64 k] (128-byte
//               swizzle; tokens beyond M read as zero), packed words [8 x 128];
//               cp.async of the group's steps and zero words.
//   warp 1      allocates 128 TMEM columns (the accumulator and a 2-slot ring
//               of dequantized A tiles); one lane issues
//               tcgen05.mma.cta_group::1.kind::f16 with A from tensor memory
//               (M = 128, N = Nt, K = 16) x 4 per stage and commits each stage
//               back to both rings.
//   warps 2..5  dequantize: warp w owns TMEM lanes 32 (w % 4) .. +31 (one
//               output column per lane) and writes the stage's 32 columns of
//               (q - z) * step binary16 pairs into the A slot (tcgen05.st); then read the accumulator (tcgen05.ld) and
//               push it to the cluster CTA that owns those columns (st.async);
//               each CTA adds the k-split partials of its columns in rank order
//               and writes Y.
// The dequantized weights never pass through shared memory, which then
// carries only the TMA loads and the MMA's reads of the X' tile.
// Within each 8-channel chunk the contraction runs in the pair order
// (0,4),(1,5),(2,6),(3,7) on both operands (X' is stored that way by the
// pre-pass), which leaves the sum unchanged.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kBN = 128;               // output columns per CTA (MMA M)
constexpr int kBK = 64;                // k per stage
constexpr int kLoadStages = 4;
constexpr int kASlots = 2;             // dequantized A tiles in tensor memory
constexpr int kASlotCols = kBK / 2;    // 32 TMEM columns: 64 binary16 per lane
constexpr int kDequantWarps = 4;
// A CTA issues one tcgen05.mma (1 KB of packed weights at M = 128, K = 16)
// every ~140 cycles whatever N is, so at a few dozen tokens the MMA issue rate
// of a CTA, not the tensor core, bounds its stream: four small CTAs per SM.
constexpr int kThreads = 32 * (2 + kDequantWarps);
constexpr int kQBytes = (kBK / 8) * kBN * 4;  // 4 KB of packed words
constexpr int kMetaBytes = 1024;              // 256 B steps + 64 B zero words, padded
constexpr int kAccCols = 64;                  // the accumulator: up to 64 token columns
constexpr int kACol = kAccCols;               // A slots after the accumulator
constexpr int kTmemCols = 128;                // four CTAs per SM share the 512 columns
constexpr int kCtasPerSm = 4;
constexpr size_t kSmemPerSm = 233472;         // shared memory of an SM
constexpr size_t kMinSmem = kSmemPerSm / (kCtasPerSm + 1) + 1024;  // a fifth CTA never fits

struct Params {
    const __half *scales;
    const int32_t *zeros;
    __half *Y;
    int32_t *status;
    int M, K, N;
    int nt;           // tokens padded to a multiple of 16 (MMA N)
    int splits;       // cluster size along K
    int stage_bytes;  // X' tile + packed words + metadata
    UnpackConsts uk;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__global__ void __launch_bounds__(kThreads, 1)
    tcs_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
               const Params p)
{
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    uint64_t *full_load = reinterpret_cast<uint64_t *>(smem + kLoadStages * p.stage_bytes);
    uint64_t *empty_load = full_load + kLoadStages;
    uint64_t *full_a = empty_load + kLoadStages;
    uint64_t *empty_a = full_a + kASlots;
    uint64_t *tmem_full = empty_a + kASlots;
    uint64_t *recv_bar = tmem_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(recv_bar + 1);
    // after the main loop the load ring is idle: it receives the pushed partials
    float *recv = reinterpret_cast<float *>(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;  // == rank in the cluster
    const int n0 = blockIdx.y * kBN;
    const int KB = p.K / kBK;
    const int kb_begin = static_cast<int>(static_cast<int64_t>(split) * KB / p.splits);
    const int kb_end = static_cast<int>(static_cast<int64_t>(split + 1) * KB / p.splits);
    const int nkb = kb_end - kb_begin;
    const int cpo = kBN / p.splits;  // columns each cluster rank owns in the epilogue
    const int xbytes = p.nt * 128;

    pdl_launch_dependents();

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
        mbar_init(recv_bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(p.splits * p.nt * cpo * 4));
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
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmQ);
        }
        pdl_wait();  // X' comes from the pre-pass kernel
        for (int i = 0; i < nkb; ++i) {
            const int kb = kb_begin + i;
            const int st = i % kLoadStages;
            if (i >= kLoadStages && !mbar_wait(&empty_load[st], ((i / kLoadStages) - 1) & 1)) {
                ok = false;
                break;
            }
            uint8_t *stg = smem + st * p.stage_bytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full_load[st], static_cast<uint32_t>(xbytes + kQBytes));
                tma_load_2d(stg, &tmX, &full_load[st], kb * kBK, 0);
                tma_load_2d(stg + xbytes, &tmQ, &full_load[st], n0, kb * (kBK / 8));
            }
            uint8_t *meta = stg + xbytes + kQBytes;
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
                           zero_word_src(p.zeros, g, p.N / 8, in ? wi : 0, lane), in ? 4u : 0u);
            }
            cp_async_arrive_noinc(&full_load[st]);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = tc_idesc_f16(kBN, p.nt);
        for (int i = 0; i < nkb; ++i) {
            const int st = i % kLoadStages;
            const int as = i % kASlots;
            // the outcome is voted so that the warp leaves the loop as one
            bool w = mbar_wait(&full_load[st], (i / kLoadStages) & 1);
            if (w) w = mbar_wait(&full_a[as], (i / kASlots) & 1);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a0 = tmem_base + kACol + as * kASlotCols;
                const uint32_t b0 = smem_u32(smem + st * p.stage_bytes);
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    tc_mma_ta(tmem_base, a0 + 8 * k, sw128_desc(b0 + 32 * k), idesc, (i > 0 || k > 0) ? 1u : 0u);
                tc_commit(&empty_load[st]);
                tc_commit(&empty_a[as]);
            }
            __syncwarp();
        }
        if (lane == 0) {
            // tmem_full completes once every MMA issued has completed; after a
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
        // warp w: TMEM lanes 32 (w % 4) .. +31 = output columns, every packed
        // row of the stage
        const int quarter = warp & 3;
        const int c = 32 * quarter + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const UnpackConsts uk = p.uk;
        for (int i = 0; i < nkb; ++i) {
            const int st = i % kLoadStages;
            const int as = i % kASlots;
            bool w = mbar_wait(&full_load[st], (i / kLoadStages) & 1);
            if (w && i >= kASlots) w = mbar_wait(&empty_a[as], ((i / kASlots) - 1) & 1);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint8_t *q = smem + st * p.stage_bytes + xbytes;
            const uint8_t *meta = q + kQBytes;
            const uint16_t sbits = reinterpret_cast<const uint16_t *>(meta)[c];
            const uint32_t sc2 = static_cast<uint32_t>(sbits) | (static_cast<uint32_t>(sbits) << 16);
            const uint32_t zw = reinterpret_cast<const uint32_t *>(meta + 256)[c >> 3];
            uint32_t za, zb;
            zero_constants((zw >> (4 * (c & 7))) & 15u, za, zb);
            uint32_t wv[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) wv[r] = reinterpret_cast<const uint32_t *>(q + r * (kBN * 4))[c];
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint32_t o[16];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    uint32_t d[4];
                    unpack_minus_zero(wv[4 * part + r], za, zb, d, uk);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[4 * r + j]) : "r"(d[j]), "r"(sc2));
                }
                tmem_st16(tmem_base + lane_addr + kACol + as * kASlotCols + 16 * part, o);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_a[as]);
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    }

    // ---------------------------------------------------------------- epilogue
    // Dequant warps read the accumulator: warp w reaches TMEM lanes
    // 32 (w % 4) .. +31 (output columns), every token column.
    // Every partial goes to the cluster rank owning its column: rank c / cpo,
    // laid out there as [source rank][token][owned column].
    const bool dq = warp >= 2;  // a dequantization warp
    const bool have_acc = dq && __all_sync(0xffffffffu, ok && mbar_wait(tmem_full, 0));
    if (dq && !have_acc && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    // Every CTA of the cluster is past its main loop (its load ring, which
    // receives the partials, is idle) and has initialized its barriers.
    cluster_arrive_release();
    cluster_wait_acquire();
    if (dq) {
        tc_fence_after();
        const int quarter = warp & 3;
        const int col = quarter * 32 + lane;
        const uint32_t owner = static_cast<uint32_t>(col / cpo);
        const int lc = col - static_cast<int>(owner) * cpo;
        const uint32_t rbar = map_to_rank(smem_u32(recv_bar), owner);
        const uint32_t rbase = map_to_rank(smem_u32(recv), owner);
        for (int t0 = 0; t0 < p.nt; t0 += 8) {
            uint32_t v[8];
            tmem_ld8(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + t0, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float x = have_acc ? __uint_as_float(v[j]) : 0.0f;
                const int off = ((split * p.nt + t0 + j) * cpo + lc) * 4;
                st_async_f32(rbase + off, x, rbar);
            }
        }
    }
    // Arrive once the pushes are issued (no fence: every owner waits for all
    // the bytes pushed to it before it reduces, hence before it exits).
    cluster_arrive_relaxed();
    if (!mbar_wait(recv_bar, 0) && threadIdx.x == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    for (int e = threadIdx.x; e < p.M * cpo; e += kThreads) {
        const int tok = e / cpo;
        const int lc = e - tok * cpo;
        const int n = n0 + split * cpo + lc;
        if (n >= p.N) continue;
        float v = 0.0f;
        for (int r = 0; r < p.splits; ++r) v += recv[(r * p.nt + tok) * cpo + lc];
        p.Y[static_cast<size_t>(tok) * p.N + n] = __float2half_rn(v);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
    cluster_wait_acquire();
}

}  // namespace

TcsPlan plan_tcs(int M, int K, int N, int num_sms)
{
    TcsPlan pl{};
    pl.nt = (M + 15) / 16 * 16;
    pl.n_tiles = (N + kBN - 1) / kBN;
    const int KB = K / kBK;
    // Four CTAs per SM fit; the largest power-of-two split that keeps one wave
    // and leaves every CTA at least four stages.
    int splits = 1;
    while (splits * 2 <= 8 && pl.n_tiles * splits * 2 <= kCtasPerSm * num_sms && KB / (splits * 2) >= 4)
        splits *= 2;
    pl.splits = splits;
    pl.stage_bytes = pl.nt * 128 + kQBytes + kMetaBytes;
    pl.smem = 1024 + static_cast<size_t>(kLoadStages) * pl.stage_bytes + 256;
    // At most four CTAs per SM: each holds 128 of the SM's 512 TMEM columns,
    // and a fifth would block in tcgen05.alloc while its cluster peers wait
    // for it.  The shared-memory request enforces that.
    if (pl.smem < kMinSmem) pl.smem = kMinSmem;
    return pl;
}

cudaError_t configure_tcs()
{
    return cudaFuncSetAttribute(tcs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(plan_tcs(64, 128, 128, 1).smem));
}

cudaError_t launch_tcs(const TcsPlan &plan, const CUtensorMap &tmX, const CUtensorMap &tmQ,
                       const __half *scales, const int32_t *zeros, __half *Y, int M, int K, int N,
                       int32_t *status, cudaStream_t st)
{
    Params prm{scales, zeros, Y, status, M, K, N, plan.nt, plan.splits, plan.stage_bytes, unpack_consts()};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.splits, plan.n_tiles, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = plan.splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, tcs_kernel, tmX, tmQ, prm);
}

}  // namespace awq
