// matmul_small.cu -- Y = (X / s) . dequant(Q) for M < 64 tokens (decode and
// small batches), the HBM-bound regime of the W4A16 linear layer.
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (a GEMV kernel for batch size 1, a GEMM kernel for batches) and
// "Group Size Configuration" / "Zero-Point Quantization" (4-bit codes, group
// 128, zero point).
//
// Design (B200):
//  * Weights stream once from HBM: a producer warp issues TMA tile loads of
//    the packed words (one 16-row x 32-column box per consumer warp, 128-byte
//    swizzled so the consumers' 16-byte shared loads are conflict free) plus
//    cp.async copies of the group's scales and zero points into a ring of
//    mbarrier-guarded stages; one stage is one 128-row group.
//  * Four consumer warps each own 32 output columns.  A lane unpacks one
//    16-byte load (4 columns x 8 consecutive k) into exact (q - z) binary16
//    pairs with integer ops and two f16x2 instructions per pair, and feeds
//    them straight from registers to mma.sync m16n8k16 (fp32 accumulate) in
//    swap-AB form: the output columns are the MMA rows, the tokens its 8
//    columns.  The contraction order inside each 8-k word is permuted
//    (k pairs (0,4),(1,5),(2,6),(3,7)); X / s is stored with the same
//    permutation, so the sum is unchanged.
//  * The MMA gives each group's partial sum_k x'_k (q_k - z) in fp32; the
//    group step is applied once per group (distributivity), y += step * part.
//  * Split-K across the CTAs of a thread-block cluster; the partial tiles are
//    reduced through distributed shared memory in a fixed rank order
//    (deterministic), each rank finishing a slice of the columns.
//  * X / s: for M <= 8 each CTA computes it for its own k range into shared
//    memory (no workspace, no extra launch); otherwise a pre-pass writes it
//    once to the workspace and the producer TMA-loads it per stage.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kBN = 128;            // output columns per CTA
constexpr int kQStage = 4 * 2048;   // 4 boxes of [16 rows x 32 words]
constexpr int kMetaBytes = 256 + 64;  // 128 scales + 16 zero words
constexpr int kRedPitch = 132;      // floats per token row of the reduction tile
constexpr size_t kPrologueMax = 64 * 1024;
constexpr int kSmemOptIn = 232448;  // 227 KB, the per-block opt-in maximum

constexpr int stages_for(int mt) { return mt <= 2 ? 8 : 4; }

struct Params {
    const __half *X;
    const __half *s;
    const __half *scales;
    const int32_t *zeros;
    __half *Y;
    int32_t *status;
    int M, K, N, G, splits;
    int xbox;          // bytes reserved per staged X' box (0 with the prologue)
    int stage_bytes;
    int prologue_bytes;
    UnpackConsts uk;
};

// x / s for 8 consecutive channels, rounded to binary16, stored in the
// pair order (0,4),(1,5),(2,6),(3,7) that the MMA fragments use.
__device__ __forceinline__ uint4 prescale8(uint4 xv, uint4 sv)
{
    const __half *x = reinterpret_cast<const __half *>(&xv);
    const __half *s = reinterpret_cast<const __half *>(&sv);
    __half o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = __float2half_rn(__fdiv_rn(__half2float(x[j]), __half2float(s[j])));
    uint4 r;
    r.x = __half_as_ushort(o[0]) | (static_cast<uint32_t>(__half_as_ushort(o[4])) << 16);
    r.y = __half_as_ushort(o[1]) | (static_cast<uint32_t>(__half_as_ushort(o[5])) << 16);
    r.z = __half_as_ushort(o[2]) | (static_cast<uint32_t>(__half_as_ushort(o[6])) << 16);
    r.w = __half_as_ushort(o[3]) | (static_cast<uint32_t>(__half_as_ushort(o[7])) << 16);
    return r;
}

__global__ void __launch_bounds__(256) prescale_kernel(const __half *__restrict__ X,
                                                      const __half *__restrict__ s, int64_t chunks,
                                                      int kchunks, __half *__restrict__ Xp)
{
    pdl_launch_dependents();
    pdl_wait();  // X may come from the previous kernel on the stream
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= chunks) return;
    const int kc = static_cast<int>(i % kchunks);
    const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(X) + i);
    const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(s) + kc);
    reinterpret_cast<uint4 *>(Xp)[i] = prescale8(xv, sv);
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// KH = warps per 32-column slab: with KH = 2 a warp pair splits each group's
// 128 rows (k 0..63 and 64..127), doubling the warps that hide MMA and
// shared-memory latency; the halves are summed in the epilogue.
template <int MT, bool PRO, int S, int KH>
__global__ void __launch_bounds__(32 * (4 * KH + 1), 1)
    small_m_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmX,
                   const Params p)
{
    constexpr int kConsumers = 4 * KH;
    constexpr int kCThreads = 32 * kConsumers;
    constexpr int kAllThreads = kCThreads + 32;
    constexpr int kSteps = 4 / KH;  // 32-row steps per warp per group

    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;  // == rank in the cluster
    const int n0 = blockIdx.y * kBN;
    const int g_begin = static_cast<int>(static_cast<int64_t>(split) * p.G / p.splits);
    const int g_end = static_cast<int>(static_cast<int64_t>(split + 1) * p.G / p.splits);
    const int ng = g_end - g_begin;
    const int chunks = ng * 16;  // 8-channel chunks of this CTA's k range

    // the next kernel on the stream may begin its own prologue now
    pdl_launch_dependents();

    uint8_t *xpro = smem + S * p.stage_bytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(xpro + p.prologue_bytes);
    uint64_t *empty = full + S;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1 + 32);     // expect_tx arrival + 32 cp.async arrivals
            mbar_init(&empty[i], kConsumers);  // one per consumer warp
        }
        fence_barrier_init();
    }
    __syncthreads();

    float acc[2][MT][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[a][j][i] = 0.0f;

    if (warp == kConsumers) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            if (!PRO) prefetch_tmap(&tmX);
            // Warm L2 with this CTA's packed weights while the previous kernel
            // on the stream finishes; the real loads below come after the wait.
            const int npf = ng < 64 ? ng : 64;
            for (int it = 0; it < npf; ++it)
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    tma_prefetch_l2_2d(&tmQ, n0 + 32 * w, (g_begin + it) * 16);
        }
        pdl_wait();
        const uint32_t tx = kQStage + (PRO ? 0 : 2 * p.M * 128);
        bool ok = true;
        for (int it = 0; it < ng; ++it) {
            const int st = it % S;
            if (it >= S && !mbar_wait(&empty[st], ((it / S) - 1) & 1)) {
                ok = false;
                break;
            }
            uint8_t *stg = smem + st * p.stage_bytes;
            const int g = g_begin + it;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[st], tx);
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    tma_load_2d(stg + w * 2048, &tmQ, &full[st], n0 + 32 * w, g * 16);
                if (!PRO) {
                    tma_load_2d(stg + kQStage, &tmX, &full[st], g * kGroup, 0);
                    tma_load_2d(stg + kQStage + p.xbox, &tmX, &full[st], g * kGroup + 64, 0);
                }
            }
            uint8_t *meta = stg + kQStage + 2 * p.xbox;
            if (lane < 16) {
                const int n = n0 + 8 * lane;
                const bool in = n < p.N;
                cp_async_16(meta + 16 * lane, p.scales + static_cast<size_t>(g) * p.N + (in ? n : 0),
                            in ? 16u : 0u);
            } else {
                const int wi = n0 / 8 + (lane - 16);
                const bool in = wi < p.N / 8;
                cp_async_4(meta + 256 + 4 * (lane - 16),
                           p.zeros + static_cast<size_t>(g) * (p.N / 8) + (in ? wi : 0), in ? 4u : 0u);
            }
            cp_async_arrive_noinc(&full[st]);
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    } else {
        // ------------------------------------------------------------ consumers
        const int gq = lane >> 2;
        const int t = lane & 3;
        const int slab = warp & 3;
        const int khalf = warp >> 2;            // 0 when KH == 1
        const int colw = 32 * slab + 4 * gq;    // my 4 columns: colw .. colw+3 (tile-local)
        pdl_wait();
        if (PRO) {
            const int total = p.M * chunks;
            for (int idx = threadIdx.x; idx < total; idx += kCThreads) {
                const int tok = idx / chunks;
                const int ch = idx - tok * chunks;
                const int k = g_begin * kGroup + ch * 8;
                const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(p.X + static_cast<size_t>(tok) * p.K + k));
                const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(p.s + k));
                *reinterpret_cast<uint4 *>(xpro + (static_cast<size_t>(tok) * chunks + (ch ^ (tok & 7))) * 16) =
                    prescale8(xv, sv);
            }
            named_bar_sync(1, kCThreads);
        }
        const uint32_t xpro_base = smem_u32(xpro);
        const UnpackConsts uk = p.uk;
        bool ok = true;
        for (int it = 0; it < ng; ++it) {
            const int st = it % S;
            if (!mbar_wait(&full[st], (it / S) & 1)) {
                ok = false;
                break;
            }
            const uint8_t *stg = smem + st * p.stage_bytes;
            const uint8_t *meta = stg + kQStage + 2 * p.xbox;
            const uint2 sc = *reinterpret_cast<const uint2 *>(meta + 2 * colw);
            const uint32_t zw = *reinterpret_cast<const uint32_t *>(meta + 256 + 4 * (colw >> 3));
            const int zsh = (colw & 7) * 4;
            uint32_t za[4], zb[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) zero_constants((zw >> (zsh + 4 * c)) & 15u, za[c], zb[c]);

            // with few token tiles, two accumulator sets (even / odd step) halve the
            // MMA dependency chains; more token tiles already give independent chains
            constexpr int kSets = MT <= 2 ? 2 : 1;
            float grp[kSets][2][MT][4];
#pragma unroll
            for (int b = 0; b < kSets; ++b)
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int j = 0; j < MT; ++j)
#pragma unroll
                        for (int i = 0; i < 4; ++i) grp[b][a][j][i] = 0.0f;

            const uint32_t qslab = smem_u32(stg) + slab * 2048;
            const uint32_t xstage = smem_u32(stg) + kQStage;
#pragma unroll
            for (int ss = 0; ss < kSteps; ++ss) {
                const int sidx = khalf * kSteps + ss;
                const int r = 8 * (sidx >> 1) + 2 * t + (sidx & 1);  // packed row in the group
                const uint4 wq = lds128(qslab + r * 128 + ((gq ^ (r & 7)) << 4));
                uint32_t bx[MT][4];
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    const int tok = 8 * j + gq;
                    if (tok < p.M) {
                        uint32_t addr;
                        if (PRO)
                            addr = xpro_base + ((tok * chunks) + ((it * 16 + r) ^ (tok & 7))) * 16;
                        else
                            addr = xstage + (sidx >> 1) * p.xbox + tok * 128 + (((r & 7) ^ (tok & 7)) << 4);
                        const uint4 v = lds128(addr);
                        bx[j][0] = v.x;
                        bx[j][1] = v.y;
                        bx[j][2] = v.z;
                        bx[j][3] = v.w;
                    } else {
                        bx[j][0] = bx[j][1] = bx[j][2] = bx[j][3] = 0u;
                    }
                }
                uint32_t d[4][4];
                unpack_minus_zero(wq.x, za[0], zb[0], d[0], uk);
                unpack_minus_zero(wq.y, za[1], zb[1], d[1], uk);
                unpack_minus_zero(wq.z, za[2], zb[2], d[2], uk);
                unpack_minus_zero(wq.w, za[3], zb[3], d[3], uk);
#pragma unroll
                for (int tile = 0; tile < 2; ++tile) {
                    const uint32_t a0[4] = {d[2 * tile][0], d[2 * tile + 1][0], d[2 * tile][1],
                                            d[2 * tile + 1][1]};
                    const uint32_t a1[4] = {d[2 * tile][2], d[2 * tile + 1][2], d[2 * tile][3],
                                            d[2 * tile + 1][3]};
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        mma_16816(grp[ss % kSets][tile][j], a0, bx[j][0], bx[j][1]);
                        mma_16816(grp[ss % kSets][tile][j], a1, bx[j][2], bx[j][3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
            const float2 s01 = __half22float2(*reinterpret_cast<const __half2 *>(&sc.x));
            const float2 s23 = __half22float2(*reinterpret_cast<const __half2 *>(&sc.y));
#pragma unroll
            for (int j = 0; j < MT; ++j) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float f0 = i < 2 ? s01.x : s01.y;
                    const float f1 = i < 2 ? s23.x : s23.y;
                    float p0 = grp[0][0][j][i], p1 = grp[0][1][j][i];
                    if (kSets == 2) {
                        p0 += grp[kSets - 1][0][j][i];
                        p1 += grp[kSets - 1][1][j][i];
                    }
                    acc[0][j][i] = fmaf(f0, p0, acc[0][j][i]);
                    acc[1][j][i] = fmaf(f1, p1, acc[1][j][i]);
                }
            }
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    }

    // ---------------------------------------------------------------- epilogue
    __syncthreads();  // every stage consumed: the ring can hold the partial tiles
    // red[khalf][token][column]
    float *red = reinterpret_cast<float *>(smem);
    constexpr int kHalfStride = 8 * MT * kRedPitch;
    if (warp < kConsumers) {
        const int gq = lane >> 2, t = lane & 3;
        const int colw = 32 * (warp & 3) + 4 * gq;
        float *rh = red + (warp >> 2) * kHalfStride;
#pragma unroll
        for (int tile = 0; tile < 2; ++tile)
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                const int tok = 8 * j + 2 * t;
                const int col = colw + 2 * tile;
                rh[tok * kRedPitch + col] = acc[tile][j][0];
                rh[(tok + 1) * kRedPitch + col] = acc[tile][j][1];
                rh[tok * kRedPitch + col + 1] = acc[tile][j][2];
                rh[(tok + 1) * kRedPitch + col + 1] = acc[tile][j][3];
            }
    }
    cluster_sync_all();
    // this rank finishes the 8-column chunks ch with ch % splits == rank,
    // summing the partials in (rank, k-half) order
    const uint32_t red_base = smem_u32(red);
    for (int e = threadIdx.x; e < p.M * 16; e += kAllThreads) {
        const int tok = e >> 4;
        const int ch = e & 15;
        const int n = n0 + ch * 8;
        if (ch % p.splits != split || n >= p.N) continue;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        for (int r = 0; r < p.splits; ++r) {
#pragma unroll
            for (int h = 0; h < KH; ++h) {
                const uint32_t off = red_base + (h * kHalfStride + tok * kRedPitch + ch * 8) * 4;
                const uint32_t a = map_to_rank(off, r);
                const float4 lo = ld_cluster_f4(a);
                const float4 hi = ld_cluster_f4(a + 16);
                v[0] += lo.x; v[1] += lo.y; v[2] += lo.z; v[3] += lo.w;
                v[4] += hi.x; v[5] += hi.y; v[6] += hi.z; v[7] += hi.w;
            }
        }
        uint4 o;
        o.x = __half_as_ushort(__float2half_rn(v[0])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[1]))) << 16);
        o.y = __half_as_ushort(__float2half_rn(v[2])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[3]))) << 16);
        o.z = __half_as_ushort(__float2half_rn(v[4])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[5]))) << 16);
        o.w = __half_as_ushort(__float2half_rn(v[6])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[7]))) << 16);
        *reinterpret_cast<uint4 *>(p.Y + static_cast<size_t>(tok) * p.N + n) = o;
    }
    cluster_sync_all();  // keep this CTA's partials alive until every rank has read them
}

template <int MT, bool PRO, int S, int KH>
cudaError_t launch_one(const SmallMPlan &plan, const CUtensorMap &tmQ, const CUtensorMap &tmX,
                       const Params &prm, cudaStream_t st)
{
    auto kern = small_m_kernel<MT, PRO, S, KH>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.splits, plan.n_tiles, 1);
    cfg.blockDim = dim3(32 * (4 * KH + 1), 1, 1);
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
    return cudaLaunchKernelEx(&cfg, kern, tmQ, tmX, prm);
}

template <int MT, bool PRO, int S, int KH>
cudaError_t configure_one()
{
    return cudaFuncSetAttribute(small_m_kernel<MT, PRO, S, KH>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemOptIn);
}

}  // namespace

cudaError_t configure_small_m()
{
    cudaError_t e = cudaSuccess;
    const cudaError_t r[] = {
        configure_one<1, true, stages_for(1), 2>(),  configure_one<1, true, stages_for(1), 1>(),
        configure_one<1, false, stages_for(1), 2>(), configure_one<2, false, stages_for(2), 2>(),
        configure_one<3, false, stages_for(3), 2>(), configure_one<4, false, stages_for(4), 2>(),
        configure_one<5, false, stages_for(5), 2>(), configure_one<6, false, stages_for(6), 2>(),
        configure_one<7, false, stages_for(7), 2>(), configure_one<8, false, stages_for(8), 2>()};
    for (cudaError_t x : r)
        if (x != cudaSuccess) e = x;
    return e;
}

#ifdef AWQ_TUNING
static int tune_env(const char *name, int dflt)
{
    const char *v = getenv(name);
    return v ? atoi(v) : dflt;
}
#endif

SmallMPlan plan_small_m(int M, int K, int N, int num_sms)
{
    SmallMPlan pl{};
    pl.mt = (M + 7) / 8;
    pl.n_tiles = (N + kBN - 1) / kBN;
    pl.stages = stages_for(pl.mt);
    pl.kh = 2;
    const int G = K / kGroup;
    const int max_split = G < 8 ? G : 8;
    const int target = 2 * num_sms;
    int splits = max_split;
    for (int sp = 1; sp <= max_split; ++sp) {
        if (pl.n_tiles * sp >= target && (G % sp == 0)) {
            splits = sp;
            break;
        }
    }
#ifdef AWQ_TUNING
    splits = tune_env("AWQ_TUNE_SPLITS", splits);
    if (splits > max_split) splits = max_split;
    if (splits < 1) splits = 1;
    if (pl.mt == 1) pl.kh = tune_env("AWQ_TUNE_KH", pl.kh);
#endif
    pl.prologue = false;
    if (pl.mt == 1) {
        // X / s in shared memory needs M * (groups per split) * 256 bytes
        for (int sp = splits; sp <= max_split; ++sp) {
            const int gmax = (G + sp - 1) / sp;
            if (static_cast<size_t>(M) * gmax * 256 <= kPrologueMax) {
                pl.prologue = true;
                splits = sp;
                break;
            }
        }
    }
    if (!pl.prologue) pl.kh = 2;
    pl.splits = splits;
    const int xbox = pl.prologue ? 0 : ((M * 128 + 1023) & ~1023);
    const int stage_bytes = (kQStage + 2 * xbox + kMetaBytes + 1023) & ~1023;
    const int gmax = (G + splits - 1) / splits;
    const size_t pro = pl.prologue ? static_cast<size_t>(M) * gmax * 256 : 0;
    pl.smem = 1024 /* alignment slack */ + static_cast<size_t>(pl.stages) * stage_bytes + pro +
              2 * pl.stages * sizeof(uint64_t);
    return pl;
}

cudaError_t launch_prescale(const __half *X, const __half *s, int M, int K, __half *Xp,
                            cudaStream_t st)
{
    const int64_t chunks = static_cast<int64_t>(M) * (K / 8);
    const int64_t blocks = (chunks + 255) / 256;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prescale_kernel, X, s, chunks, K / 8, Xp);
}

cudaError_t launch_small_m(const SmallMPlan &plan, const CUtensorMap &tmQ, const CUtensorMap &tmX,
                           const __half *X, const __half *s, const __half *scales,
                           const int32_t *zeros, __half *Y, int M, int K, int N,
                           int32_t *status, cudaStream_t st)
{
    Params prm{};
    prm.X = X;
    prm.s = s;
    prm.scales = scales;
    prm.zeros = zeros;
    prm.Y = Y;
    prm.status = status;
    prm.M = M;
    prm.K = K;
    prm.N = N;
    prm.G = K / kGroup;
    prm.splits = plan.splits;
    prm.xbox = plan.prologue ? 0 : ((M * 128 + 1023) & ~1023);
    prm.stage_bytes = (kQStage + 2 * prm.xbox + kMetaBytes + 1023) & ~1023;
    const int gmax = (prm.G + plan.splits - 1) / plan.splits;
    prm.prologue_bytes = plan.prologue ? M * gmax * 256 : 0;
    prm.uk = unpack_consts();
    switch (plan.mt) {
    case 1:
        if (plan.prologue)
            return plan.kh == 1 ? launch_one<1, true, stages_for(1), 1>(plan, tmQ, tmX, prm, st)
                                : launch_one<1, true, stages_for(1), 2>(plan, tmQ, tmX, prm, st);
        return launch_one<1, false, stages_for(1), 2>(plan, tmQ, tmX, prm, st);
    case 2: return launch_one<2, false, stages_for(2), 2>(plan, tmQ, tmX, prm, st);
    case 3: return launch_one<3, false, stages_for(3), 2>(plan, tmQ, tmX, prm, st);
    case 4: return launch_one<4, false, stages_for(4), 2>(plan, tmQ, tmX, prm, st);
    case 5: return launch_one<5, false, stages_for(5), 2>(plan, tmQ, tmX, prm, st);
    case 6: return launch_one<6, false, stages_for(6), 2>(plan, tmQ, tmX, prm, st);
    case 7: return launch_one<7, false, stages_for(7), 2>(plan, tmQ, tmX, prm, st);
    case 8: return launch_one<8, false, stages_for(8), 2>(plan, tmQ, tmX, prm, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace awq
