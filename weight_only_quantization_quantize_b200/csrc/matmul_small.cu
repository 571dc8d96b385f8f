// matmul_small.cu -- Y = (X / s) . dequant(Q) for M < 64 tokens (decode and
// small batches), the HBM-bound regime of the W4A16 linear layer.
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (a GEMV kernel for batch size 1, a GEMM kernel for batches) and
// "Group Size Configuration" / "Zero-Point Quantization" (4-bit codes, group
// 128, zero point).
//
// Design (B200), for 1 <= M < 64 tokens (the single-token GEMV with small K
// uses gemv.cu instead):
//  * Weights stream once from HBM: a producer warp issues TMA tile loads of
//    the packed words (one 16-row x 32-column box per consumer warp, 128-byte
//    swizzled so the consumers' 16-byte shared loads are conflict free), of the
//    group's X / s rows (written once by a pre-pass), plus cp.async copies of
//    the group's scales and zero points, into a ring of mbarrier-guarded
//    stages; one stage is one 128-row group.
//  * Four consumer warps each own 32 output columns.  A lane turns one 16-byte
//    load (4 columns x 8 consecutive k) into binary16 (q - z) * step values
//    (two LOP3 masks + f16x2 ops per pair, the step applied in binary16 as in
//    the tensor-core GEMM) and feeds them from registers to mma.sync m16n8k16
//    (fp32 accumulate) in swap-AB form: output columns are the MMA rows, the
//    M tokens (up to 8 tiles of 8) its columns.  The contraction order inside
//    each 8-k word is permuted (pairs (0,4),(1,5),(2,6),(3,7)); X / s is stored
//    with the same permutation.
//  * Split-K across the CTAs of a thread-block cluster; each CTA pushes its
//    partial columns into the shared memory of the rank that owns them
//    (st.async, completion counted on the owner's mbarrier) and the owner sums
//    them in rank order (deterministic).
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kBN = 128;            // output columns per CTA
constexpr int kQStage = 4 * 2048;   // 4 boxes of [16 rows x 32 words]
constexpr int kMetaGroups = 64;      // the steps and zero words of up to this many groups live in shared memory
constexpr int kSmemOptIn = 232448;  // 227 KB, the per-block opt-in maximum


struct Params {
    const __half *X;
    const __half *s;
    const __half *scales;
    const int32_t *zeros;
    __half *Y;
    int32_t *status;
    int M, K, N, G, splits;
    int xbox;          // bytes reserved per staged X' box
    int stage_bytes;
    int cmeta_bytes;   // the CTA's steps [group][128] binary16, then zero words [group][16]
    int meta_smem;     // 1: those are staged in shared memory; 0 (longer k ranges): read from global memory
    int recv_bytes;    // partials pushed to this CTA: [src rank][8 * MT tokens][128 / splits]
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
    // s == NULL: X already holds X/s; dividing by 1 leaves it bit for bit
    const uint4 sv = s ? __ldg(reinterpret_cast<const uint4 *>(s) + kc)
                       : make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
    reinterpret_cast<uint4 *>(Xp)[i] = prescale8(xv, sv);
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

template <int MT, int S>
__global__ void __launch_bounds__(160, 1)
    small_m_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmX,
                   const Params p)
{
    constexpr int kConsumers = 4;
    constexpr int kAllThreads = 160;

    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;  // == rank in the cluster
    const int n0 = blockIdx.y * kBN;
    const int g_begin = static_cast<int>(static_cast<int64_t>(split) * p.G / p.splits);
    const int g_end = static_cast<int>(static_cast<int64_t>(split + 1) * p.G / p.splits);
    const int ng = g_end - g_begin;
    const int cpo = kBN / p.splits;

    pdl_launch_dependents();

    uint8_t *csteps = smem + S * p.stage_bytes;
    uint8_t *czeros = csteps + ng * 256;
    float *recv = reinterpret_cast<float *>(csteps + p.cmeta_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(csteps + p.cmeta_bytes + p.recv_bytes);
    uint64_t *empty = full + S;
    uint64_t *recv_bar = empty + S;
    uint64_t *meta_bar = recv_bar + 1;  // the CTA's steps and zero words have landed

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);  // expect_tx arrival
            mbar_init(&empty[i], kConsumers);
        }
        mbar_init(recv_bar, 1);
        mbar_init(meta_bar, 32);
        fence_barrier_init();
        mbar_arrive_expect_tx(recv_bar, p.M * cpo * p.splits * 4);
    }
    __syncthreads();
    cluster_arrive_relaxed();  // the init fence above releases the barriers

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
            prefetch_tmap(&tmX);
        }
        // The steps and zero words of all of the CTA's groups, once (layer
        // state, so before the wait on the previous kernel).
        for (int c = lane; p.meta_smem && c < ng * 16; c += 32) {
            const int gi = c >> 4, c16 = c & 15;
            const int gg = g_begin + gi;
            const int n = n0 + 8 * c16;
            const bool in_s = n < p.N;
            cp_async_16(csteps + gi * 256 + 16 * c16, p.scales + static_cast<size_t>(gg) * p.N + (in_s ? n : 0),
                        in_s ? 16u : 0u);
            const int wi = n0 / 8 + c16;
            const bool in_z = wi < p.N / 8;
            cp_async_4(czeros + gi * 64 + 4 * c16, zero_word_src(p.zeros, gg, p.N / 8, in_z ? wi : 0, c16),
                       in_z ? 4u : 0u);
        }
        cp_async_arrive_noinc(meta_bar);
        pdl_wait();
        // the X' boxes hold 8 MT token rows (rows at and beyond M read as zero)
        const uint32_t tx = kQStage + 2 * (8 * MT) * 128;
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
                tma_load_2d(stg + kQStage, &tmX, &full[st], g * kGroup, 0);
                tma_load_2d(stg + kQStage + p.xbox, &tmX, &full[st], g * kGroup + 64, 0);
            }
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    } else {
        // ------------------------------------------------------------ consumers
        const int gq = lane >> 2;
        const int t = lane & 3;
        const int colw = 32 * warp + 4 * gq;  // my 4 columns: colw .. colw+3 (tile-local)
        const UnpackConsts uk = p.uk;
        // this lane's shared-memory offsets within a stage, computed once:
        // packed row r = 8 (sidx / 2) + 2 t + sidx % 2, chunk gq XOR-swizzled by
        // the row; X' row of token 8 j + gq, chunk r % 8 XOR-swizzled by the token
        uint32_t qoff[4], xoff[4][MT];
#pragma unroll
        for (int sidx = 0; sidx < 4; ++sidx) {
            const int r = 8 * (sidx >> 1) + 2 * t + (sidx & 1);
            qoff[sidx] = static_cast<uint32_t>(warp * 2048 + r * 128 + ((gq ^ (r & 7)) << 4));
#pragma unroll
            for (int j = 0; j < MT; ++j)
                xoff[sidx][j] = static_cast<uint32_t>(kQStage + (sidx >> 1) * p.xbox + (8 * j + gq) * 128 +
                                                      (((r & 7) ^ gq) << 4));
        }
        bool ok = __all_sync(0xffffffffu, mbar_wait(meta_bar, 0));
        for (int it = 0; ok && it < ng; ++it) {
            const int st = it % S;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (it / S) & 1))) {
                ok = false;
                break;
            }
            const uint8_t *stg = smem + st * p.stage_bytes;
            uint2 sc;
            uint32_t zw;
            if (p.meta_smem) {
                sc = *reinterpret_cast<const uint2 *>(csteps + it * 256 + 2 * colw);
                zw = *reinterpret_cast<const uint32_t *>(czeros + it * 64 + 4 * (colw >> 3));
            } else {
                // long k ranges: straight from global memory (L2); columns past N read as zero
                const int g = g_begin + it, n = n0 + colw;
                const bool in = n < p.N;
                sc = in ? __ldg(reinterpret_cast<const uint2 *>(p.scales + static_cast<size_t>(g) * p.N + n))
                        : make_uint2(0u, 0u);
                zw = !in ? 0u
                         : (p.zeros ? static_cast<uint32_t>(__ldg(p.zeros + static_cast<size_t>(g) * (p.N / 8) + n / 8))
                                    : kSymmetricZeroWords[0]);
            }
            const int zsh = (colw & 7) * 4;
            uint32_t za[4], zb[4], st2[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) zero_constants((zw >> (zsh + 4 * c)) & 15u, za[c], zb[c]);
            {
                const uint32_t s01 = sc.x, s23 = sc.y;
                st2[0] = (s01 & 0xFFFFu) * 0x10001u;
                st2[1] = (s01 >> 16) * 0x10001u;
                st2[2] = (s23 & 0xFFFFu) * 0x10001u;
                st2[3] = (s23 >> 16) * 0x10001u;
            }
            const uint32_t sbase = smem_u32(stg);
#pragma unroll
            for (int sidx = 0; sidx < 4; ++sidx) {
                uint32_t w[4];
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                             : "r"(sbase + qoff[sidx]));
                uint4 bx[MT];
#pragma unroll
                for (int j = 0; j < MT; ++j)
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(bx[j].x), "=r"(bx[j].y), "=r"(bx[j].z), "=r"(bx[j].w)
                                 : "r"(sbase + xoff[sidx][j]));
                uint32_t d[4][4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t e[4];
                    unpack_minus_zero(w[c], za[c], zb[c], e, uk);
#pragma unroll
                    for (int i = 0; i < 4; ++i) asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d[c][i]) : "r"(e[i]), "r"(st2[c]));
                }
#pragma unroll
                for (int tile = 0; tile < 2; ++tile) {
                    const uint32_t a0[4] = {d[2 * tile][0], d[2 * tile + 1][0], d[2 * tile][1], d[2 * tile + 1][1]};
                    const uint32_t a1[4] = {d[2 * tile][2], d[2 * tile + 1][2], d[2 * tile][3], d[2 * tile + 1][3]};
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        mma_16816(acc[tile][j], a0, bx[j].x, bx[j].y);
                        mma_16816(acc[tile][j], a1, bx[j].z, bx[j].w);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    }

    // ---------------------------------------------------------------- epilogue
    // Push: a consumer thread holds columns colw .. colw+3 (one 8-column chunk)
    // for tokens 8j + 2t, 8j + 2t + 1; the chunk's owner is rank chunk % splits.
    cluster_wait_acquire();
    if (warp < kConsumers) {
        const int gq = lane >> 2, t = lane & 3;
        const int colw = 32 * warp + 4 * gq;
        const int chunk = colw >> 3;
        const uint32_t owner = static_cast<uint32_t>(chunk % p.splits);
        const int lc = (chunk / p.splits) * 8 + (colw & 7);
        const uint32_t rbar = map_to_rank(smem_u32(recv_bar), owner);
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
            for (int tk = 0; tk < 2; ++tk) {
                const int tok = 8 * j + 2 * t + tk;
                if (tok < p.M) {
                    const float4 v = make_float4(acc[0][j][tk], acc[0][j][2 + tk], acc[1][j][tk], acc[1][j][2 + tk]);
                    const int off = ((split * 8 * MT + tok) * cpo + lc) * 4;
                    st_async_f4(map_to_rank(smem_u32(recv) + off, owner), v, rbar);
                }
            }
    }
    // Arrive once the pushes are issued (no fence: every owner waits for all
    // the bytes pushed to it before it reduces, hence before it exits).
    cluster_arrive_relaxed();
    if (!mbar_wait(recv_bar, 0) && threadIdx.x == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    const int lchunks = cpo / 8;
    for (int e = threadIdx.x; e < p.M * lchunks; e += kAllThreads) {
        const int tok = e / lchunks;
        const int lch = e - tok * lchunks;
        const int n = n0 + (lch * p.splits + split) * 8;
        if (n >= p.N) continue;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        for (int r = 0; r < p.splits; ++r) {
            const float4 *src = reinterpret_cast<const float4 *>(recv + ((r * 8 * MT) + tok) * cpo + lch * 8);
            const float4 lo = src[0], hi = src[1];
            v[0] += lo.x; v[1] += lo.y; v[2] += lo.z; v[3] += lo.w;
            v[4] += hi.x; v[5] += hi.y; v[6] += hi.z; v[7] += hi.w;
        }
        uint4 o;
        o.x = __half_as_ushort(__float2half_rn(v[0])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[1]))) << 16);
        o.y = __half_as_ushort(__float2half_rn(v[2])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[3]))) << 16);
        o.z = __half_as_ushort(__float2half_rn(v[4])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[5]))) << 16);
        o.w = __half_as_ushort(__float2half_rn(v[6])) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v[7]))) << 16);
        *reinterpret_cast<uint4 *>(p.Y + static_cast<size_t>(tok) * p.N + n) = o;
    }
    cluster_wait_acquire();
}

template <int MT, int S>
cudaError_t launch_one(const SmallMPlan &plan, const CUtensorMap &tmQ, const CUtensorMap &tmX,
                       const Params &prm, cudaStream_t st)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.splits, plan.n_tiles, 1);
    cfg.blockDim = dim3(160, 1, 1);
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
    return cudaLaunchKernelEx(&cfg, small_m_kernel<MT, S>, tmQ, tmX, prm);
}

template <int MT, int S>
cudaError_t configure_one()
{
    return cudaFuncSetAttribute(small_m_kernel<MT, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemOptIn);
}

// steps (256 B) and zero words (64 B) per group of the largest k range, when
// they are staged in shared memory
int cmeta_bytes_for(int G, int splits)
{
    const int gmax = (G + splits - 1) / splits;
    return gmax <= kMetaGroups ? gmax * 320 : 0;
}

int stage_bytes_for(int M)
{
    const int xbox = (((M + 7) / 8) * 8 * 128 + 1023) & ~1023;
    return (kQStage + 2 * xbox + 1023) & ~1023;
}

}  // namespace

cudaError_t configure_small_m()
{
    const cudaError_t r[] = {configure_one<1, 4>(), configure_one<2, 4>(), configure_one<3, 4>(), configure_one<4, 4>(),
                             configure_one<5, 4>(), configure_one<6, 4>(), configure_one<7, 4>(),
                             configure_one<8, 4>(), configure_one<1, 3>(), configure_one<2, 3>(),
                             configure_one<3, 3>()};
    for (cudaError_t x : r)
        if (x != cudaSuccess) return x;
    return cudaSuccess;
}


SmallMPlan plan_small_m(int M, int K, int N, int num_sms)
{
    SmallMPlan pl{};
    pl.mt = (M + 7) / 8;
    pl.n_tiles = (N + kBN - 1) / kBN;
    pl.prologue = false;
    pl.kh = 1;
    // A 4-deep ring, or 3-deep (up to 24 tokens) when that lets more CTAs
    // share an SM and so a finer split fit in one wave: measured on the 13B
    // set, resident CTAs beat ring depth (8 deep lost 8% at 8 tokens and 30%
    // at 16 against 4 deep).
    const int G = K / kGroup;
    int max_pow2 = 1;
    while (max_pow2 * 2 <= 8 && max_pow2 * 2 <= G) max_pow2 *= 2;
    const int stage_bytes = stage_bytes_for(M);
    const int recv_bytes = 8 * pl.mt * kBN * 4;
    int best_splits = 0;
    for (int stages = 4; stages >= (pl.mt <= 3 ? 3 : 4); --stages) {
        // one wave: the largest power-of-two split with n_tiles * splits <= CTAs
        // resident (the steps and zero words of a CTA's groups shrink as the
        // split grows)
        int splits = 1;
        size_t smem = 0;
        for (;;) {
            const int s2 = splits * 2;
            const size_t sm2 = 1024 + static_cast<size_t>(stages) * stage_bytes + cmeta_bytes_for(G, s2) + recv_bytes +
                               (2 * stages + 2) * 8;
            const int per_sm = static_cast<int>(228 * 1024 / (sm2 + 1024));
            if (s2 > max_pow2 || pl.n_tiles * s2 > (per_sm < 1 ? 1 : per_sm) * num_sms) break;
            splits = s2;
        }
        smem = 1024 + static_cast<size_t>(stages) * stage_bytes + cmeta_bytes_for(G, splits) + recv_bytes +
               (2 * stages + 2) * 8;
        if (splits > best_splits) {
            best_splits = splits;
            pl.splits = splits;
            pl.stages = stages;
            pl.smem = smem;
        }
    }
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
    prm.xbox = (((M + 7) / 8) * 8 * 128 + 1023) & ~1023;
    prm.stage_bytes = stage_bytes_for(M);
    prm.cmeta_bytes = cmeta_bytes_for(K / kGroup, plan.splits);
    prm.meta_smem = prm.cmeta_bytes > 0 ? 1 : 0;
    prm.recv_bytes = 8 * plan.mt * kBN * 4;
    prm.uk = unpack_consts();
    if (plan.stages == 3) {
        switch (plan.mt) {
        case 1: return launch_one<1, 3>(plan, tmQ, tmX, prm, st);
        case 2: return launch_one<2, 3>(plan, tmQ, tmX, prm, st);
        case 3: return launch_one<3, 3>(plan, tmQ, tmX, prm, st);
        default: return cudaErrorInvalidValue;
        }
    }
    switch (plan.mt) {
    case 1: return launch_one<1, 4>(plan, tmQ, tmX, prm, st);
    case 2: return launch_one<2, 4>(plan, tmQ, tmX, prm, st);
    case 3: return launch_one<3, 4>(plan, tmQ, tmX, prm, st);
    case 4: return launch_one<4, 4>(plan, tmQ, tmX, prm, st);
    case 5: return launch_one<5, 4>(plan, tmQ, tmX, prm, st);
    case 6: return launch_one<6, 4>(plan, tmQ, tmX, prm, st);
    case 7: return launch_one<7, 4>(plan, tmQ, tmX, prm, st);
    case 8: return launch_one<8, 4>(plan, tmQ, tmX, prm, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace awq
