// gemv.cu -- Y = (X / s) . dequant(Q) for M <= 2 tokens: the single-token
// decode GEMV, the HBM-bound regime.
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (a GEMV kernel for batch size 1), "Group Size Configuration" and
// "Zero-Point Quantization" (4-bit codes, groups of 128, zero point).
//
// Every packed weight is read once from HBM.  To keep the per-weight work at a
// handful of integer ops, the zero point and the step leave the inner loop:
// with S0 / S1 the sums of X' over the group's even / odd k (k mod 8), and
// R0 = sum_{k even} x'_k (1024 + q_k),  R1 = sum_{k odd} x'_k (1024 + 16 q_k)
// (what the tensor cores produce when fed the raw OR-ed nibbles),
//   sum_k x'_k (q_k - z) = R0 + R1 / 16 - (1024 S0 + 64 S1) - z (S0 + S1),
// and the group's step multiplies that once.  S0, S1 are computed per CTA in
// the prologue together with X' = fp16(X / s), from the same rounded values.
//
// Schedule (persistent, stream-K).  A unit is one 128-column tile x one
// 128-row group (8 KB of packed words).  Units are numbered tile-major and cut
// into equal contiguous ranges, one per worker; a worker is a group of four
// warps with its own TMA ring, and a CTA (one per SM) holds kWorkers of them.
// Every CTA asks for the same fixed shared-memory footprint, under half of an
// SM, so the next call on the stream (programmatic dependent launch) finds a
// free slot on every SM while this one streams: its workers fetch their first
// weights before they wait on this call, and the per-call prologue and tail
// overlap the neighbouring calls' streaming.
//   workers     a lane of the first warp refills the worker's ring (four
//               16 x 32-word boxes, 128-byte swizzle, plus cp.async of the
//               group's steps and zero words); each warp owns 32 columns; a
//               lane turns one 16-byte load (4 columns x 8 k) into four
//               even-form and four odd-form f16x2 operands with LOP3 only and
//               feeds mma.sync m16n8k16 in swap-AB form (columns are MMA rows,
//               tokens MMA columns).
//   tiles       a tile inside one worker's range is written to Y directly.  A
//               tile split between workers leaves one float partial per worker
//               in the workspace; the worker that arrives last on the tile's
//               counter adds the partials in worker order (deterministic),
//               writes Y and resets the counter to zero.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kBN = 128;
constexpr int kQStage = 4 * 2048;   // packed words of one unit
constexpr int kMetaStage = 320;     // 256 B steps + 64 B zero words
constexpr int kWorkers = 3;         // four-warp workers per CTA
constexpr int kThreads = kWorkers * 128;
constexpr int kMaxStages = 4;
constexpr int kPrefetch = 8;        // units fetched into L2 ahead of their ring stage
// Fixed per-CTA footprint: two CTAs (with the 1 KB the system reserves for
// each) fit in an SM's 228 KB, whatever the shape.
constexpr int kFootprint = 112 * 1024;

struct GemvParams {
    const __half *X;
    const __half *s;
    const __half *scales;
    const int32_t *zeros;
    __half *Y;
    int32_t *status;
    uint32_t *counters;  // [n_tiles] arrivals on split tiles (zero between calls)
    float *part;         // [workers][2][M][128] partial sums of split tiles
    int M, K, N, G, n_tiles;
    int64_t units;       // n_tiles * G
    int workers;         // gridDim.x * kWorkers
    int stages;          // ring depth per worker
    int win;             // X' window capacity (groups per token)
    // Unpack constants, passed at run time: as compile-time literals the
    // compiler re-materializes them before every use (a LOP3 encodes only one
    // 32-bit immediate), which nearly doubles the integer-pipe work per weight.
    uint32_t mask_lo;  // 0x000F000F: nibbles 0 and 4 (after >> 8: 2 and 6)
    uint32_t mask_hi;  // 0x00F000F0: nibbles 1 and 5 (after >> 8: 3 and 7)
    uint32_t magic;    // 0x64006400: binary16 1024.0 in both halves
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// First unit of worker w (units cut into W equal contiguous ranges).
__host__ __device__ __forceinline__ int64_t range_begin(int64_t w, int64_t U, int64_t W)
{
    return w * U / W;
}

// The worker whose (non-empty) range holds unit u.
__device__ __forceinline__ int worker_of(int64_t u, int64_t U, int W)
{
    int w = static_cast<int>(u * W / U);
    while (w + 1 < W && range_begin(w + 1, U, W) <= u) ++w;
    while (w > 0 && range_begin(w, U, W) > u) --w;
    return w;
}

__device__ __forceinline__ uint32_t atomic_add_acq_rel(uint32_t *p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ uint2 pack4_half(float a, float b, float c, float d)
{
    uint2 o;
    o.x = __half_as_ushort(__float2half_rn(a)) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(b))) << 16);
    o.y = __half_as_ushort(__float2half_rn(c)) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(d))) << 16);
    return o;
}

// Finalize split tile t: add the partials of its workers in worker order and
// write Y.  Called by one worker's 128 threads, thread c owning column c of
// the tile; the partials are loaded eight workers at a time, then added in
// order, so the L2 round trips overlap.
__device__ __forceinline__ void finalize_tile(const GemvParams &p, int t, int c)
{
    const int64_t U = p.units;
    const int W = p.workers;
    const int64_t first = static_cast<int64_t>(t) * p.G, last = first + p.G - 1;
    const int wlo = worker_of(first, U, W), whi = worker_of(last, U, W);
    float v0 = 0.0f, v1 = 0.0f;
    for (int w0 = wlo; w0 <= whi; w0 += 8) {
        float a0[8], a1[8];
        bool use[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int w = w0 + j;
            a0[j] = 0.0f;
            a1[j] = 0.0f;
            use[j] = false;
            if (w <= whi) {
                const int64_t b = range_begin(w, U, W);
                if (range_begin(w + 1, U, W) > b) {  // non-empty range
                    use[j] = true;
                    const int side = (b / p.G == t) ? 0 : 1;
                    const float *slot = p.part + static_cast<size_t>(w * 2 + side) * p.M * kBN;
                    a0[j] = __ldcg(slot + c);
                    if (p.M > 1) a1[j] = __ldcg(slot + kBN + c);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (use[j]) {
                v0 += a0[j];
                v1 += a1[j];
            }
    }
    const int n = t * kBN + c;
    if (n < p.N) {
        p.Y[n] = __float2half_rn(v0);
        if (p.M > 1) p.Y[p.N + n] = __float2half_rn(v1);
    }
}

__device__ __forceinline__ int parts_of_tile(const GemvParams &p, int t)
{
    const int64_t U = p.units;
    const int W = p.workers;
    const int64_t first = static_cast<int64_t>(t) * p.G, last = first + p.G - 1;
    const int wlo = worker_of(first, U, W), whi = worker_of(last, U, W);
    int parts = 0;
    for (int w = wlo; w <= whi; ++w) parts += range_begin(w + 1, U, W) > range_begin(w, U, W) ? 1 : 0;
    return parts;
}

__global__ void __launch_bounds__(kThreads, 2) gemv_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                          const GemvParams p)
{
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wk = warp >> 2;   // worker in this CTA
    const int wig = warp & 3;   // warp in the worker: 32-column slab
    const int S = p.stages;
    const int G = p.G;

    uint8_t *words = smem;                                        // [kWorkers][S][8 KB]
    uint8_t *metas = words + kWorkers * S * kQStage;              // [kWorkers][S][320 B]
    uint8_t *xpro = metas + kWorkers * S * kMetaStage;            // [M][win][16 chunks][16 B]
    float2 *gmeta = reinterpret_cast<float2 *>(xpro + p.M * p.win * 256);  // [M][win]
    uint64_t *full = reinterpret_cast<uint64_t *>(gmeta + p.M * p.win);
    uint64_t *empty = full + kWorkers * kMaxStages;
    int *bcast = reinterpret_cast<int *>(empty + kWorkers * kMaxStages);

    pdl_launch_dependents();

    const int64_t U = p.units;
    const int W = p.workers;
    const int w = blockIdx.x * kWorkers + wk;
    const int64_t u0 = range_begin(w, U, W), u1 = range_begin(w + 1, U, W);
    const int nu = static_cast<int>(u1 - u0);
    // X' window of this CTA: the groups its units touch, kept as (g - wa) mod G
    const int64_t cu0 = range_begin(static_cast<int64_t>(blockIdx.x) * kWorkers, U, W);
    const int64_t cu1 = range_begin(static_cast<int64_t>(blockIdx.x + 1) * kWorkers, U, W);
    const int wa = (cu1 - cu0 >= G) ? 0 : static_cast<int>(cu0 % G);
    const int wsz = (cu1 - cu0 >= G) ? G : static_cast<int>(cu1 - cu0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kWorkers * kMaxStages; ++i) {
            mbar_init(&full[i], 1 + 32);  // expect_tx arrival + 32 cp.async arrivals
            mbar_init(&empty[i], 4);      // the worker's four warps
        }
        fence_barrier_init();
    }
    __syncthreads();

    uint8_t *wwords = words + wk * S * kQStage;
    uint8_t *wmeta = metas + wk * S * kMetaStage;
    uint64_t *wfull = full + wk * kMaxStages;
    uint64_t *wempty = empty + wk * kMaxStages;

    // Unit `it` of this worker's range into L2 (packed words by TMA prefetch,
    // steps and zero words by line prefetch), kPrefetch units ahead of its
    // ring stage, so that a ring refill waits on L2 rather than on DRAM.
    auto prefetch_unit = [&](int it) {
        const int64_t u = u0 + it;
        const int t = static_cast<int>(u / G);
        const int g = static_cast<int>(u - static_cast<int64_t>(t) * G);
        const int n0 = t * kBN;
        if (lane < 4) tma_prefetch_2d(&tmQ, n0 + 32 * lane, g * 16);
        else if (lane < 6) prefetch_l2(p.scales + static_cast<size_t>(g) * p.N + n0 + 64 * (lane - 4));
        else if (lane == 6 && p.zeros) prefetch_l2(p.zeros + static_cast<size_t>(g) * (p.N / 8) + n0 / 8);
    };

    // Stage `it` of this worker's range into ring slot it % S (whole warp 0).
    auto issue = [&](int it) {
        if (it >= S && it + kPrefetch < nu) prefetch_unit(it + kPrefetch);
        const int st = it % S;
        const int64_t u = u0 + it;
        const int t = static_cast<int>(u / G);
        const int g = static_cast<int>(u - static_cast<int64_t>(t) * G);
        const int n0 = t * kBN;
        uint8_t *stg = wwords + st * kQStage;
        if (lane == 0) {
            mbar_arrive_expect_tx(&wfull[st], kQStage);
#pragma unroll
            for (int b = 0; b < 4; ++b) tma_load_2d(stg + b * 2048, &tmQ, &wfull[st], n0 + 32 * b, g * 16);
        }
        uint8_t *meta = wmeta + st * kMetaStage;
        if (lane < 16) {
            const int n = n0 + 8 * lane;
            const bool in = n < p.N;
            cp_async_16(meta + 16 * lane, p.scales + static_cast<size_t>(g) * p.N + (in ? n : 0), in ? 16u : 0u);
        } else {
            const int wi = n0 / 8 + (lane - 16);
            const bool in = wi < p.N / 8;
            cp_async_4(meta + 256 + 4 * (lane - 16), zero_word_src(p.zeros, g, p.N / 8, in ? wi : 0, lane),
                       in ? 4u : 0u);
        }
        cp_async_arrive_noinc(&wfull[st]);
    };

    // The packed words, steps and zero words are layer state: no kernel that
    // triggers its dependents early writes them (the quantization kernels run
    // to completion first), which the C header states for callers.  The first
    // ring's worth is therefore fetched before the wait on the previous kernel.
    int issued = 0;
    if (wig == 0) {
        if (lane == 0) prefetch_tmap(&tmQ);
        const int pre = nu < S ? nu : S;
        for (int it = 0; it < pre; ++it) issue(it);
        for (int it = S; it < S + kPrefetch && it < nu; ++it) prefetch_unit(it);
        issued = pre;
    }
    pdl_wait();

    // ---------------------------------------------------------------- prologue
    // X' = fp16(X / s) for the CTA's window, stored per 8-channel chunk in the
    // order (0,4),(2,6),(1,5),(3,7) (even-form pairs, then odd-form pairs),
    // plus the per-(token, group) sums of X'.
    {
        const int sub = lane >> 4;  // two (token, slot) pairs per warp pass
        const int c16 = lane & 15;
        const int pairs = p.M * wsz;
        constexpr int kBatch = 2;
        for (int base = warp * 2; base < pairs; base += 2 * (kThreads / 32) * kBatch) {
            uint4 xv[kBatch], sv[kBatch];
            bool valid[kBatch];
            int tok[kBatch], sl[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int pair = base + b * 2 * (kThreads / 32) + sub;
                valid[b] = pair < pairs;
                tok[b] = valid[b] ? pair / wsz : 0;
                sl[b] = valid[b] ? pair - tok[b] * wsz : 0;
                xv[b] = make_uint4(0u, 0u, 0u, 0u);
                sv[b] = xv[b];
                if (valid[b]) {
                    int g = wa + sl[b];
                    if (g >= G) g -= G;
                    const int k = g * kGroup + c16 * 8;
                    xv[b] = __ldg(reinterpret_cast<const uint4 *>(p.X + static_cast<size_t>(tok[b]) * p.K + k));
                    // s == NULL: X already holds X/s (division by 1 is exact)
                    sv[b] = p.s ? __ldg(reinterpret_cast<const uint4 *>(p.s + k))
                                : make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
                }
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                float e = 0.0f, o = 0.0f;
                if (valid[b]) {
                    const __half *xh = reinterpret_cast<const __half *>(&xv[b]);
                    const __half *sh = reinterpret_cast<const __half *>(&sv[b]);
                    __half q[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        q[j] = __float2half_rn(__fdiv_rn(__half2float(xh[j]), __half2float(sh[j])));
                    e = (__half2float(q[0]) + __half2float(q[2])) + (__half2float(q[4]) + __half2float(q[6]));
                    o = (__half2float(q[1]) + __half2float(q[3])) + (__half2float(q[5]) + __half2float(q[7]));
                    uint4 r;
                    r.x = __half_as_ushort(q[0]) | (static_cast<uint32_t>(__half_as_ushort(q[4])) << 16);
                    r.y = __half_as_ushort(q[2]) | (static_cast<uint32_t>(__half_as_ushort(q[6])) << 16);
                    r.z = __half_as_ushort(q[1]) | (static_cast<uint32_t>(__half_as_ushort(q[5])) << 16);
                    r.w = __half_as_ushort(q[3]) | (static_cast<uint32_t>(__half_as_ushort(q[7])) << 16);
                    *reinterpret_cast<uint4 *>(
                        xpro + ((static_cast<size_t>(tok[b]) * p.win + sl[b]) * 16 + (c16 ^ (tok[b] & 7))) * 16) = r;
                }
                // butterfly over the 16 lanes of one (token, slot) pair (fixed order)
#pragma unroll
                for (int off = 8; off > 0; off >>= 1) {
                    e += __shfl_xor_sync(0xffffffffu, e, off);
                    o += __shfl_xor_sync(0xffffffffu, o, off);
                }
                if (valid[b] && c16 == 0)
                    gmeta[tok[b] * p.win + sl[b]] = make_float2(fmaf(1024.0f, e, 64.0f * o), e + o);
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- main loop
    const int gq = lane >> 2;
    const int t4 = lane & 3;
    const int colw = 32 * wig + 4 * gq;
    const int tok0 = 2 * t4;
    // This lane's X' row (tokens beyond M never load it).  A chunk index
    // slot * 16 + r XOR-swizzled by gq < 8 equals slot * 16 + (r ^ gq).
    const uint8_t *xrow = xpro + static_cast<size_t>(gq) * p.win * 256;
    const uint32_t mlo = p.mask_lo, mhi = p.mask_hi, magic = p.magic;
    const uint32_t bar_id = 1 + wk;
    const int t_first = static_cast<int>(u0 / G);
    bool ok = true;
    int split_head = -1, split_tail = -1;  // first / last tile, when shared with other workers

    float acc[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[a][i] = 0.0f;

    for (int it = 0; it < nu; ++it) {
        const int st = it % S;
        const int64_t u = u0 + it;
        const int t = static_cast<int>(u / G);
        const int g = static_cast<int>(u - static_cast<int64_t>(t) * G);
        if (ok && !mbar_wait(&wfull[st], (it / S) & 1)) ok = false;
        if (ok) {
            const uint8_t *stg = wwords + st * kQStage;
            const uint8_t *meta = wmeta + st * kMetaStage;
            const uint2 sc = *reinterpret_cast<const uint2 *>(meta + 2 * colw);
            const uint32_t zw = *reinterpret_cast<const uint32_t *>(meta + 256 + 4 * (colw >> 3));
            int sl = g - wa;
            if (sl < 0) sl += G;

            float R[2][2][4];  // [tile][form][c]
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int f = 0; f < 2; ++f)
#pragma unroll
                    for (int i = 0; i < 4; ++i) R[a][f][i] = 0.0f;

            const uint8_t *qslab = stg + wig * 2048;
            const uint8_t *xs = xrow + sl * 256;
#pragma unroll
            for (int ss = 0; ss < 4; ++ss) {
                const int r = 8 * (ss >> 1) + 2 * t4 + (ss & 1);
                const uint4 wq = *reinterpret_cast<const uint4 *>(qslab + r * 128 + ((gq ^ (r & 7)) << 4));
                uint4 bx = make_uint4(0u, 0u, 0u, 0u);
                if (gq < p.M) bx = *reinterpret_cast<const uint4 *>(xs + ((r ^ gq) << 4));
                const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
                uint32_t ev0[4], ev2[4], od1[4], od3[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t w8 = wv[c] >> 8;
                    ev0[c] = (wv[c] & mlo) | magic;  // 1024 + q0, 1024 + q4
                    ev2[c] = (w8 & mlo) | magic;     // 1024 + q2, 1024 + q6
                    od1[c] = (wv[c] & mhi) | magic;  // 1024 + 16 q1, 1024 + 16 q5
                    od3[c] = (w8 & mhi) | magic;     // 1024 + 16 q3, 1024 + 16 q7
                }
#pragma unroll
                for (int tile = 0; tile < 2; ++tile) {
                    const int c0 = 2 * tile, c1 = 2 * tile + 1;
                    const uint32_t ae[4] = {ev0[c0], ev0[c1], ev2[c0], ev2[c1]};
                    const uint32_t ao[4] = {od1[c0], od1[c1], od3[c0], od3[c1]};
                    mma_16816(R[tile][0], ae, bx.x, bx.y);
                    mma_16816(R[tile][1], ao, bx.z, bx.w);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&wempty[st]);

            // group epilogue: y += step * (R0 + R1/16 - (1024 S0 + 64 S1) - z (S0 + S1))
            const float2 gm0 = tok0 < p.M ? gmeta[tok0 * p.win + sl] : make_float2(0.f, 0.f);
            const float2 gm1 = tok0 + 1 < p.M ? gmeta[(tok0 + 1) * p.win + sl] : make_float2(0.f, 0.f);
            const int zsh = (colw & 7) * 4;
            const __half2 s01 = *reinterpret_cast<const __half2 *>(&sc.x);
            const __half2 s23 = *reinterpret_cast<const __half2 *>(&sc.y);
            const float stp[4] = {__low2float(s01), __high2float(s01), __low2float(s23), __high2float(s23)};
#pragma unroll
            for (int tile = 0; tile < 2; ++tile)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = 2 * tile + (i >> 1);
                    // the 4-bit zero as a float: 2^23 + z exactly, minus 2^23
                    const float z = __int_as_float(((zw >> (zsh + 4 * c)) & 15u) | 0x4B000000u) - 8388608.0f;
                    const float2 gm = (i & 1) ? gm1 : gm0;
                    float pgrp = fmaf(R[tile][1][i], 0.0625f, R[tile][0][i]) - gm.x;
                    pgrp = fmaf(-z, gm.y, pgrp);
                    acc[tile][i] = fmaf(stp[c], pgrp, acc[tile][i]);
                }
            // refill the slot just released, once all four warps are done with it
            if (wig == 0 && it + S < nu) {
                if (mbar_wait(&wempty[st], (it / S) & 1)) {
                    issue(it + S);
                    issued = it + S + 1;
                } else {
                    ok = false;
                }
            }
        }

        // ------------------------------------------------------------ tile end
        if (g == G - 1 || it == nu - 1) {
            const bool whole = static_cast<int64_t>(t) * G >= u0 && static_cast<int64_t>(t + 1) * G <= u1;
            if (whole) {
                const int n = t * kBN + colw;
                if (ok && t4 == 0 && n < p.N) {
                    *reinterpret_cast<uint2 *>(p.Y + n) = pack4_half(acc[0][0], acc[0][2], acc[1][0], acc[1][2]);
                    if (p.M > 1)
                        *reinterpret_cast<uint2 *>(p.Y + p.N + n) =
                            pack4_half(acc[0][1], acc[0][3], acc[1][1], acc[1][3]);
                }
            } else {
                // split tile: publish this worker's partial; the arrivals on the
                // tiles' counters happen once, after the range
                const int side = (t == t_first) ? 0 : 1;
                float *slot = p.part + static_cast<size_t>(w * 2 + side) * p.M * kBN;
                if (t4 == 0) {
                    __stcg(reinterpret_cast<float4 *>(slot + colw),
                           make_float4(acc[0][0], acc[0][2], acc[1][0], acc[1][2]));
                    if (p.M > 1)
                        __stcg(reinterpret_cast<float4 *>(slot + kBN + colw),
                               make_float4(acc[0][1], acc[0][3], acc[1][1], acc[1][3]));
                }
                if (side == 0)
                    split_head = t;
                else
                    split_tail = t;
            }
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[a][i] = 0.0f;
        }
    }

    // Arrive on the split tiles (the partial writes of all four warps are
    // ordered before the arrival by the named barrier); whoever arrives last
    // on a tile adds its partials and writes Y.
    if (split_head >= 0 || split_tail >= 0) {
        named_bar_sync(bar_id, 128);
        if (wig == 0 && lane == 0) {
            uint32_t old0 = 0, old1 = 0;
            if (split_head >= 0) old0 = atomic_add_acq_rel(p.counters + split_head, 1u);
            if (split_tail >= 0) old1 = atomic_add_acq_rel(p.counters + split_tail, 1u);
            bcast[2 * wk] = split_head >= 0 && static_cast<int>(old0) == parts_of_tile(p, split_head) - 1;
            bcast[2 * wk + 1] = split_tail >= 0 && static_cast<int>(old1) == parts_of_tile(p, split_tail) - 1;
        }
        named_bar_sync(bar_id, 128);
        const int c = 32 * wig + lane;
        if (bcast[2 * wk]) {
            if (ok) finalize_tile(p, split_head, c);
            if (wig == 0 && lane == 0) p.counters[split_head] = 0u;
        }
        if (bcast[2 * wk + 1]) {
            if (ok) finalize_tile(p, split_tail, c);
            if (wig == 0 && lane == 0) p.counters[split_tail] = 0u;
        }
    }

    // After a wait ran out, let the copies already issued land before exiting
    // (each wait bounded again).
    if (wig == 0) {
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (!ok) {
            for (int it = 0; it < issued; ++it) {
                // only the slots still holding an unconsumed stage matter; the
                // last S issued stages cover them
                if (it + S < issued) continue;
                mbar_wait_for(&wfull[it % S], (it / S) & 1, kDrainLimitNs);
            }
        }
    }
    if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
}

}  // namespace

cudaError_t configure_gemv()
{
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFootprint);
    if (e != cudaSuccess) return e;
    // all of the SM's unified memory as shared memory: two CTAs per SM
    return cudaFuncSetAttribute(gemv_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared);
}

size_t gemv_part_bytes(int M)
{
    return static_cast<size_t>(kGemvMaxCtas) * kWorkers * 2 * M * kBN * sizeof(float);
}

bool plan_gemv(int M, int K, int N, int num_sms, GemvPlan *pl)
{
    if (M < 1 || M > 2 || K < kGroup || K % kGroup != 0) return false;
    const int G = K / kGroup;
    const int n_tiles = (N + kBN - 1) / kBN;
    const int64_t U = static_cast<int64_t>(n_tiles) * G;
    int ctas = num_sms < kGemvMaxCtas ? num_sms : kGemvMaxCtas;
    const int64_t need = (U + kWorkers - 1) / kWorkers;  // at least one unit per worker
    if (need < ctas) ctas = static_cast<int>(need);
    if (ctas < 1) ctas = 1;
    // the largest X' window any CTA needs (groups per token)
    int win = 0;
    for (int c = 0; c < ctas; ++c) {
        const int64_t cnt = range_begin(c + 1, U, ctas) - range_begin(c, U, ctas);
        const int wsz = cnt >= G ? G : static_cast<int>(cnt);
        if (wsz > win) win = wsz;
    }
    if (win < 1) win = 1;
    for (int S = kMaxStages; S >= 2; --S) {
        const size_t bytes = 1024 + static_cast<size_t>(kWorkers) * S * (kQStage + kMetaStage) +
                             static_cast<size_t>(M) * win * (256 + 8) +
                             2 * kWorkers * kMaxStages * sizeof(uint64_t) + 16 * sizeof(int);
        if (bytes <= static_cast<size_t>(kFootprint)) {
            pl->ctas = ctas;
            pl->stages = S;
            pl->win = win;
            pl->n_tiles = n_tiles;
            pl->smem = kFootprint;
            return true;
        }
    }
    return false;
}

cudaError_t launch_gemv(const GemvPlan &plan, const CUtensorMap &tmQ, const __half *X,
                        const __half *s, const __half *scales, const int32_t *zeros, __half *Y,
                        int M, int K, int N, uint32_t *counters, float *part, int32_t *status,
                        cudaStream_t st)
{
    GemvParams prm{};
    prm.X = X;
    prm.s = s;
    prm.scales = scales;
    prm.zeros = zeros;
    prm.Y = Y;
    prm.status = status;
    prm.counters = counters;
    prm.part = part;
    prm.M = M;
    prm.K = K;
    prm.N = N;
    prm.G = K / kGroup;
    prm.n_tiles = plan.n_tiles;
    prm.units = static_cast<int64_t>(plan.n_tiles) * prm.G;
    prm.workers = plan.ctas * kWorkers;
    prm.stages = plan.stages;
    prm.win = plan.win;
    prm.mask_lo = 0x000F000Fu;
    prm.mask_hi = 0x00F000F0u;
    prm.magic = 0x64006400u;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.ctas, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_kernel, tmQ, prm);
}

}  // namespace awq
