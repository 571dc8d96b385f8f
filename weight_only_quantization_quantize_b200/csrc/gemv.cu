// gemv.cu -- Y = (X / s) . dequant(Q) for M <= 2 tokens: the single-token
// decode GEMV (and two-token steps), the HBM-bound regime.
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (a GEMV kernel for batch size 1), "Group Size Configuration" and
// "Zero-Point Quantization" (4-bit codes, groups of 128, zero point).
//
// Every packed weight is read once from HBM.  To keep the per-weight work at a
// handful of integer ops, the zero point and the step leave the inner loop:
// the tensor cores are fed the raw OR-ed nibbles (1024 + q_k for even k mod 8,
// 1024 + 16 q_k for odd k) against x'_k and x'_k / 16, so that with S0 / S1
// the sums of those x' over the group's even / odd k,
//   R = sum_{k even} x'_k (1024 + q_k) + sum_{k odd} (x'_k / 16)(1024 + 16 q_k)
//   sum_k x'_k (q_k - z) = R - (1024 S0 + 64 S1) - z (S0 + S1),
// and the group's step multiplies that once.  S0, S1 are computed per CTA in
// the prologue together with X' = fp16(X / s), from the same rounded values.
//
// The MMA (m16n8k16, swap-AB: columns are MMA rows) has 8 token columns; with
// one or two tokens, the spare columns carry further groups: column c of the
// accumulator is (group c / M of a batch of 8 / M groups, token c % M).  A
// lane's B operand is X' where its column's group is the stage's group and
// zero elsewhere, so one accumulator fragment collects a whole batch and the
// step / zero point arithmetic runs once per batch instead of once per group.
//
// Structure (one CTA = 128 output columns x a k range; clusters split K):
//   producer warp   cp.async of the steps and zero words of all of the CTA's
//                   groups (once), then a TMA ring of 128-row groups (four
//                   16 x 32-word boxes, 128-byte swizzle); ring depth 8, 6 or 4
//                   (see plan_gemv).
//   4 consumers     32 columns per warp; a lane turns one 16-byte load
//                   (4 columns x 8 k) into four even-form and four odd-form
//                   f16x2 operands with LOP3 only and feeds mma.sync.
//   epilogue        each CTA pushes its partial columns into the shared memory
//                   of the cluster CTA that owns them (st.async, completion as
//                   transaction bytes on the owner's mbarrier); owners sum the
//                   K-split partials locally in fixed rank order and write Y.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kBN = 128;
constexpr int kQStage = 4 * 2048;  // one unit: 16 packed rows x 128 columns
constexpr int kStageBytes = kQStage;
constexpr int kSmemOptIn = 232448;
constexpr int kConsumers = 4;  // one warp per 32-column slab of the 128-column tile

struct GemvParams {
    const __half *X;
    const __half *s;
    const __half *scales;
    const int32_t *zeros;
    __half *Y;
    int32_t *status;
    int M, K, N, G, splits;
    int xpro_bytes;   // X' buffer: M * chunks * 16
    int gmeta_bytes;  // per (token, group, half): {1024 S0 + 64 S1, S0 + S1}
    int cmeta_bytes;  // the CTA's steps [group][128] binary16, then zero words [group][16]
    int recv_bytes;   // partials pushed to this CTA: [src rank][k half][8 tokens][128 / splits]
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

template <int S, int MT>
__global__ void __launch_bounds__(32 * (kConsumers + 1), 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmQ, const GemvParams p)
{
    constexpr int kCThreads = 32 * kConsumers;
    constexpr int kAllThreads = kCThreads + 32;
    // The MMA's 8 token columns carry (group, token) slots: slot = MT * (group
    // within a batch of kGPB groups) + token, so one accumulator fragment holds
    // kGPB groups' sums and the step / zero point are applied once per batch.
    constexpr int kGPB = 8 / MT;
    static_assert(MT == 1 || MT == 2, "the decode GEMV takes one or two tokens");

    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int n0 = blockIdx.y * kBN;
    const int g_begin = static_cast<int>(static_cast<int64_t>(split) * p.G / p.splits);
    const int g_end = static_cast<int>(static_cast<int64_t>(split + 1) * p.G / p.splits);
    const int ng = g_end - g_begin;
    const int chunks = ng * 16;

    pdl_launch_dependents();

    uint8_t *xpro = smem + S * kStageBytes;
    float2 *gmeta = reinterpret_cast<float2 *>(xpro + p.xpro_bytes);
    uint8_t *csteps = xpro + p.xpro_bytes + p.gmeta_bytes;
    uint8_t *czeros = csteps + ng * 256;
    float *recv = reinterpret_cast<float *>(csteps + p.cmeta_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(csteps + p.cmeta_bytes + p.recv_bytes);
    uint64_t *empty = full + S;
    uint64_t *recv_bar = empty + S;
    uint64_t *meta_bar = recv_bar + 1;  // the CTA's steps and zero words have landed
    // 256 zero bytes: the B operand of lanes whose token column is not the
    // stage's group reads them (one address select per stage, no per-load
    // predication)
    uint8_t *zchunk = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(meta_bar + 1) + 15) & ~uintptr_t(15));
    if (threadIdx.x < 64) reinterpret_cast<uint32_t *>(zchunk)[threadIdx.x] = 0u;
    const int cpo = kBN / p.splits;  // columns each cluster rank owns in the epilogue

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumers);
        }
        mbar_init(recv_bar, 1);
        mbar_init(meta_bar, 32);
        fence_barrier_init();
        // expect every rank's partials for the columns this CTA owns
        mbar_arrive_expect_tx(recv_bar, MT * cpo * p.splits * 4);
    }
    __syncthreads();
    // Barriers initialized; waited on before the first push.  The init fence
    // above already releases them to the cluster, so the arrival is relaxed.
    cluster_arrive_relaxed();

    float acc[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[a][i] = 0.0f;

    if (warp == kConsumers) {
        // ------------------------------------------------------------ producer
        if (lane == 0) prefetch_tmap(&tmQ);
        // The packed words, steps and zero words are layer state: no kernel that
        // triggers its dependents early writes them (the quantization kernels
        // run to completion first).  The first ring's worth is therefore issued
        // before the wait on the previous kernel, so this call's weights stream
        // while that kernel finishes.
        const int pre = ng < S ? ng : S;
        bool ok = true;
        int issued = 0;
        for (int it = 0; it < ng; ++it) {
            if (it == pre) pdl_wait();
            const int st = it % S;
            if (it >= S && !mbar_wait(&empty[st], ((it / S) - 1) & 1)) {
                ok = false;
                break;
            }
            issued = it + 1;
            uint8_t *stg = smem + st * kStageBytes;
            const int g = g_begin + it;
            if (lane == 0) {
                // four 16 x 32-word boxes (one per consumer warp's slab), 128-byte swizzle
                mbar_arrive_expect_tx(&full[st], kQStage);
#pragma unroll
                for (int w = 0; w < 4; ++w) tma_load_2d(stg + w * 2048, &tmQ, &full[st], n0 + 32 * w, g * 16);
            }
            if (it == pre - 1) {
                // The steps and zero words of all of the CTA's groups, once,
                // behind the first ring's worth of packed words.
                for (int c = lane; c < ng * 16; c += 32) {
                    const int gi = c >> 4, c16 = c & 15;
                    const int gg = g_begin + gi;
                    const int n = n0 + 8 * c16;
                    const bool in_s = n < p.N;
                    cp_async_16(csteps + gi * 256 + 16 * c16,
                                p.scales + static_cast<size_t>(gg) * p.N + (in_s ? n : 0), in_s ? 16u : 0u);
                    const int wi = n0 / 8 + c16;
                    const bool in_z = wi < p.N / 8;
                    cp_async_4(czeros + gi * 64 + 4 * c16, zero_word_src(p.zeros, gg, p.N / 8, in_z ? wi : 0, c16),
                               in_z ? 4u : 0u);
                }
                cp_async_arrive_noinc(meta_bar);
            }
        }
        pdl_wait();  // before this warp writes Y in the epilogue
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
        // Every copy this warp issued lands before the CTA can exit: after a
        // consumer's wait ran out, stages may still be in flight (the waits
        // here have their own limit).
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0)
            for (int it = issued > S ? issued - S : 0; it < issued; ++it)
                mbar_wait_for(&full[it % S], (it / S) & 1, kDrainLimitNs);
    } else {
        // ------------------------------------------------------------ consumers
        pdl_wait();
        // Prologue: X' = fp16(X / s) for this CTA's k range, stored per 8-channel
        // chunk in the order (0,4),(2,6),(1,5),(3,7) (even-form pairs, then
        // odd-form pairs), the odd-form values divided by 16 (exact unless the
        // quotient is subnormal, and the sums below use the same rounded
        // values), plus the per-(token, group) sums of X'.
        {
            constexpr int kLanesPerGroup = 16;  // 8-channel chunks per group
            const int sub = lane >> 4;              // two (token, group) pairs per warp pass
            const int c16 = lane & 15;
            const int pairs = p.M * ng;
            // Two passes' X and s loads are issued before either is used, so a CTA
            // with up to 16 (token, group) pairs waits for one load latency.
            constexpr int kBatch = 2;
            for (int base = warp * 2; base < pairs; base += 2 * kConsumers * kBatch) {
                uint4 xv[kBatch], sv[kBatch];
                bool valid[kBatch];
                int tok[kBatch], gl[kBatch];
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    const int pair = base + b * 2 * kConsumers + sub;
                    valid[b] = pair < pairs;
                    tok[b] = valid[b] ? pair / ng : 0;
                    gl[b] = valid[b] ? pair - tok[b] * ng : 0;
                    xv[b] = make_uint4(0u, 0u, 0u, 0u);
                    sv[b] = xv[b];
                    if (valid[b]) {
                        const int k = (g_begin + gl[b]) * kGroup + c16 * 8;
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
                        const int ch = gl[b] * 16 + c16;
                        const __half *xh = reinterpret_cast<const __half *>(&xv[b]);
                        const __half *sh = reinterpret_cast<const __half *>(&sv[b]);
                        __half q[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            q[j] = __float2half_rn(__fdiv_rn(__half2float(xh[j]), __half2float(sh[j])));
                            if (j & 1) q[j] = __float2half_rn(__half2float(q[j]) * 0.0625f);
                        }
                        e = (__half2float(q[0]) + __half2float(q[2])) + (__half2float(q[4]) + __half2float(q[6]));
                        o = 16.0f * ((__half2float(q[1]) + __half2float(q[3])) + (__half2float(q[5]) + __half2float(q[7])));
                        uint4 r;
                        r.x = __half_as_ushort(q[0]) | (static_cast<uint32_t>(__half_as_ushort(q[4])) << 16);
                        r.y = __half_as_ushort(q[2]) | (static_cast<uint32_t>(__half_as_ushort(q[6])) << 16);
                        r.z = __half_as_ushort(q[1]) | (static_cast<uint32_t>(__half_as_ushort(q[5])) << 16);
                        r.w = __half_as_ushort(q[3]) | (static_cast<uint32_t>(__half_as_ushort(q[7])) << 16);
                        *reinterpret_cast<uint4 *>(xpro + (static_cast<size_t>(tok[b]) * chunks + (ch ^ (tok[b] & 7))) * 16) = r;
                    }
                    // butterfly over the lanes of one group (fixed order)
#pragma unroll
                    for (int off = kLanesPerGroup / 2; off > 0; off >>= 1) {
                        e += __shfl_xor_sync(0xffffffffu, e, off);
                        o += __shfl_xor_sync(0xffffffffu, o, off);
                    }
                    if (valid[b] && c16 == 0)
                        gmeta[tok[b] * ng + gl[b]] = make_float2(fmaf(1024.0f, e, 64.0f * o), e + o);
                }
            }
            named_bar_sync(1, kCThreads);
        }

        const int gq = lane >> 2;
        const int t = lane & 3;
        const int colw = 32 * warp + 4 * gq;  // this lane's 4 columns (A rows gq, gq + 8 of 2 tiles)
        // This lane's B column (MMA token column gq) is slot gq: group gq / MT
        // of each batch, token gq % MT.  Its accumulator columns 2t, 2t + 1
        // are slots of group(s) (2t) / MT, (2t + 1) / MT.
        const int b_group = gq / MT;
        const int b_tok = gq % MT;
        // This lane's X' row.  A chunk index it * 16 + r XOR-swizzled by the
        // token (< 8) equals it * 16 + (r ^ token).
        const uint32_t xrow = smem_u32(xpro) + static_cast<uint32_t>(b_tok * chunks * 16);
        const uint32_t zrow = smem_u32(zchunk);
        const uint32_t qwarp = smem_u32(smem) + static_cast<uint32_t>(warp * 2048);
        // this lane's shared-memory offsets of its four 16-byte loads per stage:
        // packed row r = 8 (ss / 2) + 2 t + ss % 2 of the warp's 2 KB slab,
        // chunk gq XOR-swizzled by the row (128-byte TMA swizzle); X' chunk r
        // XOR-swizzled by the token
        uint32_t offq[4], offx[4];
#pragma unroll
        for (int ss = 0; ss < 4; ++ss) {
            const int r = 8 * (ss >> 1) + 2 * t + (ss & 1);
            offq[ss] = static_cast<uint32_t>(r * 128 + ((gq ^ (r & 7)) << 4));
            offx[ss] = static_cast<uint32_t>((r ^ b_tok) << 4);
        }
        const uint32_t mlo = p.mask_lo, mhi = p.mask_hi, magic = p.magic;
        float R[2][4];  // [tile][fragment element], one batch of groups
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int i = 0; i < 4; ++i) R[a][i] = 0.0f;
        bool ok = true;
        bool meta_ready = false;  // the CTA's steps and zero words have landed
        int st = 0;          // ring slot of the stage
        uint32_t ph = 0;     // its phase parity
        int j = 0;           // group within the batch
        for (int it = 0; it < ng; ++it) {
            // the outcome is voted so that the warp leaves the loop as one
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], ph))) {
                ok = false;
                break;
            }
            const uint32_t qbase = qwarp + static_cast<uint32_t>(st * kStageBytes);
            const uint32_t xbase = b_group == j ? xrow + static_cast<uint32_t>(it * 256) : zrow;
#pragma unroll
            for (int ss = 0; ss < 4; ++ss) {
                uint32_t w[4], bx[4];
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                             : "r"(qbase + offq[ss]));
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(bx[0]), "=r"(bx[1]), "=r"(bx[2]), "=r"(bx[3])
                             : "r"(xbase + offx[ss]));
                uint32_t ev0[4], ev2[4], od1[4], od3[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t w8 = w[c] >> 8;
                    ev0[c] = (w[c] & mlo) | magic;  // 1024 + q0, 1024 + q4
                    ev2[c] = (w8 & mlo) | magic;    // 1024 + q2, 1024 + q6
                    od1[c] = (w[c] & mhi) | magic;  // 1024 + 16 q1, 1024 + 16 q5
                    od3[c] = (w8 & mhi) | magic;    // 1024 + 16 q3, 1024 + 16 q7
                }
#pragma unroll
                for (int tile = 0; tile < 2; ++tile) {
                    const int c0 = 2 * tile, c1 = 2 * tile + 1;
                    const uint32_t ae[4] = {ev0[c0], ev0[c1], ev2[c0], ev2[c1]};
                    const uint32_t ao[4] = {od1[c0], od1[c1], od3[c0], od3[c1]};
                    mma_16816(R[tile], ae, bx[0], bx[1]);
                    mma_16816(R[tile], ao, bx[2], bx[3]);  // X' / 16 on the odd form
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);

            if (j == kGPB - 1 || it == ng - 1) {
                // the steps and zero words (loaded once by the producer) are
                // first needed here
                if (!meta_ready) {
                    if (!__all_sync(0xffffffffu, mbar_wait(meta_bar, 0))) {
                        ok = false;
                        break;
                    }
                    meta_ready = true;
                }
                // batch epilogue: fragment column 2t + u is slot 2t + u = group
                // g = (2t + u) / MT of the batch, token (2t + u) % MT;
                // y += step * (R - (1024 S0 + 64 S1) - z (S0 + S1))
                const int base = it - j;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int slot = 2 * t + u;
                    const int gb = slot / MT;
                    const int tk = slot % MT;
                    const bool valid = gb <= j;
                    const int gi = valid ? base + gb : base;
                    const float2 gm = valid ? gmeta[tk * ng + gi] : make_float2(0.f, 0.f);
                    const uint2 sc = *reinterpret_cast<const uint2 *>(csteps + gi * 256 + 2 * colw);
                    const uint32_t zw = *reinterpret_cast<const uint32_t *>(czeros + gi * 64 + 4 * (colw >> 3));
                    const float stp[4] = {__half2float(__ushort_as_half(static_cast<unsigned short>(sc.x & 0xFFFFu))),
                                          __half2float(__ushort_as_half(static_cast<unsigned short>(sc.x >> 16))),
                                          __half2float(__ushort_as_half(static_cast<unsigned short>(sc.y & 0xFFFFu))),
                                          __half2float(__ushort_as_half(static_cast<unsigned short>(sc.y >> 16)))};
                    const int zsh = (colw & 7) * 4;
#pragma unroll
                    for (int tile = 0; tile < 2; ++tile)
#pragma unroll
                        for (int row = 0; row < 2; ++row) {
                            const int c = 2 * tile + row;
                            // the 4-bit zero as a float: 2^23 + z exactly, minus 2^23
                            const float z =
                                __int_as_float(((zw >> (zsh + 4 * c)) & 15u) | 0x4B000000u) - 8388608.0f;
                            float pgrp = R[tile][2 * row + u] - gm.x;
                            pgrp = fmaf(-z, gm.y, pgrp);
                            if (valid) acc[tile][2 * row + tk] = fmaf(stp[c], pgrp, acc[tile][2 * row + tk]);
                        }
                }
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int i = 0; i < 4; ++i) R[a][i] = 0.0f;
                j = 0;
            } else {
                ++j;
            }
            if (++st == S) {
                st = 0;
                ph ^= 1u;
            }
        }
        // Sum the lanes' group partials (fixed butterfly order): lane t = 0 of
        // each quad then holds columns colw.. for tokens 0 .. MT - 1 in the
        // fragment layout [tile][2 row + token] that the push below expects.
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[a][i] += __shfl_xor_sync(0xffffffffu, acc[a][i], 1);
                acc[a][i] += __shfl_xor_sync(0xffffffffu, acc[a][i], 2);
            }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    }

    // ---------------------------------------------------------------- epilogue
    // Push: a consumer thread holds 4 consecutive columns (one 8-column chunk)
    // for tokens 2t, 2t+1; the chunk's owner is rank chunk % splits.
    cluster_wait_acquire();  // every CTA of the cluster has initialized its barriers
    if (warp < kConsumers) {
        const int gq = lane >> 2, t = lane & 3;
        const int colw = 32 * warp + 4 * gq;
        const int chunk = colw >> 3;
        const uint32_t owner = static_cast<uint32_t>(chunk % p.splits);
        const int lc = (chunk / p.splits) * 8 + (colw & 7);
        const uint32_t rbar = map_to_rank(smem_u32(recv_bar), owner);
#pragma unroll
        for (int tk = 0; tk < 2; ++tk) {
            const int tok = 2 * t + tk;
            if (tok < p.M) {
                const float4 v = make_float4(acc[0][tk], acc[0][2 + tk], acc[1][tk], acc[1][2 + tk]);
                const int off = ((split * 8 + tok) * cpo + lc) * 4;
                st_async_f4(map_to_rank(smem_u32(recv) + off, owner), v, rbar);
            }
        }
    }
    // Arrive once this thread's pushes are issued; the matching wait is the last
    // thing a CTA does, so every CTA has issued its pushes before any exits.
    // No release is needed: each owner waits on its own mbarrier for every
    // byte pushed to it before it reduces, so no push into a CTA is in flight
    // when that CTA leaves.  (A release here fenced on the pushes' completion.)
    cluster_arrive_relaxed();
    // Reduce the columns this rank owns, partials summed in (rank, k-half) order.
    if (!mbar_wait(recv_bar, 0)) {
        if (threadIdx.x == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
        // the partials pushed into this CTA still land before it exits
        mbar_wait_for(recv_bar, 0, kDrainLimitNs);
    }
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
            const float4 *src = reinterpret_cast<const float4 *>(recv + (r * 8 + tok) * cpo + lch * 8);
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

template <int S, int MT>
cudaError_t launch_gemv_one(const GemvPlan &plan, const CUtensorMap &tmQ, const GemvParams &prm,
                            cudaStream_t st)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.splits, plan.n_tiles, 1);
    cfg.blockDim = dim3(32 * (kConsumers + 1), 1, 1);
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
    return cudaLaunchKernelEx(&cfg, gemv_kernel<S, MT>, tmQ, prm);
}

template <int S, int MT>
cudaError_t configure_gemv_one()
{
    return cudaFuncSetAttribute(gemv_kernel<S, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemOptIn);
}

}  // namespace

cudaError_t configure_gemv()
{
    const cudaError_t r[] = {configure_gemv_one<8, 1>(), configure_gemv_one<8, 2>(),
                             configure_gemv_one<6, 1>(), configure_gemv_one<6, 2>(),
                             configure_gemv_one<4, 1>(), configure_gemv_one<4, 2>()};
    for (cudaError_t x : r)
        if (x != cudaSuccess) return x;
    return cudaSuccess;
}


bool plan_gemv(int M, int K, int N, int num_sms, GemvPlan *pl)
{
    if (M < 1 || M > 2) return false;
    const int G = K / kGroup;
    const int max_split = G < 8 ? G : 8;
    pl->n_tiles = (N + kBN - 1) / kBN;
    // splits is a power of two so each cluster rank owns 128 / splits columns.
    // Measured on the decode shapes (K 4096..14336, N 4096..28672): with at
    // most one 128-column tile per SM, an 8-deep ring and the largest split
    // that still fits one wave at two CTAs per SM, or one split more with a
    // 6-deep ring when that fits one wave at three CTAs per SM (the QKV shape:
    // 5.8 us against 6.5); with more tiles than SMs, a 4-deep ring and splits
    // up to about six CTAs per SM for load balance.
    int max_pow2 = 1;
    while (max_pow2 * 2 <= max_split) max_pow2 *= 2;
    int splits = 1;
    if (pl->n_tiles <= num_sms) {
        pl->stages = 8;
        while (splits * 2 <= max_pow2 && pl->n_tiles * splits * 2 <= 2 * num_sms) splits *= 2;
        if (splits * 2 <= max_pow2 && pl->n_tiles * splits * 2 <= 3 * num_sms) {
            splits *= 2;
            pl->stages = 6;
        }
    } else {
        pl->stages = 4;
        while (splits * 2 <= max_pow2 && pl->n_tiles * splits < 6 * num_sms) splits *= 2;
    }
    // X' and the group sums live in shared memory: M * (groups per CTA) * 256 B
    // (+ 8 B per group half); find the smallest split at or above the choice that fits
    for (; splits <= max_pow2; splits *= 2) {
        const int gmax = (G + splits - 1) / splits;
        if (static_cast<size_t>(M) * gmax * (256 + 8) + static_cast<size_t>(gmax) * 320 <= 80 * 1024) break;
    }
    if (splits > max_pow2) return false;
    pl->splits = splits;
    const int gmax = (G + splits - 1) / splits;
    pl->xpro_bytes = M * gmax * 256;
    pl->gmeta_bytes = (M * gmax * 8 + 15) & ~15;
    pl->cmeta_bytes = gmax * 320;
    pl->recv_bytes = 8 * kBN * 4;
    pl->smem = 1024 + static_cast<size_t>(pl->stages) * kStageBytes + pl->xpro_bytes + pl->gmeta_bytes +
               pl->cmeta_bytes + pl->recv_bytes + (2 * pl->stages + 2) * sizeof(uint64_t) + 16 + 256;  // + zero chunk
    return true;
}

cudaError_t launch_gemv(const GemvPlan &plan, const CUtensorMap &tmQ, const __half *X,
                        const __half *s, const __half *scales, const int32_t *zeros, __half *Y,
                        int M, int K, int N, int32_t *status, cudaStream_t st)
{
    GemvParams prm{};
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
    prm.xpro_bytes = plan.xpro_bytes;
    prm.gmeta_bytes = plan.gmeta_bytes;
    prm.cmeta_bytes = plan.cmeta_bytes;
    prm.recv_bytes = plan.recv_bytes;
    prm.mask_lo = 0x000F000Fu;
    prm.mask_hi = 0x00F000F0u;
    prm.magic = 0x64006400u;
    if (plan.stages == 6)
        return M == 2 ? launch_gemv_one<6, 2>(plan, tmQ, prm, st) : launch_gemv_one<6, 1>(plan, tmQ, prm, st);
    if (plan.stages == 4)
        return M == 2 ? launch_gemv_one<4, 2>(plan, tmQ, prm, st) : launch_gemv_one<4, 1>(plan, tmQ, prm, st);
    return M == 2 ? launch_gemv_one<8, 2>(plan, tmQ, prm, st) : launch_gemv_one<8, 1>(plan, tmQ, prm, st);
}

}  // namespace awq
