// matmul_tsk.cu -- Y = (X / s) . dequant(Q) for M >= 64 tokens when a grid of
// one CTA per output tile would leave SMs idle (few tiles, or a last wave that
// fills few SMs): the prefill kernel's tile, split along K by stream-K.
//
// Sources: lansai AWQ explainer (ai.lansai.wang/107648), "AWQ 的四步链路"
// (Y = (X/s)(sW)); "Awq Quantization" (skillselion.com), "WQLinear Kernel
// Variants" (GEMM kernel for batch sizes > 1), "Group Size Configuration",
// "Zero-Point Quantization".
//
// The tile and its pipeline are those of matmul_tct.cu (transposed tile
// Y^T = dequant(W)^T . X'^T, the dequantized weights written into tensor memory
// as the MMA's A operand, X' by TMA into shared memory): 128 output columns x
// BT tokens (BT = 128 or 256).  The grid is persistent: the call's work is
// tiles x (K / 64) units (one 64-k stage of one tile, token tile fastest), and
// CTA c takes the contiguous units [c U / G, (c + 1) U / G), so every CTA does
// the same amount of MMA work whatever the number of tiles.  A CTA's range
// falls into segments, one per tile it touches.  The segment that holds the
// tile's first stage (the "owner") writes Y; any other segment of that tile
// stores its fp32 partial tile in the workspace and raises a flag, and the
// owner adds those partials, in the order of their k ranges, before it writes
// Y (the same summation order on every call).  Every CTA of the grid is
// resident at once (at most one 256-token or two 128-token CTAs per SM, and
// no more CTAs than that), since an owner waits for CTAs after it.
//   warp 0      TMA ring (5 stages): X' tile [BT x 64], packed words [8 x 128]
//               (4 KB), cp.async of the group's steps and zero words.
//   warp 1      allocates TMEM (accumulator + a 4-slot ring of 32-column A
//               tiles); one lane issues tcgen05.mma.cta_group::1.kind::f16
//               (M = 128, N = BT, K = 16, A from TMEM) x 4 per stage, and
//               signals the end of each segment.
//   warps 2..9  dequantize: warp w owns TMEM lanes 32 (w % 4) .. +31 (one output
//               column per lane) and half of a stage's packed rows; it writes
//               16 columns of (q - z) * step binary16 pairs per stage; at the
//               end of each segment the same warps read the accumulator and
//               write Y or the partial tile.
// Within each 8-channel chunk the contraction runs in the pair order
// (0,4),(1,5),(2,6),(3,7) on both operands (X' is stored that way by the
// pre-pass, the unpack produces the weights that way), which leaves the sum
// unchanged.
#include "awq_kernels.cuh"

namespace awq {

namespace {

constexpr int kCols = 128;            // output columns per CTA (MMA M, TMEM lanes)
constexpr int kBK = 64;               // k per stage
constexpr int kASlots = 4;            // TMEM slots of dequantized weights
constexpr int kASlotCols = kBK / 2;   // 32 TMEM columns: 64 binary16 per lane
constexpr int kDequantWarps = 8;
constexpr int kThreads = 64 + 32 * kDequantWarps;
constexpr int kQBytes = (kBK / 8) * kCols * 4;  // 4 KB of packed words
constexpr int kMetaBytes = 1024;                // 256 B steps + 64 B zero words, padded
// A CTA's range is at least this many stages (fewer CTAs for small problems):
// every segment ends with an accumulator read-out.
constexpr int64_t kMinUnits = 16;
// Partial tiles the workspace holds: one per CTA, at most 160 CTAs of 256
// tokens or 320 of 128 (20 MB either way).
constexpr int kMaxPartials256 = 160;

template <int BT>
struct TskCfg {
    static constexpr int kXBytes = BT * kBK * 2;                    // 16 or 32 KB
    static constexpr int kStageBytes = kXBytes + kQBytes + kMetaBytes;  // a multiple of 1 KB
    static constexpr int kStages = 5;                               // load ring depth
    static constexpr int kACol = BT;                                // A slots after the accumulator
    static constexpr int kTmemCols = BT == 256 ? 512 : 256;
    static constexpr size_t kSmem = 1024 + static_cast<size_t>(kStages) * kStageBytes + 256;
};

struct TskParams {
    const __half *scales;
    const int32_t *zeros;
    __half *Y;
    int32_t *status;
    float *partials;   // one 128 x BT fp32 slot per CTA: [token][column]
    uint32_t *flags;   // kDequantWarps per CTA; zero at rest
    int M, K, N;
    int n_tiles, m_tiles;
    UnpackConsts uk;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// First unit of CTA c when U units are shared by G CTAs.
__device__ __forceinline__ int64_t unit_begin(int c, int64_t U, int G)
{
    return static_cast<int64_t>(c) * U / G;
}

// The segment of a CTA's range that starts at unit u: tile and stages
// [s0, s1) of it.
struct Segment {
    int tile, s0, s1;
};

__device__ __forceinline__ Segment segment_at(int64_t u, int64_t u_end, int S)
{
    const int64_t t = u / S;
    const int64_t tile_end = (t + 1) * S;
    Segment g;
    g.tile = static_cast<int>(t);
    g.s0 = static_cast<int>(u - t * S);
    g.s1 = static_cast<int>((tile_end < u_end ? tile_end : u_end) - t * S);
    return g;
}

__device__ __forceinline__ void flag_release(uint32_t *f, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t flag_acquire(const uint32_t *f)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}

// Wait until *f == 1; false once the limit has passed.  Each lane polls the
// flag of one contributor, so a tile's contributors are waited for together,
// with a short sleep between polls.
__device__ __forceinline__ bool flag_wait(const uint32_t *f)
{
    if (flag_acquire(f) == 1u) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(64);
        if (flag_acquire(f) == 1u) return true;
        if ((i & kWaitPollMask) == 0 && globaltimer() - t0 > kWaitLimitNs) return false;
    }
}

// v[i] += the partials of NB contributors (in the order given) for tokens
// c0 + i < c0 + mrem of this lane's column: the NB x 32 loads are issued
// before any is added, so they share one round trip.
template <int NB>
__device__ __forceinline__ void add_partials(float (&v)[32], const float *const (&slot)[NB], int c0, int mrem)
{
    float q[NB][32];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int i = 0; i < 32; ++i) q[b][i] = i < mrem ? __ldcg(slot[b] + (c0 + i) * kCols) : 0.0f;
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += q[b][i];
}

template <int BT>
__global__ void __launch_bounds__(kThreads, BT == 128 ? 2 : 1)
    tsk_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
               const TskParams p)
{
    using C = TskCfg<BT>;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *smem = align1024(smem_dyn);
    uint64_t *full_load = reinterpret_cast<uint64_t *>(smem + C::kStages * C::kStageBytes);
    uint64_t *empty_load = full_load + C::kStages;
    uint64_t *full_a = empty_load + C::kStages;
    uint64_t *empty_a = full_a + kASlots;
    uint64_t *tmem_full = empty_a + kASlots;
    uint64_t *drain = tmem_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = p.K / kBK;  // stages per tile
    const int G = static_cast<int>(gridDim.x);
    const int cta = static_cast<int>(blockIdx.x);
    const int64_t U = static_cast<int64_t>(p.n_tiles) * p.m_tiles * S;
    const int64_t u_begin = unit_begin(cta, U, G);
    const int64_t u_end = unit_begin(cta + 1, U, G);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&full_load[i], 1 + 32);  // expect_tx + 32 cp.async arrivals
            mbar_init(&empty_load[i], 1);      // MMA commit
        }
        for (int i = 0; i < kASlots; ++i) {
            mbar_init(&full_a[i], kDequantWarps);
            mbar_init(&empty_a[i], 1);         // MMA commit
        }
        mbar_init(tmem_full, 1);               // one MMA commit per segment
        mbar_init(drain, 1);
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
        int it = 0;        // stages issued
        int st = 0;        // ring slot of stage `it`
        uint32_t ph = 0;   // parity of the slot's current use
        for (int64_t u = u_begin; u < u_end && ok;) {
            const Segment sg = segment_at(u, u_end, S);
            const int n0 = (sg.tile / p.m_tiles) * kCols;
            const int m0 = (sg.tile % p.m_tiles) * BT;
            for (int kb = sg.s0; kb < sg.s1; ++kb) {
                const bool w = it < C::kStages || mbar_wait(&empty_load[st], ph ^ 1u);
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
                ++it;
                if (++st == C::kStages) {
                    st = 0;
                    ph ^= 1u;
                }
            }
            u += sg.s1 - sg.s0;
        }
        if (!ok) {
            // let the copies already issued land before the CTA exits
            asm volatile("cp.async.wait_all;" ::: "memory");
            if (lane == 0) {
                report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
                const int first = it > C::kStages ? it - C::kStages : 0;
                for (int j = first; j < it; ++j)
                    mbar_wait_for(&full_load[j % C::kStages], (j / C::kStages) & 1, kDrainLimitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The first MMA of a segment overwrites the accumulator; the dequant
        // warps have read the previous segment's sums out of it before they
        // hand over that segment's first A tile (full_a).
        const uint32_t idesc = tc_idesc_f16(kCols, BT);
        bool ok = true;
        int st = 0, as = 0;        // load slot and A slot of the current stage
        uint32_t ph = 0, pa = 0;   // their parities
        for (int64_t u = u_begin; u < u_end && ok;) {
            const Segment sg = segment_at(u, u_end, S);
            for (int kb = sg.s0; kb < sg.s1; ++kb) {
                bool w = mbar_wait(&full_load[st], ph);
                if (w) w = mbar_wait(&full_a[as], pa);
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
                                  (kb > sg.s0 || s > 0) ? 1u : 0u);
                    tc_commit(&empty_load[st]);
                    tc_commit(&empty_a[as]);
                }
                __syncwarp();
                if (++st == C::kStages) {
                    st = 0;
                    ph ^= 1u;
                }
                if (++as == kASlots) {
                    as = 0;
                    pa ^= 1u;
                }
            }
            if (ok && lane == 0) tc_commit(tmem_full);  // the segment's sums are complete
            __syncwarp();
            u += sg.s1 - sg.s0;
        }
        if (!ok && lane == 0) {
            // every MMA issued completes before tensor memory is freed
            report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
            tc_commit(drain);
            mbar_wait_for(drain, 0, kDrainLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dequant
        // warp w: TMEM lanes 32 (w % 4) .. +31 = output columns; packed rows
        // 4 h .. 4 h + 3 of each stage (h = 0 for warps 2..5, 1 for 6..9)
        const int dw = warp - 2;
        const int quarter = warp & 3;
        const int h = dw >> 2;
        const int col = quarter * 32 + lane;  // column within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const UnpackConsts uk = p.uk;
        bool ok = true;
        int it = 0;                // stages consumed
        int st = 0, as = 0;        // load slot and A slot of stage `it`
        uint32_t ph = 0, pa = 0;   // their parities
        int seg = 0;
        for (int64_t u = u_begin; u < u_end && ok; ++seg) {
            const Segment sg = segment_at(u, u_end, S);
            for (int kb = sg.s0; kb < sg.s1; ++kb) {
                bool w = mbar_wait(&full_load[st], ph);
                if (w && it >= kASlots) w = mbar_wait(&empty_a[as], pa ^ 1u);
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
                ++it;
                if (++st == C::kStages) {
                    st = 0;
                    ph ^= 1u;
                }
                if (++as == kASlots) {
                    as = 0;
                    pa ^= 1u;
                }
            }
            if (!ok) break;

            // -------------------------------------------------------- segment end
            // lane = output column n0 + col, TMEM column c = token m0 + c; warp
            // half h handles tokens h BT/2 .. (h + 1) BT/2 - 1 of the tile
            if (!__all_sync(0xffffffffu, mbar_wait(tmem_full, seg & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int n0 = (sg.tile / p.m_tiles) * kCols;
            const int m0 = (sg.tile % p.m_tiles) * BT;
            if (sg.s0 > 0) {
                // a later k range of the tile: hand the partial sums to the
                // owner (slot layout [token][column]: each store instruction
                // writes 128 contiguous bytes)
                float *slot = p.partials + static_cast<size_t>(cta) * (kCols * BT) + col;
#pragma unroll 1
                for (int c0 = h * (BT / 2); c0 < (h + 1) * (BT / 2); c0 += 32) {
                    const int mrem = p.M - (m0 + c0);  // the same on every lane
                    if (mrem <= 0) break;
                    uint32_t v[32];
                    tmem_ld32(tmem_base + lane_addr + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < mrem) __stcg(slot + (c0 + i) * kCols, __uint_as_float(v[i]));
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) flag_release(p.flags + cta * kDequantWarps + dw, 1u);
            } else {
                // the tile's first k range: add the later ranges' partial sums
                // (CTAs cta + 1, ... in order) and write Y
                const int64_t tile_end = static_cast<int64_t>(sg.tile + 1) * S;
                int last = cta;  // the last CTA holding a range of this tile
                while (last + 1 < G && unit_begin(last + 1, U, G) < tile_end) ++last;
                // lane j waits for contributor cta + 1 + j (+ 32 ...), the warp for all
                bool have = true;
                for (int cb = cta + 1; cb <= last; cb += 32) {
                    const int c = cb + lane;
                    const bool mine = c > last || flag_wait(p.flags + c * kDequantWarps + dw);
                    have = __all_sync(0xffffffffu, mine) && have;
                }
                if (!have) {
                    if (lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
                    last = cta;  // Y is unspecified after a device error
                }
                const int n = n0 + col;
#pragma unroll 1
                for (int c0 = h * (BT / 2); c0 < (h + 1) * (BT / 2); c0 += 32) {
                    const int mrem = p.M - (m0 + c0);  // the same on every lane
                    if (mrem <= 0) break;
                    uint32_t vb[32];
                    tmem_ld32(tmem_base + lane_addr + c0, vb);
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(vb[i]);
                    // contributors in order, up to three per round trip (one
                    // for 128-token tiles, whose CTAs have half the registers)
                    const float *base = p.partials + col;
                    constexpr size_t kSlot = static_cast<size_t>(kCols) * BT;
                    int c = cta + 1;
                    if constexpr (BT == 256) {
#pragma unroll 1
                        for (; c + 2 <= last; c += 3) {
                            const float *const sl[3] = {base + c * kSlot, base + (c + 1) * kSlot, base + (c + 2) * kSlot};
                            add_partials<3>(v, sl, c0, mrem);
                        }
                        if (c + 1 == last) {
                            const float *const sl[2] = {base + c * kSlot, base + (c + 1) * kSlot};
                            add_partials<2>(v, sl, c0, mrem);
                            c += 2;
                        }
                    }
#pragma unroll 1
                    for (; c <= last; ++c) {
                        const float *const sl[1] = {base + c * kSlot};
                        add_partials<1>(v, sl, c0, mrem);
                    }
                    if (n < p.N) {
                        __half *dst = p.Y + static_cast<size_t>(m0 + c0) * p.N + n;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < mrem) dst[static_cast<size_t>(i) * p.N] = __float2half_rn(v[i]);
                    }
                }
                // the partials are read (their values are in registers): set
                // the flags back to zero for the next call
                __syncwarp();
                if (lane == 0)
                    for (int c = cta + 1; c <= last; ++c) p.flags[c * kDequantWarps + dw] = 0u;
            }
            u += sg.s1 - sg.s0;
        }
        if (!ok && lane == 0) report(p.status, AWQ_ERR_DEVICE_TIMEOUT);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::kTmemCols)
                     : "memory");
    }
}

int tsk_bt(int M) { return M <= 128 ? 128 : 256; }

int64_t tsk_units(int M, int K, int N)
{
    const int bt = tsk_bt(M);
    return static_cast<int64_t>((N + kCols - 1) / kCols) * ((M + bt - 1) / bt) * (K / kBK);
}

// CTAs for U units with at most `slots` of them: every CTA at least
// kMinUnits stages.
int tsk_grid(int64_t U, int64_t slots)
{
    int64_t g = U / kMinUnits;
    if (g < 1) g = 1;
    if (g > slots) g = slots;
    return static_cast<int>(g);
}

int max_partials(int bt) { return bt == 256 ? kMaxPartials256 : 2 * kMaxPartials256; }

// CTAs of each tile size that fit on one SM (measured by the occupancy
// calculator when the library configures a device; every CTA of a call must
// be resident at once, since a tile's first CTA waits for the others).
int g_ctas_per_sm[2] = {1, 1};  // [0]: 128 tokens, [1]: 256 tokens

}  // namespace

// 128-token tiles for at most 128 tokens (a 256-token tile would be half
// padding), 256-token tiles otherwise (the MMA issue cost per instruction is
// the same for N = 128 and 256); two 128-token CTAs fit on an SM, one 256.
TskPlan plan_tsk(int M, int K, int N, int num_sms)
{
    TskPlan pl{};
    pl.bt = tsk_bt(M);
    pl.n_tiles = (N + kCols - 1) / kCols;
    pl.m_tiles = (M + pl.bt - 1) / pl.bt;
    const int sms = num_sms > 0 ? num_sms : 148;
    int64_t slots = static_cast<int64_t>(sms) * g_ctas_per_sm[pl.bt == 256 ? 1 : 0];
    if (slots > max_partials(pl.bt)) slots = max_partials(pl.bt);
    pl.grid = tsk_grid(tsk_units(M, K, N), slots);
    pl.smem = pl.bt == 256 ? TskCfg<256>::kSmem : TskCfg<128>::kSmem;
    return pl;
}

// Relative time of one 64-k stage of one tile: a 128-token tile does half the
// MMA work of a 256-token one with the same dequantization (6 against 10, the
// weights the one-tile-per-CTA planner uses), and a stream-K stage costs about
// a fifth more (segment ends, partial tiles; measured on the 7B and 70B
// prefill shapes).  Stream-K is chosen when its per-CTA share of the stages
// costs less than the waves of the one-tile-per-CTA grid.
bool tsk_preferred(const TctPlan &dp, const TskPlan &sk, int K, int num_sms)
{
    const int64_t S = K / kBK;
    const int64_t sms = num_sms > 0 ? num_sms : 148;
    const int64_t tiles = static_cast<int64_t>(dp.m_tiles) * dp.n_tiles;
    const int64_t dp_cost = (tiles + sms - 1) / sms * S * (dp.bt == 256 ? 10 : 6);
    const int64_t U = static_cast<int64_t>(sk.m_tiles) * sk.n_tiles * S;
    const int64_t sk_cost = (U + sk.grid - 1) / sk.grid * (sk.bt == 256 ? 12 : 7);
    return sk_cost < dp_cost;
}

size_t tsk_partial_bytes(int M, int K, int N)
{
    const int bt = tsk_bt(M);
    const int g = tsk_grid(tsk_units(M, K, N), max_partials(bt));
    return static_cast<size_t>(g) * kCols * bt * sizeof(float);
}

cudaError_t configure_tsk()
{
    cudaError_t e = cudaFuncSetAttribute(tsk_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(TskCfg<256>::kSmem));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(tsk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(TskCfg<128>::kSmem));
    int n128 = 0, n256 = 0;
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n128, tsk_kernel<128>, kThreads, TskCfg<128>::kSmem);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n256, tsk_kernel<256>, kThreads, TskCfg<256>::kSmem);
    if (e != cudaSuccess) return e;
    if (n128 < 1 || n256 < 1) return cudaErrorInvalidConfiguration;
    // at most two 128-token CTAs (their TMEM takes 256 of the SM's 512 columns)
    g_ctas_per_sm[0] = n128 < 2 ? n128 : 2;
    g_ctas_per_sm[1] = 1;
    return cudaSuccess;
}

cudaError_t launch_tsk(const TskPlan &plan, const CUtensorMap &tmX, const CUtensorMap &tmQ, const __half *scales,
                       const int32_t *zeros, __half *Y, int M, int K, int N, float *partials, uint32_t *flags,
                       int32_t *status, cudaStream_t st)
{
    TskParams prm{scales, zeros, Y, status, partials, flags, M, K, N, plan.n_tiles, plan.m_tiles, unpack_consts()};
    if (plan.bt == 256)
        tsk_kernel<256><<<plan.grid, kThreads, plan.smem, st>>>(tmX, tmQ, prm);
    else
        tsk_kernel<128><<<plan.grid, kThreads, plan.smem, st>>>(tmX, tmQ, prm);
    return cudaGetLastError();
}

}  // namespace awq
