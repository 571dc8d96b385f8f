// awq_common.cuh -- device helpers shared by the AWQ W4A16 kernels (sm_100a).
//
// Thin inline-PTX wrappers: mbarriers with bounded waits, TMA tile loads,
// cp.async with mbarrier completion, warp-level tensor-core MMA, cluster
// (distributed shared memory) access and the device status word.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "awq_b200.h"

namespace awq {

constexpr int kGroup = 128;

// Every wait inside a kernel is bounded by wall time (%globaltimer, ns).  A
// wait that runs out records AWQ_ERR_DEVICE_TIMEOUT and returns false; the
// caller then skips its remaining work but still reaches every block- and
// cluster-wide barrier, so the context survives and the host can read the
// status word.
// AWQ_WAIT_LIMIT_NS, AWQ_WAIT_POLL_MASK and AWQ_WAIT_NONBLOCKING_POLL exist for
// the test build that checks the timeout path (limit 0, timer read on every
// poll, polls that never suspend: a wait that does not complete at its first
// poll runs out); the library itself is always built with the defaults.
#ifndef AWQ_WAIT_LIMIT_NS
#define AWQ_WAIT_LIMIT_NS 1000000000ull
#endif
constexpr uint64_t kWaitLimitNs = AWQ_WAIT_LIMIT_NS;  // 1 s
#ifndef AWQ_WAIT_POLL_MASK
#define AWQ_WAIT_POLL_MASK 255u
#endif
constexpr uint32_t kWaitPollMask = AWQ_WAIT_POLL_MASK;  // read the timer every 256 polls
// After a wait has run out, a kernel still lets the copies it issued land
// before it exits; those waits use their own limit.
constexpr uint64_t kDrainLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ void report(int32_t *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity)
{
    uint32_t done;
#ifdef AWQ_WAIT_NONBLOCKING_POLL
    // test build: a poll that never suspends the thread
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar_addr), "r"(parity)
        : "memory");
#else
    // may suspend the thread for a while until the phase completes
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar_addr), "r"(parity)
        : "memory");
#endif
    return done != 0;
}

// Wait for the phase with the given parity to complete; false once
// `limit_ns` has passed.
__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(a, parity)) return true;
        if ((i & kWaitPollMask) == 0 && globaltimer() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled bulk-tensor load into this CTA's shared memory; completion is
// signalled as transaction bytes on `bar`.  x is the innermost coordinate.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *m, uint64_t *bar, int x,
                                            int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// ---------------------------------------------------------------- programmatic dependent launch
// Allow the next kernel on the stream to start launching (its own prologue
// then overlaps this kernel's tail).
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Wait until the grids this kernel depends on have completed and their memory
// is visible.  No global memory written by a predecessor may be read before.
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- cp.async
// src_bytes == 0 zero-fills the destination without reading global memory.
__device__ __forceinline__ void cp_async_4(void *dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_16(void *dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed.
// The arrival is counted in the barrier's initial count (.noinc).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// ---------------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- zero points
// Symmetric weights ("Zero-Point Quantization" with zero_point False) come
// without a zeros tensor: their zero point is 8 in every nibble.  Producers
// copy these constant words in its place, so the consumers are the same for
// both kinds of weights.
__device__ __align__(16) const uint32_t kSymmetricZeroWords[32] = {
    0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u,
    0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u,
    0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u,
    0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u,
    0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u};

// Address of zero-point word `wi` of group g (zeros is [G, N/8]), or of a
// constant word of 8s when zeros is NULL (`slot` < 32 picks one of them).
__device__ __forceinline__ const int32_t *zero_word_src(const int32_t *zeros, int g, int words_per_row,
                                                        int wi, int slot)
{
    return zeros ? zeros + static_cast<size_t>(g) * words_per_row + wi
                 : reinterpret_cast<const int32_t *>(kSymmetricZeroWords) + (slot & 31);
}

// ---------------------------------------------------------------- cluster / DSMEM
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Split cluster barrier: arrive (release) now, wait (acquire) later.
__device__ __forceinline__ void cluster_arrive_release()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

// Arrival with no memory ordering of its own (no fence on the arriving thread).
__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait_acquire()
{
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Asynchronous 16-byte store into another CTA's shared memory (cluster
// addresses from mapa); its bytes complete transactions on that CTA's mbarrier.
__device__ __forceinline__ void st_async_f4(uint32_t remote_addr, float4 v, uint32_t remote_bar)
{
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
            remote_addr),
        "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(remote_bar)
        : "memory");
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

// ---------------------------------------------------------------- tensor cores (warp MMA)
// D = A * B + C, A 16x16 f16 (row), B 16x8 f16 (col), C/D 16x8 f32.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- tensor cores (tcgen05)
// Shared-memory operand descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset unused (1),
// descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: A = B = binary16, D = f32,
// both operands K-major; m rows (M) by n columns (N).
__host__ __device__ constexpr uint32_t tc_idesc_f16(int m, int n)
{
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// D[tmem] (+)= A * B^T, one CTA, operands in shared memory (descriptors).
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B^T, one CTA: the A operand (M rows in the TMEM
// lanes, K along the columns, two binary16 per 32-bit column) in tensor
// memory, B in shared memory (descriptor).
__device__ __forceinline__ void tc_mma_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier when every MMA issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns of tensor memory into registers.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 8 consecutive 32-bit columns of tensor memory into registers.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes from registers;
// complete (tcgen05.wait::st) before the values are handed to an MMA.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Asynchronous 4-byte store into another cluster CTA's shared memory; its
// bytes complete transactions on that CTA's mbarrier.
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(remote_addr),
                 "f"(v), "r"(remote_bar)
                 : "memory");
}

// ---------------------------------------------------------------- binary16 rounding
// Round a positive finite double to the nearest binary16, ties to even, in a
// single rounding (IEEE 754 binary16: quantum 2^(e-10) in the binade
// [2^e, 2^(e+1)), never finer than the subnormal quantum 2^-24).
__device__ __forceinline__ uint16_t double_to_half_rn(double x)
{
    if (!(x < 65520.0)) return 0x7C00;  // rounds to +inf (x >= 65520)
    if (x == 0.0) return 0;
    const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
    int e = static_cast<int>((b >> 52) & 0x7FF) - 1023;  // x normal in double here
    int q = e - 10;
    if (q < -24) q = -24;
    const double inv_quantum = __longlong_as_double(static_cast<long long>(1023 - q) << 52);
    const double n = rint(__dmul_rn(x, inv_quantum));  // exact scaling, then RNE
    return static_cast<uint16_t>(((q + 24) << 10) + static_cast<int>(n));
}

// ---------------------------------------------------------------- 4-bit unpack
// One packed word holds 8 consecutive-k codes of one column (nibble j = row
// 8*k8 + j).  OR-ing a nibble into the mantissa of binary16 1024.0 (0x6400)
// yields exactly 1024 + q (or 1024 + 16 q for the odd nibbles); subtracting
// 1024 + z (or scaling by 1/16 and subtracting 64 + z) leaves q - z exactly.
// Output pairs (low, high half): d[0] = (q0, q4), d[1] = (q1, q5),
// d[2] = (q2, q6), d[3] = (q3, q7), each minus z.
// The masks, the magic and 1/16 arrive as run-time values (UnpackConsts in
// the kernel parameters): as literals the compiler re-materializes them before
// every use, since a LOP3 encodes only one 32-bit immediate.
struct UnpackConsts {
    uint32_t mask_lo;    // 0x000F000F
    uint32_t mask_hi;    // 0x00F000F0
    uint32_t magic;      // 0x64006400 = (1024, 1024)
    uint32_t sixteenth;  // 0x2C002C00 = (1/16, 1/16)
};

__host__ __device__ inline UnpackConsts unpack_consts()
{
    return UnpackConsts{0x000F000Fu, 0x00F000F0u, 0x64006400u, 0x2C002C00u};
}

__device__ __forceinline__ void unpack_minus_zero(uint32_t w, uint32_t za, uint32_t zb,
                                                  uint32_t (&d)[4], const UnpackConsts &k)
{
    const uint32_t w8 = w >> 8;
    const uint32_t v0 = (w & k.mask_lo) | k.magic;
    const uint32_t v1 = (w & k.mask_hi) | k.magic;
    const uint32_t v2 = (w8 & k.mask_lo) | k.magic;
    const uint32_t v3 = (w8 & k.mask_hi) | k.magic;
    const uint32_t sixteenth = k.sixteenth;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d[0]) : "r"(v0), "r"(za));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d[1]) : "r"(v1), "r"(sixteenth), "r"(zb));
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d[2]) : "r"(v2), "r"(za));
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d[3]) : "r"(v3), "r"(sixteenth), "r"(zb));
}

// (-(1024 + z), -(1024 + z)) and (-(64 + z), -(64 + z)) as f16x2 bit patterns.
__device__ __forceinline__ void zero_constants(uint32_t z, uint32_t &za, uint32_t &zb)
{
    // -(1024 + z): sign | exponent of 1024 | mantissa z
    const uint32_t a = 0xE400u | z;
    // -(64 + z) = -(1 + z/64) * 2^6: exponent 6+15 = 21 (0x5400), mantissa z*16
    const uint32_t b = 0xD400u | (z << 4);
    za = a | (a << 16);
    zb = b | (b << 16);
}

}  // namespace awq
