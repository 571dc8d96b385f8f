// abi.cu -- the extern "C" boundary of libawq_b200.so (declared in awq_b200.h).
//
// Host-side work only: argument validation (returned before any launch), a
// one-time per-device architecture check, TMA descriptor encoding, workspace
// accounting and the choice of tile path.  Every step of the computation runs
// in the kernels of quantize.cu, fold.cu, gemv.cu, matmul_small.cu,
// matmul_tcs.cu, matmul_tct.cu, matmul_tsk.cu, search.cu and clip.cu.
#include <mutex>

#include "awq_kernels.cuh"

namespace {

using awq::kGroup;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
    bool checked = false;
    bool supported = false;
    int sms = 0;
};

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
DeviceState g_devices[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

awq_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Checks (once per device) that the current device is an sm_100 part and
// prepares the kernels' shared-memory limits and the TMA encoder.
awq_status_t device_ready(int *sms)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return AWQ_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_ARCH;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState &d = g_devices[dev];
    if (!d.checked) {
        int major = 0, minor = 0, count = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return AWQ_ERR_CUDA;
        }
        d.supported = (major == 10 && minor == 0);
        d.sms = count;
        if (d.supported) {
            if (!g_encode) {
                void *fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                        cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || fn == nullptr) {
                    cudaGetLastError();
                    return AWQ_ERR_CUDA;
                }
                g_encode = reinterpret_cast<EncodeTiledFn>(fn);
            }
            if (awq::configure_tct() != cudaSuccess || awq::configure_tsk() != cudaSuccess ||
                awq::configure_small_m() != cudaSuccess ||
                awq::configure_gemv() != cudaSuccess || awq::configure_quantize() != cudaSuccess ||
                awq::configure_tcs() != cudaSuccess || awq::configure_search() != cudaSuccess ||
                awq::configure_clip() != cudaSuccess) {
                cudaGetLastError();
                return AWQ_ERR_CUDA;
            }
        }
        d.checked = true;
    }
    if (!d.supported) return AWQ_ERR_ARCH;
    *sms = d.sms;
    return AWQ_OK;
}

// 2-D tiled tensor map over a row-major [outer, inner] array.  Encoded maps
// are cached per host thread (a map is a pure function of these arguments and
// the device), so a layer called again with the same tensors skips the
// encoder.
struct MapKey {
    const void *base;
    uint64_t inner, outer, row_bytes;
    uint32_t box_inner, box_outer;
    int dtype, swizzle, device;
    bool operator==(const MapKey &o) const
    {
        return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
               box_inner == o.box_inner && box_outer == o.box_outer && dtype == o.dtype &&
               swizzle == o.swizzle && device == o.device;
    }
};

constexpr int kMapCache = 64;
struct MapCache {
    MapKey key[kMapCache];
    CUtensorMap map[kMapCache];
    int used = 0;
    int next = 0;
};
thread_local MapCache t_maps;

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    const MapKey k{base, inner, outer, row_bytes, box_inner, box_outer, static_cast<int>(dtype),
                   static_cast<int>(swizzle), dev};
    MapCache &c = t_maps;
    for (int i = 0; i < c.used; ++i)
        if (c.key[i] == k) {
            *map = c.map[i];
            return true;
        }
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t elem[2] = {1, 1};
    if (g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, elem,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    int slot;
    if (c.used < kMapCache) {
        slot = c.used++;
    } else {
        slot = c.next;
        c.next = (c.next + 1) % kMapCache;
    }
    c.key[slot] = k;
    c.map[slot] = *map;
    return true;
}

bool matmul_shape_ok(int64_t M, int64_t K, int64_t N)
{
    return M >= 1 && M <= AWQ_MAX_M && K >= kGroup && K % kGroup == 0 && K <= AWQ_MAX_K && N >= 8 &&
           N % 8 == 0 && N <= AWQ_MAX_N;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace layout of every matmul call:
//   [0, 32 KB)              a counter block (AWQ_MAX_N / 128 uint32 words) for
//                           kernels that signal between CTAs (the stream-K
//                           prefill kernel's partial-tile flags); zero between calls
//   [32 KB, +2MK)           X / s (binary16, pair-permuted) for the small-batch
//                           and tcgen05 paths
//   then, for M >= 64       the stream-K prefill kernel's fp32 partial tiles
//                           (one per CTA whose k range starts inside a tile)
constexpr size_t kCounterBytes = static_cast<size_t>(AWQ_MAX_N / 128) * sizeof(uint32_t);
constexpr int64_t kPrefillMinM = 64;  // from here on the prefill kernel runs

size_t xp_bytes(int64_t M, int64_t K) { return round_up(static_cast<size_t>(2 * M * K), 256); }

size_t workspace_bytes(int64_t M, int64_t K, int64_t N)
{
    size_t b = kCounterBytes + xp_bytes(M, K);
    if (M >= kPrefillMinM)
        b += awq::tsk_partial_bytes(static_cast<int>(M), static_cast<int>(K), static_cast<int>(N));
    return b;
}

awq_status_t run_matmul(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                        const uint16_t *scales, const int32_t *zeros, int64_t M, int64_t K,
                        int64_t N, uint16_t *Y, void *ws, size_t ws_bytes, int32_t *dev_status,
                        awq_stream_t stream)
{
    // zeros == NULL: symmetric weights (zero point 8); s == NULL: X holds X/s
    if (!X || !Q || !scales || !Y) return AWQ_ERR_NULL;
    if (!matmul_shape_ok(M, K, N)) return AWQ_ERR_SHAPE;
    if (!aligned16(X) || (s && !aligned16(s)) || !aligned16(Q) || !aligned16(scales) ||
        (zeros && !aligned16(zeros)) || !aligned16(Y) || (ws && !aligned16(ws)) ||
        (dev_status && !aligned4(dev_status)))
        return AWQ_ERR_ALIGN;
    if (ws == nullptr || ws_bytes < workspace_bytes(M, K, N)) return AWQ_ERR_WORKSPACE;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int m = static_cast<int>(M), k = static_cast<int>(K), n = static_cast<int>(N);
    const __half *hX = reinterpret_cast<const __half *>(X);
    const __half *hs = reinterpret_cast<const __half *>(s);
    const __half *hsc = reinterpret_cast<const __half *>(scales);
    __half *hY = reinterpret_cast<__half *>(Y);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    __half *Xp = reinterpret_cast<__half *>(wsb + kCounterBytes);

    CUtensorMap tmQ, tmX;
    awq::GemvPlan gplan;
    // The decode GEMV (X / s and its group sums in shared memory) wins for one
    // or two tokens; from three tokens on, the small-batch kernel with the
    // X / s pre-pass is faster (measured on the 7B and 13B layer shapes).
    if (M <= 2 && awq::plan_gemv(m, k, n, sms, &gplan)) {
        if (!encode_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_INT32, Q, N, K / 8, N * 4, 32, 16,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return AWQ_ERR_CUDA;
        return from_cuda(awq::launch_gemv(gplan, tmQ, hX, hs, hsc, zeros, hY, m, k, n, dev_status, st));
    }
    // From about 24 tokens the small-batch layer needs more MMA rate than
    // mma.sync gives: tcgen05 with the dequantized weights in tensor memory as
    // the 128-row operand (measured on the 13B shapes: as fast at 24 tokens,
    // faster from 32, slower at 8 and 16).
    if (M >= 24 && M < kPrefillMinM) {
        const awq::TcsPlan plan = awq::plan_tcs(m, k, n, sms);
        if (!encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Xp, K, M, K * 2, 64,
                       static_cast<uint32_t>(plan.nt), CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_INT32, Q, N, K / 8, N * 4, 128, 8,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
            return AWQ_ERR_CUDA;
        e = from_cuda(awq::launch_prescale(hX, hs, m, k, Xp, st));
        if (e != AWQ_OK) return e;
        return from_cuda(awq::launch_tcs(plan, tmX, tmQ, hsc, zeros, hY, m, k, n, dev_status, st));
    }
    if (M < kPrefillMinM) {
        const awq::SmallMPlan plan = awq::plan_small_m(m, k, n, sms);
        if (!encode_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_INT32, Q, N, K / 8, N * 4, 32, 16,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return AWQ_ERR_CUDA;
        // boxes of 8 * mt token rows: rows at and beyond M read as zero
        if (!encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Xp, K, M, K * 2, 64,
                       static_cast<uint32_t>(8 * plan.mt), CU_TENSOR_MAP_SWIZZLE_128B))
            return AWQ_ERR_CUDA;
        e = from_cuda(awq::launch_prescale(hX, hs, m, k, Xp, st));
        if (e != AWQ_OK) return e;
        return from_cuda(awq::launch_small_m(plan, tmQ, tmX, hX, hs, hsc, zeros, hY, m, k, n,
                                             dev_status, st));
    }
    // One tile per CTA, or stream-K over the tiles' k stages where that grid
    // would leave SMs idle (few tiles, or a last wave that fills few SMs).
    const awq::TctPlan plan = awq::plan_tct(m, k, n, sms);
    const awq::TskPlan skplan = awq::plan_tsk(m, k, n, sms);
    const bool sk = awq::tsk_preferred(plan, skplan, k, sms);
    if (!encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Xp, K, M, K * 2, 64,
                   static_cast<uint32_t>(sk ? skplan.bt : plan.bt), CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_INT32, Q, N, K / 8, N * 4, 128, 8,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
        return AWQ_ERR_CUDA;
    e = from_cuda(awq::launch_prescale(hX, hs, m, k, Xp, st));
    if (e != AWQ_OK) return e;
    if (!sk) return from_cuda(awq::launch_tct(plan, tmX, tmQ, hsc, zeros, hY, m, k, n, dev_status, st));
    float *partials = reinterpret_cast<float *>(wsb + kCounterBytes + xp_bytes(M, K));
    uint32_t *flags = reinterpret_cast<uint32_t *>(wsb);
    return from_cuda(
        awq::launch_tsk(skplan, tmX, tmQ, hsc, zeros, hY, m, k, n, partials, flags, dev_status, st));
}

}  // namespace

namespace awq {
// The host-side argument checks of the matmul (null, shape, alignment), for
// entry points that must reject bad arguments before any device query.
awq_status_t matmul_args_status(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                                const uint16_t *scales, const int32_t *zeros, int64_t M,
                                int64_t K, int64_t N, const uint16_t *Y, const int32_t *dev_status)
{
    if (!X || !Q || !scales || !Y) return AWQ_ERR_NULL;
    if (!matmul_shape_ok(M, K, N)) return AWQ_ERR_SHAPE;
    if (!aligned16(X) || (s && !aligned16(s)) || !aligned16(Q) || !aligned16(scales) ||
        (zeros && !aligned16(zeros)) || !aligned16(Y) || (dev_status && !aligned4(dev_status)))
        return AWQ_ERR_ALIGN;
    return AWQ_OK;
}

// The workspace-taking matmul, for the library's other entry points.
awq_status_t matmul_with_workspace(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                                   const uint16_t *scales, const int32_t *zeros, int64_t M,
                                   int64_t K, int64_t N, uint16_t *Y, void *ws, size_t ws_bytes,
                                   int32_t *dev_status, awq_stream_t stream)
{
    return run_matmul(X, s, Q, scales, zeros, M, K, N, Y, ws, ws_bytes, dev_status, stream);
}
}  // namespace awq

extern "C" {

const char *awq_status_string(awq_status_t status)
{
    switch (status) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_NULL: return "AWQ_ERR_NULL: a required pointer is NULL";
    case AWQ_ERR_SHAPE: return "AWQ_ERR_SHAPE: unsupported shape";
    case AWQ_ERR_ALIGN: return "AWQ_ERR_ALIGN: device pointer not 16-byte aligned";
    case AWQ_ERR_NONFINITE: return "AWQ_ERR_NONFINITE: NaN or Inf in the input";
    case AWQ_ERR_ARCH: return "AWQ_ERR_ARCH: device is not sm_100 (B200)";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA: CUDA call or launch failed";
    case AWQ_ERR_DEVICE_TIMEOUT: return "AWQ_ERR_DEVICE_TIMEOUT: a kernel wait ran out";
    case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE: workspace missing or too small";
    }
    return "AWQ_ERR_UNKNOWN";
}

int awq_abi_version(void) { return AWQ_ABI_VERSION; }

awq_status_t awq_act_stats(const uint16_t *xcal, int64_t R, int64_t K, float *m,
                           int32_t *dev_status, awq_stream_t stream)
{
    if (!xcal || !m) return AWQ_ERR_NULL;
    if (R < 1 || R > AWQ_MAX_CALIB_ROWS || K < 8 || K % 8 != 0 || K > AWQ_MAX_K) return AWQ_ERR_SHAPE;
    if (!aligned16(xcal) || !aligned16(m) || (dev_status && !aligned4(dev_status))) return AWQ_ERR_ALIGN;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;
    return from_cuda(awq::launch_act_stats(reinterpret_cast<const __half *>(xcal), static_cast<int>(R),
                                           static_cast<int>(K), m, dev_status,
                                           static_cast<cudaStream_t>(stream)));
}

awq_status_t awq_compute_scales(const float *m, int64_t K, uint16_t *s, int32_t *dev_status,
                                awq_stream_t stream)
{
    if (!m || !s) return AWQ_ERR_NULL;
    if (K < 1 || K > AWQ_MAX_K) return AWQ_ERR_SHAPE;
    if (!aligned16(m) || !aligned16(s) || (dev_status && !aligned4(dev_status))) return AWQ_ERR_ALIGN;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;
    return from_cuda(awq::launch_compute_scales(m, static_cast<int>(K), s, dev_status,
                                                static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {
// Both quantizers: zeros == NULL selects the symmetric grid, for which the
// kernel writes no zero points.
awq_status_t quantize_pack_any(const uint16_t *W, const uint16_t *s, int64_t K, int64_t N, int32_t *Q,
                               uint16_t *scales, int32_t *zeros, int32_t *dev_status, awq_stream_t stream)
{
    if (!W || !s || !Q || !scales) return AWQ_ERR_NULL;
    if (K < kGroup || K % kGroup != 0 || K > AWQ_MAX_K || N < 8 || N % 8 != 0 || N > AWQ_MAX_N)
        return AWQ_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(s) || !aligned16(Q) || !aligned16(scales) ||
        (zeros && !aligned16(zeros)) || (dev_status && !aligned4(dev_status)))
        return AWQ_ERR_ALIGN;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;
    CUtensorMap tmW;
    if (!encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, W, N, K, N * 2, 128, kGroup,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
        return AWQ_ERR_CUDA;
    return from_cuda(awq::launch_quantize_pack(tmW, reinterpret_cast<const __half *>(s), static_cast<int>(K),
                                               static_cast<int>(N), Q, reinterpret_cast<__half *>(scales),
                                               zeros, dev_status, sms, static_cast<cudaStream_t>(stream)));
}
}  // namespace

extern "C" {

awq_status_t awq_quantize_pack(const uint16_t *W, const uint16_t *s, int64_t K, int64_t N,
                               int32_t *Q, uint16_t *scales, int32_t *zeros, int32_t *dev_status,
                               awq_stream_t stream)
{
    if (!zeros) return AWQ_ERR_NULL;
    return quantize_pack_any(W, s, K, N, Q, scales, zeros, dev_status, stream);
}

awq_status_t awq_quantize_pack_symmetric(const uint16_t *W, const uint16_t *s, int64_t K, int64_t N,
                                         int32_t *Q, uint16_t *scales, int32_t *dev_status,
                                         awq_stream_t stream)
{
    return quantize_pack_any(W, s, K, N, Q, scales, nullptr, dev_status, stream);
}

awq_status_t awq_quantize_pack_clip(const uint16_t *W, const uint16_t *s, const uint16_t *xcal, int64_t R,
                                    int64_t K, int64_t N, int32_t n_cand, int32_t *Q, uint16_t *scales,
                                    int32_t *zeros, int32_t *ratio_index, int32_t *dev_status,
                                    awq_stream_t stream)
{
    if (!W || !s || !xcal || !Q || !scales || !zeros) return AWQ_ERR_NULL;
    if (R < 1 || R > AWQ_MAX_CALIB_ROWS || K < kGroup || K % kGroup != 0 || K > AWQ_MAX_K || N < 8 ||
        N % 8 != 0 || N > AWQ_MAX_N || n_cand < 1 || n_cand > 11)
        return AWQ_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(s) || !aligned16(xcal) || !aligned16(Q) || !aligned16(scales) ||
        !aligned16(zeros) || (ratio_index && !aligned4(ratio_index)) || (dev_status && !aligned4(dev_status)))
        return AWQ_ERR_ALIGN;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;
    return from_cuda(awq::launch_clip(reinterpret_cast<const __half *>(W), reinterpret_cast<const __half *>(s),
                                      reinterpret_cast<const __half *>(xcal), static_cast<int>(R),
                                      static_cast<int>(K), static_cast<int>(N), n_cand, Q,
                                      reinterpret_cast<__half *>(scales), zeros, ratio_index, dev_status,
                                      static_cast<cudaStream_t>(stream)));
}

awq_status_t awq_fold_inverse_scale(const uint16_t *a, int64_t rows, int64_t K, const uint16_t *s,
                                    uint16_t *out, int32_t *dev_status, awq_stream_t stream)
{
    if (!a || !s || !out) return AWQ_ERR_NULL;
    if (rows < 1 || rows > AWQ_MAX_M || K < 8 || K % 8 != 0 || K > AWQ_MAX_K) return AWQ_ERR_SHAPE;
    if (!aligned16(a) || !aligned16(s) || !aligned16(out) || (dev_status && !aligned4(dev_status)))
        return AWQ_ERR_ALIGN;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;
    return from_cuda(awq::launch_fold_inverse_scale(reinterpret_cast<const __half *>(a), rows,
                                                    static_cast<int>(K), reinterpret_cast<const __half *>(s),
                                                    reinterpret_cast<__half *>(out), dev_status, sms,
                                                    static_cast<cudaStream_t>(stream)));
}

size_t awq_w4a16_gemv_workspace_size(int64_t K, int64_t N)
{
    return matmul_shape_ok(1, K, N) ? workspace_bytes(1, K, N) : 0;
}

awq_status_t awq_w4a16_gemv(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                            const uint16_t *scales, const int32_t *zeros, int64_t K, int64_t N,
                            uint16_t *Y, void *workspace, size_t workspace_bytes_, int32_t *dev_status,
                            awq_stream_t stream)
{
    return run_matmul(X, s, Q, scales, zeros, 1, K, N, Y, workspace, workspace_bytes_, dev_status,
                      stream);
}

size_t awq_w4a16_gemm_workspace_size(int64_t M, int64_t K, int64_t N)
{
    return matmul_shape_ok(M, K, N) ? workspace_bytes(M, K, N) : 0;
}

awq_status_t awq_w4a16_gemm(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                            const uint16_t *scales, const int32_t *zeros, int64_t M, int64_t K,
                            int64_t N, uint16_t *Y, void *workspace, size_t workspace_bytes_,
                            int32_t *dev_status, awq_stream_t stream)
{
    return run_matmul(X, s, Q, scales, zeros, M, K, N, Y, workspace, workspace_bytes_, dev_status,
                      stream);
}


}  // extern "C"

namespace {
// Workspace of the scale search, every part 256-byte aligned:
//   the matmul's own workspace (its counter block first), m, s(j), Q, steps,
//   zero points, W transposed, Y = X W (float), Yq (binary16), loss partials.
enum { kSmm, kSm, kSs, kSQ, kSsc, kSz, kSWT, kSYr, kSYq, kSpart, kSparts };

void search_layout(int64_t R, int64_t K, int64_t N, size_t off[kSparts + 1])
{
    const size_t G = static_cast<size_t>(K / kGroup);
    const size_t sz[kSparts] = {workspace_bytes(R, K, N),
                                4 * static_cast<size_t>(K),
                                2 * static_cast<size_t>(K),
                                4 * static_cast<size_t>(K / 8) * N,
                                2 * G * N,
                                4 * G * static_cast<size_t>(N / 8),
                                2 * static_cast<size_t>(N) * K,
                                4 * static_cast<size_t>(R) * N,
                                2 * static_cast<size_t>(R) * N,
                                awq::loss_partial_bytes()};
    off[0] = 0;
    for (int i = 0; i < kSparts; ++i) off[i + 1] = off[i] + round_up(sz[i], 256);
}

bool search_shape_ok(int64_t R, int64_t K, int64_t N)
{
    return R >= 1 && R <= AWQ_MAX_CALIB_ROWS && matmul_shape_ok(R, K, N);
}
}  // namespace

extern "C" {

awq_status_t awq_scales_alpha(const float *m, int64_t K, int32_t j, uint16_t *s, int32_t *dev_status,
                              awq_stream_t stream)
{
    if (!m || !s) return AWQ_ERR_NULL;
    if (K < 1 || K > AWQ_MAX_K || j < 0 || j > 8) return AWQ_ERR_SHAPE;
    if (!aligned16(m) || !aligned16(s) || (dev_status && !aligned4(dev_status))) return AWQ_ERR_ALIGN;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;
    return from_cuda(awq::launch_scales_alpha(m, static_cast<int>(K), j, nullptr, s, dev_status,
                                              static_cast<cudaStream_t>(stream)));
}

size_t awq_scale_search_workspace_size(int64_t R, int64_t K, int64_t N)
{
    if (!search_shape_ok(R, K, N)) return 0;
    size_t off[kSparts + 1];
    search_layout(R, K, N, off);
    return off[kSparts];
}

awq_status_t awq_scale_search(const uint16_t *xcal, int64_t R, int64_t K, const uint16_t *W, int64_t N,
                              double *losses, uint16_t *s_best, int32_t *j_best, void *workspace,
                              size_t workspace_bytes_, int32_t *dev_status, awq_stream_t stream)
{
    if (!xcal || !W || !losses || !s_best || !j_best) return AWQ_ERR_NULL;
    if (!search_shape_ok(R, K, N)) return AWQ_ERR_SHAPE;
    if (!aligned16(xcal) || !aligned16(W) || !aligned16(s_best) || !aligned16(losses) || !aligned4(j_best) ||
        (workspace && !aligned16(workspace)) || (dev_status && !aligned4(dev_status)))
        return AWQ_ERR_ALIGN;
    size_t off[kSparts + 1];
    search_layout(R, K, N, off);
    if (workspace == nullptr || workspace_bytes_ < off[kSparts]) return AWQ_ERR_WORKSPACE;
    int sms = 0;
    awq_status_t e = device_ready(&sms);
    if (e != AWQ_OK) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *m = reinterpret_cast<float *>(ws + off[kSm]);
    uint16_t *sj = reinterpret_cast<uint16_t *>(ws + off[kSs]);
    int32_t *Q = reinterpret_cast<int32_t *>(ws + off[kSQ]);
    uint16_t *sc = reinterpret_cast<uint16_t *>(ws + off[kSsc]);
    int32_t *z = reinterpret_cast<int32_t *>(ws + off[kSz]);
    uint16_t *WT = reinterpret_cast<uint16_t *>(ws + off[kSWT]);
    float *Yr = reinterpret_cast<float *>(ws + off[kSYr]);
    uint16_t *Yq = reinterpret_cast<uint16_t *>(ws + off[kSYq]);
    double *part = reinterpret_cast<double *>(ws + off[kSpart]);
    const int r = static_cast<int>(R), k = static_cast<int>(K), n = static_cast<int>(N);

    CUtensorMap tmX, tmWT, tmW;
    if (!encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xcal, K, R, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&tmWT, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, WT, K, N, K * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, W, N, K, N * 2, 128, kGroup, CU_TENSOR_MAP_SWIZZLE_NONE))
        return AWQ_ERR_CUDA;
    // statistics, then Y = X W once
    e = from_cuda(awq::launch_act_stats(reinterpret_cast<const __half *>(xcal), r, k, m, dev_status, st));
    if (e == AWQ_OK) e = from_cuda(awq::launch_transpose(W, k, n, WT, st));
    if (e == AWQ_OK) e = from_cuda(awq::launch_dense_gemm(tmX, tmWT, Yr, r, k, n, dev_status, st));
    // each grid point: scales, the library's quantizer and matmul, the loss
    for (int j = 0; j <= 8 && e == AWQ_OK; ++j) {
        e = from_cuda(awq::launch_scales_alpha(m, k, j, nullptr, sj, dev_status, st));
        if (e == AWQ_OK)
            e = from_cuda(awq::launch_quantize_pack(tmW, reinterpret_cast<const __half *>(sj), k, n, Q,
                                                    reinterpret_cast<__half *>(sc), z, dev_status, sms, st));
        if (e == AWQ_OK)
            e = run_matmul(xcal, sj, Q, sc, z, R, K, N, Yq, ws + off[kSmm], off[kSm] - off[kSmm], dev_status,
                           stream);
        if (e == AWQ_OK)
            e = from_cuda(awq::launch_sq_err(reinterpret_cast<const __half *>(Yq), Yr, R * N, part, losses + j, st));
    }
    if (e == AWQ_OK) e = from_cuda(awq::launch_pick_best(losses, j_best, st));
    if (e == AWQ_OK) e = from_cuda(awq::launch_scales_alpha(m, k, 0, j_best, s_best, dev_status, st));
    return e;
}

}  // extern "C"
