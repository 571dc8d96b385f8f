/*
 * awq_b200.h -- C ABI of libawq_b200.so, the AWQ W4A16 group-quantized linear
 * layer for NVIDIA B200 (sm_100a).
 *
 * The operations restate the activation-aware weight quantization described
 * on the AWQ pages:
 *   - lansai AWQ explainer (ai.lansai.wang/107648), section "AWQ 的四步链路":
 *     Y = XW is rewritten with a positive per-input-channel scale s as
 *     Y = (X/s)(sW); calibration activations give per-channel magnitudes;
 *     the scaled weights are quantized by group and packed with their
 *     scale and zero point;
 *   - "Awq Quantization" (skillselion.com), "How AWQ Works" (objective
 *     ||Q(W*s)(s^-1*X) - W*X||), "Group Size Configuration" (groups of 128,
 *     4 bits), "Zero-Point Quantization" (asymmetric codes with an offset),
 *     "WQLinear Kernel Variants" (a GEMV kernel for single-token decode and
 *     a GEMM kernel for batches).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE memory owned by the caller, on the
 *     current CUDA device; the library allocates nothing on these calls and
 *     keeps no pointer after it returns.
 *   - float16 data are passed as IEEE binary16 bit patterns (uint16_t).
 *   - Every tensor is dense row-major; device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on that stream.
 *   - Errors detectable on the host (null pointers, shapes, alignment,
 *     device architecture, workspace size) are returned before anything is
 *     launched.  Errors found on the device (non-finite inputs, a bounded wait
 *     that ran out) are written as an awq_status_t value into *dev_status if
 *     dev_status is not NULL; the first error wins, the library never clears
 *     it: the caller zeroes it and reads it after synchronizing the stream.
 *   - Outputs must not alias inputs.
 *   - The library keeps per-device state (device checks, kernel attributes,
 *     encoded tensor maps, the no-allocation scratch address): do not use it
 *     on a device after cudaDeviceReset in the same process.
 *
 * Data layout (K input channels, N output channels, G = K/128 groups)
 *   W       binary16 [K, N]     Y = X W
 *   s       binary16 [K]        per-input-channel scale
 *   Q       int32 [K/8, N]      bits [4j, 4j+4) of Q[k8, n] hold the 4-bit code
 *                               of row 8*k8 + j, column n (sequential nibbles)
 *   scales  binary16 [G, N]     per-group step of the 4-bit grid
 *   zeros   int32 [G, N/8]      bits [4j, 4j+4) of zeros[g, n8] hold the zero
 *                               point of column 8*n8 + j; absent (NULL) for
 *                               symmetric weights, whose zero point is 8
 *   X       binary16 [M, K]     activations;  Y binary16 [M, N]
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define AWQ_API __attribute__((visibility("default")))
#else
#define AWQ_API
#endif

#define AWQ_GROUP_SIZE 128      /* q_group_size ("Group Size Configuration") */
#define AWQ_W_BIT 4             /* w_bit: codes 0..15                          */
#define AWQ_MAX_CALIB_ROWS 8192 /* keeps the double sum of |x| exact           */
#define AWQ_MAX_K 262144
#define AWQ_MAX_N 1048576
#define AWQ_MAX_M 1048576
#define AWQ_ABI_VERSION 5  /* 2: symmetric weights; 3: 1/s folded upstream;
                               4: every matmul takes a zero-filled workspace;
                               scale search over alpha; weight clipping;
                               5: matmul workspaces for M >= 64 hold the
                               prefill kernel's partial tiles */

typedef enum {
    AWQ_OK = 0,
    AWQ_ERR_NULL = 1,           /* a required pointer is NULL                      */
    AWQ_ERR_SHAPE = 2,          /* K % 128, N % 8, M < 1, R < 1, or above a limit  */
    AWQ_ERR_ALIGN = 3,          /* a device pointer is not 16-byte aligned         */
    AWQ_ERR_NONFINITE = 4,      /* NaN/Inf in W, s, X_cal or the statistics        */
    AWQ_ERR_ARCH = 5,           /* the current device is not sm_100 (B200)         */
    AWQ_ERR_CUDA = 6,           /* a CUDA runtime/driver call or launch failed     */
    AWQ_ERR_DEVICE_TIMEOUT = 7, /* a bounded wait inside a kernel ran out          */
    AWQ_ERR_WORKSPACE = 8       /* workspace NULL or smaller than required         */
} awq_status_t;

typedef void *awq_stream_t; /* a cudaStream_t */

/* Human-readable name of a status code (static storage). */
AWQ_API const char *awq_status_string(awq_status_t status);

/* AWQ_ABI_VERSION of the loaded library. */
AWQ_API int awq_abi_version(void);

/*
 * Activation statistics -- lansai explainer, "AWQ 的四步链路", row "采集激活"
 * (collect the layer-input magnitude on calibration data).
 *   m[k] = (1/R) * sum_r |xcal[r, k]|
 * The sum is exact (double; every binary16 is a multiple of 2^-24), divided
 * once in double and rounded once to float, so the result does not depend on
 * the reduction order.
 *   xcal  binary16 [R, K], 1 <= R <= AWQ_MAX_CALIB_ROWS ("Calibration samples
 *         are empty" is AWQ_ERR_SHAPE), K % 8 == 0
 *   m     float [K] (output)
 * Device errors: AWQ_ERR_NONFINITE if xcal holds NaN/Inf (m is still written).
 */
AWQ_API awq_status_t awq_act_stats(const uint16_t *xcal, int64_t R, int64_t K, float *m,
                           int32_t *dev_status, awq_stream_t stream);

/*
 * Per-channel scale -- lansai explainer, "AWQ 的四步链路" (Y = (X/s)(sW));
 * "Awq Quantization", "How AWQ Works" (s lowers ||Q(W*s)(s^-1*X) - W*X||).
 * One point of the scale family: s = m^0.5, normalised by the geometric
 * centre of its extremes:
 *   t_k = sqrt(max(m_k, 1e-8)),  c = sqrt(max_j t_j * min_j t_j),
 *   s_k = binary16_RNE(t_k / c)          (double arithmetic, IEEE rounding)
 *   m  float [K] (K >= 1);  s  binary16 [K] (output)
 * Device errors: AWQ_ERR_NONFINITE if some m_k is NaN/Inf/negative (s is
 * then left unspecified).
 */
AWQ_API awq_status_t awq_compute_scales(const float *m, int64_t K, uint16_t *s, int32_t *dev_status,
                                awq_stream_t stream);

/*
 * Fold, quantize and pack -- lansai explainer, "AWQ 的四步链路" (enlarge the
 * salient channels' weights, sW, then quantize by group; row "真实量化/打包");
 * "Awq Quantization", "Group Size Configuration", "Zero-Point Quantization".
 * Per group g (rows 128g..128g+127) and column n, with w' = float(w) * float(s_k):
 *   r       = max(max w' - min w', 1e-5f)
 *   scale_h = binary16_RNE(r / 15)  (the smallest subnormal if that is 0)
 *   z       = clamp(rint(-min w' / scale_h), 0, 15)
 *   q       = clamp(rint(w' / scale_h) + z, 0, 15)   (rint: ties to even)
 * all in IEEE float arithmetic; the outputs are bit-exact functions of W, s.
 *   W binary16 [K, N], s binary16 [K] (> 0), K % 128 == 0, N % 8 == 0
 *   Q int32 [K/8, N], scales binary16 [K/128, N], zeros int32 [K/128, N/8] (outputs)
 * Device errors: AWQ_ERR_NONFINITE if W or s holds NaN/Inf or s <= 0
 * ("NaN detected in weights", "Awq Quantization", Troubleshooting Guide).
 */
AWQ_API awq_status_t awq_quantize_pack(const uint16_t *W, const uint16_t *s, int64_t K, int64_t N,
                               int32_t *Q, uint16_t *scales, int32_t *zeros,
                               int32_t *dev_status, awq_stream_t stream);

/*
 * Symmetric variant -- "Awq Quantization", "Zero-Point Quantization"
 * (zero_point False: no per-group offset, for symmetric weight distributions
 * and for kernels without zero points).  The page names only the flag; this
 * library reads it as a grid centred at zero whose largest level is 7 steps:
 *   a       = max(max |w'|, 1e-5f)
 *   scale_h = binary16_RNE(a / 7)  (the smallest subnormal if that is 0)
 *   q       = clamp(rint(w' / scale_h), -8, 7) + 8          (rint: ties to even)
 * i.e. the asymmetric codes with z = 8.  No zeros tensor is written; pass
 * zeros = NULL to the matmul entry points for these weights.
 *   W, s, K, N, Q, scales as for awq_quantize_pack.
 * Device errors: as for awq_quantize_pack.
 */
AWQ_API awq_status_t awq_quantize_pack_symmetric(const uint16_t *W, const uint16_t *s, int64_t K,
                                         int64_t N, int32_t *Q, uint16_t *scales,
                                         int32_t *dev_status, awq_stream_t stream);

/*
 * Fold, quantize and pack with weight clipping -- "Awq Quantization",
 * calibration parameters: apply_clip ("Apply weight clipping"); the page names
 * only the flag.  This library reads it, per group g (rows 128g..128g+127)
 * and column n with w' = float(w) * float(s_k), as:
 *   candidates  c_i = 1 - i/20, i = 0 .. n_cand-1 (1 <= n_cand <= 11, down to
 *               c = 1/2; c_0 = 1 is no clipping)
 *   clipped     lo = c * min w', hi = c * max w' (float); step and zero point
 *               from [lo, hi] as in awq_quantize_pack (r = max(hi - lo, 1e-5f),
 *               scale_h = binary16_RNE(r / 15), z = clamp(rint(-lo / scale_h),
 *               0, 15)); every weight of the group coded on that grid,
 *               q = clamp(rint(w' / scale_h) + z, 0, 15)
 *   loss        sum over the R calibration rows of
 *               (sum_{k in g} (xcal[r,k] / s_k) ((q - z) scale_h - w'))^2
 *               (float arithmetic)
 *   choice      the first candidate (largest c) with the minimum loss.
 * With n_cand = 1 the outputs equal awq_quantize_pack's bit for bit.  The
 * step, zero point and codes of a chosen candidate are bit-exact functions of
 * W, s and that candidate; the choice itself rests on float losses, so it can
 * differ from an exact (double) evaluation only between candidates whose
 * losses agree to float rounding.
 *   W binary16 [K, N], s binary16 [K] (> 0), xcal binary16 [R, K]
 *   (1 <= R <= AWQ_MAX_CALIB_ROWS), K % 128 == 0, N % 8 == 0
 *   Q, scales, zeros as for awq_quantize_pack (outputs); ratio_index int32
 *   [K/128, N] receives the chosen i (may be NULL)
 * Device errors: AWQ_ERR_NONFINITE for NaN/Inf in W, s or xcal, or s <= 0.
 */
AWQ_API awq_status_t awq_quantize_pack_clip(const uint16_t *W, const uint16_t *s, const uint16_t *xcal,
                                            int64_t R, int64_t K, int64_t N, int32_t n_cand, int32_t *Q,
                                            uint16_t *scales, int32_t *zeros, int32_t *ratio_index,
                                            int32_t *dev_status, awq_stream_t stream);

/*
 * Fused-dequantization matmul -- lansai explainer, "AWQ 的四步链路"
 * (Y = (X/s)(sW)); "Awq Quantization", "WQLinear Kernel Variants" (GEMV for
 * batch size 1, GEMM for batches).
 *   Y[m, n] = sum_k (X[m, k] / s_k) * (q[k, n] - z[g(k), n]) * scale_h[g(k), n]
 * with the nibble unpack and (q - z) * scale dequantisation done inside the
 * kernel (no dequantised weight matrix is ever written to memory), X / s
 * rounded to binary16 for the tensor cores, float accumulation, Y rounded to
 * binary16.  Results agree with the exact definition within
 * max|dY| <= 1e-2 * max|Y| and ||dY||_F <= 5e-3 * ||Y||_F.
 *
 * awq_w4a16_gemv is the M = 1 (single-token decode) entry point:
 *   X binary16 [1, K], Y binary16 [1, N].
 * awq_w4a16_gemm takes any 1 <= M <= AWQ_MAX_M and picks its tile path
 * internally: the decode GEMV for M <= 2, register-fed tensor cores for
 * 3 <= M < 24, tcgen05/TMEM for M >= 24 (small batch from 24, prefill from 64).
 *   K % 128 == 0, N % 8 == 0, Q/scales/zeros as produced by awq_quantize_pack;
 *   zeros = NULL for weights from awq_quantize_pack_symmetric (zero point 8).
 *   s = NULL when X already holds X/s (1/s folded into the operator that
 *   produced X, e.g. by awq_fold_inverse_scale): X is then used as it is, and
 *   with X = awq_fold_inverse_scale(X, s) the result equals, bit for bit,
 *   the call with the original X and s.
 * Workspace: caller-owned device memory of at least *_workspace_size() bytes,
 * never NULL.  It must be zero-filled (e.g. cudaMemsetAsync) before its first
 * use: its first 32 KB are a counter block that a call expects at zero and
 * leaves at zero when it completes without a device error.  The rest holds
 * X / s and, for M >= 64, the partial sums of output tiles whose k range is
 * split between CTAs (at most 20 MB); it is overwritten.  The size depends on
 * M, K and N, not on the device.  Calls on one stream may share a
 * workspace; calls that can run at the same time need separate ones.  After a
 * device error (AWQ_ERR_DEVICE_TIMEOUT) zero the workspace again.
 * Device errors: AWQ_ERR_DEVICE_TIMEOUT if an internal pipeline wait ran out
 * (Y is then unspecified).  For M >= 64 with few output tiles the call may run
 * a grid whose CTAs wait (up to 1 s) for partial sums from later CTAs of the
 * same grid; the grid is sized so that all of its CTAs fit on the GPU at once,
 * so a kernel on another stream that keeps SMs occupied for longer than that
 * can make such a call report AWQ_ERR_DEVICE_TIMEOUT instead of finishing.
 * Stream ordering: these kernels use programmatic dependent launch, so a call
 * may start while the previous kernel on the stream is still finishing.  X and
 * the workspace are touched only after that kernel has completed.  Q, scales
 * and zeros are treated as layer state and may be read before it completes:
 * they must not be written by a kernel that triggers programmatic dependent
 * launch early.  Ordinary kernels, copies and awq_quantize_pack complete before
 * any dependent starts, so writing the weights with them is safe.
 */
/*
 * Fold 1/s upstream -- lansai explainer, "AWQ 的四步链路": Y = XW = (X/s)(sW),
 * with the X/s side carried by the operator that produces X (a normalisation
 * weight: rows = 1; or activations divided once for several projections).
 *   out[r, k] = binary16_RNE(float(a[r, k]) / float(s_k))   (IEEE division)
 * the same operations the matmul applies to X when it is given s.
 *   a    binary16 [rows, K], 1 <= rows <= AWQ_MAX_M, K % 8 == 0
 *   s    binary16 [K] (> 0);  out binary16 [rows, K] (output, not aliasing a)
 * Device errors: AWQ_ERR_NONFINITE if some s_k is NaN/Inf or <= 0 (out is
 * still written).
 */
AWQ_API awq_status_t awq_fold_inverse_scale(const uint16_t *a, int64_t rows, int64_t K,
                                    const uint16_t *s, uint16_t *out, int32_t *dev_status,
                                    awq_stream_t stream);

AWQ_API size_t awq_w4a16_gemv_workspace_size(int64_t K, int64_t N);
AWQ_API awq_status_t awq_w4a16_gemv(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                            const uint16_t *scales, const int32_t *zeros, int64_t K, int64_t N,
                            uint16_t *Y, void *workspace, size_t workspace_bytes,
                            int32_t *dev_status, awq_stream_t stream);

AWQ_API size_t awq_w4a16_gemm_workspace_size(int64_t M, int64_t K, int64_t N);
AWQ_API awq_status_t awq_w4a16_gemm(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                            const uint16_t *scales, const int32_t *zeros, int64_t M, int64_t K,
                            int64_t N, uint16_t *Y, void *workspace, size_t workspace_bytes,
                            int32_t *dev_status, awq_stream_t stream);

/*
 * Scales of one grid point of the scale search (below): alpha = j/8,
 * 0 <= j <= 8, by the same fixed chain of IEEE double operations,
 *   s = binary16_RNE(t / sqrt(max t * min t)),  t = m^(j/8)
 * (j = 4 gives awq_compute_scales bit for bit, j = 0 gives s = 1).
 *   m float [K] (K >= 1); s binary16 [K] (output)
 * Device errors: AWQ_ERR_NONFINITE if some m_k is NaN/Inf/negative.
 */
AWQ_API awq_status_t awq_scales_alpha(const float *m, int64_t K, int32_t j, uint16_t *s,
                                      int32_t *dev_status, awq_stream_t stream);

/*
 * Scale search over alpha -- "Awq Quantization", "How AWQ Works" (s is chosen
 * to make L(s) = ||Q(W*s)(s^-1*X) - W*X|| small); lansai explainer, "AWQ 的四步
 * 链路", row "搜索缩放" (try channel scalings, keep the one with the smallest
 * reconstruction error).  The pages give neither the family nor the grid;
 * this library reads them as:
 *   family  s(alpha) = m^alpha normalised as in awq_compute_scales (whose scale
 *           is the alpha = 1/2 point), m = awq_act_stats(xcal)
 *   grid    alpha = j/8, j = 0..8, m^alpha by one fixed chain of IEEE double
 *           operations: u = max(m, 1e-8), r1 = sqrt(u), r2 = sqrt(r1),
 *           r3 = sqrt(r2); t = u for j = 8, else the product of r1, r2, r3
 *           selected by the bits 4, 2, 1 of j, in that order;
 *           s = binary16_RNE(t / sqrt(max t * min t))
 *   loss    losses[j] = sum over the R calibration rows and N outputs of
 *           (Yq - Y)^2 (double), Yq = awq_w4a16_gemm(xcal, s(j), awq_quantize_pack(W, s(j)))
 *           and Y = xcal W (tensor cores, float accumulation)
 *   choice  *j_best = the smallest j with the minimum loss; s_best = s(j_best),
 *           bit for bit the scale of that grid point.
 *   xcal  binary16 [R, K], 1 <= R <= AWQ_MAX_CALIB_ROWS; W binary16 [K, N],
 *         K % 128 == 0, N % 8 == 0
 *   losses double [9], s_best binary16 [K], j_best int32 [1] (device outputs)
 *   workspace  at least awq_scale_search_workspace_size(R, K, N) bytes,
 *         zero-filled before its first use (it embeds a matmul workspace)
 * Device errors: AWQ_ERR_NONFINITE for NaN/Inf in xcal or W (the outputs are
 * then unspecified); AWQ_ERR_DEVICE_TIMEOUT as for the matmul.
 */
AWQ_API size_t awq_scale_search_workspace_size(int64_t R, int64_t K, int64_t N);
AWQ_API awq_status_t awq_scale_search(const uint16_t *xcal, int64_t R, int64_t K, const uint16_t *W,
                                      int64_t N, double *losses, uint16_t *s_best, int32_t *j_best,
                                      void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                      awq_stream_t stream);

/*
 * awq_w4a16_gemm_noalloc -- awq_w4a16_gemm for callers that cannot hand the
 * library a workspace.  No counterpart in the AWQ paper or pages: this is an
 * integration entry point of this library only.
 *
 * Who needs it: code that is not allowed to allocate device memory at the point
 * where it runs the layer -- for example an inference-engine plugin whose
 * execute callback may only use memory the engine planned beforehand, a
 * real-time or fixed-budget deployment that allocates everything at start-up,
 * or a plain C caller that has no device allocator of its own.  Instead of a
 * caller-provided workspace, X / s is staged in a fixed scratch array that is
 * part of the library's device image: AWQ_NOALLOC_SCRATCH_BYTES on every GPU
 * that loads the library, held until the process exits.  The call itself
 * allocates nothing (no cudaMalloc, no allocating library routine).
 *
 * Arguments, layouts, tolerance and errors are those of awq_w4a16_gemm, minus
 * the workspace.  Limit: awq_w4a16_gemm_workspace_size(M, K, N) must not exceed
 * AWQ_NOALLOC_SCRATCH_BYTES (32 KB of counters + 2 * M * K bytes of X / s +
 * for M >= 64 up to 20 MB of partial tiles; M * K <= 2 Mi - 16 Ki elements
 * always fits); larger problems return AWQ_ERR_WORKSPACE before anything runs.
 * Set-up: the first call on each device (with that device current) looks up
 * the scratch array's device address; make that first call before any stream
 * capture begins.
 * Sharing: every call on a device uses the same scratch array, which keeps the
 * last call's contents.  Its counter block starts at zero (the array is
 * zero-initialised when the library is loaded) and every call that completes
 * without a device error leaves it at zero; the rest is written before it is
 * read.  Calls whose executions overlap on the GPU (different streams without
 * ordering between them) race on the scratch array and give undefined
 * results; order them on one stream or with events.
 */
#define AWQ_NOALLOC_SCRATCH_BYTES ((size_t)24 << 20)
AWQ_API awq_status_t awq_w4a16_gemm_noalloc(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                                            const uint16_t *scales, const int32_t *zeros,
                                            int64_t M, int64_t K, int64_t N, uint16_t *Y,
                                            int32_t *dev_status, awq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
