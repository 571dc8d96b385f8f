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
#define AWQ_ABI_VERSION 3  /* 2: symmetric weights; 3: 1/s folded upstream */

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
 * 3 <= M < 40, tcgen05/TMEM for M >= 40 (small batch from 40, prefill from 64).
 *   K % 128 == 0, N % 8 == 0, Q/scales/zeros as produced by awq_quantize_pack;
 *   zeros = NULL for weights from awq_quantize_pack_symmetric (zero point 8).
 *   s = NULL when X already holds X/s (1/s folded into the operator that
 *   produced X, e.g. by awq_fold_inverse_scale): X is then used as it is, and
 *   with X = awq_fold_inverse_scale(X, s) the result equals, bit for bit,
 *   the call with the original X and s.
 * Workspace: caller-owned device memory of at least *_workspace_size() bytes
 * (may be NULL when that size is 0); it holds X / s and is overwritten.
 * Device errors: AWQ_ERR_DEVICE_TIMEOUT if an internal pipeline wait ran out
 * (Y is then unspecified).
 * Stream ordering: these kernels use programmatic dependent launch, so a call
 * may start while the previous kernel on the stream is still finishing.  X is
 * read only after that kernel has completed.  Q, scales and zeros are treated
 * as layer state and may be read before it completes: they must not be
 * written by a kernel that triggers programmatic dependent launch early.
 * Ordinary kernels, copies and awq_quantize_pack complete before any
 * dependent starts, so writing the weights with them is safe.
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
 * AWQ_NOALLOC_SCRATCH_BYTES (2 * M * K bytes for M > 1, i.e. M * K <= 2 Mi
 * elements); larger problems return AWQ_ERR_WORKSPACE before anything runs.
 * Set-up: the first call on each device (with that device current) looks up
 * the scratch array's device address; make that first call before any stream
 * capture begins.
 * Sharing: every call on a device uses the same scratch array, which keeps the
 * last call's contents (nothing in it needs to start at zero: each call writes
 * the part it reads).  Calls whose executions overlap on the GPU (different
 * streams without ordering between them) race on the scratch array and give
 * undefined results; order them on one stream or with events.
 */
#define AWQ_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
AWQ_API awq_status_t awq_w4a16_gemm_noalloc(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                                            const uint16_t *scales, const int32_t *zeros,
                                            int64_t M, int64_t K, int64_t N, uint16_t *Y,
                                            int32_t *dev_status, awq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
