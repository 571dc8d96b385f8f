// awq_kernels.cuh -- kernel launchers of libawq_b200 (internal, C++ only).
#pragma once

#include "awq_common.cuh"

namespace awq {

// quantize.cu
cudaError_t launch_act_stats(const __half *xcal, int R, int K, float *m, int32_t *status,
                             cudaStream_t st);
cudaError_t launch_compute_scales(const float *m, int K, uint16_t *s, int32_t *status,
                                  cudaStream_t st);
cudaError_t configure_quantize();
cudaError_t launch_quantize_pack(const CUtensorMap &tmW, const __half *s, int K, int N, int32_t *Q,
                                 __half *scales, int32_t *zeros, int32_t *status, int num_sms,
                                 cudaStream_t st);

// fold.cu -- out = fp16(a / s) per channel (1/s folded upstream)
cudaError_t launch_fold_inverse_scale(const __half *a, int64_t rows, int K, const __half *s,
                                      __half *out, int32_t *status, int num_sms, cudaStream_t st);

// gemv.cu -- M <= 2: decode GEMV, zero point and step applied once per group
struct GemvPlan {
    int splits;       // CTAs per cluster along K
    int n_tiles;      // 128-column tiles
    int stages;
    int xpro_bytes;
    int gmeta_bytes;
    int cmeta_bytes;  // the CTA's steps and zero words
    int recv_bytes;
    size_t smem;
};
bool plan_gemv(int M, int K, int N, int num_sms, GemvPlan *plan);
cudaError_t configure_gemv();
cudaError_t launch_gemv(const GemvPlan &plan, const CUtensorMap &tmQ, const __half *X,
                        const __half *s, const __half *scales, const int32_t *zeros, __half *Y,
                        int M, int K, int N, int32_t *status, cudaStream_t st);

// matmul_small.cu -- M < 64: register-fed tensor cores, TMA weight stream
struct SmallMPlan {
    int mt;          // token tiles of 8
    bool prologue;   // X / s computed inside the kernel (no workspace)
    int splits;      // CTAs per cluster along K
    int n_tiles;     // 128-column tiles
    int stages;
    int kh;          // consumer warps per 32-column slab (k split inside a group)
    size_t smem;     // dynamic shared memory bytes
};
SmallMPlan plan_small_m(int M, int K, int N, int num_sms);
cudaError_t configure_small_m();
cudaError_t launch_prescale(const __half *X, const __half *s, int M, int K, __half *Xp,
                            cudaStream_t st);
cudaError_t launch_small_m(const SmallMPlan &plan, const CUtensorMap &tmQ, const CUtensorMap &tmX,
                           const __half *X, const __half *s, const __half *scales,
                           const int32_t *zeros, __half *Y, int M, int K, int N,
                           int32_t *status, cudaStream_t st);

// matmul_tct.cu -- M >= 64: tcgen05 with the dequantized weights in TMEM
// (transposed tile: 128 output columns x bt tokens), one tile per CTA
struct TctPlan {
    int bt;        // tokens per tile: 128 or 256
    int m_tiles, n_tiles;
    size_t smem;
};
TctPlan plan_tct(int M, int K, int N, int num_sms);
cudaError_t configure_tct();
cudaError_t launch_tct(const TctPlan &plan, const CUtensorMap &tmX, const CUtensorMap &tmQ,
                       const __half *scales, const int32_t *zeros, __half *Y, int M, int K, int N,
                       int32_t *status, cudaStream_t st);

// matmul_tsk.cu -- the same tile split along K by stream-K, for grids that
// one tile per CTA would leave partly idle
struct TskPlan {
    int bt;        // tokens per tile: 128 or 256
    int m_tiles, n_tiles;
    int grid;      // CTAs, each a contiguous range of the tiles' 64-k stages
    size_t smem;
};
TskPlan plan_tsk(int M, int K, int N, int num_sms);
// True when the stream-K grid is expected to finish before the one-tile-per-CTA grid.
bool tsk_preferred(const TctPlan &dp, const TskPlan &sk, int K, int num_sms);
// Workspace bytes for the partial tiles (one slot per CTA of the largest grid
// any device gets for this problem).
size_t tsk_partial_bytes(int M, int K, int N);
cudaError_t configure_tsk();
// partials: tsk_partial_bytes(M, K, N) bytes; flags: 8 zero words per CTA,
// left at zero by a call that completes without a device error.
cudaError_t launch_tsk(const TskPlan &plan, const CUtensorMap &tmX, const CUtensorMap &tmQ,
                       const __half *scales, const int32_t *zeros, __half *Y, int M, int K, int N,
                       float *partials, uint32_t *flags, int32_t *status, cudaStream_t st);

// matmul_tcs.cu -- 24 <= M < 64: tcgen05 with the weights as the 128-row operand in TMEM
struct TcsPlan {
    int nt;        // tokens padded to a multiple of 16
    int n_tiles;   // 128-column tiles
    int splits;    // cluster size along K
    int stage_bytes;
    size_t smem;
};
TcsPlan plan_tcs(int M, int K, int N, int num_sms);
cudaError_t configure_tcs();
cudaError_t launch_tcs(const TcsPlan &plan, const CUtensorMap &tmX, const CUtensorMap &tmQ,
                       const __half *scales, const int32_t *zeros, __half *Y, int M, int K, int N,
                       int32_t *status, cudaStream_t st);

// search.cu -- scale search over alpha: scales of one grid point, transpose,
// unquantized X W (tcgen05, float out), fixed-order loss, argmin
size_t loss_partial_bytes();
cudaError_t configure_search();
cudaError_t launch_scales_alpha(const float *m, int K, int j, const int32_t *jptr, uint16_t *s, int32_t *status,
                                cudaStream_t st);
cudaError_t launch_transpose(const uint16_t *W, int K, int N, uint16_t *WT, cudaStream_t st);
cudaError_t launch_dense_gemm(const CUtensorMap &tmX, const CUtensorMap &tmWT, float *Y, int R, int K, int N,
                              int32_t *status, cudaStream_t st);
cudaError_t launch_sq_err(const __half *Yq, const float *Yr, int64_t n, double *partial, double *loss,
                          cudaStream_t st);
cudaError_t launch_pick_best(const double *losses, int32_t *j_best, cudaStream_t st);

// clip.cu -- weight clipping: per (group, column) the range shrink with the
// smallest output error on calibration rows, then its codes
cudaError_t configure_clip();
cudaError_t launch_clip(const __half *W, const __half *s, const __half *xcal, int R, int K, int N, int n_cand,
                        int32_t *Q, __half *scales, int32_t *zeros, int32_t *ratio, int32_t *status,
                        cudaStream_t st);

// abi.cu -- host-side argument checks of the matmul (null, shape, alignment)
awq_status_t matmul_args_status(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                                const uint16_t *scales, const int32_t *zeros, int64_t M,
                                int64_t K, int64_t N, const uint16_t *Y, const int32_t *dev_status);

// abi.cu -- the matmul behind awq_w4a16_gemm, with an explicit workspace
awq_status_t matmul_with_workspace(const uint16_t *X, const uint16_t *s, const int32_t *Q,
                                   const uint16_t *scales, const int32_t *zeros, int64_t M,
                                   int64_t K, int64_t N, uint16_t *Y, void *ws, size_t ws_bytes,
                                   int32_t *dev_status, awq_stream_t stream);

}  // namespace awq
