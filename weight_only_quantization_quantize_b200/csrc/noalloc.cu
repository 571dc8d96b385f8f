// noalloc.cu -- awq_w4a16_gemm_noalloc: the batched matmul for callers that
// cannot allocate device memory (see awq_b200.h for who they are and why).
//
// The X / s staging buffer that awq_w4a16_gemm takes as a caller workspace is
// here a fixed array in the library's device image.  Host code cannot use the
// array's name as a device address (on the host it names a stand-in object),
// so the address is looked up once per device with cudaGetSymbolAddress while
// that device is current, cached, and passed to the kernels like any other
// workspace pointer.
#include <mutex>

#include "awq_kernels.cuh"

namespace {

// One copy per device that loads the library; lives until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[AWQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of this device's scratch array (looked up on first use).
awq_status_t scratch_for_current_device(void **addr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return AWQ_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_ARCH;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return AWQ_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return AWQ_OK;
}

}  // namespace

extern "C" awq_status_t awq_w4a16_gemm_noalloc(const uint16_t *X, const uint16_t *s,
                                               const int32_t *Q, const uint16_t *scales,
                                               const int32_t *zeros, int64_t M, int64_t K,
                                               int64_t N, uint16_t *Y, int32_t *dev_status,
                                               awq_stream_t stream)
{
    // Bad arguments, then problems whose X / s staging does not fit the fixed
    // array, are refused before anything is looked up or launched.
    awq_status_t e = awq::matmul_args_status(X, s, Q, scales, zeros, M, K, N, Y, dev_status);
    if (e != AWQ_OK) return e;
    if (awq_w4a16_gemm_workspace_size(M, K, N) > AWQ_NOALLOC_SCRATCH_BYTES) return AWQ_ERR_WORKSPACE;
    void *scratch = nullptr;
    e = scratch_for_current_device(&scratch);
    if (e != AWQ_OK) return e;
    return awq::matmul_with_workspace(X, s, Q, scales, zeros, M, K, N, Y, scratch,
                                      AWQ_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
