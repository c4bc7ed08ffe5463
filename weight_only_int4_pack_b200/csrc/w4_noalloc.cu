// w4_noalloc.cu -- w4a16_gemm_noalloc: the decode (M <= 32) W4A16 layer for
// callers that cannot allocate device memory.
//
// w4a16_gemm asks its caller for a workspace (split-K partial sums and
// arrival counters).  Some callers have no way to provide one: a plugin
// running inside a host application that owns every device allocation, or a
// latency-critical path where a cudaMalloc (and the device synchronization it
// may imply) is not allowed.  This entry point runs the same decode kernel
// with its workspace in a file-scope device array of fixed size, so it
// allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
//
// Costs and limits:
//   * every GPU that loads the library holds kScratchBytes for the array until
//     the process exits;
//   * shapes whose workspace would exceed kScratchBytes are rejected with
//     W4_ERR_UNSUPPORTED (w4_last_error() says so);
//   * all calls on a device share the one array, so calls that may overlap on
//     the GPU (different streams, or several host threads) race and give
//     wrong results; issue them one after another on one stream;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current; make that first call
//     before any stream capture.

#include <mutex>

#include "w4_internal.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB per device

__device__ __align__(256) unsigned char g_w4_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_w4_scratch on the current device.  In host code the
// name g_w4_scratch only stands in for the symbol; the address a kernel can
// use has to be asked for, once per device, with that device current.
int scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return w4::cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices)
        return w4::set_error(W4_ERR_CUDA, "w4a16_gemm_noalloc", "device ordinal out of range");
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_w4_scratch);
        if (e != cudaSuccess) return w4::cuda_fail("cudaGetSymbolAddress(scratch)", e);
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return W4_OK;
}

}  // namespace

extern "C" int w4a16_gemm_noalloc(const void *X, int xt, int64_t M, const uint8_t *packed,
                                  const float *scales, const float *zeros, int64_t K, int64_t N,
                                  int group, void *Y, void *stream) {
    const char *fn = "w4a16_gemm_noalloc";
    if (xt != W4_F16 && xt != W4_BF16) return w4::set_error(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (M < 0 || K <= 0 || N < 0 || group <= 0 || K % group != 0 || K % 8 != 0)
        return w4::set_error(W4_ERR_INVALID_ARG, fn, "bad shape (see w4a16_gemm)");
    if (M > 32)
        return w4::set_error(W4_ERR_UNSUPPORTED, fn,
                             "only M <= 32 (the M > 32 path of w4a16_gemm needs no workspace)");
    if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
        return w4::set_error(W4_ERR_INVALID_ARG, fn, "N and K must be below 2^31");
    if (M == 0 || N == 0) return W4_OK;
    if (!X || !packed || !scales || !Y) return w4::set_error(W4_ERR_INVALID_ARG, fn, "null pointer");
    if (group != 128) return w4::set_error(W4_ERR_UNSUPPORTED, fn, "group must be 128");
    if (!w4::aligned16(X) || !w4::aligned16(packed) || !w4::aligned16(scales) ||
        (zeros && !w4::aligned16(zeros)) || !w4::aligned16(Y))
        return w4::set_error(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    const size_t need = w4::decode_workspace_bytes(M, K, N, group);
    if (need > kScratchBytes)
        return w4::set_error(W4_ERR_UNSUPPORTED, fn,
                             "this shape needs more than the 4 MiB static workspace; use w4a16_gemm");
    void *ws = nullptr;
    size_t ws_bytes = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (need > 0) {
        int st = scratch_address(&ws);
        if (st != W4_OK) return st;
        ws_bytes = kScratchBytes;
        // The array keeps whatever the previous call left; the counters must
        // start at zero.
        const size_t zeroed = w4::decode_counter_bytes();
        cudaError_t e = cudaMemsetAsync(ws, 0, need < zeroed ? need : zeroed, s);
        if (e != cudaSuccess) return w4::cuda_fail("cudaMemsetAsync(scratch counters)", e);
    }
    return w4::launch_decode(X, xt, M, packed, scales, zeros, K, N, Y, ws, ws_bytes, s);
}
