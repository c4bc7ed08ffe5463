// w4_api.cu -- the extern "C" entry points of libw4a16.so (declared in
// include/w4a16.h): host-side argument validation, dispatch to the kernels,
// the per-device attribute cache and the device status word.

#include <mutex>

#include "w4_internal.cuh"

namespace {

// Set by kernels (atomicOr) when a bounded wait runs out.
__device__ unsigned g_w4_status = 0;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
w4::DeviceInfo g_info[kMaxDevices];
bool g_info_ok[kMaxDevices] = {};
unsigned *g_status_ptr[kMaxDevices] = {};

bool valid_dtype(int t) { return t == W4_F16 || t == W4_BF16; }

}  // namespace

namespace w4 {

int device_info(DeviceInfo *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_info_ok[dev]) {
        DeviceInfo d;
        int l2 = 0;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
            return W4_ERR_CUDA;
        d.l2_bytes = static_cast<size_t>(l2);
        g_info[dev] = d;
        g_info_ok[dev] = true;
    }
    *out = g_info[dev];
    return W4_OK;
}

unsigned *device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_w4_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<unsigned *>(p);
    }
    return g_status_ptr[dev];
}

}  // namespace w4

extern "C" {

int w4_abi_version(void) { return W4A16_ABI_VERSION; }

const char *w4_status_string(int status) {
    switch (status) {
        case W4_OK: return "W4_OK";
        case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG";
        case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED";
        case W4_ERR_CUDA: return "W4_ERR_CUDA";
        case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT";
        default: return "W4_ERR_UNKNOWN";
    }
}

int w4_quantize(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                const float *col_scale, uint8_t *packed, float *scales, float *zeros,
                void *stream) {
    if (!valid_dtype(wt) || K <= 0 || N < 0 || group <= 0) return W4_ERR_INVALID_ARG;
    if (K % group != 0 || K % 8 != 0) return W4_ERR_INVALID_ARG;
    if (N > (int64_t(1) << 40) / K) return W4_ERR_INVALID_ARG;
    if (N == 0) return W4_OK;
    if (!W || !packed || !scales || !zeros) return W4_ERR_INVALID_ARG;
    if (group != 32 && group != 64 && group != 128 && group != 256) return W4_ERR_UNSUPPORTED;
    if (!w4::aligned16(W) || !w4::aligned16(packed) || !w4::aligned16(scales) ||
        !w4::aligned16(zeros) || (col_scale && !w4::aligned16(col_scale)))
        return W4_ERR_UNSUPPORTED;
    return w4::launch_quantize(W, wt, K, N, group, sym, col_scale, packed, scales, zeros,
                               static_cast<cudaStream_t>(stream));
}

size_t w4a16_workspace_bytes(int64_t M, int64_t K, int64_t N, int group) {
    if (M <= 0 || K <= 0 || N <= 0 || group != 128 || K % group != 0) return 0;
    if (M <= 32) return w4::decode_workspace_bytes(M, K, N, group);
    return 0;
}

int w4a16_gemm(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
               const float *zeros, int64_t K, int64_t N, int group, void *Y, void *workspace,
               size_t workspace_bytes, void *stream) {
    if (!valid_dtype(xt) || M < 0 || K <= 0 || N < 0 || group <= 0) return W4_ERR_INVALID_ARG;
    if (K % group != 0 || K % 8 != 0) return W4_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
        return W4_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return W4_OK;
    if (!X || !packed || !scales || !Y) return W4_ERR_INVALID_ARG;
    if (group != 128) return W4_ERR_UNSUPPORTED;
    if (!w4::aligned16(X) || !w4::aligned16(packed) || !w4::aligned16(scales) ||
        (zeros && !w4::aligned16(zeros)) || !w4::aligned16(Y))
        return W4_ERR_UNSUPPORTED;
    const size_t need = w4a16_workspace_bytes(M, K, N, group);
    if (need > 0 && (!workspace || workspace_bytes < need || !w4::aligned16(workspace)))
        return W4_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= 32)
        return w4::launch_decode(X, xt, M, packed, scales, zeros, K, N, Y, workspace,
                                 workspace_bytes, s);
    return w4::launch_prefill(X, xt, M, packed, scales, zeros, K, N, Y, s);
}

int w4_device_status(int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return W4_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_w4_status, sizeof v) != cudaSuccess) return W4_ERR_CUDA;
    if (reset) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_w4_status, &zero, sizeof zero) != cudaSuccess) return W4_ERR_CUDA;
    }
    return v ? W4_ERR_TIMEOUT : W4_OK;
}

}  // extern "C"
