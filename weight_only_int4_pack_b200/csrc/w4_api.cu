// w4_api.cu -- the extern "C" entry points of libw4a16.so (declared in
// include/w4a16.h): host-side argument validation, dispatch to the kernels,
// the per-device attribute cache, the device status word and the
// thread-local description of the last failure.

#include <stdio.h>

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

thread_local char g_last_error[320] = "";

// One warp; lane 0 waits on an mbarrier that nothing arrives on, bounded by
// limit_ns of the global timer, then records the timeout in the status word.
__global__ void selftest_wait_kernel(unsigned long long limit_ns, unsigned *status) {
    __shared__ uint64_t bar;
    const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        unsigned long long t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        while (true) {
            uint32_t ok;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(ok)
                : "r"(b)
                : "memory");
            if (ok) break;  // cannot happen: nothing arrives
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > limit_ns) {
                atomicOr(status, 1u);
                break;
            }
        }
    }
    __syncwarp();
}

bool valid_dtype(int t) { return t == W4_F16 || t == W4_BF16; }

int reject(int status, const char *fn, const char *why) { return w4::set_error(status, fn, why); }

}  // namespace

namespace w4 {

int set_error(int status, const char *what, const char *detail) {
    if (status != W4_OK)
        snprintf(g_last_error, sizeof g_last_error, "%s: %s%s%s", w4_status_string(status), what,
                 detail ? ": " : "", detail ? detail : "");
    return status;
}

int cuda_fail(const char *what, cudaError_t e) {
    return set_error(W4_ERR_CUDA, what, cudaGetErrorString(e));
}

int device_info(DeviceInfo *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return set_error(W4_ERR_CUDA, "device ordinal", "out of range");
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_info_ok[dev]) {
        DeviceInfo d;
        int l2 = 0;
        if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                        dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev)) != cudaSuccess)
            return cuda_fail("cudaDeviceGetAttribute", e);
        d.l2_bytes = static_cast<size_t>(l2);
        g_info[dev] = d;
        g_info_ok[dev] = true;
    }
    *out = g_info[dev];
    return W4_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    if (!fn) set_error(W4_ERR_CUDA, "cuTensorMapEncodeTiled", "driver entry point not found");
    return fn;
}

// Encoded tensor maps are cached per host thread, direct-mapped by a hash of
// everything the encoding depends on (the map holds only the address, the
// extents, the stride, the box and the modes), so a layer called again with
// the same buffers skips the driver call.  A buffer freed and another
// allocated at the same address with the same extents gets the same map,
// which is exactly the map it needs.
struct MapKey {
    const void *ptr;
    uint64_t inner, outer, row_bytes;
    uint32_t box_inner, box_outer;
    int dt, swz;
    bool operator==(const MapKey &o) const {
        return ptr == o.ptr && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
               box_inner == o.box_inner && box_outer == o.box_outer && dt == o.dt && swz == o.swz;
    }
};
struct MapEntry {
    CUtensorMap map;
    MapKey key;
    bool valid;
};
constexpr int kMapCache = 64;
thread_local MapEntry t_maps[kMapCache];

int make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *ptr, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                CUtensorMapSwizzle swz, const char *what) {
    const MapKey key = {ptr, inner, outer, row_bytes, box_inner, box_outer, (int)dt, (int)swz};
    uint64_t h = reinterpret_cast<uintptr_t>(ptr) >> 8;
    h = h * 0x9E3779B97F4A7C15ull ^ inner ^ (outer << 20) ^ (row_bytes << 7) ^
        (uint64_t(box_inner) << 40) ^ (uint64_t(box_outer) << 48) ^ (uint64_t(dt) << 56) ^
        (uint64_t(swz) << 60);
    MapEntry &slot = t_maps[(h ^ (h >> 29)) % kMapCache];
    if (slot.valid && slot.key == key) {
        *map = slot.map;
        return W4_OK;
    }
    auto fn = tensor_map_encoder();
    if (!fn) return W4_ERR_CUDA;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[64];
        snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled returned CUresult %d", (int)r);
        return set_error(W4_ERR_CUDA, what, buf);
    }
    slot.map = *map;
    slot.key = key;
    slot.valid = true;
    return W4_OK;
}

unsigned *device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_w4_status);
        if (e != cudaSuccess) {
            cuda_fail("cudaGetSymbolAddress(status word)", e);
            return nullptr;
        }
        g_status_ptr[dev] = static_cast<unsigned *>(p);
    }
    return g_status_ptr[dev];
}

}  // namespace w4

namespace {

int quantize_impl(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                  const float *col_scale, uint8_t *packed, float *scales, float *zeros,
                  void *stream) {
    const char *fn = "w4_quantize";
    if (!valid_dtype(wt)) return reject(W4_ERR_INVALID_ARG, fn, "wt is not W4_F16 or W4_BF16");
    if (K <= 0 || N < 0) return reject(W4_ERR_INVALID_ARG, fn, "K must be > 0 and N >= 0");
    if (group <= 0 || K % group != 0)
        return reject(W4_ERR_INVALID_ARG, fn, "K must be a positive multiple of group");
    if (K % 8 != 0) return reject(W4_ERR_INVALID_ARG, fn, "K must be a multiple of 8");
    if (N > (int64_t(1) << 40) / K) return reject(W4_ERR_INVALID_ARG, fn, "N * K too large");
    if (N == 0) return W4_OK;
    if (!W || !packed || !scales || !zeros) return reject(W4_ERR_INVALID_ARG, fn, "null pointer");
    if (group != 32 && group != 64 && group != 128 && group != 256)
        return reject(W4_ERR_UNSUPPORTED, fn, "group must be 32, 64, 128 or 256");
    if (!w4::aligned16(W) || !w4::aligned16(packed) || !w4::aligned16(scales) ||
        !w4::aligned16(zeros) || (col_scale && !w4::aligned16(col_scale)))
        return reject(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    return w4::launch_quantize(W, wt, K, N, group, sym, col_scale, packed, scales, zeros,
                               static_cast<cudaStream_t>(stream));
}

int gemm_impl(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
              const float *zeros, int64_t K, int64_t N, int group, void *Y, void *workspace,
              size_t workspace_bytes, void *stream) {
    const char *fn = "w4a16_gemm";
    if (!valid_dtype(xt)) return reject(W4_ERR_INVALID_ARG, fn, "xt is not W4_F16 or W4_BF16");
    if (M < 0 || K <= 0 || N < 0) return reject(W4_ERR_INVALID_ARG, fn, "need M >= 0, K > 0, N >= 0");
    if (group <= 0 || K % group != 0)
        return reject(W4_ERR_INVALID_ARG, fn, "K must be a positive multiple of group");
    if (K % 8 != 0) return reject(W4_ERR_INVALID_ARG, fn, "K must be a multiple of 8");
    if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
        return reject(W4_ERR_INVALID_ARG, fn, "M, N and K must be below 2^31");
    if (M == 0 || N == 0) return W4_OK;
    if (!X || !packed || !scales || !Y) return reject(W4_ERR_INVALID_ARG, fn, "null pointer");
    if (group != 128) return reject(W4_ERR_UNSUPPORTED, fn, "group must be 128");
    if (!w4::aligned16(X) || !w4::aligned16(packed) || !w4::aligned16(scales) ||
        (zeros && !w4::aligned16(zeros)) || !w4::aligned16(Y))
        return reject(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= 32) {
        const size_t need = w4::decode_workspace_bytes(M, K, N, group);
        if (need > 0 && (!workspace || workspace_bytes < need || !w4::aligned16(workspace)))
            return reject(W4_ERR_INVALID_ARG, fn,
                          "workspace missing, misaligned or smaller than w4a16_workspace_bytes");
        return w4::launch_decode(X, xt, M, packed, scales, zeros, K, N, Y, workspace,
                                 workspace_bytes, s);
    }
    return w4::launch_prefill(X, xt, M, packed, scales, zeros, K, N, Y, s);
}

}  // namespace

extern "C" {

int w4_abi_version(void) { return W4A16_ABI_VERSION; }

const char *w4_last_error(void) { return g_last_error; }

const char *w4_status_string(int status) {
    switch (status) {
        case W4_OK: return "W4_OK";
        case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG";
        case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED";
        case W4_ERR_CUDA: return "W4_ERR_CUDA";
        case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT";
        case W4_ERR_BOUNDS: return "W4_ERR_BOUNDS";
        default: return "W4_ERR_UNKNOWN";
    }
}

int w4_quantize(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                const float *col_scale, uint8_t *packed, float *scales, float *zeros,
                void *stream) {
    return quantize_impl(W, wt, K, N, group, sym, col_scale, packed, scales, zeros, stream);
}

size_t w4a16_workspace_bytes(int64_t M, int64_t K, int64_t N, int group) {
    if (M <= 0 || K <= 0 || N <= 0 || group != 128 || K % group != 0) return 0;
    if (M <= 32) return w4::decode_workspace_bytes(M, K, N, group);
    return 0;
}

int w4a16_gemm(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
               const float *zeros, int64_t K, int64_t N, int group, void *Y, void *workspace,
               size_t workspace_bytes, void *stream) {
    return gemm_impl(X, xt, M, packed, scales, zeros, K, N, group, Y, workspace, workspace_bytes,
                     stream);
}

int w4_selftest_wait_timeout(unsigned timeout_us, void *stream) {
    if (timeout_us < 1 || timeout_us > 1000000)
        return w4::set_error(W4_ERR_INVALID_ARG, "w4_selftest_wait_timeout",
                             "timeout_us must be 1 .. 1000000");
    unsigned *status = w4::device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<unsigned long long>(timeout_us) * 1000ull, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return w4::cuda_fail("selftest_wait_kernel launch", e);
    return W4_OK;
}

int w4_device_status(int reset) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return w4::cuda_fail("cudaDeviceSynchronize", e);
    unsigned v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_w4_status, sizeof v)) != cudaSuccess)
        return w4::cuda_fail("read status word", e);
    if (reset) {
        const unsigned zero = 0;
        if ((e = cudaMemcpyToSymbol(g_w4_status, &zero, sizeof zero)) != cudaSuccess)
            return w4::cuda_fail("clear status word", e);
    }
    if (v & 2u) return W4_ERR_BOUNDS;
    return v ? W4_ERR_TIMEOUT : W4_OK;
}

int w4_debug_build(void) {
#ifdef W4_DEBUG
    return 1;
#else
    return 0;
#endif
}

int w4_debug_first_failure(int *file_id, int *line) {
    if (!file_id || !line) return w4::set_error(W4_ERR_INVALID_ARG, "w4_debug_first_failure", "null pointer");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return w4::cuda_fail("cudaDeviceSynchronize", e);
    unsigned v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_w4_status, sizeof v)) != cudaSuccess)
        return w4::cuda_fail("read status word", e);
    *file_id = static_cast<int>((v >> 2) & 63u);
    *line = static_cast<int>(v >> 8);
    return W4_OK;
}

}  // extern "C"
