// w4_libs.cu -- the one NVIDIA library call of the library, opened on first
// use: a cuBLAS GEMM with fp32 output for the unquantized layer's output
// X W^T that the AWQ search compares against (computed once per search, a
// few percent of its time).
//
// The library does not link cuBLAS: only w4_awq_search uses it, and the
// other entry points must load where it is absent.  The first use on a
// device opens libcublas.so.12 (the process's copy when one is already
// loaded, e.g. by PyTorch) and creates one handle per device, kept for the
// life of the process.  Calls are serialized by a process-wide lock (a
// handle is bound to one stream at a time).

#include <cublas_v2.h>
#include <dlfcn.h>

#include <mutex>

#include "w4_internal.cuh"

namespace w4 {
namespace {

using PFN_blas_create = cublasStatus_t (*)(cublasHandle_t *);
using PFN_blas_set_stream = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
using PFN_gemm_ex = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int,
                                       int, int, const void *, const void *, cudaDataType, int,
                                       const void *, cudaDataType, int, const void *, void *,
                                       cudaDataType, int, cublasComputeType_t, cublasGemmAlgo_t);

constexpr int kMaxDevices = 64;
std::mutex g_mu;

PFN_blas_create g_blas_create = nullptr;
PFN_blas_set_stream g_blas_set_stream = nullptr;
PFN_gemm_ex g_gemm_ex = nullptr;
cublasHandle_t g_blas[kMaxDevices] = {};


int current_device(const char *fn, int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (*dev < 0 || *dev >= kMaxDevices) return set_error(W4_ERR_CUDA, fn, "device ordinal out of range");
    return W4_OK;
}

// Caller holds g_mu.
int blas_handle(const char *fn, cublasHandle_t *out) {
    int dev = 0, st = current_device(fn, &dev);
    if (st != W4_OK) return st;
    if (!g_gemm_ex) {
        void *h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
        if (!h) return set_error(W4_ERR_UNSUPPORTED, fn, "libcublas.so.12 could not be loaded");
        g_blas_create = reinterpret_cast<PFN_blas_create>(dlsym(h, "cublasCreate_v2"));
        g_blas_set_stream = reinterpret_cast<PFN_blas_set_stream>(dlsym(h, "cublasSetStream_v2"));
        g_gemm_ex = reinterpret_cast<PFN_gemm_ex>(dlsym(h, "cublasGemmEx"));
        if (!g_blas_create || !g_blas_set_stream || !g_gemm_ex) {
            g_gemm_ex = nullptr;
            return set_error(W4_ERR_UNSUPPORTED, fn, "libcublas.so.12 lacks cublasGemmEx");
        }
    }
    if (!g_blas[dev]) {
        cublasHandle_t h = nullptr;
        if (g_blas_create(&h) != CUBLAS_STATUS_SUCCESS)
            return set_error(W4_ERR_CUDA, fn, "cublasCreate failed");
        g_blas[dev] = h;
    }
    *out = g_blas[dev];
    return W4_OK;
}

}  // namespace

int blas_gemm_f32(const char *fn, bool trans_a, bool trans_b, int m, int n, int k, float alpha,
                  const void *A, int at, int lda, const void *B, int bt, int ldb, float beta,
                  float *C, int ldc, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    cublasHandle_t h = nullptr;
    int st = blas_handle(fn, &h);
    if (st != W4_OK) return st;
    if (g_blas_set_stream(h, stream) != CUBLAS_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cublasSetStream failed");
    const cudaDataType ta = at == W4_F16 ? CUDA_R_16F : CUDA_R_16BF;
    const cudaDataType tb = bt == W4_F16 ? CUDA_R_16F : CUDA_R_16BF;
    const cublasStatus_t bs =
        g_gemm_ex(h, trans_a ? CUBLAS_OP_T : CUBLAS_OP_N, trans_b ? CUBLAS_OP_T : CUBLAS_OP_N, m, n,
                  k, &alpha, A, ta, lda, B, tb, ldb, &beta, C, CUDA_R_32F, ldc, CUBLAS_COMPUTE_32F,
                  CUBLAS_GEMM_DEFAULT);
    if (bs != CUBLAS_STATUS_SUCCESS) return set_error(W4_ERR_CUDA, fn, "cublasGemmEx failed");
    return W4_OK;
}

}  // namespace w4
