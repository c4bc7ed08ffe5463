// w4_libs.cu -- the two NVIDIA libraries the calibration entry points call
// for plain dense linear algebra, opened on first use: cuBLAS (a GEMM with
// fp32 output: the unquantized layer's output in the AWQ search, the Hessian
// 2 X^T X of GPTQ) and cuSOLVER (Cholesky factorization and inversion of the
// GPTQ Hessian).
//
// The library does not link them: only these calibration entry points use
// them, and the quantizer and GEMM entry points must load where they are
// absent.  The first use on a device opens libcublas.so.12 /
// libcusolver.so.11 (the process's copy when one is already loaded, e.g. by
// PyTorch) and creates one handle per device, kept for the life of the
// process.  Calls are serialized by a process-wide lock (a handle is bound
// to one stream at a time).

#include <cublas_v2.h>
#include <cusolverDn.h>
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
using PFN_solver_create = cusolverStatus_t (*)(cusolverDnHandle_t *);
using PFN_solver_set_stream = cusolverStatus_t (*)(cusolverDnHandle_t, cudaStream_t);
using PFN_potrf_bufsize = cusolverStatus_t (*)(cusolverDnHandle_t, cublasFillMode_t, int, float *,
                                               int, int *);
using PFN_potrf = cusolverStatus_t (*)(cusolverDnHandle_t, cublasFillMode_t, int, float *, int,
                                       float *, int, int *);

constexpr int kMaxDevices = 64;
std::mutex g_mu;

PFN_blas_create g_blas_create = nullptr;
PFN_blas_set_stream g_blas_set_stream = nullptr;
PFN_gemm_ex g_gemm_ex = nullptr;
cublasHandle_t g_blas[kMaxDevices] = {};

PFN_solver_create g_solver_create = nullptr;
PFN_solver_set_stream g_solver_set_stream = nullptr;
PFN_potrf_bufsize g_potrf_bufsize = nullptr, g_potri_bufsize = nullptr;
PFN_potrf g_potrf = nullptr, g_potri = nullptr;
cusolverDnHandle_t g_solver[kMaxDevices] = {};

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

// Caller holds g_mu.
int solver_handle(const char *fn, cusolverDnHandle_t *out) {
    int dev = 0, st = current_device(fn, &dev);
    if (st != W4_OK) return st;
    if (!g_potri) {
        void *h = dlopen("libcusolver.so.11", RTLD_NOW | RTLD_LOCAL);
        if (!h) return set_error(W4_ERR_UNSUPPORTED, fn, "libcusolver.so.11 could not be loaded");
        g_solver_create = reinterpret_cast<PFN_solver_create>(dlsym(h, "cusolverDnCreate"));
        g_solver_set_stream =
            reinterpret_cast<PFN_solver_set_stream>(dlsym(h, "cusolverDnSetStream"));
        g_potrf_bufsize = reinterpret_cast<PFN_potrf_bufsize>(dlsym(h, "cusolverDnSpotrf_bufferSize"));
        g_potri_bufsize = reinterpret_cast<PFN_potrf_bufsize>(dlsym(h, "cusolverDnSpotri_bufferSize"));
        g_potrf = reinterpret_cast<PFN_potrf>(dlsym(h, "cusolverDnSpotrf"));
        g_potri = reinterpret_cast<PFN_potrf>(dlsym(h, "cusolverDnSpotri"));
        if (!g_solver_create || !g_solver_set_stream || !g_potrf_bufsize || !g_potri_bufsize ||
            !g_potrf || !g_potri) {
            g_potri = nullptr;
            return set_error(W4_ERR_UNSUPPORTED, fn, "libcusolver.so.11 lacks potrf / potri");
        }
    }
    if (!g_solver[dev]) {
        cusolverDnHandle_t h = nullptr;
        if (g_solver_create(&h) != CUSOLVER_STATUS_SUCCESS)
            return set_error(W4_ERR_CUDA, fn, "cusolverDnCreate failed");
        g_solver[dev] = h;
    }
    *out = g_solver[dev];
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

size_t solver_work_bytes(int64_t n) {
    // potrf / potri of an fp32 n x n matrix ask for far less (a few panel
    // widths times n); the run-time query is checked against this.
    const size_t v = sizeof(float) * size_t(n) * 512;
    return v < (size_t(1) << 22) ? (size_t(1) << 22) : v;
}

int solver_inverse_factor(const char *fn, float *H, int n, void *work, size_t work_bytes,
                          int *info_dev, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    cusolverDnHandle_t h = nullptr;
    int st = solver_handle(fn, &h);
    if (st != W4_OK) return st;
    if (g_solver_set_stream(h, stream) != CUSOLVER_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cusolverDnSetStream failed");
    int l1 = 0, l2 = 0;
    if (g_potrf_bufsize(h, CUBLAS_FILL_MODE_LOWER, n, H, n, &l1) != CUSOLVER_STATUS_SUCCESS ||
        g_potri_bufsize(h, CUBLAS_FILL_MODE_LOWER, n, H, n, &l2) != CUSOLVER_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cuSOLVER buffer size query failed");
    const int lwork = l1 > l2 ? l1 : l2;
    if (size_t(lwork) * sizeof(float) > work_bytes)
        return set_error(W4_ERR_UNSUPPORTED, fn, "cuSOLVER asks for more work space than reserved");
    float *w = static_cast<float *>(work);
    // H = L L^T (lower, column-major); H^-1 from L (lower triangle); the lower
    // Cholesky factor of H^-1, which read row-major is the upper factor U with
    // H^-1 = U^T U.  A symmetric row-major matrix is its own column-major view.
    if (g_potrf(h, CUBLAS_FILL_MODE_LOWER, n, H, n, w, lwork, info_dev) != CUSOLVER_STATUS_SUCCESS ||
        g_potri(h, CUBLAS_FILL_MODE_LOWER, n, H, n, w, lwork, info_dev + 1) != CUSOLVER_STATUS_SUCCESS ||
        g_potrf(h, CUBLAS_FILL_MODE_LOWER, n, H, n, w, lwork, info_dev + 2) != CUSOLVER_STATUS_SUCCESS)
        return set_error(W4_ERR_CUDA, fn, "cuSOLVER potrf / potri failed to launch");
    int info[3] = {0, 0, 0};
    cudaError_t e = cudaMemcpyAsync(info, info_dev, sizeof info, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail("reading the factorization status", e);
    if (info[0] != 0 || info[1] != 0 || info[2] != 0)
        return set_error(W4_ERR_INVALID_ARG, fn,
                         "the damped Hessian is not positive definite (raise the damping)");
    return W4_OK;
}

}  // namespace w4
