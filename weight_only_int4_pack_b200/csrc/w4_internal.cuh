// w4_internal.cuh -- declarations shared by the CUDA translation units of
// libw4a16.so.  Host-side launchers return w4_status codes; nothing here is
// part of the public ABI (that is include/w4a16.h).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "w4a16.h"

namespace w4 {

// Per-device attributes cached on first use.
struct DeviceInfo {
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    int max_smem_optin = 0;
    size_t l2_bytes = 0;
};
int device_info(DeviceInfo *out);  // W4_OK or W4_ERR_CUDA

// Device address of the library's status word for the current device
// (kernels set W4_ERR_TIMEOUT into it when a bounded wait runs out).
unsigned *device_status_ptr();

// Records a description of the failing call for w4_last_error() and
// returns the status.  `what` names the call; `detail` may be null.
int set_error(int status, const char *what, const char *detail);
int cuda_fail(const char *what, cudaError_t e);  // W4_ERR_CUDA with the runtime's text

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? W4_OK : cuda_fail("kernel launch", e); }

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library does not link libcuda); records an error and returns null if absent.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Encodes a 2-D tiled tensor map; W4_OK or W4_ERR_CUDA (with a message).
int make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *ptr, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                CUtensorMapSwizzle swz, const char *what);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- launchers (one per translation unit) ----
int launch_quantize(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                    const float *col_scale, uint8_t *packed, float *scales, float *zeros,
                    cudaStream_t stream);

// decode path, M <= 32
size_t decode_workspace_bytes(int64_t M, int64_t K, int64_t N, int group);
size_t decode_counter_bytes();  // leading workspace bytes that must read as zero
int launch_decode(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                  const float *zeros, int64_t K, int64_t N, void *Y, void *workspace,
                  size_t workspace_bytes, cudaStream_t stream);

// M = 1, K % 512 == 0, K <= 4096: the CUDA-core GEMV; needs no workspace
bool gemv1_supported(int64_t M, int64_t K);
int launch_gemv1(const void *X, int xt, const uint8_t *packed, const float *scales,
                 const float *zeros, int64_t K, int64_t N, void *Y, cudaStream_t stream);

// decode path for M <= 8, K <= 4096 (warp-level tensor-core GEMV); needs no workspace
bool gemv_supported(int64_t M, int64_t K);
int launch_gemv(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                const float *zeros, int64_t K, int64_t N, void *Y, cudaStream_t stream);

// prefill path, M > 32 (tcgen05)
int launch_prefill(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                   const float *zeros, int64_t K, int64_t N, void *Y, cudaStream_t stream);

// ---- GPTQ's dense linear algebra on the device (w4_linalg.cu) ----
// H = 2 X^T X (fp32, [K][K] row-major; only the tiles on and above the
// diagonal are written) from X [Mc][K] (W4_F16 / W4_BF16).
int hessian(const void *X, int xt, int64_t Mc, int64_t K, float *H, cudaStream_t stream);
// fp32 words of scratch inverse_factor needs for an n x n matrix.
size_t linalg_scratch_floats(int64_t n);
// In place: H (n x n fp32, the upper triangle read) -> U, the upper Cholesky
// factor of H^-1 (row-major, zeros below the diagonal).  n % 64 == 0.
// Synchronizes `stream` once to read the factorization status (info_dev: one
// int of device memory); W4_ERR_INVALID_ARG if H is not positive definite.
int inverse_factor(const char *fn, float *H, int64_t n, float *scratch, int *info_dev,
                   cudaStream_t stream);

// ---- NVIDIA libraries for plain dense linear algebra (w4_libs.cu) ----
// C [m x n] fp32 (column-major, ldc) = alpha * op(A) op(B) + beta * C with
// 16-bit A and B (types W4_F16 / W4_BF16), fp32 accumulation (cuBLAS GemmEx).
int blas_gemm_f32(const char *fn, bool trans_a, bool trans_b, int m, int n, int k, float alpha,
                  const void *A, int at, int lda, const void *B, int bt, int ldb, float beta,
                  float *C, int ldc, cudaStream_t stream);
}  // namespace w4
