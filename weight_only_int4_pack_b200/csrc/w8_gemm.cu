// w8_gemm.cu -- the 8-bit GEMM of the W8A8 layer on the 5th-generation
// tensor cores of B200: Y = (Xq Wq^T) * fl32(sx * sw) with per-tensor scales,
// INT8 (tcgen05.mma kind::i8, exact int32 accumulation) or FP8 E4M3
// (kind::f8f6f4, fp32 accumulation).
//
// Method: "LLM quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §4.3 (W8A8: both operands INT8 per
// tensor, the matmul on INT8 tensor cores) and §4.6 (FP8 E4M3 operands);
// "Quantization method families" (inference-learning-path.pages.dev) §3.3-§3.4.
//
// Tile: 128 weight rows (n) x 256 activation rows (m), persistent over all
// tiles, "swap-AB" like the W4A16 prefill kernel: Wq is the M = 128 operand A
// and Xq the N = 256 operand B, so TMEM lane = weight row and the epilogue of
// a warp writes 32 consecutive n of one output row per store.  Both operands
// arrive by TMA with the 128-byte swizzle, 128 k (bytes) per stage: 16 KB of
// Wq + 32 KB of Xq, four stages.  One stage is four MMAs of 128 x 256 x 32.
// Two accumulators of 256 columns in TMEM (512 columns): the epilogue of
// tile t drains one while the MMAs of tile t + 1 fill the other.
//
// Warp roles (192 threads): warp 0 TMA producer (one thread), warp 1 TMEM
// allocator and MMA issuer (one thread), warps 2..5 epilogue (warp w reads
// TMEM lane quarter w % 4).  Every mbarrier wait is bounded (kWaitNs); a
// wait that runs out sets the library's status word and a shared abort
// flag, every role leaves its loop, the producer and the issuer wait
// (bounded) for their copies / MMAs in flight, and TMEM is freed.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_internal.cuh"
#include "w4_tc.cuh"
#include "w8a8.h"

namespace w4 {
namespace {

constexpr int kBM = 128;     // weight rows per tile (MMA M)
constexpr int kBN = 256;     // activation rows per tile (MMA N)
constexpr int kBK = 128;     // k per stage: one 128-byte swizzle row of 8-bit values
constexpr int kMmaK = 32;    // k per tcgen05.mma for 8-bit operands
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kTmemCols = 2 * kBN;

constexpr int kATileBytes = kBM * kBK;  // 16 KB
constexpr int kBTileBytes = kBN * kBK;  // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

using namespace tc;

// Instruction descriptor, both operands K-major:
//   INT8: D s32 (2), A and B signed 8-bit (1);  E4M3: D f32 (1), A and B E4M3 (0).
template <int FMT>
__host__ __device__ constexpr uint32_t instr_desc() {
    return ((FMT == W8_INT8 ? 2u : 1u) << 4)          // D format
           | ((FMT == W8_INT8 ? 1u : 0u) << 7)        // A format
           | ((FMT == W8_INT8 ? 1u : 0u) << 10)       // B format
           | (static_cast<uint32_t>(kBN >> 3) << 17)  // N
           | (static_cast<uint32_t>(kBM >> 4) << 24); // M
}

template <int FMT>
__device__ __forceinline__ void mma8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                     uint32_t idesc, uint32_t accumulate) {
    if (FMT == W8_INT8)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

template <int YT>
__device__ __forceinline__ void store_y(void *Y, int64_t idx, float v) {
    if (YT == W4_F16)
        reinterpret_cast<__half *>(Y)[idx] = __float2half_rn(v);
    else
        reinterpret_cast<__nv_bfloat16 *>(Y)[idx] = __float2bfloat16_rn(v);
}

struct Smem {
    uint64_t full[kStages];   // TMA bytes of the stage landed
    uint64_t empty[kStages];  // MMAs of the stage done
    uint64_t tfull[2];        // accumulator b holds a finished tile
    uint64_t tempty[2];       // accumulator b drained by the epilogue
    uint32_t tmem_base;
    int abort_flag;
};

template <int FMT, int YT>
__global__ void __launch_bounds__(kThreads, 1)
w8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
               const float *__restrict__ x_scale, const float *__restrict__ w_scale, int M, int N,
               int K, void *__restrict__ Y, unsigned *__restrict__ status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *as = base;                          // kStages x 16 KB (Wq)
    uint8_t *bs = base + kStages * kATileBytes;  // kStages x 32 KB (Xq)
    Smem *sm = reinterpret_cast<Smem *>(bs + kStages * kBTileBytes);
    volatile int *abort_flag = &sm->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_tiles = (N + kBM - 1) / kBM;
    const int m_tiles = (M + kBN - 1) / kBN;
    const int tiles = n_tiles * m_tiles;
    const int kblocks = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&sm->full[s]), 1);
            mbar_init(smem_u32(&sm->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm->tfull[b]), 1);
            mbar_init(smem_u32(&sm->tempty[b]), 32 * 4);
        }
        sm->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm->tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int nt = tile % n_tiles, mt = tile / n_tiles;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(smem_u32(&sm->empty[s]), ph ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&sm->full[s]);
                    mbar_arrive_tx(fb, kStageBytes);
                    tma_load_2d(smem_u32(as + s * kATileBytes), &tmap_w, kb * kBK, nt * kBM, fb);
                    tma_load_2d(smem_u32(bs + s * kBTileBytes), &tmap_x, kb * kBK, mt * kBN, fb);
                }
            }
            // drain: wait (bounded) for the copies already issued
            for (uint32_t j = (it >= kStages ? it - kStages : 0); j < it; ++j) {
                const unsigned long long t0 = globaltimer();
                while (!mbar_try(smem_u32(&sm->full[j % kStages]), (j / kStages) & 1) &&
                       globaltimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc<FMT>();
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
                const int b = tc & 1;
                const uint32_t tph = (tc >> 1) & 1;
                if (!mbar_wait(smem_u32(&sm->tempty[b]), tph ^ 1, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem + b * kBN;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(smem_u32(&sm->full[s]), ph, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(as + s * kATileBytes);
                    const uint32_t b0 = smem_u32(bs + s * kBTileBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / kMmaK; ++kk)
                        // advance 32 elements (32 bytes) inside the swizzle row
                        mma8<FMT>(dcol, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(smem_u32(&sm->empty[s]));
                }
                if (ok) mma_commit(smem_u32(&sm->tfull[b]));
            }
            // drain: wait (bounded) until the last issued MMAs have completed
            if (it > 0) {
                const uint32_t j = it - 1;
                const unsigned long long t0 = globaltimer();
                while (!mbar_try(smem_u32(&sm->empty[j % kStages]), (j / kStages) & 1) &&
                       globaltimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;             // TMEM lane quarter of this warp
        const int er = 32 * q + lane;       // TMEM lane = weight row of the tile
        const float alpha = __fmul_rn(__ldg(x_scale), __ldg(w_scale));
        uint32_t tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            const int nt = tile % n_tiles, mt = tile / n_tiles;
            const int b = tc & 1;
            const uint32_t tph = (tc >> 1) & 1;
            if (!__all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&sm->tfull[b]), tph, abort_flag, status)))
                break;
            tc_fence_after();
            const int n = nt * kBM + er;
            const uint32_t taddr =
                tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * kBN);
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(taddr + 32 * c, r);
                tmem_wait_ld();
                const int m0 = mt * kBN + 32 * c;
                if (n < N) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int m = m0 + i;
                        const float acc = FMT == W8_INT8
                                              ? __int2float_rn(static_cast<int>(r[i]))
                                              : __uint_as_float(r[i]);
                        if (m < M) store_y<YT>(Y, static_cast<int64_t>(m) * N + n, __fmul_rn(acc, alpha));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sm->tempty[b]));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols));
    }
}

template <int FMT, int YT>
int launch_t(const void *Xq, const float *x_scale, const void *Wq, const float *w_scale, int64_t M,
             int64_t K, int64_t N, void *Y, cudaStream_t stream) {
    const char *fn = "w8_gemm";
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    if (di.cc_major != 10) return set_error(W4_ERR_UNSUPPORTED, fn, "needs an sm_100 GPU");
    if (di.max_smem_optin < kSmemBytes)
        return set_error(W4_ERR_UNSUPPORTED, fn, "not enough shared memory");
    unsigned *status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    CUtensorMap mw, mx;
    if ((st = make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                          (uint64_t)K, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B, "tensor map of Wq")) !=
        W4_OK)
        return st;
    if ((st = make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, (uint64_t)K, (uint64_t)M,
                          (uint64_t)K, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B, "tensor map of Xq")) !=
        W4_OK)
        return st;
    auto kern = w8_gemm_kernel<FMT, YT>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(W4_ERR_CUDA, "cudaGetDevice", nullptr);
    static bool attr_done[64][2][2] = {};
    if (!attr_done[dev][FMT][YT]) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(w8_gemm smem)", e);
        attr_done[dev][FMT][YT] = true;
    }
    const int64_t tiles = ((N + kBM - 1) / kBM) * ((M + kBN - 1) / kBN);
    const int grid = (int)(tiles < di.sm_count ? tiles : di.sm_count);
    kern<<<grid, kThreads, kSmemBytes, stream>>>(mw, mx, x_scale, w_scale, (int)M, (int)N, (int)K,
                                                 Y, status);
    return cuda_status(cudaGetLastError());
}

}  // namespace
}  // namespace w4

extern "C" int w8_gemm(const void *Xq, const float *x_scale, const void *Wq, const float *w_scale,
                       int fmt, int64_t M, int64_t K, int64_t N, void *Y, int yt, void *stream) {
    const char *fn = "w8_gemm";
    if (fmt != W8_INT8 && fmt != W8_E4M3)
        return w4::set_error(W4_ERR_INVALID_ARG, fn, "fmt is not W8_INT8 or W8_E4M3");
    if (yt != W4_F16 && yt != W4_BF16) return w4::set_error(W4_ERR_INVALID_ARG, fn, "bad dtype");
    if (M <= 0 || N <= 0 || K <= 0) return w4::set_error(W4_ERR_INVALID_ARG, fn, "need M, N, K >= 1");
    if (K % 16 != 0) return w4::set_error(W4_ERR_INVALID_ARG, fn, "K must be a multiple of 16");
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return w4::set_error(W4_ERR_INVALID_ARG, fn, "M, N and K must be below 2^31");
    if (fmt == W8_INT8 && K > 133000)
        return w4::set_error(W4_ERR_UNSUPPORTED, fn, "INT8 needs K <= 133000 (int32 accumulator)");
    if (!Xq || !x_scale || !Wq || !w_scale || !Y)
        return w4::set_error(W4_ERR_INVALID_ARG, fn, "null pointer");
    if (!w4::aligned16(Xq) || !w4::aligned16(Wq) || !w4::aligned16(Y))
        return w4::set_error(W4_ERR_UNSUPPORTED, fn, "pointers must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (fmt == W8_INT8)
        return yt == W4_F16
                   ? w4::launch_t<W8_INT8, W4_F16>(Xq, x_scale, Wq, w_scale, M, K, N, Y, s)
                   : w4::launch_t<W8_INT8, W4_BF16>(Xq, x_scale, Wq, w_scale, M, K, N, Y, s);
    return yt == W4_F16 ? w4::launch_t<W8_E4M3, W4_F16>(Xq, x_scale, Wq, w_scale, M, K, N, Y, s)
                        : w4::launch_t<W8_E4M3, W4_BF16>(Xq, x_scale, Wq, w_scale, M, K, N, Y, s);
}
