// w4_gemv1.cu -- the W4A16 linear layer at M = 1 (one-token decode) on the CUDA
// cores.
//
// y[n] = sum_g scale[n][g] * sum_{k in g} x[k] * (u[n][k] - zero[n][g]): the
// "dequant -> 16-bit matmul" of W4A16 ("Quantization method families",
// inference-learning-path.pages.dev, §2), dequantization as in "LLM
// quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2-§2.3.  A GEMV moves 0.5 byte
// of codes per weight and does one multiply-add per weight, so it is bound by
// HBM, not by any arithmetic pipe; the kernel is shaped for that:
//
//   * No split-K, no workspace.  Three CTAs of four warps per SM (so that a
//     CTA of the next launch in the stream can be resident, and start its
//     weight copies, while this launch's last CTAs finish); each CTA owns an
//     equal contiguous range of weight rows and its warps take the rows
//     round robin.  A row's codes, scales
//     and zero points are contiguous in HBM and come in with three 1-D bulk
//     copies (cp.async.bulk) into a per-warp ring of shared-memory stages, so
//     every warp has four rows in flight without holding them in registers,
//     and the copies of the first rows are issued before anything else.
//   * Exact products, fp32 sums: the sm_100 mixed-precision fma
//     (fma.rn.f32.f16 / .bf16) multiplies two 16-bit operands exactly and adds
//     in fp32 (measured on B200 it costs two issue slots, about three per
//     weight in all, so the kernel runs near its issue limit; at M = 1 it
//     still beats the warp-level tensor-core GEMV of w4_gemv.cu, whose warps
//     must meet per 16-row tile, because every warp here streams its own rows
//     on its own).  The codes become 16-bit operands with one lop3 per pair: the
//     code bits OR-ed into the mantissa of 1024.0 (fp16) or 128.0 (bf16) give
//     1024 + u or 128 + u exactly (and 1024 + 16u for the high nibble of a
//     byte in fp16, so only half the nibbles need a shift).  The offsets are
//     removed per group with sums of x computed once per CTA:
//       sum x (u - z) = sum x (1024 + u) - (1024 + z) sum x.
//     Products are exact and every sum is fp32; no weight is rounded to 16 bits.
//   * Each lane keeps its own 32-k slices of x in registers for the whole
//     kernel (K <= 4096: at most 128 k, 64 registers), so the only per-weight
//     shared-memory traffic is the code stream itself.
//   * Row sums are reduced across the warp four rows at a time (six shuffles
//     for four rows) and rounded once to the output dtype.
//   * Programmatic dependent launch: the first rows' copies are issued, and
//     dependents are released, before griddepcontrol.wait; x and y are touched
//     only after it.
//
// Every mbarrier wait is bounded; a wait that runs out sets the library's
// status word (W4_ERR_TIMEOUT), the warp stops, and it waits (bounded) for its
// copies in flight before it exits.  The W4_DEBUG build checks every global
// and shared-memory index and every copy against its buffer (w4_debug.cuh).

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_debug.cuh"
#include "w4_half.cuh"
#include "w4_internal.cuh"
#include "w4_tc.cuh"

namespace w4 {
namespace {

[[maybe_unused]] constexpr unsigned kDbgFile = 5;  // W4_DEBUG file id

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 4;      // rows in flight per warp
constexpr int kBatch = 4;       // rows reduced together
constexpr int kMaxK = 4096;     // x slices held in registers: K / 64 words per lane
constexpr int kGroup = 128;
constexpr int kCtasPerSm = 3;  // 12 warps per SM; a CTA of the next launch can join early

static_assert(kBatch == kStages, "a batch uses every stage once");

__host__ __device__ constexpr int stage_bytes_for(int K, bool asym) {
    return K / 2 + (asym ? 2 : 1) * (K / kGroup) * 4;
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}

__device__ __forceinline__ float lds32f(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t lop_or(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
    return d;
}

// acc += lo(a) * lo(x) + hi(a) * hi(x): two mixed-precision fmas (16-bit
// operands, exact product, fp32 add).
template <int XT>
__device__ __forceinline__ void fma2(float &acc, uint32_t a, uint32_t x) {
    if (XT == W4_F16)
        asm("{\n\t.reg .b16 al, ah, xl, xh;\n\t"
            "mov.b32 {al, ah}, %1;\n\t"
            "mov.b32 {xl, xh}, %2;\n\t"
            "fma.rn.f32.f16 %0, al, xl, %0;\n\t"
            "fma.rn.f32.f16 %0, ah, xh, %0;\n\t}"
            : "+f"(acc)
            : "r"(a), "r"(x));
    else
        asm("{\n\t.reg .b16 al, ah, xl, xh;\n\t"
            "mov.b32 {al, ah}, %1;\n\t"
            "mov.b32 {xl, xh}, %2;\n\t"
            "fma.rn.f32.bf16 %0, al, xl, %0;\n\t"
            "fma.rn.f32.bf16 %0, ah, xh, %0;\n\t}"
            : "+f"(acc)
            : "r"(a), "r"(x));
}

// sum over one 32-k slice of x * (offset + code), into two accumulators.
// Code word j of the slice holds k = 8j + {0,2,4,6,1,3,5,7} in nibbles 0..7,
// so masking with 0x000F000F yields the pair (8j, 8j+1) in the two halves,
// 0x00F000F0 the pair (8j+2, 8j+3) shifted up by four bits, and the same on
// the word shifted right by 8 the pairs (8j+4, 8j+5) and (8j+6, 8j+7).
// fp16: accA collects x * (1024 + u) of k = 8j + {0,1,4,5}, accB collects
// x * (1024 + 16u) of k = 8j + {2,3,6,7}.  bf16: every pair needs a shift;
// both accumulators collect x * (128 + u).
template <int XT>
__device__ __forceinline__ void slice_dot(const uint4 c, const uint4 (&x)[4], float &accA,
                                          float &accB) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 xv = x[j];
        if (XT == W4_F16) {
            const uint32_t m = 0x64006400u;
            const uint32_t w8 = w[j] >> 8;
            fma2<XT>(accA, lop_or(w[j], 0x000F000Fu, m), xv.x);
            fma2<XT>(accB, lop_or(w[j], 0x00F000F0u, m), xv.y);
            fma2<XT>(accA, lop_or(w8, 0x000F000Fu, m), xv.z);
            fma2<XT>(accB, lop_or(w8, 0x00F000F0u, m), xv.w);
        } else {
            const uint32_t m = 0x43004300u;
            fma2<XT>(accA, lop_or(w[j], 0x000F000Fu, m), xv.x);
            fma2<XT>(accB, lop_or(w[j] >> 4, 0x000F000Fu, m), xv.y);
            fma2<XT>(accA, lop_or(w[j] >> 8, 0x000F000Fu, m), xv.z);
            fma2<XT>(accB, lop_or(w[j] >> 12, 0x000F000Fu, m), xv.w);
        }
    }
}

// Sum of 4 per-lane values over the warp: after the call lane l holds the
// full sum of value ((l >> 3) & 3).
__device__ __forceinline__ float reduce4(const float (&v)[kBatch], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8;
    float u[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const float send = b4 ? v[t] : v[t + 2];
        const float keep = b4 ? v[t + 2] : v[t];
        u[t] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    const float send = b3 ? u[0] : u[1];
    float r = (b3 ? u[1] : u[0]) + __shfl_xor_sync(0xffffffffu, send, 8);
    r += __shfl_xor_sync(0xffffffffu, r, 4);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    return r;
}

// Bounded wait of the whole warp on a stage barrier.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, unsigned *status) {
    bool ok = tc::mbar_try(bar, parity);
    if (!ok) {
        const unsigned long long t0 = tc::globaltimer();
        while (!(ok = tc::mbar_try(bar, parity))) {
            if (tc::globaltimer() - t0 > tc::kWaitNs) {
                atomicOr(status, 1u);
                break;
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// C = 32-k slices per lane = ceil(K / 1024).
template <int XT, int C>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    gemv1_kernel(const uint8_t *__restrict__ packed, const float *__restrict__ scales,
                const float *__restrict__ zeros, const uint16_t *__restrict__ X,
                uint16_t *__restrict__ Y, int K, int N, unsigned *status) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int G = K / kGroup;
    const int KW = K / 32;  // 32-k slices of a row (16 code bytes each)
    const bool asym = zeros != nullptr;
    const uint32_t sbytes = static_cast<uint32_t>(stage_bytes_for(K, asym));
    const uint32_t cbytes = static_cast<uint32_t>(K / 2);
    const uint32_t gbytes = static_cast<uint32_t>(G * 4);

    // shared memory: x [K] (swizzled 16-byte pieces), then per warp kStages
    // stages, then the stage barriers
    const uint32_t sx = tc::smem_u32(smem);
    const uint32_t sstage = sx + static_cast<uint32_t>(K) * 2 + warp * kStages * sbytes;
    const uint32_t sbar = sx + static_cast<uint32_t>(K) * 2 + kWarps * kStages * sbytes +
                          warp * kStages * 8;

    // rows of this CTA and of this warp
    const int64_t P = gridDim.x;
    const int r0 = static_cast<int>(static_cast<int64_t>(N) * blockIdx.x / P);
    const int r1 = static_cast<int>(static_cast<int64_t>(N) * (blockIdx.x + 1) / P);
    const int nrows = r1 - r0 > warp ? (r1 - r0 - warp + kWarps - 1) / kWarps : 0;
    auto row_of = [&](int j) { return r0 + warp + j * kWarps; };

    auto issue = [&](int j, int d) {  // lane 0: row j into stage d
        const int64_t r = row_of(j);
        const uint32_t st = sstage + d * sbytes;
        const uint32_t bar = sbar + d * 8;
        if (!W4_CHECK(r >= 0 && r < N && d >= 0 && d < kStages &&
                          in_range(st, sbytes, sx, dyn_smem_bytes()) &&
                          in_range(bar, 8, sx, dyn_smem_bytes()),
                      status))
            return;
        tc::mbar_arrive_tx(bar, sbytes);
        bulk_g2s(st, packed + r * cbytes, cbytes, bar);
        bulk_g2s(st + cbytes, scales + r * G, gbytes, bar);
        if (asym) bulk_g2s(st + cbytes + gbytes, zeros + r * G, gbytes, bar);
    };

    if (lane == 0) {
#pragma unroll
        for (int d = 0; d < kStages; ++d) tc::mbar_init(sbar + d * 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
#pragma unroll
        for (int d = 0; d < kStages; ++d)
            if (d < nrows) issue(d, d);
    }
    // the next kernel of the stream may launch now; this one waits for the
    // previous kernel before it reads x
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // x -> shared memory.  16-byte piece p of slice i (p = 0..3) is stored at
    // slice*64 + 16*(p ^ ((i >> 1) & 3)), so that the 8 lanes of a quarter warp
    // reading piece p of slices i..i+7 hit 8 different bank quads.
    for (int t = threadIdx.x; t < K / 8; t += kThreads) {
        const int i = t >> 2, p = t & 3;
        const uint32_t a = sx + i * 64 + ((p ^ ((i >> 1) & 3)) << 4);
        if (!W4_CHECK(t >= 0 && in_range(a, 16, sx, static_cast<uint64_t>(K) * 2), status)) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X) + t);
        sts128(a, v);
    }
    __syncthreads();

    // this lane's x slices, their sums S and the offset sums T
    uint4 xr[C][4];
    float S[C], T[C];
#pragma unroll
    for (int q = 0; q < C; ++q) {
        const int i = lane + 32 * q;
        const bool on = i < KW;
        const int ic = on ? i : 0;
        float s = 0.f, tb = 0.f;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const uint32_t a = sx + ic * 64 + ((p ^ ((ic >> 1) & 3)) << 4);
            xr[q][p] = on && W4_CHECK(in_range(a, 16, sx, static_cast<uint64_t>(K) * 2), status)
                           ? lds128(a)
                           : make_uint4(0, 0, 0, 0);
            float f[8];
            widen8<XT>(xr[q][p], f);
            // fp16: k = 8p + {0,1,4,5} carry offset 1024, k = 8p + {2,3,6,7}
            // carry 1024 / 16 after the accB rescale; bf16: all carry 128
            s += ((f[0] + f[1]) + (f[4] + f[5])) + ((f[2] + f[3]) + (f[6] + f[7]));
            tb += (f[2] + f[3]) + (f[6] + f[7]);
        }
        S[q] = s;
        // fp16: T = 1024 * (sum_A x + sum_B x / 16); bf16: T = 128 * sum x
        T[q] = XT == W4_F16 ? 1024.f * (s - tb) + 64.f * tb : 128.f * s;
    }

    // main loop: batches of kBatch rows, each row from its stage
    for (int jb = 0; jb < nrows; jb += kBatch) {
        float part[kBatch];
#pragma unroll
        for (int t = 0; t < kBatch; ++t) {
            const int j = jb + t;
            part[t] = 0.f;
            if (j < nrows) {
                const int d = t;
                const uint32_t st = sstage + d * sbytes;
                if (!warp_wait(sbar + d * 8, (jb / kStages) & 1, status)) {
                    // drain this warp's copies in flight, then stop
                    if (lane == 0) {
                        for (int jj = j; jj < nrows && jj < j + kStages; ++jj) {
                            const int dd = jj % kStages;
                            const uint32_t par = (jj / kStages) & 1;
                            const unsigned long long t0 = tc::globaltimer();
                            while (!tc::mbar_try(sbar + dd * 8, par) &&
                                   tc::globaltimer() - t0 < tc::kWaitNs) {
                            }
                        }
                    }
                    __syncwarp();
                    return;
                }
                float y = 0.f;
#pragma unroll
                for (int q = 0; q < C; ++q) {
                    const int i = lane + 32 * q;
                    const int ic = i < KW ? i : KW - 1;
                    if (!W4_CHECK(in_range(st + ic * 16, 16, st, cbytes) &&
                                      in_range(st + cbytes + (ic >> 2) * 4, 4, st + cbytes, gbytes) &&
                                      (!asym || in_range(st + cbytes + gbytes + (ic >> 2) * 4, 4,
                                                         st + cbytes + gbytes, gbytes)) &&
                                      in_range(st, sbytes, sx, dyn_smem_bytes()),
                                  status))
                        continue;  // per-lane work only: no collective until reduce4
                    const uint4 cw = lds128(st + ic * 16);
                    const float sc = lds32f(st + cbytes + (ic >> 2) * 4);
                    const float zc = asym ? lds32f(st + cbytes + gbytes + (ic >> 2) * 4) : 8.f;
                    float a = -T[q], b = 0.f;
                    slice_dot<XT>(cw, xr[q], a, b);
                    float v = XT == W4_F16 ? fmaf(b, 0.0625f, a) : a + b;
                    v = fmaf(-zc, S[q], v);
                    y = fmaf(sc, v, y);
                }
                // every lane has used its reads of the stage: refill it
                __syncwarp();
                if (lane == 0 && j + kStages < nrows) {
                    tc::fence_proxy_async();
                    issue(j + kStages, d);
                }
                part[t] = y;
            }
        }
        const float r = reduce4(part, lane);
        const int t = (lane >> 3) & 3;
        if ((lane & 7) == 0 && jb + t < nrows &&
            W4_CHECK(row_of(jb + t) >= 0 && row_of(jb + t) < N, status))
            Y[row_of(jb + t)] = narrow1<XT>(r);
    }
}

template <int XT, int C>
int launch_t(const uint8_t *packed, const float *scales, const float *zeros, const void *X,
             void *Y, int K, int N, int grid, size_t smem, cudaStream_t stream) {
    auto kern = gemv1_kernel<XT, C>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(W4_ERR_CUDA, "cudaGetDevice", nullptr);
    static bool attr_done[64] = {};
    if (!attr_done[dev]) {
        // the largest configuration (K = 4096, asymmetric)
        const size_t most = static_cast<size_t>(kMaxK) * 2 +
                            static_cast<size_t>(kWarps) * kStages * (stage_bytes_for(kMaxK, true) + 8);
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(gemv1 smem)", e);
        attr_done[dev] = true;
    }
    unsigned *status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, packed, scales, zeros,
                                       static_cast<const uint16_t *>(X), static_cast<uint16_t *>(Y),
                                       K, N, status);
    if (e != cudaSuccess) return cuda_fail("cudaLaunchKernelEx(gemv1)", e);
    return W4_OK;
}

}  // namespace

bool gemv1_supported(int64_t M, int64_t K) {
    return M == 1 && K % 512 == 0 && K >= 512 && K <= kMaxK;
}

int launch_gemv1(const void *X, int xt, const uint8_t *packed, const float *scales,
                const float *zeros, int64_t K, int64_t N, void *Y, cudaStream_t stream) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    if (di.cc_major != 10) return set_error(W4_ERR_UNSUPPORTED, "w4a16_gemm", "needs an sm_100 GPU");
    const int k = static_cast<int>(K), n = static_cast<int>(N);
    const int64_t most = static_cast<int64_t>(kCtasPerSm) * di.sm_count;
    const int grid = static_cast<int>(N < most ? N : most);
    const size_t smem = static_cast<size_t>(k) * 2 +
                        static_cast<size_t>(kWarps) * kStages * (stage_bytes_for(k, zeros != nullptr) + 8);
    const int C = (k + 1023) / 1024;
#define W4_GEMV_CASE(XTV, CV)                                                                  \
    if (xt == XTV && C == CV)                                                                  \
        return launch_t<XTV, CV>(packed, scales, zeros, X, Y, k, n, grid, smem, stream);
    W4_GEMV_CASE(W4_F16, 1)
    W4_GEMV_CASE(W4_F16, 2)
    W4_GEMV_CASE(W4_F16, 3)
    W4_GEMV_CASE(W4_F16, 4)
    W4_GEMV_CASE(W4_BF16, 1)
    W4_GEMV_CASE(W4_BF16, 2)
    W4_GEMV_CASE(W4_BF16, 3)
    W4_GEMV_CASE(W4_BF16, 4)
#undef W4_GEMV_CASE
    return set_error(W4_ERR_UNSUPPORTED, "w4a16_gemm", "gemv1 shape");
}

}  // namespace w4
