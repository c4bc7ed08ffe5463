// w4_prefill.cu -- the W4A16 linear layer for large M (prefill) on the
// 5th-generation tensor cores of B200 (tcgen05, TMEM, TMA).
//
// Y[m][n] = sum_g scale[n][g] * sum_{k in g} X[m][k] * (u[n][k] - zero[n][g]):
// "dequant -> 16-bit matmul" ("Quantization method families",
// inference-learning-path.pages.dev, §2), dequantization as in "LLM
// quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2-§2.3.
//
// Tile: 128 weight rows (n) x 256 activation rows (m) per CTA, persistent
// over all tiles.  The MMA runs "swap-AB": the dequantized weights are the
// M = 128 operand A and X is the N = 256 operand B, so the accumulator in
// tensor memory holds D[n][m] with one weight row per TMEM lane.  That makes
// each group's scale a single scalar per epilogue thread.
//
// Exactness: the A operand holds (u - zero), an integer in [-15, 15] that is
// exact in bf16/fp16; tcgen05.mma accumulates each 128-wide group into an
// fp32 partial in TMEM, and the epilogue adds scale * partial into fp32
// registers.  No weight is rounded to 16 bits.
//
// Warp roles (512 threads, four warpgroups):
//   warp 0       TMA producer: X tile (256 x 64, 128B swizzle) and the packed
//                codes of 128 rows x 64 k into a 4-stage shared-memory ring.
//   warp 1       TMEM allocator and MMA issuer (one thread): 4 x
//                tcgen05.mma.kind::f16 (128 x 256 x 16) per stage into the
//                group's partial buffer P[b] (2 x 256 TMEM columns).
//   warps 2, 3   no role (they only give their registers back).
//   warps 4..7   dequantize: thread t writes row t of each stage's A tile
//                (the bf16/fp16 values of 64 k, 128B-swizzled K-major, the
//                layout the MMA descriptor names), as soon as the stage's
//                codes have landed -- up to the whole ring ahead of the MMAs.
//   warps 8..15  fold: per group, read P[b] with tcgen05.ld and accumulate
//                acc += scale * P into registers (two warps per TMEM lane
//                quarter, 128 columns each).  After the last group of a tile
//                they round acc to the output dtype and store Y.
// Dequantization and folding are separate warps so that the A tile of group
// g + 2 never waits for the fold of group g.
//
// Registers: the CTA is launched with 128 a thread (512 x 128 = the SM's 64K);
// warpgroups 0 and 1 give back to 88 and warpgroups 2 and 3 (the fold warps,
// which keep 128 fp32 accumulators) take 168: 2 x 128 x 88 + 2 x 128 x 168 =
// 65536, exactly what the CTA was launched with.
//
// Every wait on an mbarrier is bounded (kWaitNs); a wait that runs out sets
// the library's device status word to W4_ERR_TIMEOUT and a shared abort
// flag, every role then leaves its loop, the producer and the MMA issuer
// wait (bounded) for their copies / MMAs in flight, and TMEM is freed before
// the CTA exits.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <stdio.h>


#include "w4_debug.cuh"
#include "w4_internal.cuh"
#include "w4_tc.cuh"

namespace w4 {
namespace {

[[maybe_unused]] constexpr unsigned kDbgFile = 3;  // W4_DEBUG file id

constexpr int kBM = 128;       // weight rows per tile (MMA M)
constexpr int kBN = 256;       // activation rows per tile (MMA N)
constexpr int kBK = 64;        // k per pipeline stage (one 128-byte swizzle row of 16-bit)
constexpr int kStages = 4;
constexpr int kGroup = 128;
constexpr int kFoldWarps = 8;
constexpr int kThreads = 512;
constexpr int kDequantWarp0 = 4;
constexpr int kFoldWarp0 = 8;
constexpr int kTmemCols = 512;                  // 2 partial buffers x 256 columns

constexpr int kXTileBytes = kBN * kBK * 2;      // 32 KB
constexpr int kATileBytes = kBM * kBK * 2;      // 16 KB
constexpr int kCodeTileBytes = kBM * kBK / 2;   // 4 KB
constexpr int kStageBytes = kXTileBytes + kATileBytes + kCodeTileBytes;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

using namespace tc;

// kind::f16 instruction descriptor: D f32, A/B bf16 (or f16), both K-major.
template <int XT>
__host__ __device__ constexpr uint32_t instr_desc() {
    return (1u << 4)                                  // D format f32
           | ((XT == W4_BF16 ? 1u : 0u) << 7)         // A format
           | ((XT == W4_BF16 ? 1u : 0u) << 10)        // B format
           | (static_cast<uint32_t>(kBN >> 3) << 17)  // N
           | (static_cast<uint32_t>(kBM >> 4) << 24); // M
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}


// ---- dequantization of one packed word into the A tile ------------------------------

// Four registers holding the exact pairs (u - z) of k = {0,1},{2,3},{4,5},{6,7}.
// zb = {bias+z, bias+z} in the operand type; for fp16 zq = {-(64+z), -(64+z)}.
template <int XT>
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t zb, uint32_t zq) {
    uint32_t p[4];
    if (XT == W4_F16) {
        const uint32_t magic = 0x64006400u;      // {1024, 1024}
        const uint32_t sixteenth = 0x2C002C00u;  // {1/16, 1/16}
        const uint32_t lo0 = (w & 0x000F000Fu) | magic;
        const uint32_t hi0 = (w & 0x00F000F0u) | magic;
        const uint32_t w8 = w >> 8;
        const uint32_t lo1 = (w8 & 0x000F000Fu) | magic;
        const uint32_t hi1 = (w8 & 0x00F000F0u) | magic;
        asm("sub.f16x2 %0, %1, %2;" : "=r"(p[0]) : "r"(lo0), "r"(zb));
        asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[1]) : "r"(hi0), "r"(sixteenth), "r"(zq));
        asm("sub.f16x2 %0, %1, %2;" : "=r"(p[2]) : "r"(lo1), "r"(zb));
        asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[3]) : "r"(hi1), "r"(sixteenth), "r"(zq));
    } else {
        const uint32_t magic = 0x43004300u;  // {128, 128} in bf16
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | magic;
            asm("sub.bf16x2 %0, %1, %2;" : "=r"(p[i]) : "r"(v), "r"(zb));
        }
    }
    return make_uint4(p[0], p[1], p[2], p[3]);
}

template <int XT>
__device__ __forceinline__ void zero_bias(float z, uint32_t &zb, uint32_t &zq) {
    if (XT == W4_F16) {
        __half2 a = __float2half2_rn(1024.0f + z);
        __half2 b = __float2half2_rn(-(64.0f + z));
        zb = *reinterpret_cast<uint32_t *>(&a);
        zq = *reinterpret_cast<uint32_t *>(&b);
    } else {
        __nv_bfloat162 a = __float2bfloat162_rn(128.0f + z);
        zb = *reinterpret_cast<uint32_t *>(&a);
        zq = 0;
    }
}

template <int XT>
__device__ __forceinline__ void store_y(void *Y, int64_t idx, float v) {
    if (XT == W4_F16)
        reinterpret_cast<__half *>(Y)[idx] = __float2half_rn(v);
    else
        reinterpret_cast<__nv_bfloat16 *>(Y)[idx] = __float2bfloat16_rn(v);
}

struct Smem {
    uint64_t full[kStages];    // TMA bytes of X + codes landed
    uint64_t empty[kStages];   // MMAs of the stage done (stage may be refilled)
    uint64_t aready[kStages];  // dequantized A tile written
    uint64_t pfull[2];         // group partial P[b] complete in TMEM
    uint64_t pempty[2];        // P[b] read by the epilogue
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Smem) <= 256, "the barrier area of kSmemBytes");

// Dequantizes the two stages of group g of the current tile (stage counter
// base `it`) for this thread's A-tile row dr: waits for the codes, writes the
// row's 8 swizzled 16-byte chunks per stage, fences them for the tensor core
// and arrives on the stage's A-ready barrier.
template <int XT>
__device__ __forceinline__ bool dequant_group(int g, uint32_t it, int n_d, int G,
                                              const float *__restrict__ zeros, const uint8_t *cs,
                                              uint8_t *as, int dr, Smem *sm,
                                              volatile int *abort_flag, unsigned *status) {
    if (!W4_CHECK_WARP(n_d >= 0 && g >= 0 && g < G, status)) return false;
    const float z = zeros ? __ldg(zeros + (int64_t)n_d * G + g) : 8.0f;
    uint32_t zb, zq;
    zero_bias<XT>(z, zb, zq);
#pragma unroll
    for (int h = 0; h < kGroup / kBK; ++h) {
        const uint32_t j = it + (uint32_t)(g * (kGroup / kBK) + h);
        const int s = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        // warp-uniform outcome: the warp either goes on together or leaves together
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm->full[s]), ph, abort_flag, status)))
            return false;
        const uint8_t *crow = cs + s * kCodeTileBytes + dr * (kBK / 2);
        if (!W4_CHECK_WARP(in_range(smem_u32(crow), kBK / 2, smem_u32(cs), uint64_t(kStages) * kCodeTileBytes) &&
                               in_range(smem_u32(as + s * kATileBytes + dr * 128), 128, smem_u32(as),
                                        uint64_t(kStages) * kATileBytes),
                           status))
            return false;
        const uint4 w0 = *reinterpret_cast<const uint4 *>(crow);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(crow + 16);
        uint8_t *arow = as + s * kATileBytes + dr * 128;
        const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const int chunk = jj ^ (dr & 7);
            *reinterpret_cast<uint4 *>(arow + chunk * 16) = dequant_word<XT>(ws[jj], zb, zq);
        }
        fence_proxy_async();
        mbar_arrive(smem_u32(&sm->aready[s]));
    }
    return true;
}

template <int XT>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               const float *__restrict__ scales, const float *__restrict__ zeros, int M, int N,
               int K, void *__restrict__ Y, unsigned *__restrict__ status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned stage ring, then the barriers
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *xs = base;                                // kStages x 32 KB
    uint8_t *as = base + kStages * kXTileBytes;        // kStages x 16 KB
    uint8_t *cs = as + kStages * kATileBytes;          // kStages x 4 KB
    Smem *sm = reinterpret_cast<Smem *>(cs + kStages * kCodeTileBytes);
    volatile int *abort_flag = &sm->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = K / kGroup;
    const int n_tiles = (N + kBM - 1) / kBM;
    const int m_tiles = (M + kBN - 1) / kBN;
    const int tiles = n_tiles * m_tiles;
    const int kstages_per_tile = K / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&sm->full[s]), 1);
            mbar_init(smem_u32(&sm->empty[s]), 1);
            mbar_init(smem_u32(&sm->aready[s]), kBM);  // one dequant thread per row
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm->pfull[b]), 1);
            mbar_init(smem_u32(&sm->pempty[b]), 32 * kFoldWarps);
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

    // Register split (see the header): each warpgroup's branch starts with its
    // setmaxnreg, executed by all four of its warps.
    if (warp < 4) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
      if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int nt = tile % n_tiles, mt = tile / n_tiles;
                for (int ks = 0; ks < kstages_per_tile; ++ks, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(smem_u32(&sm->empty[s]), ph ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&sm->full[s]);
                    // W4_DEBUG: 16-byte aligned box starts inside the tensors, and the
                    // stage ring (then the barriers) inside this launch's shared memory
                    if (!W4_CHECK((ks * kBK) % 8 == 0 && ks * kBK < K && mt * kBN < M &&
                                      (ks * (kBK / 2)) % 16 == 0 && nt * kBM < N &&
                                      in_range(smem_u32(sm), sizeof(Smem), smem_u32(smem_raw),
                                               dyn_smem_bytes()),
                                  status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_tx(fb, kXTileBytes + kCodeTileBytes);
                    tma_load_2d(smem_u32(xs + s * kXTileBytes), &tmap_x, ks * kBK, mt * kBN, fb);
                    tma_load_2d(smem_u32(cs + s * kCodeTileBytes), &tmap_w, ks * (kBK / 2),
                                nt * kBM, fb);
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
        __syncwarp();  // the whole warp reconverges before the CTA barrier
      } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc<XT>();
            uint32_t it = 0, gc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                for (int g = 0; g < G && ok; ++g, ++gc) {
                    const int b = gc & 1;
                    const uint32_t pph = (gc >> 1) & 1;
                    if (!mbar_wait(smem_u32(&sm->pempty[b]), pph ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dcol = tmem + b * kBN;
                    for (int h = 0; h < kGroup / kBK; ++h, ++it) {
                        const int s = it % kStages;
                        const uint32_t ph = (it / kStages) & 1;
                        if (!mbar_wait(smem_u32(&sm->full[s]), ph, abort_flag, status) ||
                            !mbar_wait(smem_u32(&sm->aready[s]), ph, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(as + s * kATileBytes);
                        const uint32_t b0 = smem_u32(xs + s * kXTileBytes);
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            // advance 16 elements (32 bytes) inside the swizzle row
                            mma_f16(dcol, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                                    (h > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(smem_u32(&sm->empty[s]));
                    }
                    if (ok) mma_commit(smem_u32(&sm->pfull[gc & 1]));
                }
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
        __syncwarp();  // the whole warp reconverges before the CTA barrier
      }
    } else if (warp < kFoldWarp0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 88;" ::: "memory");
        // ---------------- dequantize: thread = A-tile row ----------------
        const int dr = threadIdx.x - 32 * kDequantWarp0;  // 0..127
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int nt = tile % n_tiles;
            const int n_d = min(nt * kBM + dr, N - 1);  // clamped: rows past N are never stored
            bool ok = true;
            for (int g = 0; g < G && ok; ++g)
                ok = dequant_group<XT>(g, it, n_d, G, zeros, cs, as, dr, sm, abort_flag, status);
            if (!ok) break;
            it += (uint32_t)kstages_per_tile;
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 168;" ::: "memory");
        // ---------------- fold + epilogue ----------------
        const int fw = warp - kFoldWarp0;  // 0..7
        const int q = warp & 3;            // TMEM lane quarter this warp may access
        const int colhalf = fw >> 2;       // 0: columns 0..127, 1: 128..255
        const int er = 32 * q + lane;      // TMEM lane = weight row of the tile

        float acc[128];
        uint32_t gc = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            const int nt = tile % n_tiles, mt = tile / n_tiles;
            const int n_e = nt * kBM + er;
            const int n_ec = min(n_e, N - 1);
            if (!W4_CHECK_WARP(n_ec >= 0 && G >= 1, status)) break;
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            float s_next = __ldg(scales + (int64_t)n_ec * G + 0);
            for (int g = 0; g < G; ++g, ++gc) {
                const float sg = s_next;
                if (g + 1 < G) s_next = __ldg(scales + (int64_t)n_ec * G + g + 1);
                const int b = gc & 1;
                const uint32_t pph = (gc >> 1) & 1;
                if (!__all_sync(0xffffffffu,
                                mbar_wait(smem_u32(&sm->pfull[b]), pph, abort_flag, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) +
                                       static_cast<uint32_t>(b * kBN + colhalf * 128);
                // two 16-column loads in flight per wait
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    uint32_t r0[16], r1[16];
                    tmem_ld16(taddr + 16 * c, r0);
                    tmem_ld16(taddr + 16 * (c + 1), r1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        acc[16 * c + i] = fmaf(sg, __uint_as_float(r0[i]), acc[16 * c + i]);
                        acc[16 * (c + 1) + i] = fmaf(sg, __uint_as_float(r1[i]), acc[16 * (c + 1) + i]);
                    }
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&sm->pempty[b]));
            }
            if (!ok) break;
            // store this thread's row n_e for its 128 columns m
            if (n_e < N && W4_CHECK(n_e >= 0 && mt * kBN < M, status)) {
                const int m0 = mt * kBN + colhalf * 128;
#pragma unroll
                for (int i = 0; i < 128; ++i) {
                    const int m = m0 + i;
                    if (m < M) store_y<XT>(Y, (int64_t)m * N + n_e, acc[i]);
                }
            }
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

// ---- host side --------------------------------------------------------------------------

template <int XT>
int launch_t(const void *X, int64_t M, const uint8_t *packed, const float *scales,
             const float *zeros, int64_t K, int64_t N, void *Y, cudaStream_t stream) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    if (di.cc_major != 10)
        return set_error(W4_ERR_UNSUPPORTED, "w4a16_gemm (M > 32)", "needs an sm_100 GPU");
    if (di.max_smem_optin < kSmemBytes)
        return set_error(W4_ERR_UNSUPPORTED, "w4a16_gemm (M > 32)", "not enough shared memory");
    unsigned *status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    CUtensorMap mx, mw;
    if ((st = make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT16, X, (uint64_t)K, (uint64_t)M,
                          (uint64_t)K * 2, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B, "tensor map of X")) !=
        W4_OK)
        return st;
    if ((st = make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)K / 2, (uint64_t)N,
                          (uint64_t)K / 2, kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_NONE,
                          "tensor map of packed")) != W4_OK)
        return st;
    auto kern = prefill_kernel<XT>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(W4_ERR_CUDA, "cudaGetDevice", nullptr);
    static bool attr_done[64][2] = {};
    if (!attr_done[dev][XT]) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(prefill smem)", e);
        attr_done[dev][XT] = true;
    }
    static int threads_ok[64][2] = {};
    if (!threads_ok[dev][XT]) {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return cuda_fail("cudaFuncGetAttributes(prefill)", e);
        if (fa.maxThreadsPerBlock < kThreads) {
            char buf[96];
            snprintf(buf, sizeof buf, "%d registers per thread allow only %d threads", fa.numRegs,
                     fa.maxThreadsPerBlock);
            return set_error(W4_ERR_CUDA, "prefill kernel resources", buf);
        }
        threads_ok[dev][XT] = 1;
    }
    const int64_t tiles = ((N + kBM - 1) / kBM) * ((M + kBN - 1) / kBN);
    const int grid = (int)(tiles < di.sm_count ? tiles : di.sm_count);
    kern<<<grid, kThreads, kSmemBytes, stream>>>(mx, mw, scales, zeros, (int)M, (int)N, (int)K, Y,
                                                 status);
    return cuda_status(cudaGetLastError());
}

}  // namespace

int launch_prefill(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                   const float *zeros, int64_t K, int64_t N, void *Y, cudaStream_t stream) {
    if (xt == W4_F16) return launch_t<W4_F16>(X, M, packed, scales, zeros, K, N, Y, stream);
    return launch_t<W4_BF16>(X, M, packed, scales, zeros, K, N, Y, stream);
}

}  // namespace w4
