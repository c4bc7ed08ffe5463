// w4_decode.cu -- the W4A16 linear layer for small M (decode, M <= 32).
//
// Y[m][n] = sum_g scale[n][g] * sum_{k in g} X[m][k] * (u[n][k] - zero[n][g]):
// the "dequant -> 16-bit matmul" of W4A16 ("Quantization method families",
// inference-learning-path.pages.dev, §2), dequantization as in "LLM
// quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2-§2.3.  At small M the layer is
// bound by streaming the packed weights from HBM, so the kernel is built to
// keep HBM busy from the first cycle to the last and to spend as few issue
// slots per weight as possible:
//
//   * Persistent, one CTA per SM.  The packed matrix is cut into units of
//     128 weight rows x 256 k (16 KB of codes, two groups).  The units, in
//     row-block-major order, are split into equal contiguous ranges, one per
//     CTA ("stream-K"): every SM streams the same number of bytes.
//   * Warp 0 streams each unit into a shared-memory ring: the codes and the
//     unit's X slice with TMA (128-byte swizzle), the unit's scales and zero
//     points with cp.async from its 32 lanes; one mbarrier covers all three.
//   * Tensor cores (tcgen05): two warpgroups, one per group of the unit, and
//     one thread per weight row (= TMEM lane).  Each thread dequantizes its
//     row's 128 codes into the exact integers (u - zero), 16 at a time, and
//     stores them with tcgen05.st into tensor memory, where they form the A
//     operand (M = 128 rows) of tcgen05.mma.kind::f16; B is the X slice in
//     shared memory (N = 16 or 32 columns of X rows, zero past M).  The MMA
//     of each group goes to its own fp32 partial in TMEM; the same thread then
//     reads its row of that partial (tcgen05.ld) and adds scale * partial to
//     its fp32 accumulators.  No weight is rounded to 16 bits: (u - zero) is an
//     integer in [-15, 15], exact in fp16/bf16.
//   * Warp 1 allocates TMEM and issues the MMAs (one thread).
//   * A row block whose units all fall in one CTA's range is written to Y
//     directly (the two warpgroups add their halves through shared memory).
//     A row block split between CTAs: each warp stores its partial (32 rows)
//     to its CTA's slot in the caller's workspace, and after its last unit
//     arrives on a (row block, warp) counter; the last warp to arrive adds the
//     slots in CTA order, writes Y and re-arms the counter (deterministic).
//   * Programmatic dependent launch: the kernel may start while the preceding
//     kernel of the stream finishes; the first ring of packed codes is
//     requested at once, everything else (X, scales, zeros, Y, workspace) is
//     touched only after griddepcontrol.wait.
//
// Every mbarrier wait is bounded; a wait that runs out sets the library's
// status word (W4_ERR_TIMEOUT) and an abort flag, every role leaves its loop,
// the producer and the MMA issuer wait (bounded) for their copies and MMAs in
// flight, and TMEM is freed before the CTA exits.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdio.h>

#include "w4_internal.cuh"

namespace w4 {
namespace {

constexpr int kGroup = 128;
constexpr int kUnitRows = 128;                      // weight rows per unit (= TMEM lanes)
constexpr int kUnitK = 256;                         // k per unit: two groups, 128 bytes per row
constexpr int kUnitBytes = kUnitRows * kUnitK / 2;  // 16 KB of codes
constexpr int kSZBytes = kUnitRows * 2 * 4;         // scales (or zeros) of a unit: [128][2] fp32
constexpr int kThreads = 320;                       // producer, MMA, two dequant warpgroups
constexpr int kTmemCols = 512;
// TMEM columns: A operand [group][buffer] 64 columns each (128 k of 16-bit
// pairs), then the fp32 partials [group][buffer] of N columns each.
constexpr int kAColsPerGroup = 64;
constexpr int kDBase = 256;
// Workspace: arrival counters (one per row block and 32-row warp) first,
// then two partial slots per CTA ([2 * ctas][128 rows][M] fp32).  The counter
// area is fixed so that one workspace serves calls of any shape; row-block
// counts beyond it switch to whole-row-block ranges, which need no workspace.
constexpr int kMaxRowBlocks = 2048;
constexpr int kMaxCounters = kMaxRowBlocks * 8;
constexpr size_t kCounterBytes = kMaxCounters * sizeof(unsigned);
constexpr unsigned long long kWaitNs = 2000000000ull;

// ---- PTX wrappers -------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: true once the phase with `parity` has completed; false if the
// CTA aborted or the wait ran out (then the abort flag and status are set).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned *status) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitNs) {
            *abort_flag = 1;
            atomicOr(status, 1u);
            return false;
        }
    }
}

// The same, with one outcome for the whole warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned *status) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status));
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// The mbarrier gets one arrival once all of this thread's cp.async copies landed.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand, 128-byte swizzle, 128-byte rows, 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFF) >> 4);  // start address
    d |= static_cast<uint64_t>(1) << 16;                 // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;         // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                 // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                 // SWIZZLE_128B
    return d;
}

// kind::f16 instruction descriptor: D f32, A and B of type XT, K-major, M = 128.
template <int XT, int NN>
__host__ __device__ constexpr uint32_t instr_desc() {
    return (1u << 4) | ((XT == W4_BF16 ? 1u : 0u) << 7) | ((XT == W4_BF16 ? 1u : 0u) << 10) |
           (static_cast<uint32_t>(NN >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// D[128 x NN] (+)= A[128 x 16] (TMEM) * B[NN x 16]^T (shared memory)
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
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

// ---- dequantization -----------------------------------------------------------------------

// Biased zero point in the operand type, from integer ops: z is an integer
// 0..15, and 1024 + z (fp16), 128 + z (bf16) and 64 + z (fp16, mantissa step
// 1/16) are exact with z in the low mantissa bits.
// fp16: zb = {1024+z, 1024+z}, zq = {-(64+z), -(64+z)}; bf16: zb = {128+z, 128+z}.
template <int XT>
__device__ __forceinline__ void zero_bias(float z, uint32_t &zb, uint32_t &zq) {
    const uint32_t zi = static_cast<uint32_t>(__float2int_rn(z));
    if (XT == W4_F16) {
        zb = (0x6400u + zi) * 0x10001u;
        zq = (0xD400u + (zi << 4)) * 0x10001u;
    } else {
        zb = (0x4300u + zi) * 0x10001u;
        zq = 0;
    }
}

// One packed word (k = 8j..8j+7 of a row) -> four registers holding the exact
// pairs (u - z) of k = {0,1}, {2,3}, {4,5}, {6,7} (low half = even k).  The
// packed layout keeps k = 8j+{2i, 2i+1} in nibbles i and i+4 of the word.
template <int XT>
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t zb, uint32_t zq, uint32_t *p) {
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
}

template <int XT>
__device__ __forceinline__ void store_out(void *Y, int64_t idx, float v) {
    if (XT == W4_F16)
        reinterpret_cast<__half *>(Y)[idx] = __float2half_rn(v);
    else
        reinterpret_cast<__nv_bfloat16 *>(Y)[idx] = __float2bfloat16_rn(v);
}

// ---- work split ---------------------------------------------------------------------------

struct Work {
    int U;       // units in total
    int KS;      // units per row block
    int G;       // groups per row
    int RB;      // row blocks
    int P;       // CTAs
    int aligned; // 1: ranges are whole row blocks (no partials)
};

__host__ __device__ inline int range_start(const Work &w, int c) {
    if (w.aligned) return (int)((int64_t)c * w.RB / w.P) * w.KS;
    return (int)((int64_t)c * w.U / w.P);
}

// CTA whose range holds unit u (stream-K ranges only).
__device__ __forceinline__ int owner(const Work &w, int u) {
    return (int)(((int64_t)(u + 1) * w.P - 1) / w.U);
}

// ---- kernel -------------------------------------------------------------------------------

// NN: MMA N (16 or 32) = X rows staged per unit (rows >= M are zero).
// Stage: codes [128][128 B] (swizzled) | X: four 64-k boxes [NN][128 B]
// (swizzled) | scales [128][2] | zeros [128][2].
template <int NN>
struct Cfg {
    static constexpr int kXBox = NN * 128;
    static constexpr int kSZ = kUnitBytes + 4 * kXBox;
    static constexpr int kBytes = kSZ + 2 * kSZBytes;
    static constexpr int kTmaBytes = kUnitBytes + 4 * kXBox;
    static constexpr int kStages = (176 * 1024) / kBytes < 8 ? (176 * 1024) / kBytes : 8;
    static constexpr int kXchg = kUnitRows * NN * 4;  // second warpgroup's half at a flush
    static constexpr int kSmem = kStages * kBytes + 1024 + 512 + kXchg;
};

struct Shared {
    uint64_t full[8];      // codes + X (TMA bytes) and scales/zeros (cp.async) landed
    uint64_t empty[8];     // both groups' MMAs of the stage done
    uint64_t afull[2][2];  // [group][buffer] A operand stored in TMEM (128 threads)
    uint64_t afree[2][2];  // its MMAs done (commit)
    uint64_t dfull[2][2];  // [group][buffer] partial complete (commit)
    uint64_t dfree[2][2];  // partial read (128 threads)
    uint64_t xfull, xfree; // warpgroup 1 -> 0 exchange at a flush (128 threads each)
    uint32_t tmem_base;
    int abort_flag;
};

template <int XT, int NN>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
              int M, const float *__restrict__ scales, const float *__restrict__ zeros, int K, int N,
              void *__restrict__ Y, unsigned *__restrict__ counters, float *__restrict__ partial,
              const Work wk, unsigned *__restrict__ status) {
    using C = Cfg<NN>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    Shared *sh = reinterpret_cast<Shared *>(ring + S * C::kBytes);
    float *xchg = reinterpret_cast<float *>(ring + S * C::kBytes + 512);
    volatile int *abort_flag = &sh->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int u0 = range_start(wk, c);
    const int u1 = range_start(wk, c + 1);
    const int G = wk.G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&sh->full[s]), 1 + 32);  // TMA arrive_tx + 32 cp.async arrivals
            mbar_init(smem_u32(&sh->empty[s]), 1);
        }
        for (int h = 0; h < 2; ++h)
            for (int b = 0; b < 2; ++b) {
                mbar_init(smem_u32(&sh->afull[h][b]), 128);
                mbar_init(smem_u32(&sh->afree[h][b]), 1);
                mbar_init(smem_u32(&sh->dfull[h][b]), 1);
                mbar_init(smem_u32(&sh->dfree[h][b]), 128);
            }
        mbar_init(smem_u32(&sh->xfull), 128);
        mbar_init(smem_u32(&sh->xfree), 128);
        sh->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh->tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    // let the next kernel in the stream start its prologue as SMs free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // ---------------- producer ----------------
        // Codes and X by TMA (lane 0), the unit's scales and zero points by
        // cp.async (four rows per lane); every lane arrives on the stage's full
        // barrier once its copies have landed.
        auto issue_sz = [&](int u, uint8_t *st, uint32_t fb) {
            const int rb = u / wk.KS, ks = u % wk.KS;
            const int g0 = 2 * ks, g1 = min(2 * ks + 1, G - 1);
            float *ss = reinterpret_cast<float *>(st + C::kSZ);
            float *zz = ss + 2 * kUnitRows;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = lane + 32 * q;
                const int64_t n = min(rb * kUnitRows + r, N - 1);
                cp_async4(smem_u32(ss + 2 * r), scales + n * G + g0);
                cp_async4(smem_u32(ss + 2 * r + 1), scales + n * G + g1);
                if (zeros) {
                    cp_async4(smem_u32(zz + 2 * r), zeros + n * G + g0);
                    cp_async4(smem_u32(zz + 2 * r + 1), zeros + n * G + g1);
                }
            }
            cp_async_arrive(fb);
        };
        auto issue_x = [&](int u, uint8_t *st, uint32_t fb) {
            const int ks = u % wk.KS;
#pragma unroll
            for (int b = 0; b < 4; ++b)
                tma_load_2d(smem_u32(st + kUnitBytes + b * C::kXBox), &tmap_x, ks * kUnitK + 64 * b, 0,
                            fb);
        };
        // The packed weights are inputs no earlier kernel writes: the first ring
        // of codes is requested before waiting for the preceding kernel.
        const int pre = min(S, u1 - u0);
        if (lane == 0) {
            for (int it = 0; it < pre; ++it) {
                const int u = u0 + it;
                const uint32_t fb = smem_u32(&sh->full[it]);
                mbar_arrive_tx(fb, C::kTmaBytes);
                tma_load_2d(smem_u32(ring + it * C::kBytes), &tmap_w, (u % wk.KS) * (kUnitK / 2),
                            (u / wk.KS) * kUnitRows, fb);
            }
        }
        __syncwarp();
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int it = 0; it < pre; ++it) {
            uint8_t *st = ring + it * C::kBytes;
            const uint32_t fb = smem_u32(&sh->full[it]);
            if (lane == 0) issue_x(u0 + it, st, fb);
            issue_sz(u0 + it, st, fb);
        }
        int u = u0 + pre;
        for (; u < u1; ++u) {
            const int it = u - u0;
            const int s = it % S;
            const uint32_t ph = (it / S) & 1;
            if (!warp_wait(smem_u32(&sh->empty[s]), ph ^ 1, abort_flag, status)) break;
            uint8_t *st = ring + s * C::kBytes;
            const uint32_t fb = smem_u32(&sh->full[s]);
            if (lane == 0) {
                mbar_arrive_tx(fb, C::kTmaBytes);
                tma_load_2d(smem_u32(st), &tmap_w, (u % wk.KS) * (kUnitK / 2), (u / wk.KS) * kUnitRows,
                            fb);
                issue_x(u, st, fb);
            }
            issue_sz(u, st, fb);
        }
        // wait (bounded) for the copies still in flight before the CTA may exit
        if (lane == 0) {
            for (int j = (u - u0 > S ? u - u0 - S : 0); j < u - u0; ++j) {
                const unsigned long long t0 = globaltimer();
                while (!mbar_try(smem_u32(&sh->full[j % S]), (j / S) & 1) &&
                       globaltimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc<XT, NN>();
            uint32_t n_mma[2] = {0, 0};  // group MMAs issued, per warpgroup
            bool ok = true;
            int u = u0;
            for (; u < u1 && ok; ++u) {
                const int it = u - u0;
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                const int ks = u % wk.KS;
                if (!mbar_wait(smem_u32(&sh->full[s]), ph, abort_flag, status)) break;
                const uint32_t xs = smem_u32(ring + s * C::kBytes + kUnitBytes);
                for (int h = 0; h < 2; ++h) {
                    if (2 * ks + h >= G) break;  // a last unit with one group
                    const uint32_t b = n_mma[h] & 1, pb = (n_mma[h] >> 1) & 1;
                    if (!mbar_wait(smem_u32(&sh->afull[h][b]), pb, abort_flag, status) ||
                        !mbar_wait(smem_u32(&sh->dfree[h][b]), pb ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ta = tmem + (uint32_t)((2 * h + b) * kAColsPerGroup);
                    const uint32_t td = tmem + (uint32_t)(kDBase + (2 * h + b) * NN);
#pragma unroll
                    for (int kb = 0; kb < 8; ++kb) {
                        // X box 2h + kb/4, 16 k (32 bytes) per step inside the swizzle row
                        const uint32_t xa = xs + (2 * h + kb / 4) * C::kXBox + (kb % 4) * 32;
                        mma_ts(td, ta + 8 * kb, sw128_desc(xa), idesc, kb > 0 ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&sh->afree[h][b]));
                    mma_commit(smem_u32(&sh->dfull[h][b]));
                    ++n_mma[h];
                }
                if (ok) mma_commit(smem_u32(&sh->empty[s]));
            }
            // drain: wait (bounded) until the last issued MMAs have completed
            if (u > u0) {
                const int j = u - 1 - u0;
                const unsigned long long t0 = globaltimer();
                while (!mbar_try(smem_u32(&sh->empty[j % S]), (j / S) & 1) &&
                       globaltimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else {
        // ---------------- dequant + accumulate: two warpgroups ----------------
        const int h = (warp - 2) >> 2;               // group of each unit this warpgroup owns
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int r = 32 * q + lane;                 // weight row of the unit (= TMEM lane)
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        const int swz = r & 7;
        float acc[NN];
        int cur_rb = -1, first_ks = 0, last_ks = -1;
        uint32_t n_a = 0, n_d = 0, n_x = 0;          // A stores, partials read, exchanges
        int pending[2];
        int npending = 0;
        bool ok = true;

        // Reads this warpgroup's partial of its previous group and adds it.
        auto fold = [&](float sc) -> bool {
            const uint32_t b = n_d & 1, pb = (n_d >> 1) & 1;
            if (!warp_wait(smem_u32(&sh->dfull[h][b]), pb, abort_flag, status)) return false;
            tc_fence_after();
            const uint32_t td = tmem + lanebase + (uint32_t)(kDBase + (2 * h + b) * NN);
#pragma unroll
            for (int cc = 0; cc < NN / 16; ++cc) {
                uint32_t v[16];
                tmem_ld16(td + 16 * cc, v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    acc[16 * cc + i] = fmaf(sc, __uint_as_float(v[i]), acc[16 * cc + i]);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sh->dfree[h][b]));
            ++n_d;
            return true;
        };

        // Finishes row block rb for this thread's row: the two warpgroups' halves
        // are added through shared memory, then warpgroup 0 writes Y or stores a
        // partial (arrival and final sum after the loop, finish_partials).
        auto flush = [&](int rb) -> bool {
            const uint32_t px = n_x & 1;
            float *xr = xchg + r * NN;
            if (h == 1) {
                if (!warp_wait(smem_u32(&sh->xfree), px ^ 1, abort_flag, status)) return false;
#pragma unroll
                for (int i = 0; i < NN; ++i) xr[i] = acc[i];
                mbar_arrive(smem_u32(&sh->xfull));
                ++n_x;
                return true;
            }
            if (!warp_wait(smem_u32(&sh->xfull), px, abort_flag, status)) return false;
#pragma unroll
            for (int i = 0; i < NN; ++i) acc[i] += xr[i];
            mbar_arrive(smem_u32(&sh->xfree));
            ++n_x;
            const int n = rb * kUnitRows + r;
            if (first_ks == 0 && last_ks == wk.KS - 1) {
                if (n < N) {
#pragma unroll
                    for (int m = 0; m < NN; ++m)
                        if (m < M) store_out<XT>(Y, (int64_t)m * N + n, acc[m]);
                }
                return true;
            }
            const int slot = 2 * c + (rb == u0 / wk.KS ? 0 : 1);
            float *dst = partial + ((int64_t)slot * kUnitRows + r) * M;
#pragma unroll
            for (int m = 0; m < NN; ++m)
                if (m < M) dst[m] = acc[m];
            pending[npending++] = rb;
            return true;
        };

        // Arrives on the counters of the split row blocks this warp stored; the
        // last warp to arrive on one adds its partials in CTA order.
        auto finish_partials = [&]() {
            if (npending == 0) return;
            __threadfence();
            __syncwarp();
            for (int pi = 0; pi < npending; ++pi) {
                const int rb = pending[pi];
                const int cf = owner(wk, rb * wk.KS), cl = owner(wk, (rb + 1) * wk.KS - 1);
                unsigned *cnt = counters + rb * 8 + q;
                unsigned prev = 0;
                if (lane == 0) prev = atomicAdd(cnt, 1u);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev != (unsigned)(cl - cf)) continue;
                __threadfence();
                const int n = rb * kUnitRows + r;
                if (n < N) {
                    for (int m = 0; m < M; ++m) {
                        float v = 0.0f;
                        for (int cc = cf; cc <= cl; ++cc) {
                            const int sl = 2 * cc + (rb == range_start(wk, cc) / wk.KS ? 0 : 1);
                            v += __ldcg(partial + ((int64_t)sl * kUnitRows + r) * M + m);
                        }
                        store_out<XT>(Y, (int64_t)m * N + n, v);
                    }
                }
                __syncwarp();
                if (lane == 0) *cnt = 0u;  // re-arm for the next call
            }
        };

        asm volatile("griddepcontrol.wait;" ::: "memory");
        float prev_scale = 0.0f;
        bool have_prev = false;  // a partial of this warpgroup waits to be folded
        int rb = u0 / wk.KS;
        int ks = u0 - rb * wk.KS;
        for (int u = u0; u < u1; ++u) {
            const int it = u - u0;
            const int s = it % S;
            const uint32_t ph = (it / S) & 1;
            if (rb != cur_rb) {
                // the previous row block's last partial first, then finish it
                if (have_prev) {
                    if (!fold(prev_scale)) { ok = false; break; }
                    have_prev = false;
                }
                if (cur_rb >= 0 && !flush(cur_rb)) { ok = false; break; }
                cur_rb = rb;
                first_ks = ks;
#pragma unroll
                for (int i = 0; i < NN; ++i) acc[i] = 0.0f;
            }
            last_ks = ks;
            const bool mine = 2 * ks + h < G;  // this unit has a group for this warpgroup
            if (!warp_wait(smem_u32(&sh->full[s]), ph, abort_flag, status)) { ok = false; break; }
            const uint8_t *st = ring + s * C::kBytes;
            float sc = 0.0f;
            if (mine) {
                const float *ss = reinterpret_cast<const float *>(st + C::kSZ);
                const float *zz = ss + 2 * kUnitRows;
                sc = ss[2 * r + h];
                uint32_t zb, zq;
                zero_bias<XT>(zeros ? zz[2 * r + h] : 8.0f, zb, zq);
                // this row's 128 codes of group h: four swizzled 16-byte chunks
                uint32_t wv[16];
#pragma unroll
                for (int cch = 0; cch < 4; ++cch) {
                    const uint4 v =
                        *reinterpret_cast<const uint4 *>(st + r * 128 + (((4 * h + cch) ^ swz) << 4));
                    wv[4 * cch] = v.x;
                    wv[4 * cch + 1] = v.y;
                    wv[4 * cch + 2] = v.z;
                    wv[4 * cch + 3] = v.w;
                }
                const uint32_t b = n_a & 1, pb = (n_a >> 1) & 1;
                if (!warp_wait(smem_u32(&sh->afree[h][b]), pb ^ 1, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ta = tmem + lanebase + (uint32_t)((2 * h + b) * kAColsPerGroup);
#pragma unroll
                for (int kb = 0; kb < 8; ++kb) {
                    uint32_t a[8];
                    dequant_word<XT>(wv[2 * kb], zb, zq, a);
                    dequant_word<XT>(wv[2 * kb + 1], zb, zq, a + 4);
                    tmem_st8(ta + 8 * kb, a);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                mbar_arrive(smem_u32(&sh->afull[h][b]));
                ++n_a;
            }
            // fold the previous unit's partial while this unit's MMAs run
            if (have_prev) {
                if (!fold(prev_scale)) { ok = false; break; }
                have_prev = false;
            }
            if (mine) {
                prev_scale = sc;
                have_prev = true;
            }
            if (++ks == wk.KS) {
                ks = 0;
                ++rb;
            }
        }
        if (ok && have_prev) ok = fold(prev_scale);
        if (ok && cur_rb >= 0) ok = flush(cur_rb);
        if (ok && h == 0) finish_partials();
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

int make_work(int64_t M, int64_t K, int64_t N, Work *w, size_t *ws_bytes) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    w->G = (int)(K / kGroup);
    w->KS = (int)((K + kUnitK - 1) / kUnitK);
    w->RB = (int)((N + kUnitRows - 1) / kUnitRows);
    w->U = w->KS * w->RB;
    w->P = w->U < di.sm_count ? w->U : di.sm_count;
    // many row blocks per CTA (or too many for the counter area): whole row blocks
    w->aligned = (w->RB >= 8 * w->P || w->RB > kMaxRowBlocks) ? 1 : 0;
    if (w->aligned && w->P > w->RB) w->P = w->RB;
    *ws_bytes = w->aligned ? 0 : kCounterBytes + (size_t)2 * w->P * kUnitRows * M * sizeof(float);
    return W4_OK;
}

template <int XT, int NN>
int launch_t(const Work &w, const CUtensorMap &mapw, const void *X, int64_t M, const float *scales,
             const float *zeros, int64_t K, int64_t N, void *Y, void *ws, cudaStream_t stream) {
    using C = Cfg<NN>;
    auto kern = decode_kernel<XT, NN>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(W4_ERR_CUDA, "cudaGetDevice", nullptr);
    static bool attr_done[64] = {};
    if (!attr_done[dev]) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(decode smem)", e);
        attr_done[dev] = true;
    }
    unsigned *status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    CUtensorMap mapx;
    int st = make_map_2d(&mapx, CU_TENSOR_MAP_DATA_TYPE_UINT16, X, (uint64_t)K, (uint64_t)M,
                         (uint64_t)K * 2, 64, NN, CU_TENSOR_MAP_SWIZZLE_128B,
                         "tensor map of X (decode)");
    if (st != W4_OK) return st;
    unsigned *counters = nullptr;
    float *partial = nullptr;
    if (!w.aligned) {
        counters = static_cast<unsigned *>(ws);
        partial = reinterpret_cast<float *>(static_cast<char *>(ws) + kCounterBytes);
    }
    // programmatic dependent launch: this kernel may start while the previous
    // kernel of the stream finishes; it waits for it before reading X
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(w.P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mapw, mapx, (int)M, scales, zeros, (int)K, (int)N,
                                       Y, counters, partial, w, status);
    if (e != cudaSuccess) return cuda_fail("cudaLaunchKernelEx(decode)", e);
    return W4_OK;
}

}  // namespace

size_t decode_counter_bytes() { return kCounterBytes; }

size_t decode_workspace_bytes(int64_t M, int64_t K, int64_t N, int group) {
    (void)group;
    Work w;
    size_t b = 0;
    if (make_work(M, K, N, &w, &b) != W4_OK) return 0;
    return b;
}

int launch_decode(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                  const float *zeros, int64_t K, int64_t N, void *Y, void *workspace,
                  size_t workspace_bytes, cudaStream_t stream) {
    Work w;
    size_t need = 0;
    int st = make_work(M, K, N, &w, &need);
    if (st != W4_OK) return st;
    if (need > workspace_bytes || (need > 0 && !workspace))
        return set_error(W4_ERR_INVALID_ARG, "w4a16_gemm", "workspace smaller than needed");
    DeviceInfo di;
    if ((st = device_info(&di)) != W4_OK) return st;
    if (di.cc_major != 10) return set_error(W4_ERR_UNSUPPORTED, "w4a16_gemm", "needs an sm_100 GPU");
    CUtensorMap map;
    if ((st = make_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)K / 2, (uint64_t)N,
                          (uint64_t)K / 2, kUnitK / 2, kUnitRows, CU_TENSOR_MAP_SWIZZLE_128B,
                          "tensor map of packed (decode)")) != W4_OK)
        return st;
    const bool small = M <= 16;
    if (xt == W4_F16)
        return small ? launch_t<W4_F16, 16>(w, map, X, M, scales, zeros, K, N, Y, workspace, stream)
                     : launch_t<W4_F16, 32>(w, map, X, M, scales, zeros, K, N, Y, workspace, stream);
    return small ? launch_t<W4_BF16, 16>(w, map, X, M, scales, zeros, K, N, Y, workspace, stream)
                 : launch_t<W4_BF16, 32>(w, map, X, M, scales, zeros, K, N, Y, workspace, stream);
}

}  // namespace w4
