// w4_decode.cu -- the W4A16 linear layer for small M (decode, M <= 32).
//
// Y[m][n] = sum_g scale[n][g] * sum_{k in g} X[m][k] * (u[n][k] - zero[n][g]):
// the "dequant -> 16-bit matmul" of W4A16 ("Quantization method families",
// inference-learning-path.pages.dev, §2), dequantization as in "LLM
// quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2-§2.3.  At small M the layer is
// bound by streaming the packed weights from HBM, so the kernel is built to
// keep HBM busy from the first cycle to the last:
//
//   * Persistent, one CTA per SM.  The packed matrix is cut into units of
//     128 weight rows x 256 k (16 KB of codes).  The units, in row-block-major
//     order, are split into equal contiguous ranges, one per CTA ("stream-K"):
//     every SM streams the same number of bytes whatever N and K are.
//   * A producer warp streams the CTA's units into an 8-stage shared-memory
//     ring with TMA (128-byte swizzle), up to 128 KB in flight per SM.
//   * Eight consumer warps each own 16 of the unit's rows and run
//     mma.sync m16n8k16 "swap-AB": the dequantized weights are the 16-row A
//     operand, built in registers from the swizzled codes, X is the B operand
//     (M padded to 8*MT).  The A operand holds (u - zero), an integer in
//     [-15, 15], exact in fp16/bf16 (exponent-bias trick: OR the nibble into
//     the mantissa of 1024.0 or 128.0, subtract the biased zero point); the
//     fp32 partial of each group is multiplied by its scale afterwards, so no
//     weight is rounded to 16 bits.
//   * A row block whose units all fall in one CTA's range is written to Y
//     directly.  A row block split between CTAs: each warp writes its fp32
//     partial (16 rows) to its CTA's slot in the caller's workspace; the last
//     warp to arrive on that (row block, warp) counter adds the slots in CTA
//     order, writes Y and re-arms the counter.  No warp ever waits for
//     another warp, and the result is deterministic.
//   * Programmatic dependent launch: the kernel may start while the preceding
//     kernel of the stream is finishing; the producer requests the first
//     ring of packed codes at once and everything else (X, scales, zeros,
//     Y, workspace) is touched only after griddepcontrol.wait.
//   * Fragment layout: thread (g, t) holds k = 32t..32t+31 of each group, so
//     mma (word j, half h) maps the fragment's k indices {2t,2t+1,2t+8,2t+9}
//     to k = 32t + 8j + 4h + {0,1,2,3}; the packed layout puts consecutive k
//     pairs in the two halves of one masked 32-bit word, so no shuffles are
//     needed.  mma row g reads unit row 16w + ((g & 1) << 2 | g >> 1) (and
//     that + 8): the rows of one 8-lane load phase then differ in bit 2 of
//     the swizzle key, which makes the 16-byte shared-memory loads
//     conflict-free.
//
// Every mbarrier wait is bounded; a wait that runs out sets the library's
// status word (W4_ERR_TIMEOUT) and an abort flag, and all warps leave.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdio.h>


#include "w4_internal.cuh"

namespace w4 {
namespace {

constexpr int kGroup = 128;
constexpr int kUnitRows = 128;                  // weight rows per unit
constexpr int kUnitK = 256;                     // k per unit (two groups, 128 bytes of codes per row)
constexpr int kUnitBytes = kUnitRows * kUnitK / 2;  // 16 KB
// Workspace: arrival counters (one per row block and consumer warp) first,
// then two partial slots per CTA ([2 * ctas][128 rows][M] fp32).  The counter
// area is fixed so that one workspace serves calls of any shape; row-block
// counts beyond it switch to whole-row-block ranges, which need no workspace.
constexpr int kMaxRowBlocks = 2048;
constexpr int kMaxCounters = kMaxRowBlocks * 8;  // one per (row block, 16-row tile)
constexpr size_t kCounterBytes = kMaxCounters * sizeof(unsigned);
constexpr unsigned long long kWaitNs = 2000000000ull;

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

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

template <int XT>
__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    if (XT == W4_F16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// Biased zero point in the operand type, built with integer ops: the zero
// point z is an integer 0..15, and 1024 + z (fp16), 128 + z (bf16) and
// 64 + z (fp16, mantissa step 1/16) are exact with z in the low mantissa bits.
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
// pairs (u - z) of k = {0,1}, {2,3}, {4,5}, {6,7}.
template <int XT>
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t zb, uint32_t zq, uint32_t p[4]) {
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

// Kernel configuration for MT n8-tiles of X and CW consumer warps.
//   CW = 8:  warp w owns unit rows 16w..16w+15 and both groups of every unit.
//   CW = 16: warps w and w+8 own the same 16 rows; warp w + 8h takes group h
//            of every unit, and the pair adds its two halves through shared
//            memory when a row block ends (twice the warps per scheduler to
//            hide the dequant/MMA latency, at small M where registers allow).
// Stage layout: the unit's codes (128 rows x 128 B), then X[0 .. 8*MT)[k0 ..
// k0+256) as four 64-k boxes of 8*MT rows x 128 B, all with the 128-byte
// swizzle (TMA zero-fills rows >= M and k >= K).
template <int MT, int CW>
struct Cfg {
    static constexpr int kHalves = CW / 8;
    static constexpr int kThreads = 32 * (CW + 1);
    static constexpr int kXBox = 8 * MT * 128;
    static constexpr int kBytes = kUnitBytes + 4 * kXBox;  // 20..32 KB
    static constexpr int kStages = (192 * 1024) / kBytes < 8 ? (192 * 1024) / kBytes : 8;
    static constexpr int kXchgBytes = kHalves == 2 ? 8 * 32 * 4 * MT * 4 : 0;
    static constexpr int kSmem = kStages * kBytes + 1024 + 512 + kXchgBytes;
};

struct Shared {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t pair_full[8];  // CW = 16: second half of a row tile written
    uint64_t pair_free[8];  // CW = 16: first half read it
    int abort_flag;
};

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

template <int XT, int MT, int CW>
__global__ void __launch_bounds__(Cfg<MT, CW>::kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
              int M, const float *__restrict__ scales, const float *__restrict__ zeros, int K, int N,
              void *__restrict__ Y, unsigned *__restrict__ counters, float *__restrict__ partial,
              const Work wk, unsigned *__restrict__ status) {
    using C = Cfg<MT, CW>;
    constexpr int S = C::kStages;
    constexpr int H = C::kHalves;
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

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&sh->full[s]), 1);
            mbar_init(smem_u32(&sh->empty[s]), CW);
        }
        for (int r = 0; r < 8; ++r) {
            mbar_init(smem_u32(&sh->pair_full[r]), 1);
            mbar_init(smem_u32(&sh->pair_free[r]), 1);
        }
        sh->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // let the next kernel in the stream start its prologue as SMs free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == CW) {
        // ---------------- producer ----------------
        if (lane == 0) {
            // The packed weights are inputs no earlier kernel writes: the first
            // ring's worth of codes is requested before waiting for the
            // preceding kernel; X (possibly its output) only after.
            const int pre = min(S, u1 - u0);
            for (int it = 0; it < pre; ++it) {
                const int u = u0 + it;
                const uint32_t fb = smem_u32(&sh->full[it]);
                mbar_arrive_tx(fb, C::kBytes);
                tma_load_2d(smem_u32(ring + it * C::kBytes), &tmap_w, (u % wk.KS) * (kUnitK / 2),
                            (u / wk.KS) * kUnitRows, fb);
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int it = 0; it < pre; ++it) {
                const int u = u0 + it;
                uint8_t *st = ring + it * C::kBytes;
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    tma_load_2d(smem_u32(st + kUnitBytes + b * C::kXBox), &tmap_x,
                                (u % wk.KS) * kUnitK + 64 * b, 0, smem_u32(&sh->full[it]));
            }
            int u = u0 + pre;
            for (; u < u1; ++u) {
                const int it = u - u0;
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                if (!mbar_wait(smem_u32(&sh->empty[s]), ph ^ 1, abort_flag, status)) break;
                const uint32_t fb = smem_u32(&sh->full[s]);
                mbar_arrive_tx(fb, C::kBytes);
                const int rb = u / wk.KS, ks = u % wk.KS;
                uint8_t *st = ring + s * C::kBytes;
                tma_load_2d(smem_u32(st), &tmap_w, ks * (kUnitK / 2), rb * kUnitRows, fb);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    tma_load_2d(smem_u32(st + kUnitBytes + b * C::kXBox), &tmap_x,
                                ks * kUnitK + 64 * b, 0, fb);
            }
            // wait (bounded) for the copies still in flight before the CTA may exit
            for (int j = (u - u0 > S ? u - u0 - S : 0); j < u - u0; ++j) {
                const unsigned long long t0 = globaltimer();
                while (!mbar_try(smem_u32(&sh->full[j % S]), (j / S) & 1) &&
                       globaltimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
        return;
    }

    // ---------------- consumers ----------------
    const int g = lane >> 2, t = lane & 3;
    const int tile = warp % 8;                   // 16-row tile of the unit
    const int half = warp / 8;                   // CW = 16: which group of each unit
    const int rsel = ((g & 1) << 2) | (g >> 1);  // unit row of mma row g (conflict-free loads)
    const int lrow0 = 16 * tile + rsel;          // this thread's two rows in the unit
    const int lrow1 = lrow0 + 8;
    const int swz = lrow0 & 7;                   // swizzle key of both rows
    const int G = wk.G;

    float acc[MT][4];
    int cur_rb = -1, first_ks = 0, last_ks = -1;
    uint32_t xph = 0;  // flushes done (pair exchange parity)
    bool ok = true;
    int pending[2];    // row blocks whose partials this warp stored (at most 2 per CTA)
    int npending = 0;

    // Finishes row block rb for this tile's 16 rows.  Waits are bounded; no
    // step waits on a warp of another tile.  A row block split between CTAs
    // has one arrival counter per (row block, tile), and the last warp to
    // arrive adds the partials in CTA order (finish_partials).
    auto flush = [&](int rb) -> bool {
        if (H == 2) {
            float *xc = xchg + (tile * 32 + lane) * 4 * MT;
            if (half == 1) {
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sh->pair_free[tile]), xph ^ 1,
                                                        abort_flag, status)))
                    return false;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) xc[4 * mt + i] = acc[mt][i];
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sh->pair_full[tile]));
                xph ^= 1;
                return true;
            }
            if (!__all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&sh->pair_full[tile]), xph, abort_flag, status)))
                return false;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[mt][i] += xc[4 * mt + i];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh->pair_free[tile]));
            xph ^= 1;
        }
        const int n0 = rb * kUnitRows;
        if (first_ks == 0 && last_ks == wk.KS - 1) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int n = n0 + (i < 2 ? lrow0 : lrow1);
                    const int m = 8 * mt + 2 * t + (i & 1);
                    if (n < N && m < M) store_out<XT>(Y, (int64_t)m * N + n, acc[mt][i]);
                }
            return true;
        }
        // partial: slot 0 for the CTA's first row block, 1 for its last.  Only
        // the store happens here; the arrival and the final sum wait until the
        // CTA's units are all done (finish_partials), so the warp goes on.
        const int slot = 2 * c + (rb == u0 / wk.KS ? 0 : 1);
        float *dst = partial + (int64_t)slot * kUnitRows * M;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = i < 2 ? lrow0 : lrow1;
                const int m = 8 * mt + 2 * t + (i & 1);
                if (m < M) dst[r * M + m] = acc[mt][i];
            }
        pending[npending++] = rb;
        return true;
    };

    // Arrives on the counters of the row blocks whose partials this warp
    // stored; the last warp to arrive on one adds its partials in CTA order.
    auto finish_partials = [&]() {
        if (npending == 0) return;
        __threadfence();
        __syncwarp();
        for (int q = 0; q < npending; ++q) {
            const int rb = pending[q];
            const int n0 = rb * kUnitRows;
            const int cf = owner(wk, rb * wk.KS), cl = owner(wk, (rb + 1) * wk.KS - 1);
            unsigned *cnt = counters + rb * 8 + tile;
            unsigned prev = 0;
            if (lane == 0) prev = atomicAdd(cnt, 1u);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            if (prev != (unsigned)(cl - cf)) continue;
            __threadfence();
            for (int e = lane; e < 16 * M; e += 32) {
                const int r = 16 * tile + (e & 15), m = e >> 4;
                const int n = n0 + r;
                if (n >= N) continue;
                float v = 0.0f;
                for (int cc = cf; cc <= cl; ++cc) {
                    const int sl = 2 * cc + (rb == range_start(wk, cc) / wk.KS ? 0 : 1);
                    v += __ldcg(partial + ((int64_t)sl * kUnitRows + r) * M + m);
                }
                store_out<XT>(Y, (int64_t)m * N + n, v);
            }
            __syncwarp();
            if (lane == 0) *cnt = 0u;  // re-arm for the next call
        }
    };

    // scales and zero points of one unit for this thread's two rows and
    // this warp's groups
    const int64_t rowoff0 = (int64_t)lrow0 * G, rowoff1 = (int64_t)lrow1 * G;
    const int64_t blockstride = (int64_t)kUnitRows * G;
    const int64_t lastrow = (int64_t)(N - 1) * G;
    float sa[2], sb[2], za[2], zbv[2];
    auto load_sz = [&](int rb, int ks) {
        const int64_t base = rb * blockstride;
        const int64_t ia = min(base + rowoff0, lastrow), ib = min(base + rowoff1, lastrow);
#pragma unroll
        for (int q = 0; q < 2 / H; ++q) {
            const int grp = min(2 * ks + (H == 2 ? half : q), G - 1);
            sa[q] = __ldg(scales + ia + grp);
            sb[q] = __ldg(scales + ib + grp);
            za[q] = zeros ? __ldg(zeros + ia + grp) : 8.0f;
            zbv[q] = zeros ? __ldg(zeros + ib + grp) : 8.0f;
        }
    };
    int rb = u0 / wk.KS;
    int ks = u0 - rb * wk.KS;
    // everything but the packed codes is read after the preceding kernel of
    // the stream has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (u0 < u1) load_sz(rb, ks);
    // X of k = 128 gi + 32 t + 8 j sits in box 2 gi + t/2, 16-byte chunk
    // 4 (t&1) + j, row 8 mt + g of that box (swizzle key g)
    const int xoff0 = (t >> 1) * C::kXBox + g * 128;
    const int xsw = 4 * (t & 1);
    constexpr bool kSplit = MT <= 2;  // two accumulators per group: more independent MMAs

    for (int u = u0; u < u1; ++u) {
        const int it = u - u0;
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        if (rb != cur_rb) {
            if (cur_rb >= 0 && !flush(cur_rb)) { ok = false; break; }
            cur_rb = rb;
            first_ks = ks;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[mt][i] = 0.0f;
        }
        last_ks = ks;
        // this unit's scales and zero points; the next unit's are fetched
        // while this one is computed
        float cs_a[2], cs_b[2];
        uint32_t zba[2], zqa[2], zbb[2], zqb[2];
#pragma unroll
        for (int q = 0; q < 2 / H; ++q) {
            cs_a[q] = sa[q];
            cs_b[q] = sb[q];
            zero_bias<XT>(za[q], zba[q], zqa[q]);
            zero_bias<XT>(zbv[q], zbb[q], zqb[q]);
        }
        int nrb = rb, nks = ks + 1;
        if (nks == wk.KS) {
            nks = 0;
            ++nrb;
        }
        if (u + 1 < u1) load_sz(nrb, nks);
        const bool got = __all_sync(0xffffffffu,
                                    mbar_wait(smem_u32(&sh->full[s]), ph, abort_flag, status));
        if (!got) {
            ok = false;
            break;
        }
        const uint8_t *unit = ring + s * C::kBytes;
        const uint8_t *xs = unit + kUnitBytes + xoff0;
#pragma unroll
        for (int q = 0; q < 2 / H; ++q) {
            const int gi = H == 2 ? half : q;  // group of the unit
            if (2 * ks + gi >= G) break;       // a last unit with one group
            const int ch0 = ((4 * gi + t) ^ swz) << 4;
            const uint4 wa = *reinterpret_cast<const uint4 *>(unit + lrow0 * 128 + ch0);
            const uint4 wb = *reinterpret_cast<const uint4 *>(unit + lrow1 * 128 + ch0);
            const uint32_t wav[4] = {wa.x, wa.y, wa.z, wa.w};
            const uint32_t wbv[4] = {wb.x, wb.y, wb.z, wb.w};
            const uint8_t *xg = xs + 2 * gi * C::kXBox;
            float pa_[MT][4], pb_[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) pa_[mt][i] = pb_[mt][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 xv[MT];
                const int ch = ((xsw + j) ^ g) << 4;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    // rows >= M are zero: those lanes skip the shared-memory read
                    xv[mt] = make_uint4(0, 0, 0, 0);
                    if (8 * mt + g < M) xv[mt] = *reinterpret_cast<const uint4 *>(xg + mt * 1024 + ch);
                }
                uint32_t pa[4], pb[4];
                dequant_word<XT>(wav[j], zba[q], zqa[q], pa);
                dequant_word<XT>(wbv[j], zbb[q], zqb[q], pb);
                const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
                const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    mma16816<XT>(pa_[mt], a0, xv[mt].x, xv[mt].y);
                    mma16816<XT>(kSplit ? pb_[mt] : pa_[mt], a1, xv[mt].z, xv[mt].w);
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const float p0 = kSplit ? pa_[mt][0] + pb_[mt][0] : pa_[mt][0];
                const float p1 = kSplit ? pa_[mt][1] + pb_[mt][1] : pa_[mt][1];
                const float p2 = kSplit ? pa_[mt][2] + pb_[mt][2] : pa_[mt][2];
                const float p3 = kSplit ? pa_[mt][3] + pb_[mt][3] : pa_[mt][3];
                acc[mt][0] = fmaf(cs_a[q], p0, acc[mt][0]);
                acc[mt][1] = fmaf(cs_a[q], p1, acc[mt][1]);
                acc[mt][2] = fmaf(cs_b[q], p2, acc[mt][2]);
                acc[mt][3] = fmaf(cs_b[q], p3, acc[mt][3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sh->empty[s]));
        rb = nrb;
        ks = nks;
    }
    if (ok && cur_rb >= 0) ok = flush(cur_rb);
    if (ok && (H == 1 || half == 0)) finish_partials();
}

// ---- host side --------------------------------------------------------------------------

int mt_for(int64_t M) { return (int)((M + 7) / 8); }

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

template <int XT, int MT, int CW>
int launch_t(const Work &w, const CUtensorMap &mapw, const void *X, int64_t M, const float *scales,
             const float *zeros, int64_t K, int64_t N, void *Y, void *ws, cudaStream_t stream) {
    using C = Cfg<MT, CW>;
    auto kern = decode_kernel<XT, MT, CW>;
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
                         (uint64_t)K * 2, 64, 8 * MT, CU_TENSOR_MAP_SWIZZLE_128B,
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
    cfg.blockDim = dim3(C::kThreads);
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

template <int XT>
int launch_x(const Work &w, const CUtensorMap &map, const void *X, int64_t M, const float *scales,
             const float *zeros, int64_t K, int64_t N, void *Y, void *ws, cudaStream_t s) {
    switch (mt_for(M)) {
        case 1: return launch_t<XT, 1, 16>(w, map, X, M, scales, zeros, K, N, Y, ws, s);
        case 2: return launch_t<XT, 2, 16>(w, map, X, M, scales, zeros, K, N, Y, ws, s);
        case 3: return launch_t<XT, 3, 8>(w, map, X, M, scales, zeros, K, N, Y, ws, s);
        default: return launch_t<XT, 4, 8>(w, map, X, M, scales, zeros, K, N, Y, ws, s);
    }
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
    CUtensorMap map;
    if ((st = make_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)K / 2, (uint64_t)N,
                          (uint64_t)K / 2, kUnitK / 2, kUnitRows, CU_TENSOR_MAP_SWIZZLE_128B,
                          "tensor map of packed (decode)")) != W4_OK)
        return st;
    if (xt == W4_F16)
        return launch_x<W4_F16>(w, map, X, M, scales, zeros, K, N, Y, workspace, stream);
    return launch_x<W4_BF16>(w, map, X, M, scales, zeros, K, N, Y, workspace, stream);
}

}  // namespace w4
