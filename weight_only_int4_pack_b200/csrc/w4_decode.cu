// w4_decode.cu -- the W4A16 linear layer for small M (decode, M <= 32).
//
// Y[m][n] = sum_g scale[n][g] * sum_{k in g} X[m][k] * (u[n][k] - zero[n][g]):
// the "dequant -> 16-bit matmul" of W4A16 ("Quantization method families",
// inference-learning-path.pages.dev, §2), dequantization as in "LLM
// quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2-§2.3.  At small M the layer is
// bound by streaming the packed weights from HBM, so the kernel is built to
// keep HBM busy from the first cycle to the last and to spend as few issue
// slots per weight as possible.  (launch_decode, at the end, sends M = 1
// with K <= 4096 to the CUDA-core GEMV of w4_gemv1.cu and other M <= 8 with
// K <= 4096 to the warp-MMA GEMV of w4_gemv.cu; this kernel serves the rest.)
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

#include "w4_debug.cuh"
#include "w4_internal.cuh"

namespace w4 {
namespace {

[[maybe_unused]] constexpr unsigned kDbgFile = 2;  // W4_DEBUG file id

constexpr int kGroup = 128;
constexpr int kUnitRows = 128;                      // weight rows per unit (= TMEM lanes)
constexpr int kUnitK = 256;                         // k per unit: two groups, 128 bytes per row
constexpr int kUnitBytes = kUnitRows * kUnitK / 2;  // 16 KB of codes
constexpr int kSZBytes = kUnitRows * 2 * 4;         // zero points (or scales) of a unit: [128][2] fp32
constexpr int kTmemCols = 512;
constexpr int kAColsPerGroup = 64;  // A operand of one group: 128 k of 16-bit pairs
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

// Up to 64 polls of the barrier in a tight loop (five instructions a poll):
// true as soon as the phase with `parity` has completed.
__device__ __forceinline__ bool mbar_poll64(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t.reg .u32 n;\n\t"
        "mov.u32 n, 64;\n"
        "W4_POLL_%=:\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "@p bra W4_DONE_%=;\n\t"
        "sub.u32 n, n, 1;\n\t"
        "setp.ne.u32 q, n, 0;\n\t"
        "@q bra W4_POLL_%=;\n"
        "W4_DONE_%=:\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: true once the phase with `parity` has completed; false if the
// CTA aborted or the wait ran out (then the abort flag and status are set).
// The abort flag and the clock are looked at every 64 polls only, so that
// waiting warps take few issue slots from the working ones.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned *status) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_poll64(bar, parity)) return true;
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

// true in exactly one lane of the (fully active) warp
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
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

// Dequantizes 8 packed words (64 codes of one row, k = 8i .. 8i + 7 in word
// i) and stores the 32 exact pairs (u - z) to TMEM columns taddr ..
// taddr + 31 of this thread's lane, in one block: the 32 results are produced
// straight into the store's registers.  mask_lo, mask_hi and magic come in
// registers so that each nibble pair costs one LOP3.  fp16: pairs {0,1} and
// {4,5} come from the low nibbles of the word and of the word >> 8, minus
// (1024 + z); pairs {2,3} and {6,7} from the high nibbles, times 1/16 minus
// (64 + z).  bf16: nibble i of each half (word >> 4i), minus (128 + z).
template <int XT>
__device__ __forceinline__ void dequant8_store(uint32_t taddr, const uint32_t (&w)[8], uint32_t zb,
                                               uint32_t zq) {
    uint32_t mlo, mhi, magic, sixteenth;
    asm("mov.b32 %0, 0x000F000F;" : "=r"(mlo));
    asm("mov.b32 %0, 0x00F000F0;" : "=r"(mhi));
    if (XT == W4_F16) {
        asm("mov.b32 %0, 0x64006400;" : "=r"(magic));
        asm("mov.b32 %0, 0x2C002C00;" : "=r"(sixteenth));
#define W4_F16_WORD(i)                                                   \
    "lop3.b32 t" #i "a, %" #i ", mlo, magic, 0xEA;\n\t"                  \
    "lop3.b32 t" #i "b, %" #i ", mhi, magic, 0xEA;\n\t"                  \
    "shr.b32 x, %" #i ", 8;\n\t"                                         \
    "lop3.b32 t" #i "c, x, mlo, magic, 0xEA;\n\t"                        \
    "lop3.b32 t" #i "d, x, mhi, magic, 0xEA;\n\t"                        \
    "sub.f16x2 t" #i "a, t" #i "a, zb;\n\t"                               \
    "fma.rn.f16x2 t" #i "b, t" #i "b, six, zq;\n\t"                       \
    "sub.f16x2 t" #i "c, t" #i "c, zb;\n\t"                               \
    "fma.rn.f16x2 t" #i "d, t" #i "d, six, zq;\n\t"
        asm volatile(
            "{\n\t"
            ".reg .b32 t0a, t0b, t0c, t0d, t1a, t1b, t1c, t1d, t2a, t2b, t2c, t2d, t3a, t3b, t3c, t3d;\n\t"
            ".reg .b32 t4a, t4b, t4c, t4d, t5a, t5b, t5c, t5d, t6a, t6b, t6c, t6d, t7a, t7b, t7c, t7d;\n\t"
            ".reg .b32 x, mlo, mhi, magic, six, zb, zq;\n\t"
            "mov.b32 mlo, %9;\n\tmov.b32 mhi, %10;\n\tmov.b32 magic, %11;\n\t"
            "mov.b32 six, %12;\n\tmov.b32 zb, %13;\n\tmov.b32 zq, %14;\n\t"
            W4_F16_WORD(0) W4_F16_WORD(1) W4_F16_WORD(2) W4_F16_WORD(3)
            W4_F16_WORD(4) W4_F16_WORD(5) W4_F16_WORD(6) W4_F16_WORD(7)
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%8], {t0a, t0b, t0c, t0d, t1a, t1b, t1c, t1d, "
            "t2a, t2b, t2c, t2d, t3a, t3b, t3c, t3d, t4a, t4b, t4c, t4d, t5a, t5b, t5c, t5d, "
            "t6a, t6b, t6c, t6d, t7a, t7b, t7c, t7d};\n\t"
            "}" ::"r"(w[0]),
            "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(taddr),
            "r"(mlo), "r"(mhi), "r"(magic), "r"(sixteenth), "r"(zb), "r"(zq)
            : "memory");
#undef W4_F16_WORD
    } else {
        asm("mov.b32 %0, 0x43004300;" : "=r"(magic));
#define W4_BF16_WORD(i)                                                  \
    "lop3.b32 t" #i "a, %" #i ", mlo, magic, 0xEA;\n\t"                  \
    "shr.b32 x, %" #i ", 4;\n\t"                                         \
    "lop3.b32 t" #i "b, x, mlo, magic, 0xEA;\n\t"                        \
    "shr.b32 x, %" #i ", 8;\n\t"                                         \
    "lop3.b32 t" #i "c, x, mlo, magic, 0xEA;\n\t"                        \
    "shr.b32 x, %" #i ", 12;\n\t"                                        \
    "lop3.b32 t" #i "d, x, mlo, magic, 0xEA;\n\t"                        \
    "sub.bf16x2 t" #i "a, t" #i "a, zb;\n\t"                              \
    "sub.bf16x2 t" #i "b, t" #i "b, zb;\n\t"                              \
    "sub.bf16x2 t" #i "c, t" #i "c, zb;\n\t"                              \
    "sub.bf16x2 t" #i "d, t" #i "d, zb;\n\t"
        asm volatile(
            "{\n\t"
            ".reg .b32 t0a, t0b, t0c, t0d, t1a, t1b, t1c, t1d, t2a, t2b, t2c, t2d, t3a, t3b, t3c, t3d;\n\t"
            ".reg .b32 t4a, t4b, t4c, t4d, t5a, t5b, t5c, t5d, t6a, t6b, t6c, t6d, t7a, t7b, t7c, t7d;\n\t"
            ".reg .b32 x, mlo, magic, zb;\n\t"
            "mov.b32 mlo, %9;\n\tmov.b32 magic, %10;\n\tmov.b32 zb, %11;\n\t"
            W4_BF16_WORD(0) W4_BF16_WORD(1) W4_BF16_WORD(2) W4_BF16_WORD(3)
            W4_BF16_WORD(4) W4_BF16_WORD(5) W4_BF16_WORD(6) W4_BF16_WORD(7)
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%8], {t0a, t0b, t0c, t0d, t1a, t1b, t1c, t1d, "
            "t2a, t2b, t2c, t2d, t3a, t3b, t3c, t3d, t4a, t4b, t4c, t4d, t5a, t5b, t5c, t5d, "
            "t6a, t6b, t6c, t6d, t7a, t7b, t7c, t7d};\n\t"
            "}" ::"r"(w[0]),
            "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(taddr),
            "r"(mlo), "r"(magic), "r"(zb)
            : "memory");
#undef W4_BF16_WORD
        (void)zq;
        (void)mhi;
        (void)sixteenth;
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
// (swizzled) | zero points [128][2] fp32.
//
// Slots: unit `it` of a CTA's range uses TMEM slot it % kSlots, which holds
// its A operand (both groups, 2 x 64 columns) and its two fp32 partials
// (2 x NN columns).  A slot is reused by unit it + kSlots once the MMAs of
// unit it are done and its partials have been read.
template <int NN>
struct Cfg {
    static constexpr int kXBox = NN * 128;
    static constexpr int kZOff = kUnitBytes + 4 * kXBox;
    static constexpr int kBytes = kZOff + kSZBytes;
    static constexpr int kTmaBytes = kUnitBytes + 4 * kXBox;
    static constexpr int kXchgBytes = 4 * NN * 32 * 4;  // [quarter][m][lane] fp32
    static constexpr int kStages =
        (200 * 1024 - kXchgBytes) / kBytes < 8 ? (200 * 1024 - kXchgBytes) / kBytes : 8;
    static constexpr int kSmem = kStages * kBytes + 1024 + 512 + kXchgBytes;
    static constexpr int kSlots = kTmemCols / (2 * kAColsPerGroup + 2 * NN);
    static constexpr int kDBase = kSlots * 2 * kAColsPerGroup;
    static_assert(kSlots >= 2 && kSlots <= 3, "TMEM slots");
    static_assert(kDBase + kSlots * 2 * NN <= kTmemCols, "TMEM columns");
};

struct Shared {
    uint64_t full[8];   // stage: codes + X (TMA bytes) and zero points (cp.async) landed
    uint64_t empty[8];  // stage: the unit's MMAs done (commit)
    uint64_t ready[3];  // slot: A stored and the previous partials read (4 dequant warps)
    uint64_t mdone[3];  // slot: the unit's MMAs done (commit): A free, partials complete
    uint64_t xfull[4];  // lane quarter: group-1 accumulators of a row block in xbuf
    uint64_t xfree[4];  // lane quarter: xbuf read
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Shared) <= 512, "the exchange buffer starts 512 bytes after the barriers");

// Warp roles (10 warps): 0 producer, 1 TMEM allocator + MMA issuer,
// 2..9 dequant (warp w: TMEM lane quarter w % 4, the units of parity
// (w - 2) / 4), which also fold the partials of their rows.
constexpr int kDequantWarps = 8;
constexpr int kThreads = 32 * (2 + kDequantWarps);

// Launch bounds of 384 threads cap the registers at 168 a thread: up to three
// of the 10 warps share one SM sub-partition (16K registers).
template <int XT, int NN>
__global__ void __launch_bounds__(384, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
              int M, const float *__restrict__ scales, const float *__restrict__ zeros, int K, int N,
              void *__restrict__ Y, unsigned *__restrict__ counters, float *__restrict__ partial,
              const Work wk, unsigned *__restrict__ status) {
    using C = Cfg<NN>;
    constexpr int S = C::kStages;
    constexpr int R = C::kSlots;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    Shared *sh = reinterpret_cast<Shared *>(ring + S * C::kBytes);
    float *xbuf = reinterpret_cast<float *>(ring + S * C::kBytes + 512);
    volatile int *abort_flag = &sh->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int u0 = range_start(wk, c);
    const int u1 = range_start(wk, c + 1);
    const int nu = u1 - u0;
    const int G = wk.G;
    // W4_DEBUG: [p, p + bytes) inside the stage ring, itself inside this
    // launch's shared memory; a TMA box start with a 16-byte aligned x
    [[maybe_unused]] auto ring_ok = [&](const void *p, uint32_t bytes) {
        return in_range(smem_u32(p), bytes, smem_u32(ring), uint64_t(S) * C::kBytes) &&
               in_range(smem_u32(ring), uint64_t(S) * C::kBytes + 512 + 4 * NN * 32 * 4,
                        smem_u32(smem_raw), dyn_smem_bytes());
    };
    [[maybe_unused]] auto wbox_ok = [&](int x, int y) {
        return x >= 0 && x % 16 == 0 && x < K / 2 && y >= 0 && y < N;
    };
    [[maybe_unused]] auto xbox_ok = [&](int x) { return x >= 0 && x % 8 == 0; };

    // The packed weights are inputs no earlier kernel writes: thread 0 (the
    // producer's TMA lane) requests the codes of the CTA's first two units as
    // soon as the barriers exist, before anything else of the prologue.
    const int early = min(2, min(S, nu));
    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&sh->full[s]), 1 + 32);  // TMA arrive_tx + 32 cp.async arrivals
            mbar_init(smem_u32(&sh->empty[s]), 1);
        }
        for (int j = 0; j < R; ++j) {
            mbar_init(smem_u32(&sh->ready[j]), 4);  // the unit's four dequant warps
            mbar_init(smem_u32(&sh->mdone[j]), 1);
        }
        for (int q = 0; q < 4; ++q) {
            mbar_init(smem_u32(&sh->xfull[q]), 1);
            mbar_init(smem_u32(&sh->xfree[q]), 1);
        }
        sh->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        int rb = u0 / wk.KS, ks = u0 - (u0 / wk.KS) * wk.KS;
        for (int it = 0; it < early; ++it) {
            const uint32_t fb = smem_u32(&sh->full[it]);
            if (!W4_CHECK(ring_ok(ring + it * C::kBytes, C::kBytes) &&
                              wbox_ok(ks * (kUnitK / 2), rb * kUnitRows),
                          status))
                break;
            mbar_arrive_tx(fb, C::kTmaBytes);
            tma_load_2d(smem_u32(ring + it * C::kBytes), &tmap_w, ks * (kUnitK / 2), rb * kUnitRows,
                        fb);
            if (++ks == wk.KS) {
                ks = 0;
                ++rb;
            }
        }
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
        // Codes and X by TMA (lane 0); the unit's zero points by cp.async (four
        // rows per lane); every lane arrives on the stage's full barrier once
        // its copies have landed.
        auto issue_sz = [&](int rb, int ks, uint8_t *st, uint32_t fb) {
            if (zeros) {
                const int g0 = 2 * ks, g1 = min(2 * ks + 1, G - 1);
                float *zz = reinterpret_cast<float *>(st + C::kZOff);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int r = lane + 32 * q;
                    const int64_t n = min(rb * kUnitRows + r, N - 1);
                    if (!W4_CHECK(n >= 0 && g0 >= 0 && g1 < G && ring_ok(zz + 2 * r, 8), status)) continue;
                    cp_async4(smem_u32(zz + 2 * r), zeros + n * G + g0);
                    cp_async4(smem_u32(zz + 2 * r + 1), zeros + n * G + g1);
                }
            }
            cp_async_arrive(fb);
        };
        auto issue_x = [&](int ks, uint8_t *st, uint32_t fb) {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (W4_CHECK(xbox_ok(ks * kUnitK + 64 * b) && ring_ok(st + kUnitBytes + b * C::kXBox, C::kXBox),
                             status))
                    tma_load_2d(smem_u32(st + kUnitBytes + b * C::kXBox), &tmap_x, ks * kUnitK + 64 * b, 0,
                            fb);
        };
        auto issue_w = [&](int rb, int ks, uint8_t *st, uint32_t fb) {
            if (!W4_CHECK(ring_ok(st, C::kBytes) && wbox_ok(ks * (kUnitK / 2), rb * kUnitRows), status))
                return;
            mbar_arrive_tx(fb, C::kTmaBytes);
            tma_load_2d(smem_u32(st), &tmap_w, ks * (kUnitK / 2), rb * kUnitRows, fb);
        };
        // (rb, ks): row block and k step of the next unit to issue
        int rb = u0 / wk.KS, ks = u0 - (u0 / wk.KS) * wk.KS;
        // The codes of the first `early` units went out in the prologue; the
        // X slices and zero points of the first units go out before the rest
        // of the first ring, so that unit 0 lands early.
        const int pre = min(S, nu);
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int it = 0; it < pre; ++it) {
            uint8_t *st = ring + it * C::kBytes;
            const uint32_t fb = smem_u32(&sh->full[it]);
            if (lane == 0) {
                if (it >= early) issue_w(rb, ks, st, fb);
                issue_x(ks, st, fb);
            }
            issue_sz(rb, ks, st, fb);
            if (++ks == wk.KS) {
                ks = 0;
                ++rb;
            }
        }
        int it = pre;
        int s = 0;        // stage of unit it (it >= pre only runs when pre == S)
        uint32_t ph = 1;  // its fill parity
        for (; it < nu; ++it) {
            if (!warp_wait(smem_u32(&sh->empty[s]), ph ^ 1, abort_flag, status)) break;
            uint8_t *st = ring + s * C::kBytes;
            const uint32_t fb = smem_u32(&sh->full[s]);
            if (lane == 0) {
                issue_w(rb, ks, st, fb);
                issue_x(ks, st, fb);
            }
            issue_sz(rb, ks, st, fb);
            if (++ks == wk.KS) {
                ks = 0;
                ++rb;
            }
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
        }
        // wait (bounded) for the copies still in flight before the CTA may exit
        if (lane == 0) {
            for (int j = (it > S ? it - S : 0); j < it; ++j) {
                const unsigned long long t0 = globaltimer();
                while (!mbar_try(smem_u32(&sh->full[j % S]), (j / S) & 1) &&
                       globaltimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // The whole warp takes the waits (warp-uniform operands stay in
        // uniform registers); one elected lane issues.  The tensor pipe queues
        // only a few MMAs, so the wait for unit it + 1 is taken while the last
        // four MMAs of unit it are still to be issued: the pipe never runs dry
        // between units when the next unit is ready.  Each unit waits on one
        // barrier: its slot's `ready` (A stored, previous partials read).  Its
        // X comes from the stage the dequant warps waited for before they
        // arrived.
        constexpr uint32_t idesc = instr_desc<XT, NN>();
        const bool leader = elect_one();
        const uint64_t xdesc0 = sw128_desc(smem_u32(ring + kUnitBytes));
        int done = -1;  // last unit whose MMAs are tracked by its empty barrier
        bool ok = nu > 0 && warp_wait(smem_u32(&sh->ready[0]), 0, abort_flag, status);
        int ks = u0 - (u0 / wk.KS) * wk.KS;  // k step of unit it
        int s = 0, j = 0;                    // its stage and slot
        int jn = 1;                          // slot of unit it + 1 and its ready parity
        uint32_t pn = 0;
        for (int it = 0; it < nu && ok; ++it) {
            const bool two = 2 * ks + 1 < G;  // false: a last unit with one group
            tc_fence_after();
            // stage s's X boxes: descriptor start address advances in 16-byte units
            const uint64_t xd = xdesc0 + (uint64_t)((s * C::kBytes) >> 4);
            const uint32_t ta0 = tmem + (uint32_t)(2 * j * kAColsPerGroup);
            const uint32_t ta1 = ta0 + kAColsPerGroup;
            const uint32_t td0 = tmem + (uint32_t)(C::kDBase + 2 * j * NN);
            const uint32_t td1 = td0 + NN;
            // group h, k16 step kb: X box 2h + kb/4, 32 bytes per step in its swizzle row
            auto issue = [&](int kb) {
                const uint32_t off0 = (uint32_t)(((kb / 4) * C::kXBox + (kb % 4) * 32) >> 4);
                const uint32_t off1 = (uint32_t)(((2 + kb / 4) * C::kXBox + (kb % 4) * 32) >> 4);
                mma_ts(td0, ta0 + 8 * kb, xd + off0, idesc, kb > 0 ? 1u : 0u);
                if (two) mma_ts(td1, ta1 + 8 * kb, xd + off1, idesc, kb > 0 ? 1u : 0u);
            };
            if (leader) {
#pragma unroll
                for (int kb = 0; kb < 6; ++kb) issue(kb);
            }
            __syncwarp();
            bool ok_next = true;
            if (it + 1 < nu) ok_next = warp_wait(smem_u32(&sh->ready[jn]), pn, abort_flag, status);
            if (leader) {
                issue(6);
                issue(7);
                mma_commit(smem_u32(&sh->mdone[j]));
                mma_commit(smem_u32(&sh->empty[s]));
            }
            __syncwarp();
            done = it;
            ok = ok_next;
            if (++ks == wk.KS) ks = 0;
            if (++s == S) s = 0;
            j = jn;
            if (++jn == R) {
                jn = 0;
                pn ^= 1;
            }
        }
        // drain: wait (bounded) until the last issued MMAs have completed
        if (done >= 0 && lane == 0) {
            const unsigned long long t0 = globaltimer();
            while (!mbar_try(smem_u32(&sh->empty[done % S]), (done / S) & 1) &&
                   globaltimer() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else {
        // ---------------- dequant + fold: 8 warps ----------------
        // Warp (q, p) owns rows r = 32q..32q+31 (its TMEM lane quarter) and the
        // units of parity p of the CTA's range.  For such a unit it, it
        // dequantizes the row's 256 codes (both groups) into the slot's A
        // operand, after first adding scale * partial of the slot's previous
        // unit (it - R, done in the tensor pipe) into its fp32 accumulators.
        // Both warps of a quarter follow every unit's row block, so that at
        // each row-block boundary both hand over their sums: the p = 1 warp
        // through xbuf to the p = 0 warp, which writes Y (or its CTA's
        // partial of a row block split between CTAs).
        const int p = (warp - 2) >> 2;
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lanebase = (uint32_t)(32 * q) << 16;
        const int swz = r & 7;
        float acc[NN];
#pragma unroll
        for (int i = 0; i < NN; ++i) acc[i] = 0.0f;
        int cur_rb = -1;      // row block the accumulators belong to
        int pend0 = -1, pend1 = -1;
        unsigned prev0 = 0, prev1 = 0;  // their counters before this warp's arrival (lane 0)  // split row blocks stored (p == 0)
        uint32_t nflush = 0;  // row blocks flushed (xfull / xfree parity)
        bool ok = true;

        auto flush = [&](int rb) -> bool {
            float *xb = xbuf + q * NN * 32 + lane;
            const uint32_t par = nflush & 1;
            ++nflush;
            if (!W4_CHECK_WARP(in_range(smem_u32(xb), 4, smem_u32(ring) + uint64_t(S) * C::kBytes + 512,
                                        4 * NN * 32 * 4) &&
                                   in_range(smem_u32(xb + 32 * (NN - 1)), 4,
                                            smem_u32(ring) + uint64_t(S) * C::kBytes + 512, 4 * NN * 32 * 4),
                               status))
                return false;
            if (p == 1) {
                if (!warp_wait(smem_u32(&sh->xfree[q]), par ^ 1, abort_flag, status)) return false;
#pragma unroll
                for (int m = 0; m < NN; ++m) xb[32 * m] = acc[m];
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sh->xfull[q]));
                return true;
            }
            if (!warp_wait(smem_u32(&sh->xfull[q]), par, abort_flag, status)) return false;
#pragma unroll
            for (int m = 0; m < NN; ++m) acc[m] += xb[32 * m];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh->xfree[q]));
            const int n = rb * kUnitRows + r;
            if (rb * wk.KS >= u0 && (rb + 1) * wk.KS <= u1) {  // whole row block in this range
                if (n < N && W4_CHECK(n >= 0 && M <= NN, status)) {
#pragma unroll
                    for (int m = 0; m < NN; ++m)
                        if (m < M) store_out<XT>(Y, (int64_t)m * N + n, acc[m]);
                }
                return true;
            }
            const int slot = 2 * c + (rb == u0 / wk.KS ? 0 : 1);
            if (!W4_CHECK_WARP(partial != nullptr && slot >= 0 && slot < 2 * wk.P && M <= NN &&
                                   rb >= 0 && rb * 8 + q < static_cast<int>(kCounterBytes / sizeof(unsigned)),
                               status))
                return false;
            float *dst = partial + ((int64_t)slot * kUnitRows + r) * M;
#pragma unroll
            for (int m = 0; m < NN; ++m)
                if (m < M) dst[m] = acc[m];
            // Arrive on the row block's (row block, lane quarter) counter at
            // once: one acquire-release atomic orders this warp's partial
            // stores (every lane's, joined by __syncwarp) before the arrival;
            // its result (was this the last arrival?) is only looked at after
            // the CTA's last unit, so the round trip overlaps the work.
            __syncwarp();
            unsigned prev = 0;
            if (lane == 0)
                asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                             : "=r"(prev)
                             : "l"(counters + rb * 8 + q)
                             : "memory");
            if (pend0 < 0) {
                pend0 = rb;
                prev0 = prev;
            } else {
                pend1 = rb;
                prev1 = prev;
            }
            return true;
        };

        asm volatile("griddepcontrol.wait;" ::: "memory");
        int ks = u0 - (u0 / wk.KS) * wk.KS;              // unit it: k step
        int s = 0, j = 0;                                // its stage and slot
        uint32_t ph = 0, pj = 1;  // full parity; parity of the slot's previous use
        // unit it - R, the one folded at iteration it (from it = R on): row
        // block and k step
        int frb = u0 / wk.KS, fks = u0 - (u0 / wk.KS) * wk.KS;
        const int last = nu + R;  // iterations nu .. nu + R - 1 only fold
        for (int it = 0; it < last; ++it) {
            const bool mine = (it & 1) == p;
            const bool fold = it >= R;  // unit it - R exists in this range
            // row-block boundary: unit it - R opens a row block
            if (fold && frb != cur_rb) {
                if (cur_rb >= 0 && !flush(cur_rb)) {
                    ok = false;
                    break;
                }
                cur_rb = frb;
#pragma unroll
                for (int i = 0; i < NN; ++i) acc[i] = 0.0f;
            }
            if (mine) {
                const bool unit = it < nu;
                const bool two = 2 * ks + 1 < G;  // unit it has its second group
                uint32_t wv[32];
                uint32_t zb0 = 0, zq0 = 0, zb1 = 0, zq1 = 0;
                float s0 = 0.0f, s1 = 0.0f;
                if (fold) {
                    // scales of the folded unit (row r), from global memory
                    const int64_t n = min(frb * kUnitRows + r, N - 1);
                    if (!W4_CHECK_WARP(n >= 0 && fks >= 0 && 2 * fks < G, status)) {
                        ok = false;
                        break;
                    }
                    const float *sp = scales + n * G + 2 * fks;
                    s0 = __ldg(sp);
                    s1 = 2 * fks + 1 < G ? __ldg(sp + 1) : 0.0f;
                }
                if (unit) {
                    if (!warp_wait(smem_u32(&sh->full[s]), ph, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint8_t *st = ring + s * C::kBytes;
                    if (!W4_CHECK_WARP(ring_ok(st, C::kBytes) && r * 128 + 128 <= kUnitBytes &&
                                           ring_ok(st + C::kZOff + 8 * r, 8),
                                       status)) {
                        ok = false;
                        break;
                    }
                    const float *zz = reinterpret_cast<const float *>(st + C::kZOff) + 2 * r;
                    zero_bias<XT>(zeros ? zz[0] : 8.0f, zb0, zq0);
                    zero_bias<XT>(zeros ? zz[1] : 8.0f, zb1, zq1);
                    // the row's 256 codes: eight swizzled 16-byte chunks
#pragma unroll
                    for (int cch = 0; cch < 8; ++cch) {
                        const uint4 v =
                            *reinterpret_cast<const uint4 *>(st + r * 128 + ((cch ^ swz) << 4));
                        wv[4 * cch] = v.x;
                        wv[4 * cch + 1] = v.y;
                        wv[4 * cch + 2] = v.z;
                        wv[4 * cch + 3] = v.w;
                    }
                }
                // the slot is free (and its partials complete) once the MMAs of
                // unit it - R are done
                if (!warp_wait(smem_u32(&sh->mdone[j]), pj, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (fold) {
                    // partial of group 0, then (when the unit has it) of group 1
                    const uint32_t td = tmem + lanebase + (uint32_t)(C::kDBase + 2 * j * NN);
                    const int ng = 2 * fks + 1 < G ? 2 : 1;
                    for (int g = 0; g < ng; ++g) {
                        const float sg = g == 0 ? s0 : s1;
#pragma unroll
                        for (int cc = 0; cc < NN / 16; ++cc) {
                            uint32_t v[16];
                            tmem_ld16(td + g * NN + 16 * cc, v);
                            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                acc[16 * cc + i] = fmaf(sg, __uint_as_float(v[i]), acc[16 * cc + i]);
                        }
                    }
                }
                if (unit) {
                    const uint32_t ta = tmem + lanebase + (uint32_t)(2 * j * kAColsPerGroup);
                    dequant8_store<XT>(ta, *reinterpret_cast<const uint32_t(*)[8]>(wv), zb0, zq0);
                    dequant8_store<XT>(ta + 32, *reinterpret_cast<const uint32_t(*)[8]>(wv + 8), zb0,
                                       zq0);
                    if (two) {
                        dequant8_store<XT>(ta + 64, *reinterpret_cast<const uint32_t(*)[8]>(wv + 16),
                                           zb1, zq1);
                        dequant8_store<XT>(ta + 96, *reinterpret_cast<const uint32_t(*)[8]>(wv + 24),
                                           zb1, zq1);
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&sh->ready[j]));
                }
            }
            // advance the cursors of unit it and of unit it - R
            if (++ks == wk.KS) ks = 0;
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
            if (++j == R) {
                j = 0;
                pj ^= 1;
            }
            if (fold && ++fks == wk.KS) {
                fks = 0;
                ++frb;
            }
        }
        if (ok && cur_rb >= 0) ok = flush(cur_rb);
        // Arrives on the counters of the split row blocks this warp stored; the
        // last warp to arrive on one adds its partials in CTA order.
        // The last warp to arrive on a split row block's counter adds the
        // partials in CTA order, writes Y and re-arms the counter.
        if (ok && p == 0 && pend0 >= 0) {
            for (int pi = 0; pi < 2; ++pi) {
                const int prb = pi == 0 ? pend0 : pend1;
                if (prb < 0) break;
                const int cf = owner(wk, prb * wk.KS), cl = owner(wk, (prb + 1) * wk.KS - 1);
                unsigned *cnt = counters + prb * 8 + q;
                const unsigned prev = __shfl_sync(0xffffffffu, pi == 0 ? prev0 : prev1, 0);
                if (prev != (unsigned)(cl - cf)) continue;
                __syncwarp();
                const int n = prb * kUnitRows + r;
                if (n < N && W4_CHECK(n >= 0 && cf >= 0 && cl < wk.P, status)) {
                    for (int m = 0; m < M; ++m) {
                        float v = 0.0f;
                        for (int cc = cf; cc <= cl; ++cc) {
                            const int sl = 2 * cc + (prb == range_start(wk, cc) / wk.KS ? 0 : 1);
                            v += __ldcg(partial + ((int64_t)sl * kUnitRows + r) * M + m);
                        }
                        store_out<XT>(Y, (int64_t)m * N + n, v);
                    }
                }
                __syncwarp();
                if (lane == 0) *cnt = 0u;  // re-arm for the next call
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
    if (gemv1_supported(M, K) || gemv_supported(M, K)) return 0;
    Work w;
    size_t b = 0;
    if (make_work(M, K, N, &w, &b) != W4_OK) return 0;
    return b;
}

int launch_decode(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                  const float *zeros, int64_t K, int64_t N, void *Y, void *workspace,
                  size_t workspace_bytes, cudaStream_t stream) {
    if (gemv1_supported(M, K)) return launch_gemv1(X, xt, packed, scales, zeros, K, N, Y, stream);
    if (gemv_supported(M, K))
        return launch_gemv(X, xt, M, packed, scales, zeros, K, N, Y, stream);
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
