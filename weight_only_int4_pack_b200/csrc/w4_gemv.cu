// w4_gemv.cu -- the W4A16 linear layer for 1 <= M <= 8 (decode), K <= 4096.
//
// Y[m][n] = sum_g scale[n][g] * sum_{k in g} X[m][k] * (u[n][k] - zero[n][g]):
// the "dequant -> 16-bit matmul" of W4A16 ("Quantization method families",
// inference-learning-path.pages.dev, §2), dequantization as in "LLM
// quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2-§2.3.  At M <= 8 the layer
// moves 0.5 byte of codes per weight and does M multiply-adds per weight: it
// is bound by HBM.  Everything here serves that bound:
//
//   * Weight rows are split evenly over one CTA per SM (whole rows, no split
//     of K across CTAs, no workspace).  A CTA cuts its rows into tiles of 16
//     rows.  Its eight warps share each tile, each owning one eighth of K
//     (its groups), and reduce their partial sums through shared memory in
//     warp order (deterministic) once per tile.
//   * Streaming: every lane fetches exactly the code bytes its tensor-core
//     operands need (16 bytes of two rows per group) with 16-byte cp.async
//     into its warp's own four-stage shared-memory ring, together with the
//     tile's scales and zero points; a lane later reads back only what its
//     own quad loaded.  So up to four tiles per warp (144 KB per SM) are in
//     flight without holding registers and without a producer thread, and the
//     reads of a stage need no barrier beyond cp.async.wait_group and a warp
//     sync.  (Measured on B200: 16-byte per-thread copies keep HBM busier than
//     1-D bulk copies of a few KB, whose per-copy cost caps the stream.)
//   * The multiply-adds run on the tensor cores, warp by warp
//     (mma.sync m16n8k16, fp32 accumulation): A = 16 weight rows x 16 k, B =
//     16 k x 8 columns holding the M activation rows (zero past M).  Each warp
//     stays independent of the others -- no tensor-memory round trip, no
//     CTA-wide MMA issue -- so a tile's compute is one warp's instruction
//     stream.  The codes become A operands with one logic op per pair:
//       fp16: the code bits ARE an fp16 number when placed in the low mantissa
//             bits with a zero exponent: u * 2^-24 (a subnormal, exact), or
//             16u * 2^-24 for the high nibble of a byte, so no code needs a
//             shift except every second byte; the products x * u * 2^-24 are
//             exact in fp32 and the group sum is rescaled by 2^24 exactly.
//       bf16: the bits are placed in the mantissa of 128.0 (128 + u, exact)
//             and 136 is subtracted (u - 8, exact); the fold adds 8 back.
//     The zero point is applied once per group with the group sums of x:
//       sum x (u - z) = sum x u - z sum x.
//     No weight is rounded to 16 bits: (u - 8) and u * 2^-24 are exact.
//   * Per group and row the fp32 partial gets its scale (s * partial) and is
//     added to the row's fp32 sum, which is rounded once to the output dtype.
//   * Programmatic dependent launch: the first tiles are requested and the
//     next kernel is released before griddepcontrol.wait; X and Y are touched
//     only after it (weights -- codes, scales, zero points -- before).
//
// The kernel has no unbounded wait: cp.async groups complete on their own,
// the CTA-wide bar.sync are reached by every warp, and the one spin (a warp
// kSlots tiles ahead waiting for a reduction slot) is bounded: when it runs
// out it sets the library's status word (W4_ERR_TIMEOUT).  The W4_DEBUG build
// checks every global and shared-memory index and copy (w4_debug.cuh).

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_debug.cuh"
#include "w4_half.cuh"
#include "w4_internal.cuh"
#include "w4_tc.cuh"

namespace w4 {
namespace {

[[maybe_unused]] constexpr unsigned kDbgFile = 4;  // W4_DEBUG file id

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 16;          // weight rows per tile (the MMA's M)
constexpr int kDepth = 2;          // tiles in flight per warp
constexpr int kGPW = 32 / kWarps;  // groups per warp at most (K <= 4096)
constexpr int kMaxK = kGPW * kWarps * 128;
constexpr int kSlots = 4;          // tiles whose partial sums may be pending
constexpr int kMaxM = 8;
constexpr int kGroup = 128;

// Per-warp stage: codes [kGPW][16 rows][64 B], scales [kGPW][16], zeros [kGPW][16].
constexpr int kStageCodes = kGPW * kTile * 64;
constexpr int kStageBytes = kStageCodes + 2 * kGPW * kTile * 4;

// Shared-memory layout (bytes), the same on host and device.
struct Layout {
    int ring;   // kWarps x kDepth stages
    int x;      // X: M rows (permuted, see below), stride XS
    int XS;
    int tab;    // group sums of x: [G][8] fp32
    int red;    // partial sums: [kSlots][kWarps][32 lanes][4] fp32
    int sync;   // per slot: generation, arrivals (unsigned)
    int total;
};

__host__ __device__ inline Layout layout(int K, int M) {
    Layout L;
    const int G = K / kGroup;
    L.ring = 0;
    L.x = kWarps * kDepth * kStageBytes;
    L.XS = 2 * K + 32;
    L.tab = L.x + M * L.XS;
    L.red = L.tab + G * 8 * 4;
    L.sync = L.red + kSlots * kWarps * 32 * 16;
    L.total = L.sync + 2 * kSlots * 4;
    return L;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}

__device__ __forceinline__ float2 lds64f(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
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

__device__ __forceinline__ void cta_sync() { asm volatile("bar.sync 0;" ::: "memory"); }

// One step of a group: the code words w0 (row gq) and w1 (row gq + 8) of the
// lane's slice word j become the A operands of two m16n8k16 MMAs (fp32
// accumulation in place).  The word holds k = 8j + {0,2,4,6,1,3,5,7} in
// nibbles 0..7, so masking pairs (k, k+1) into the two halves of a register:
//   0x000F000F -> (8j, 8j+1), on the word >> 8 -> (8j+4, 8j+5)   [class A]
//   0x00F000F0 -> (8j+2, 8j+3), on the word >> 8 -> (8j+6, 8j+7) [class B]
// fp16: those bits, with a zero exponent, are the fp16 numbers u * 2^-24
// (class A) and 16u * 2^-24 (class B), exact subnormals; dA and dB collect
// 2^-24 sum x u and 2^-24 sum x 16u.
// bf16: the bits go into the mantissa of 128.0 (128 + u) and 136 is
// subtracted (u - 8, exact); dA and dB both collect sum x (u - 8).
// Logical k (2t, 2t+1) of the MMA is physical 32t + 8j + {0,1} (class A) or
// + {2,3} (class B); logical (2t+8, 2t+9) is + {4,5} or + {6,7}; xa / xb are
// the matching activation pairs (B operand, column gq).
template <int XT>
__device__ __forceinline__ void step(float (&dA)[4], float (&dB)[4], uint32_t w0, uint32_t w1,
                                     uint32_t xa0, uint32_t xa1, uint32_t xb0, uint32_t xb1) {
    if (XT == W4_F16)
        asm("{\n\t.reg .b32 a0, a1, a2, a3, b0, b1, b2, b3, h0, h1;\n\t"
            "shr.b32 h0, %8, 8;\n\t"
            "shr.b32 h1, %9, 8;\n\t"
            "and.b32 a0, %8, 0x000F000F;\n\t"
            "and.b32 a1, %9, 0x000F000F;\n\t"
            "and.b32 a2, h0, 0x000F000F;\n\t"
            "and.b32 a3, h1, 0x000F000F;\n\t"
            "and.b32 b0, %8, 0x00F000F0;\n\t"
            "and.b32 b1, %9, 0x00F000F0;\n\t"
            "and.b32 b2, h0, 0x00F000F0;\n\t"
            "and.b32 b3, h1, 0x00F000F0;\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {a0,a1,a2,a3}, "
            "{%10,%11}, {%0,%1,%2,%3};\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%4,%5,%6,%7}, {b0,b1,b2,b3}, "
            "{%12,%13}, {%4,%5,%6,%7};\n\t}"
            : "+f"(dA[0]), "+f"(dA[1]), "+f"(dA[2]), "+f"(dA[3]), "+f"(dB[0]), "+f"(dB[1]),
              "+f"(dB[2]), "+f"(dB[3])
            : "r"(w0), "r"(w1), "r"(xa0), "r"(xa1), "r"(xb0), "r"(xb1));
    else
        asm("{\n\t.reg .b32 a0, a1, a2, a3, b0, b1, b2, b3, h0, h1, m, o;\n\t"
            "mov.b32 m, 0x43004300;\n\t"
            "mov.b32 o, 0x43084308;\n\t"
            "lop3.b32 a0, %8, 0x000F000F, m, 0xEA;\n\t"
            "lop3.b32 a1, %9, 0x000F000F, m, 0xEA;\n\t"
            "shr.b32 h0, %8, 4;\n\t"
            "shr.b32 h1, %9, 4;\n\t"
            "lop3.b32 b0, h0, 0x000F000F, m, 0xEA;\n\t"
            "lop3.b32 b1, h1, 0x000F000F, m, 0xEA;\n\t"
            "shr.b32 h0, %8, 8;\n\t"
            "shr.b32 h1, %9, 8;\n\t"
            "lop3.b32 a2, h0, 0x000F000F, m, 0xEA;\n\t"
            "lop3.b32 a3, h1, 0x000F000F, m, 0xEA;\n\t"
            "shr.b32 h0, %8, 12;\n\t"
            "shr.b32 h1, %9, 12;\n\t"
            "lop3.b32 b2, h0, 0x000F000F, m, 0xEA;\n\t"
            "lop3.b32 b3, h1, 0x000F000F, m, 0xEA;\n\t"
            "sub.rn.bf16x2 a0, a0, o;\n\t"
            "sub.rn.bf16x2 a1, a1, o;\n\t"
            "sub.rn.bf16x2 a2, a2, o;\n\t"
            "sub.rn.bf16x2 a3, a3, o;\n\t"
            "sub.rn.bf16x2 b0, b0, o;\n\t"
            "sub.rn.bf16x2 b1, b1, o;\n\t"
            "sub.rn.bf16x2 b2, b2, o;\n\t"
            "sub.rn.bf16x2 b3, b3, o;\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {a0,a1,a2,a3}, "
            "{%10,%11}, {%0,%1,%2,%3};\n\t"
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%4,%5,%6,%7}, {b0,b1,b2,b3}, "
            "{%12,%13}, {%4,%5,%6,%7};\n\t}"
            : "+f"(dA[0]), "+f"(dA[1]), "+f"(dA[2]), "+f"(dA[3]), "+f"(dB[0]), "+f"(dB[1]),
              "+f"(dB[2]), "+f"(dB[3])
            : "r"(w0), "r"(w1), "r"(xa0), "r"(xa1), "r"(xb0), "r"(xb1));
}

template <int XT>
__global__ void __launch_bounds__(kThreads, 2)
    gemv_kernel(const uint8_t *__restrict__ packed, const float *__restrict__ scales,
                const float *__restrict__ zeros, const uint16_t *__restrict__ X,
                uint16_t *__restrict__ Y, int M, int K, int N, unsigned *status) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int G = K / kGroup;
    const int kb = K / 2;
    const bool asym = zeros != nullptr;
    const Layout L = layout(K, M);
    const uint32_t sb = tc::smem_u32(smem);

    // rows of this CTA, in tiles of 16
    const int64_t P = gridDim.x;
    const int r0 = static_cast<int>(static_cast<int64_t>(N) * blockIdx.x / P);
    const int r1 = static_cast<int>(static_cast<int64_t>(N) * (blockIdx.x + 1) / P);
    const int ntile = (r1 - r0 + kTile - 1) / kTile;

    const int gq = lane >> 2;  // A rows gq and gq + 8; B column (activation row) gq
    const int t = lane & 3;    // k slice [32t, 32t + 32) of each group
    const int gA = warp * G / kWarps;
    const int ng = (warp + 1) * G / kWarps - gA;  // groups of this warp, 0 .. kGPW
    const uint32_t ring = sb + L.ring + warp * (kDepth * kStageBytes);

    // this lane's copies: 16 bytes of rows gq and gq + 8 per group, stored at
    // [group][row][16t] (the reads of a quarter warp cover 128 contiguous
    // bytes), and, for t < ng, the scale and zero point of group gA + t
    const uint8_t *pa = packed + static_cast<int64_t>(r0 + gq) * kb + gA * 64 + 16 * t;
    const int64_t tile_bytes = static_cast<int64_t>(kTile) * kb;
    const uint32_t ca = (gq * 64 + 16 * t), cb = ca + 8 * 64;  // + gi * kTile * 64
    const float *sp = scales + static_cast<int64_t>(r0 + gq) * G + gA + t;
    const float *zp = asym ? zeros + static_cast<int64_t>(r0 + gq) * G + gA + t : nullptr;
    const int64_t tile_gs = static_cast<int64_t>(kTile) * G;
    const uint32_t sza = kStageCodes + t * kTile * 4 + gq * 4;

    auto issue = [&](int i) {
        if (i < ntile) {
            const uint32_t st = ring + (i % kDepth) * kStageBytes;
            const int ra = r0 + i * kTile + gq;
            const bool oka = ra < r1, okb = ra + 8 < r1;
            const uint8_t *qa = pa + i * tile_bytes, *qb = qa + 8 * static_cast<int64_t>(kb);
            if (!W4_CHECK(ra >= 0 && (!oka || ra < N) && (!okb || ra + 8 < N) && gA + ng <= G &&
                              in_range(st, kStageBytes, sb, dyn_smem_bytes()) &&
                              in_range(st, kStageBytes, sb + L.ring, L.x - L.ring),
                          status)) {
                cp_async_commit();
                return;
            }
#pragma unroll
            for (int gi = 0; gi < kGPW; ++gi) {
                if (gi < ng) {
                    if (oka) cp_async16(st + gi * (kTile * 64) + ca, qa + gi * 64);
                    if (okb) cp_async16(st + gi * (kTile * 64) + cb, qb + gi * 64);
                }
            }
            if (t < ng) {
                const float *s_a = sp + i * tile_gs, *s_b = s_a + 8 * static_cast<int64_t>(G);
                if (oka) cp_async4(st + sza, s_a);
                if (okb) cp_async4(st + sza + 32, s_b);
                if (asym) {
                    const float *z_a = zp + i * tile_gs, *z_b = z_a + 8 * static_cast<int64_t>(G);
                    if (oka) cp_async4(st + sza + kGPW * kTile * 4, z_a);
                    if (okb) cp_async4(st + sza + kGPW * kTile * 4 + 32, z_b);
                }
            }
        }
        cp_async_commit();
    };

    // the first tiles' weights before waiting for the previous kernel
#pragma unroll
    for (int i = 0; i < kDepth - 1; ++i) issue(i);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // X -> shared memory.  Row m at m * XS; within group g (256 bytes) the
    // 16-byte piece w4 (k 8*w4 .. +7) of lane t's 32-k slice (bytes 64t..) is
    // stored at 64t + 16 * (w4 ^ (t >> 1)), so that the lanes of a quarter
    // warp reading piece w4 of their slices hit different bank quads, with its
    // words in the order (k, k+1), (k+4, k+5), (k+2, k+3), (k+6, k+7): the
    // B operands of the two MMAs of a slice word are then adjacent.  Then
    // the group sums of x: tab[g][m] = sum_{k in g} x[m][k] (times 2^-24 for
    // fp16, the scale of the fp16 code operand); zero for m >= M.
    const int KC = K / 8;
    for (int e = threadIdx.x; e < M * KC; e += kThreads) {
        const int m = e / KC, kc = e - m * KC;
        const int g = kc >> 4, tt = (kc >> 2) & 3, w4 = kc & 3;
        const uint32_t a = sb + L.x + m * L.XS + g * 256 + tt * 64 + ((w4 ^ (tt >> 1)) << 4);
        if (!W4_CHECK(m < M && kc < KC && in_range(a, 16, sb + L.x, L.tab - L.x), status)) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<int64_t>(m) * K) + kc);
        sts128(a, make_uint4(v.x, v.z, v.y, v.w));
    }
    cta_sync();
    // entries (g, m), m < M, one thread each, from the shared copy of x (the
    // sum order is fixed: pieces in k order, pairs within a piece in k order)
    float *tab = reinterpret_cast<float *>(smem + L.tab);
    for (int e = threadIdx.x; e < G * M; e += kThreads) {
        const int g = e / M, m = e - g * M;
        float acc = 0.f;
#pragma unroll 4
        for (int c = 0; c < kGroup / 8; ++c) {
            const int tt = c >> 2, w4 = c & 3;
            const uint4 v = lds128(sb + L.x + m * L.XS + g * 256 + tt * 64 + ((w4 ^ (tt >> 1)) << 4));
            float f[8];
            widen8<XT>(v, f);  // words stored as (k,k+1), (k+4,k+5), (k+2,k+3), (k+6,k+7)
            acc += ((f[0] + f[1]) + (f[4] + f[5])) + ((f[2] + f[3]) + (f[6] + f[7]));
        }
        if (W4_CHECK(g < G && m < 8, status)) tab[g * 8 + m] = XT == W4_F16 ? acc * 0x1p-24f : acc;
    }
    for (int e = threadIdx.x; e < G * 8; e += kThreads)
        if ((e & 7) >= M) tab[e] = 0.f;
    if (threadIdx.x < 2 * kSlots) reinterpret_cast<unsigned *>(smem + L.sync)[threadIdx.x] = 0;
    cta_sync();

    // the group sums of columns 2t, 2t + 1 of the warp's groups, in registers;
    // the B fragments (activation row gq, this lane's 32-k slice) are read
    // from shared memory per group by the lanes with gq < M
    float S0[kGPW], S1[kGPW];
#pragma unroll
    for (int gi = 0; gi < kGPW; ++gi) {
        const float2 Sv = gi < ng ? lds64f(sb + L.tab + ((gA + gi) * 8 + 2 * t) * 4) : make_float2(0.f, 0.f);
        S0[gi] = Sv.x;
        S1[gi] = Sv.y;
    }
    // lanes whose activation row is past M read row 0 and zero it
    const uint32_t xmask = gq < M ? 0xFFFFFFFFu : 0u;
    const uint32_t xrow = sb + L.x + (gq < M ? gq : 0) * L.XS + t * 64;
    uint32_t xoff[4];
#pragma unroll
    for (int w4 = 0; w4 < 4; ++w4) xoff[w4] = static_cast<uint32_t>((w4 ^ (t >> 1)) << 4);

    for (int i = 0; i < ntile; ++i) {
        issue(i + kDepth - 1);
        cp_async_wait<kDepth - 1>();  // tile i has landed (this lane's copies)
        __syncwarp();                 // ... and the quad's scales / zero points
        const uint32_t st = ring + (i % kDepth) * kStageBytes;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int gi = 0; gi < kGPW; ++gi) {
            if (gi < ng) {
                const uint32_t ss = st + sza - t * kTile * 4 + gi * kTile * 4 - gq * 4;
                // the lane's code reads, its x reads (pieces xoff[0..3] = [0, 64)
                // of its slice), its scale and zero-point reads; one vote for
                // the warp, whose MMAs below are warp-collective
                if (!W4_CHECK_WARP(in_range(st + gi * (kTile * 64) + ca, 16, st, kStageCodes) &&
                                       in_range(st + gi * (kTile * 64) + cb, 16, st, kStageCodes) &&
                                       in_range(xrow + (gA + gi) * 256, 64, sb + L.x, L.tab - L.x) &&
                                       in_range(ss + gq * 4, 4, st + kStageCodes, kGPW * kTile * 4) &&
                                       in_range(ss + (gq + 8) * 4, 4, st + kStageCodes, kGPW * kTile * 4) &&
                                       in_range(ss + kGPW * kTile * 4 + (gq + 8) * 4, 4,
                                                st + kStageCodes + kGPW * kTile * 4, kGPW * kTile * 4),
                                   status))
                    continue;
                const uint4 c0 = lds128(st + gi * (kTile * 64) + ca);
                const uint4 c1 = lds128(st + gi * (kTile * 64) + cb);
                // activation pairs of the 4 slice words, stored per 16-byte
                // piece as (8j,8j+1), (8j+4,8j+5), (8j+2,8j+3), (8j+6,8j+7)
                uint4 xv[4];
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) {
                    const uint4 v = lds128(xrow + (gA + gi) * 256 + xoff[w4]);
                    xv[w4] = make_uint4(v.x & xmask, v.y & xmask, v.z & xmask, v.w & xmask);
                }
                const uint32_t cw0[4] = {c0.x, c0.y, c0.z, c0.w}, cw1[4] = {c1.x, c1.y, c1.z, c1.w};
                float dA[4] = {0.f, 0.f, 0.f, 0.f}, dB[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    step<XT>(dA, dB, cw0[j], cw1[j], xv[j].x, xv[j].y, xv[j].z, xv[j].w);
                // fold: y[r][n] += s_r * (sum x u - z_r sum x)
                const float s0 = lds32f(ss + gq * 4), s1 = lds32f(ss + (gq + 8) * 4);
                float z0 = 8.f, z1 = 8.f;
                if (asym) {
                    z0 = lds32f(ss + kGPW * kTile * 4 + gq * 4);
                    z1 = lds32f(ss + kGPW * kTile * 4 + (gq + 8) * 4);
                }
                float w[4];
                if (XT == W4_F16) {
                    // dA = 2^-24 sum x u (pairs 0, 2), dB = 2^-24 sum x 16u (pairs 1, 3)
#pragma unroll
                    for (int v = 0; v < 4; ++v) w[v] = fmaf(dB[v], 0.0625f, dA[v]);
                } else {
                    // both = sum x (u - 8)
#pragma unroll
                    for (int v = 0; v < 4; ++v) w[v] = dA[v] + dB[v];
                    z0 -= 8.f;
                    z1 -= 8.f;
                }
                const float e0 = XT == W4_F16 ? s0 * 0x1p24f : s0;
                const float e1 = XT == W4_F16 ? s1 * 0x1p24f : s1;
                y[0] = fmaf(e0, fmaf(-z0, S0[gi], w[0]), y[0]);
                y[1] = fmaf(e0, fmaf(-z0, S1[gi], w[1]), y[1]);
                y[2] = fmaf(e1, fmaf(-z1, S0[gi], w[2]), y[2]);
                y[3] = fmaf(e1, fmaf(-z1, S1[gi], w[3]), y[3]);
            }
        }
        // K-split reduction without a CTA barrier: the warp stores its partial
        // in slot i % kSlots, and the last of the kWarps warps to arrive adds
        // the partials in warp order (deterministic) and writes the tile.  A
        // slot is reused for tile i + kSlots only after that reduction has
        // read it (its generation count has advanced).
        const int slot = i % kSlots;
        volatile unsigned *gen = reinterpret_cast<volatile unsigned *>(smem + L.sync) + slot;
        unsigned *arrive = reinterpret_cast<unsigned *>(smem + L.sync) + kSlots + slot;
        const unsigned want = static_cast<unsigned>(i / kSlots);
        if (*gen != want) {  // a warp kSlots tiles ahead of the slowest one
            const unsigned long long t0 = tc::globaltimer();
            while (*gen != want) {
                if (tc::globaltimer() - t0 > tc::kWaitNs) {
                    if (lane == 0) atomicOr(status, 1u);
                    break;
                }
            }
        }
        const uint32_t sl = sb + L.red + slot * (kWarps * 32 * 16);
        if (!W4_CHECK_WARP(in_range(sl + (warp * 32 + lane) * 16, 16, sb + L.red, L.sync - L.red), status))
            continue;
        sts128(sl + (warp * 32 + lane) * 16, make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]),
                                                        __float_as_uint(y[2]), __float_as_uint(y[3])));
        __syncwarp();
        unsigned old = 0;
        if (lane == 0) {
            __threadfence_block();
            old = atomicAdd(arrive, 1u);
        }
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old % kWarps == kWarps - 1) {
            __threadfence_block();
            float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ww = 0; ww < kWarps; ++ww) {
                const uint4 v = lds128(sl + (ww * 32 + lane) * 16);
                a[0] += __uint_as_float(v.x);
                a[1] += __uint_as_float(v.y);
                a[2] += __uint_as_float(v.z);
                a[3] += __uint_as_float(v.w);
            }
            const int row0 = r0 + i * kTile;
            const int ra = row0 + gq, rbw = row0 + gq + 8;
            const int m0 = 2 * t, m1 = 2 * t + 1;
            if (ra < r1 && W4_CHECK(ra >= 0 && ra < N, status)) {
                if (m0 < M) Y[static_cast<int64_t>(m0) * N + ra] = narrow1<XT>(a[0]);
                if (m1 < M) Y[static_cast<int64_t>(m1) * N + ra] = narrow1<XT>(a[1]);
            }
            if (rbw < r1 && W4_CHECK(rbw >= 0 && rbw < N, status)) {
                if (m0 < M) Y[static_cast<int64_t>(m0) * N + rbw] = narrow1<XT>(a[2]);
                if (m1 < M) Y[static_cast<int64_t>(m1) * N + rbw] = narrow1<XT>(a[3]);
            }
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                *gen = want + 1;
            }
        }
        // this warp's reads of the stage are done before the next issue
        // overwrites it (issue(i + kDepth) targets stage i % kDepth)
        __syncwarp();
    }
    cp_async_wait<0>();
}

template <int XT>
int launch_t(const uint8_t *packed, const float *scales, const float *zeros, const void *X,
             void *Y, int M, int K, int N, int grid, cudaStream_t stream) {
    auto kern = gemv_kernel<XT>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(W4_ERR_CUDA, "cudaGetDevice", nullptr);
    static bool attr_done[64] = {};
    if (!attr_done[dev]) {
        const int most = layout(kMaxK, kMaxM).total;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(gemv smem)", e);
        attr_done[dev] = true;
    }
    unsigned *status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = layout(K, M).total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, packed, scales, zeros,
                                       static_cast<const uint16_t *>(X), static_cast<uint16_t *>(Y),
                                       M, K, N, status);
    if (e != cudaSuccess) return cuda_fail("cudaLaunchKernelEx(gemv)", e);
    return W4_OK;
}

}  // namespace

bool gemv_supported(int64_t M, int64_t K) {
    return M >= 1 && M <= kMaxM && K >= kGroup && K <= kMaxK && K % kGroup == 0;
}

int launch_gemv(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                const float *zeros, int64_t K, int64_t N, void *Y, cudaStream_t stream) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    if (di.cc_major != 10) return set_error(W4_ERR_UNSUPPORTED, "w4a16_gemm", "needs an sm_100 GPU");
    const int grid = static_cast<int>(N < di.sm_count ? N : di.sm_count);
    if (xt == W4_F16)
        return launch_t<W4_F16>(packed, scales, zeros, X, Y, (int)M, (int)K, (int)N, grid, stream);
    return launch_t<W4_BF16>(packed, scales, zeros, X, Y, (int)M, (int)K, (int)N, grid, stream);
}

}  // namespace w4
