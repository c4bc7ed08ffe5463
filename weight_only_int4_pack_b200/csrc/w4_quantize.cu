// w4_quantize.cu -- per-group INT4 round-to-nearest quantization + nibble packing.
//
// Method: "LLM quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2 (symmetric / asymmetric
// integer quantization with scale, zero point, round and clamp) and §2.3
// (one scale per group of `group` consecutive in_features), with the AWQ
// column factor of §4.2 folded in first when given.  Every weight is
// rounded on its own ("PTQ weight quantization: from GPTQ to AWQ",
// section "Round-to-Nearest").
//
// Results are bit-identical to the plain definition computed with IEEE fp32
// division: s and the zero point use correctly rounded division; each code
// is first obtained from a reciprocal multiply and is recomputed with the
// correctly rounded division whenever that product lies within DELTA of a
// rounding boundary (k + 1/2).  The bound on |fast - exact| is derived in the
// comment of `codes_fast`.
//
// Work layout: a CTA of 128 threads owns a strip of 2048 consecutive k and
// walks down RT rows of it.  Thread t covers k = 16t..16t+15 of the strip:
// two 16-byte loads of sixteen 16-bit weights and two 32-bit packed words per
// row, so the per-group work (the reduction, the scale and zero point, the
// reciprocal) is shared by sixteen weights per thread.  GROUP/16 adjacent
// lanes form one group and reduce its amax (or min/max) with butterfly
// shuffles.  A warp writes 256 contiguous bytes of codes per row; the strip's
// scales and zeros of a row are contiguous too.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <float.h>

#include "w4_debug.cuh"
#include "w4_internal.cuh"

namespace w4 {
namespace {

[[maybe_unused]] constexpr unsigned kDbgFile = 1;  // W4_DEBUG file id

constexpr int kThreads = 128;
constexpr int kPer = 16;                // consecutive k per thread
constexpr int kStripK = kThreads * kPer;  // 2048 k per CTA tile
constexpr int kRowsPerTile = 32;
constexpr int kRowUnroll = 4;

// 1.5 * 2^23: adding it to |y| < 2^22 rounds y to an integer (ties to even)
// and leaves that integer in the low mantissa bits.
constexpr float kMagic = 12582912.0f;
// Half-width of the band around k + 1/2 in which the reciprocal-multiply
// result is not trusted (see codes_fast).
constexpr float kDelta = 1.52587890625e-05f;  // 2^-16

template <int WT>
__device__ __forceinline__ void load8(const uint4 v, float w[8]) {
    const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (WT == W4_F16) {
            __half2 h = *reinterpret_cast<const __half2 *>(&r[i]);
            float2 f = __half22float2(h);
            w[2 * i] = f.x;
            w[2 * i + 1] = f.y;
        } else {
            w[2 * i] = __uint_as_float(r[i] << 16);
            w[2 * i + 1] = __uint_as_float(r[i] & 0xFFFF0000u);
        }
    }
}

// Packs the low nibbles of bits[0..7] (k = 0..7 of the word) in the library's
// order: nibble i holds k = {0,2,4,6,1,3,5,7}[i].  Byte 1 of every bits[] is
// zero (bits = 0x4B4000uu), so PRMT can pull zeros from it.
__device__ __forceinline__ uint32_t pack8(const uint32_t b[8]) {
    // x_ab = u_a | u_b << 16
    const uint32_t x01 = __byte_perm(b[0], b[1], 0x1410);
    const uint32_t x23 = __byte_perm(b[2], b[3], 0x1410);
    const uint32_t x45 = __byte_perm(b[4], b[5], 0x1410);
    const uint32_t x67 = __byte_perm(b[6], b[7], 0x1410);
    // nibbles: 0:k0 1:k2 2:k4 3:k6 4:k1 5:k3 6:k5 7:k7
    return x01 | (x23 << 4) | (x45 << 8) | (x67 << 12);
}

// Packed pairs of fp32 (the f32x2 instructions of sm_100a: one instruction,
// two independent IEEE operations rounded to nearest even, exactly as the
// scalar forms).
__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Codes of eight weights with the group's s (>= FLT_MIN), r = rcp_rn(s) and
// zero point zp (0 for symmetric, which then adds 8 through the magic).
//
// Error bound.  Let A = fl(w/s) and the exact target B = fl(A + zp) (sym: B = A).
// The fast value is y = fl(w*r + zp) (one FMA; sym: fl(w*r)), with
// r = (1/s)(1+e_r), |e_r| <= 2^-24.  Where the result can still change
// (|y| < 32), |y - B| <= 2*2^-24*|w/s| + ulp(32)/2 + ulp(32)/2
//                    <= 2*2^-24*31 + 2^-19 < 5.6e-6 < kDelta / 2.
// So if y is farther than kDelta from every k + 1/2, B lies on the same side
// of every rounding boundary and rne(B) = rne(y).  Values beyond the clamp
// range round to the clamp bound either way, so clamping y first is exact
// (rne is monotone and 0, 15 are integers).  Symmetric groups need no clamp:
// s >= amax/7 * (1 - 2^-24) keeps |y| < 7.5.
// The arithmetic runs on pairs (f32x2): y, m = y + magic and d = y - (m - magic).
template <bool SYM>
__device__ __forceinline__ bool codes_fast(const float w[8], float r, float zp, uint32_t bits[8]) {
    bool near = false;
    const float magic = SYM ? kMagic + 8.0f : kMagic;
    const uint64_t r2 = pk2(r, r), z2 = pk2(zp, zp), g2 = pk2(magic, magic);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint64_t w2 = pk2(w[2 * p], w[2 * p + 1]);
        uint64_t y2;
        if (SYM) {
            y2 = mul2(w2, r2);
        } else {
            float y0, y1;
            upk2(fma2(w2, r2, z2), y0, y1);
            y2 = pk2(fminf(fmaxf(y0, 0.0f), 15.0f), fminf(fmaxf(y1, 0.0f), 15.0f));
        }
        const uint64_t m2 = add2(y2, g2);
        float d0, d1, m0, m1;
        upk2(sub2(y2, sub2(m2, g2)), d0, d1);
        near |= fabsf(d0) > 0.5f - kDelta;
        near |= fabsf(d1) > 0.5f - kDelta;
        upk2(m2, m0, m1);
        bits[2 * p] = __float_as_uint(m0);  // 0x4B4000uu, uu = code
        bits[2 * p + 1] = __float_as_uint(m1);
    }
    return near;
}

// The plain definition with correctly rounded division (rare path).
template <bool SYM>
__device__ __forceinline__ void codes_exact(const float w[8], float s, float zp, uint32_t bits[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float a = __fdiv_rn(w[j], s);
        int u;
        if (SYM) {
            u = static_cast<int>(fminf(fmaxf(rintf(a), -7.0f), 7.0f)) + 8;
        } else {
            const float b = __fadd_rn(a, zp);
            u = static_cast<int>(fminf(fmaxf(rintf(b), 0.0f), 15.0f));
        }
        bits[j] = 0x4B400000u | static_cast<uint32_t>(u);
    }
}

template <int WT, int GROUP, bool SYM, bool FOLD>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const uint16_t *__restrict__ W, int64_t K, int64_t N,
                const float *__restrict__ col_scale, uint32_t *__restrict__ packed,
                float *__restrict__ scales, float *__restrict__ zeros, int64_t tiles_k,
                int64_t tiles, unsigned *status) {
    constexpr int LPG = GROUP / kPer;  // lanes per group (2, 4, 8 or 16)
    const int t = threadIdx.x;
    const int lane = t & 31;
    const int64_t G = K / GROUP;

    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t kb = tile % tiles_k;
        const int64_t rb = tile / tiles_k;
        const int64_t k = kb * kStripK + kPer * t;
        const bool valid_k = k < K;  // uniform over each group since K % GROUP == 0
        float cs[kPer];
        if (FOLD) {
#pragma unroll
            for (int j = 0; j < kPer; ++j) cs[j] = 1.0f;
            if (valid_k && W4_CHECK(k >= 0 && k + kPer <= K, status)) {
#pragma unroll
                for (int v = 0; v < kPer / 4; ++v) {
                    const float4 c = __ldg(reinterpret_cast<const float4 *>(col_scale + k) + v);
                    cs[4 * v] = c.x; cs[4 * v + 1] = c.y; cs[4 * v + 2] = c.z; cs[4 * v + 3] = c.w;
                }
            }
        }
        const int64_t row0 = rb * kRowsPerTile;
        for (int rr = 0; rr < kRowsPerTile; rr += kRowUnroll) {
            if (row0 + rr >= N) break;  // uniform over the CTA
            uint4 raw[kRowUnroll][2];
#pragma unroll
            for (int i = 0; i < kRowUnroll; ++i) {
                const int64_t row = row0 + rr + i;
                raw[i][0] = raw[i][1] = make_uint4(0, 0, 0, 0);
                if (valid_k && row < N &&
                    W4_CHECK(row >= 0 && k >= 0 && k + kPer <= K && (k & 7) == 0, status)) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(W + row * K + k);
                    raw[i][0] = __ldcs(src);
                    raw[i][1] = __ldcs(src + 1);
                }
            }
#pragma unroll
            for (int i = 0; i < kRowUnroll; ++i) {
                const int64_t row = row0 + rr + i;
                if (row >= N) break;  // uniform
                float w[kPer];
                load8<WT>(raw[i][0], w);
                load8<WT>(raw[i][1], w + 8);
                if (FOLD) {
#pragma unroll
                    for (int j = 0; j < kPer; j += 2)
                        upk2(mul2(pk2(w[j], w[j + 1]), pk2(cs[j], cs[j + 1])), w[j], w[j + 1]);
                }
                float s, zp;
                if (SYM) {
                    float a = fabsf(w[0]);
#pragma unroll
                    for (int j = 1; j < kPer; ++j) a = fmaxf(a, fabsf(w[j]));
#pragma unroll
                    for (int off = LPG / 2; off >= 1; off >>= 1)
                        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
                    s = __fdiv_rn(a, 7.0f);
                    zp = 8.0f;
                } else {
                    float mn = w[0], mx = w[0];
#pragma unroll
                    for (int j = 1; j < kPer; ++j) {
                        mn = fminf(mn, w[j]);
                        mx = fmaxf(mx, w[j]);
                    }
#pragma unroll
                    for (int off = LPG / 2; off >= 1; off >>= 1) {
                        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    }
                    s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
                    zp = 0.0f;
                    // "+ 0" stores an integer zero point of 0 as +0.0, never -0.0
                    if (s != 0.0f)
                        zp = __fadd_rn(fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.0f), 15.0f), 0.0f);
                }
                uint32_t bits[kPer];
                if (s == 0.0f) {
                    const uint32_t u = 0x4B400000u | static_cast<uint32_t>(zp);
#pragma unroll
                    for (int j = 0; j < kPer; ++j) bits[j] = u;
                } else {
                    const float r = __frcp_rn(s);
                    const bool fast_ok = s >= FLT_MIN;
                    const bool near0 = codes_fast<SYM>(w, r, SYM ? 0.0f : zp, bits);
                    const bool near1 = codes_fast<SYM>(w + 8, r, SYM ? 0.0f : zp, bits + 8);
                    if (near0 || !fast_ok) codes_exact<SYM>(w, s, zp, bits);
                    if (near1 || !fast_ok) codes_exact<SYM>(w + 8, s, zp, bits + 8);
                }
                if (valid_k &&
                    W4_CHECK(row >= 0 && row < N && k >= 0 && k + kPer <= K && ((row * K + k) & 15) == 0,
                             status)) {
                    reinterpret_cast<uint2 *>(packed)[(row * K + k) >> 4] =
                        make_uint2(pack8(bits), pack8(bits + 8));
                    if ((lane % LPG) == 0) {
                        const int64_t gi = row * G + k / GROUP;
                        if (W4_CHECK(gi >= 0 && gi < N * G, status)) {
                            scales[gi] = s;
                            zeros[gi] = zp;
                        }
                    }
                }
            }
        }
    }
}

template <int WT, int GROUP, bool SYM, bool FOLD>
int launch_t(const void *W, int64_t K, int64_t N, const float *col_scale, uint8_t *packed,
             float *scales, float *zeros, cudaStream_t stream) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    auto kern = quantize_kernel<WT, GROUP, SYM, FOLD>;
    static int blocks_per_sm = 0;  // same for every device of one architecture
    if (blocks_per_sm == 0) {
        int b = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, kThreads, 0);
        if (e != cudaSuccess) return cuda_fail("cudaOccupancyMaxActiveBlocksPerMultiprocessor", e);
        blocks_per_sm = b > 0 ? b : 1;
    }
    const int64_t tiles_k = (K + kStripK - 1) / kStripK;
    const int64_t tiles = tiles_k * ((N + kRowsPerTile - 1) / kRowsPerTile);
    int64_t grid = static_cast<int64_t>(di.sm_count) * blocks_per_sm;
    if (grid > tiles) grid = tiles;
    unsigned *status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    kern<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(
        static_cast<const uint16_t *>(W), K, N, col_scale, reinterpret_cast<uint32_t *>(packed),
        scales, zeros, tiles_k, tiles, status);
    return cuda_status(cudaGetLastError());
}

template <int WT, int GROUP>
int launch_g(const void *W, int64_t K, int64_t N, int sym, const float *cs, uint8_t *packed,
             float *scales, float *zeros, cudaStream_t s) {
    if (sym) {
        return cs ? launch_t<WT, GROUP, true, true>(W, K, N, cs, packed, scales, zeros, s)
                  : launch_t<WT, GROUP, true, false>(W, K, N, cs, packed, scales, zeros, s);
    }
    return cs ? launch_t<WT, GROUP, false, true>(W, K, N, cs, packed, scales, zeros, s)
              : launch_t<WT, GROUP, false, false>(W, K, N, cs, packed, scales, zeros, s);
}

template <int WT>
int launch_w(const void *W, int64_t K, int64_t N, int group, int sym, const float *cs,
             uint8_t *packed, float *scales, float *zeros, cudaStream_t s) {
    switch (group) {
        case 32: return launch_g<WT, 32>(W, K, N, sym, cs, packed, scales, zeros, s);
        case 64: return launch_g<WT, 64>(W, K, N, sym, cs, packed, scales, zeros, s);
        case 128: return launch_g<WT, 128>(W, K, N, sym, cs, packed, scales, zeros, s);
        case 256: return launch_g<WT, 256>(W, K, N, sym, cs, packed, scales, zeros, s);
        default: return W4_ERR_UNSUPPORTED;
    }
}

}  // namespace

int launch_quantize(const void *W, int wt, int64_t K, int64_t N, int group, int sym,
                    const float *col_scale, uint8_t *packed, float *scales, float *zeros,
                    cudaStream_t stream) {
    if (wt == W4_F16)
        return launch_w<W4_F16>(W, K, N, group, sym, col_scale, packed, scales, zeros, stream);
    return launch_w<W4_BF16>(W, K, N, group, sym, col_scale, packed, scales, zeros, stream);
}

}  // namespace w4
