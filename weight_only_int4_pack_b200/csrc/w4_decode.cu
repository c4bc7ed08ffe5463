// w4_decode.cu -- the W4A16 linear layer for small M (decode, M <= 32).
//
// Y[m][n] = sum_k X[m][k] * (u[n][k] - zero[n][g]) * scale[n][g]: the
// "dequant -> 16-bit matmul" of W4A16 ("Quantization method families",
// inference-learning-path.pages.dev, §2), with dequantization as in
// "LLM quantization methods: principles and implementation"
// (zhiyuanblog.org/blog/llm-quantization) §2.2.  At small M the layer is
// bound by streaming the packed weights from HBM.
//
// Design (B200, sm_100a):
//   * Swap-AB tensor-core GEMV: a warp owns RT tiles of 16 weight rows and
//     runs mma.sync m16n8k16 with the dequantized weights as the 16-row A
//     operand and X as the 8-column B operand (M padded to 8*MT).  The A
//     fragments are built in registers straight from the packed words, so
//     the weights never touch shared memory.
//   * Exact operands: (u - zero) is an integer in [-15, 15], exact in fp16
//     and bf16.  It is produced with the exponent-bias trick (OR the nibble
//     into the mantissa of 1024.0 (fp16) or 128.0 (bf16), subtract the biased
//     zero point); the group's fp32 partial sum is multiplied by the group
//     scale afterwards.  No weight is ever rounded to 16 bits.
//   * The packed layout puts k = 8j+{0,1} in nibbles 0 and 4 of word j,
//     k+{2,3} in nibbles 1 and 5, etc., so one mask pulls a pair of
//     consecutive k into the two halves of a 32-bit register.  Thread (g, t)
//     of a warp loads the 32 consecutive k = 32t..32t+31 of a group for rows
//     g and g+8 (one 16-byte load each) and the matching 16 bytes of X per
//     word, so no register shuffles are needed: mma (word j, half h) maps the
//     fragment's k indices {2t,2t+1,2t+8,2t+9} to the physical
//     k = 32t + 8j + 4h + {0,1,2,3}.
//   * Split-K: the 8 warps of a CTA split K (WK ways) and reduce through
//     shared memory in a fixed order.  When there are too few row tiles to
//     fill the GPU, the grid also splits K across CTAs: each CTA writes an
//     fp32 partial to the caller's workspace and the last CTA to arrive on a
//     tile (atomic counter) sums the partials in split order, writes Y and
//     re-arms the counter.  The result is deterministic.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "w4_internal.cuh"

namespace w4 {
namespace {

constexpr int kGroup = 128;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kBatch = 4;  // groups whose weight loads are in flight together
// Workspace layout when K is split across CTAs: a fixed area of arrival
// counters first (one per row block), then the fp32 partials.  The counters
// sit at the same place for every shape, so a workspace shared by calls of
// different shapes stays valid: every call leaves its counters at zero and
// fully overwrites the partials it reads.
constexpr int kMaxCounters = 1024;
constexpr size_t kCounterBytes = kMaxCounters * sizeof(unsigned);

struct DecodeCfg {
    int MT, RT, WN;  // n8 tiles of X rows, 16-row weight tiles per warp, warps along N
};

__host__ __device__ constexpr int rows_per_cta(int RT, int WN) { return 16 * RT * WN; }

__device__ __forceinline__ uint4 ldg_stream(const uint32_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_keep(const void *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
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

// Biased zero point of one row for the current group, in the operand type:
// fp16: zb = {1024+z, 1024+z}, zq = {-(64+z), -(64+z)}; bf16: zb = {128+z, 128+z}.
template <int XT>
struct ZeroBias {
    uint32_t zb, zq;
    __device__ __forceinline__ void set(float z) {
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
};

// One packed word (k = 8j..8j+7 of a row) -> four registers holding the
// exact pairs (u-z) of k = {0,1}, {2,3}, {4,5}, {6,7}.
template <int XT>
__device__ __forceinline__ void dequant_word(uint32_t w, const ZeroBias<XT> &zb, uint32_t p[4]) {
    if (XT == W4_F16) {
        const uint32_t magic = 0x64006400u;  // {1024.0, 1024.0}
        const uint32_t sixteenth = 0x2C002C00u;  // {1/16, 1/16}
        uint32_t lo0 = (w & 0x000F000Fu) | magic;
        uint32_t hi0 = (w & 0x00F000F0u) | magic;
        uint32_t w8 = w >> 8;
        uint32_t lo1 = (w8 & 0x000F000Fu) | magic;
        uint32_t hi1 = (w8 & 0x00F000F0u) | magic;
        asm("sub.f16x2 %0, %1, %2;" : "=r"(p[0]) : "r"(lo0), "r"(zb.zb));
        asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[1]) : "r"(hi0), "r"(sixteenth), "r"(zb.zq));
        asm("sub.f16x2 %0, %1, %2;" : "=r"(p[2]) : "r"(lo1), "r"(zb.zb));
        asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(p[3]) : "r"(hi1), "r"(sixteenth), "r"(zb.zq));
    } else {
        const uint32_t magic = 0x43004300u;  // {128.0, 128.0} in bf16
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | magic;
            asm("sub.bf16x2 %0, %1, %2;" : "=r"(p[i]) : "r"(v), "r"(zb.zb));
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

template <int XT, int MT, int RT, int WN>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const uint16_t *__restrict__ X, int M, const uint32_t *__restrict__ packed,
              const float *__restrict__ scales, const float *__restrict__ zeros, int K, int N,
              void *__restrict__ Y, float *__restrict__ ws_partial, unsigned *__restrict__ ws_count,
              int splits) {
    constexpr int WK = kWarps / WN;
    constexpr int ROWS = rows_per_cta(RT, WN);
    constexpr int MP = 8 * MT;
    __shared__ float red[WK][ROWS][MP];
    __shared__ unsigned s_last;

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int wn = warp % WN, wk = warp / WN;
    const int G = K / kGroup;
    const int KW = K / 8;  // packed words per row
    const int rb = blockIdx.x;
    const int split = blockIdx.y;
    const int n_cta = rb * ROWS;
    const int n_warp = n_cta + wn * 16 * RT;

    // groups of this split, then of this warp
    const int gs0 = (int)((int64_t)G * split / splits), gs1 = (int)((int64_t)G * (split + 1) / splits);
    const int gw0 = gs0 + (gs1 - gs0) * wk / WK, gw1 = gs0 + (gs1 - gs0) * (wk + 1) / WK;

    float acc[RT][MT][4];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][mt][i] = 0.0f;

    // row pointers of this thread (rows beyond N read row N-1 and are dropped)
    const uint32_t *wrow[RT][2];
    int nrow[RT][2];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            int n = n_warp + 16 * r + 8 * h + g;
            nrow[r][h] = n < N ? n : N - 1;
            wrow[r][h] = packed + (int64_t)nrow[r][h] * KW + 4 * t;
        }
    // X rows of this thread's B fragments (rows beyond M contribute zero columns)
    const uint16_t *xrow[MT];
    bool xval[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        int m = 8 * mt + g;
        xval[mt] = m < M;
        xrow[mt] = X + (int64_t)(xval[mt] ? m : 0) * K + 32 * t;
    }

    for (int gb = gw0; gb < gw1; gb += kBatch) {
        uint4 wv[kBatch][RT][2];
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    if (gb + b < gw1) wv[b][r][h] = ldg_stream(wrow[r][h] + (gb + b) * 16);
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int grp = gb + b;
            if (grp >= gw1) break;
            float s[RT][2];
            ZeroBias<XT> zb[RT][2];
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t gi = (int64_t)nrow[r][h] * G + grp;
                    s[r][h] = __ldg(scales + gi);
                    zb[r][h].set(zeros ? __ldg(zeros + gi) : 8.0f);
                }
            float part[RT][MT][4];
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) part[r][mt][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 xv[MT];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    xv[mt] = make_uint4(0, 0, 0, 0);
                    if (xval[mt]) xv[mt] = ldg_keep(xrow[mt] + grp * kGroup + 8 * j);
                }
#pragma unroll
                for (int r = 0; r < RT; ++r) {
                    uint32_t pa[4], pb[4];  // rows g and g+8
                    const uint32_t wa = j == 0 ? wv[b][r][0].x : j == 1 ? wv[b][r][0].y
                                      : j == 2 ? wv[b][r][0].z : wv[b][r][0].w;
                    const uint32_t wbw = j == 0 ? wv[b][r][1].x : j == 1 ? wv[b][r][1].y
                                       : j == 2 ? wv[b][r][1].z : wv[b][r][1].w;
                    dequant_word<XT>(wa, zb[r][0], pa);
                    dequant_word<XT>(wbw, zb[r][1], pb);
                    const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
                    const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        mma16816<XT>(part[r][mt], a0, xv[mt].x, xv[mt].y);
                        mma16816<XT>(part[r][mt], a1, xv[mt].z, xv[mt].w);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    acc[r][mt][0] = fmaf(s[r][0], part[r][mt][0], acc[r][mt][0]);
                    acc[r][mt][1] = fmaf(s[r][0], part[r][mt][1], acc[r][mt][1]);
                    acc[r][mt][2] = fmaf(s[r][1], part[r][mt][2], acc[r][mt][2]);
                    acc[r][mt][3] = fmaf(s[r][1], part[r][mt][3], acc[r][mt][3]);
                }
        }
    }

    // ---- reduce the WK warps of each row tile in fixed order ----
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = wn * 16 * RT + 16 * r + g + 8 * (i >> 1);
                const int m = 8 * mt + 2 * t + (i & 1);
                red[wk][row][m] = acc[r][mt][i];
            }
    __syncthreads();

    const int Mv = M < MP ? M : MP;
    if (splits == 1) {
        for (int e = threadIdx.x; e < ROWS * Mv; e += kThreads) {
            const int row = e % ROWS, m = e / ROWS;
            const int n = n_cta + row;
            if (n >= N) continue;
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < WK; ++w) v += red[w][row][m];
            store_out<XT>(Y, (int64_t)m * N + n, v);
        }
        return;
    }

    // ---- split-K across CTAs: partial to workspace, last CTA finishes ----
    for (int e = threadIdx.x; e < ROWS * Mv; e += kThreads) {
        const int row = e % ROWS, m = e / ROWS;
        const int n = n_cta + row;
        if (n >= N) continue;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < WK; ++w) v += red[w][row][m];
        ws_partial[((int64_t)split * M + m) * N + n] = v;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(ws_count + rb, 1u);
        s_last = (prev == (unsigned)(splits - 1)) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int e = threadIdx.x; e < ROWS * Mv; e += kThreads) {
        const int row = e % ROWS, m = e / ROWS;
        const int n = n_cta + row;
        if (n >= N) continue;
        float v = 0.0f;
        for (int sp = 0; sp < splits; ++sp) v += __ldcg(ws_partial + ((int64_t)sp * M + m) * N + n);
        store_out<XT>(Y, (int64_t)m * N + n, v);
    }
    if (threadIdx.x == 0) ws_count[rb] = 0u;  // re-arm for the next call
}

DecodeCfg pick_cfg(int64_t M) {
    if (M <= 8) return {1, 1, 1};
    if (M <= 16) return {2, 1, 2};
    if (M <= 24) return {3, 2, 2};
    return {4, 2, 4};
}

struct Plan {
    DecodeCfg c;
    int row_blocks, splits;
    size_t partial_bytes, count_bytes;
};

int make_plan(int64_t M, int64_t K, int64_t N, Plan *p) {
    DeviceInfo di;
    int st = device_info(&di);
    if (st != W4_OK) return st;
    p->c = pick_cfg(M);
    const int rows = rows_per_cta(p->c.RT, p->c.WN);
    p->row_blocks = (int)((N + rows - 1) / rows);
    const int G = (int)(K / kGroup);
    const int WK = kWarps / p->c.WN;
    // enough CTAs for ~2 per SM, keeping >= 2 groups per warp
    int want = (2 * di.sm_count + p->row_blocks - 1) / p->row_blocks;
    int maxs = G / (2 * WK);
    if (maxs < 1) maxs = 1;
    if (want > maxs) want = maxs;
    if (want > 16) want = 16;
    p->splits = want < 1 ? 1 : want;
    if (p->row_blocks > kMaxCounters) p->splits = 1;
    if (p->splits > 1) {
        p->partial_bytes = ((size_t)p->splits * M * N * sizeof(float) + 255) & ~(size_t)255;
        p->count_bytes = kCounterBytes;
    } else {
        p->partial_bytes = p->count_bytes = 0;
    }
    return W4_OK;
}

template <int XT, int MT, int RT, int WN>
int launch_t(const Plan &p, const void *X, int64_t M, const uint8_t *packed, const float *scales,
             const float *zeros, int64_t K, int64_t N, void *Y, void *ws, cudaStream_t stream) {
    float *partial = nullptr;
    unsigned *count = nullptr;
    if (p.splits > 1) {
        count = static_cast<unsigned *>(ws);
        partial = reinterpret_cast<float *>(static_cast<char *>(ws) + p.count_bytes);
    }
    dim3 grid(p.row_blocks, p.splits);
    decode_kernel<XT, MT, RT, WN><<<grid, kThreads, 0, stream>>>(
        static_cast<const uint16_t *>(X), (int)M, reinterpret_cast<const uint32_t *>(packed),
        scales, zeros, (int)K, (int)N, Y, partial, count, p.splits);
    return cuda_status(cudaGetLastError());
}

template <int XT>
int launch_x(const Plan &p, const void *X, int64_t M, const uint8_t *packed, const float *scales,
             const float *zeros, int64_t K, int64_t N, void *Y, void *ws, cudaStream_t s) {
    switch (p.c.MT) {
        case 1: return launch_t<XT, 1, 1, 1>(p, X, M, packed, scales, zeros, K, N, Y, ws, s);
        case 2: return launch_t<XT, 2, 1, 2>(p, X, M, packed, scales, zeros, K, N, Y, ws, s);
        case 3: return launch_t<XT, 3, 2, 2>(p, X, M, packed, scales, zeros, K, N, Y, ws, s);
        default: return launch_t<XT, 4, 2, 4>(p, X, M, packed, scales, zeros, K, N, Y, ws, s);
    }
}

}  // namespace

size_t decode_workspace_bytes(int64_t M, int64_t K, int64_t N, int group) {
    (void)group;
    Plan p;
    if (make_plan(M, K, N, &p) != W4_OK) return 0;
    return p.partial_bytes + p.count_bytes;
}

int launch_decode(const void *X, int xt, int64_t M, const uint8_t *packed, const float *scales,
                  const float *zeros, int64_t K, int64_t N, void *Y, void *workspace,
                  size_t workspace_bytes, cudaStream_t stream) {
    Plan p;
    int st = make_plan(M, K, N, &p);
    if (st != W4_OK) return st;
    if (p.partial_bytes + p.count_bytes > workspace_bytes) return W4_ERR_INVALID_ARG;
    if (xt == W4_F16)
        return launch_x<W4_F16>(p, X, M, packed, scales, zeros, K, N, Y, workspace, stream);
    return launch_x<W4_BF16>(p, X, M, packed, scales, zeros, K, N, Y, workspace, stream);
}

}  // namespace w4
