// 1x128 activation quantiser: FP32 or BF16 [M, K] -> E4M3 bytes [M, K] and
// one FP32 scale per row per 128-wide K block, written column-major
// ([K/128][ld_sa]) as the GEMM reads them.  The DeepGEMM README (usage)
// leaves the cast and the transposition of the LHS scales to a kernel before
// the GEMM; the 1x128 granularity is the DeepSeek-V3 recipe.
//
// Per block: amax = max |x| (exact), s = max(amax, 1e-4) / 448 and
// q = E4M3(clamp(x / s, +-448)), both divisions rounded to nearest (IEEE),
// the cast round-to-nearest-even.  The per-element quotient x / s comes from
// the block's correctly rounded reciprocal r = 1/s and one FMA correction
// step (Markstein's method: q0 = x * r, e = x - q0 * s exactly by FMA,
// q = q0 + e * r), which yields the correctly rounded quotient when r is the
// correctly rounded reciprocal, at three operations per element instead of a
// full division, done on packed pairs of elements.
//
// HBM-bound: one warp per 32 (BF16) or 16 (FP32) rows x 128 columns, 8
// lanes per row, each lane 16 elements of a row as 16-byte words (two of
// BF16, four of FP32): word h of lane l is the row block's 16-byte word
// 8h + l, so that each load instruction of a warp reads whole 128-byte lines;
// four rows per step, the next rows' loads in flight; the amax of a row is
// three shuffles within its 8 lanes; lane j ends up with the scale of the
// warp's row j, so a block column of the warp's scales is one coalesced store.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace fp8nt {

namespace {

constexpr int QUANT_WARPS = 8; // warps per CTA

// Two FP32 values -> two E4M3 bytes (round to nearest even, saturating),
// low byte = lo.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// 16 consecutive elements of a row: RAW 16-byte words (BF16: 2, FP32: 4)
template <bool BF16_IN>
struct Raw16 {
    static constexpr int WORDS = BF16_IN ? 2 : 4;
    uint4 w[WORDS];
};

// The lane's words of a row block starting at element `off`: word h is the
// block's 16-byte word 8h + l8.
template <bool BF16_IN>
__device__ __forceinline__ void load_raw16(const void *x, long off, int l8, Raw16<BF16_IN> &r)
{
    const uint4 *p = BF16_IN ? reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + off)
                             : reinterpret_cast<const uint4 *>(static_cast<const float *>(x) + off);
#pragma unroll
    for (int h = 0; h < Raw16<BF16_IN>::WORDS; ++h)
        r.w[h] = __ldg(p + 8 * h + l8);
}

template <bool BF16_IN>
__device__ __forceinline__ void unpack16(const Raw16<BF16_IN> &r, float (&v)[16])
{
    if constexpr (BF16_IN) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t w[4] = {r.w[h].x, r.w[h].y, r.w[h].z, r.w[h].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // a BF16 value is the high half of the FP32 with the same bits
                v[h * 8 + 2 * i] = __uint_as_float(w[i] << 16);
                v[h * 8 + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
        }
    } else {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            v[4 * h] = __uint_as_float(r.w[h].x);
            v[4 * h + 1] = __uint_as_float(r.w[h].y);
            v[4 * h + 2] = __uint_as_float(r.w[h].z);
            v[4 * h + 3] = __uint_as_float(r.w[h].w);
        }
    }
}

// x / s rounded to nearest for two elements at once, given r = 1/s rounded
// to nearest and ns = -s: one FMA correction of the product x * r
// (Markstein's method: q0 = x r, e = x - q0 s exactly by FMA, q = q0 + e r),
// on packed pairs (mul.rn / fma.rn .f32x2, rounded per element as the scalar
// operations are).  s > 0, so the quotient has the sign of x; taking the sign
// from x at the end keeps a zero quotient's sign (-0 / s is -0, which the
// correction q0 + 0 * r would turn into +0) and changes nothing else.
__device__ __forceinline__ void div2_by_scale(float x0, float x1, uint64_t r2, uint64_t ns2, float &y0,
                                              float &y1)
{
    uint64_t x, q0, e, q;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(x0), "f"(x1));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q0) : "l"(x), "l"(r2));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e) : "l"(q0), "l"(ns2), "l"(x));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(e), "l"(r2), "l"(q0));
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(q));
    y0 = copysignf(a, x0);
    y1 = copysignf(b, x1);
}

__device__ __forceinline__ uint64_t splat2(float v)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
    return r;
}

// Rows in flight per lane and CTAs per SM asked of the compiler (so, the
// registers each thread may use), measured on B200 (4096 x 7168): BF16 two
// steps in flight at four CTAs per SM, 32 rows per warp; FP32 four steps,
// 16 rows per warp (its block column of scales is then 16 rows)
template <bool BF16_IN>
struct QuantShape {
    static constexpr int ROWS = BF16_IN ? 32 : 16; // rows per warp, a multiple of 4, <= 32
    static constexpr int DEPTH = BF16_IN ? 2 : 4;  // <= ROWS / 4
    static constexpr int MIN_CTAS = BF16_IN ? 4 : 1;
    static_assert(ROWS % 4 == 0 && ROWS <= 32 && DEPTH >= 1 && DEPTH <= ROWS / 4, "row steps of 4 rows");
};

template <bool BF16_IN>
__global__ void __launch_bounds__(QUANT_WARPS * 32, QuantShape<BF16_IN>::MIN_CTAS)
    quantize_1x128_kernel(const void *x, uint8_t *q, float *sa, int M, int K, long ld_sa)
{
    const int lane = threadIdx.x & 31;
    const long wid = (long)blockIdx.x * QUANT_WARPS + (threadIdx.x >> 5);
    const int nkb = K / 128;
    constexpr int ROWS = QuantShape<BF16_IN>::ROWS;
    const long blocks = (long)((M + ROWS - 1) / ROWS) * nkb;
    if (wid >= blocks)
        return;
    // consecutive warps take consecutive K blocks of the same ROWS rows
    const int kb = (int)(wid % nkb);
    const int r0 = (int)(wid / nkb) * ROWS;
    const int sub = lane >> 3;                      // row within a step of 4
    const int l8 = lane & 7;
    const long col = (long)kb * 128;
    float my_scale = 0.0f;
    constexpr int DEPTH = QuantShape<BF16_IN>::DEPTH;
    Raw16<BF16_IN> raw[DEPTH];
    auto load_step = [&](int it, Raw16<BF16_IN> &dst) {
        const int row = r0 + it * 4 + sub;
        if (row < M) {
            load_raw16<BF16_IN>(x, (long)row * K + col, l8, dst);
        } else {
#pragma unroll
            for (int h = 0; h < Raw16<BF16_IN>::WORDS; ++h)
                dst.w[h] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
#pragma unroll
    for (int it = 0; it < DEPTH; ++it)
        load_step(it, raw[it]);
#pragma unroll
    for (int it = 0; it < ROWS / 4; ++it) {
        float w[16];
        unpack16<BF16_IN>(raw[it % DEPTH], w);
        if (it + DEPTH < ROWS / 4)
            load_step(it + DEPTH, raw[it % DEPTH]);
        float amax = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e)
            amax = fmaxf(amax, fabsf(w[e]));
#pragma unroll
        for (int d = 4; d > 0; d >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
        const float s = __fdiv_rn(fmaxf(amax, 1e-4f), 448.0f);
        const uint64_t r2 = splat2(__frcp_rn(s)), ns2 = splat2(-s);
        uint32_t packed[4];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            float y[4];
            div2_by_scale(w[e], w[e + 1], r2, ns2, y[0], y[1]);
            div2_by_scale(w[e + 2], w[e + 3], r2, ns2, y[2], y[3]);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                y[i] = fminf(fmaxf(y[i], -448.0f), 448.0f);
            packed[e / 4] = cvt_e4m3x2(y[0], y[1]) | (cvt_e4m3x2(y[2], y[3]) << 16);
        }
        const int row = r0 + it * 4 + sub;
        if (row < M) {
            // codes of word h: elements (8h + l8) * (16 / element size) on
            uint8_t *dst = q + (long)row * K + col;
            if constexpr (BF16_IN) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<uint2 *>(dst + (8 * h + l8) * 8) = make_uint2(packed[2 * h], packed[2 * h + 1]);
            } else {
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    *reinterpret_cast<uint32_t *>(dst + (8 * h + l8) * 4) = packed[h];
            }
        }
        // lane j keeps the scale of row j (rows it * 4 .. it * 4 + 3 now)
        const float sv = __shfl_sync(0xffffffffu, s, (lane & 3) * 8);
        if ((lane >> 2) == it)
            my_scale = sv;
    }
    if (lane < ROWS && r0 + lane < M)
        sa[(long)kb * ld_sa + r0 + lane] = my_scale;
}

} // namespace

cudaError_t launch_quantize_1x128(const void *x, bool bf16_in, uint8_t *q, float *sa, int M, int K,
                                  long ld_sa, cudaStream_t stream)
{
    const int rows = bf16_in ? QuantShape<true>::ROWS : QuantShape<false>::ROWS;
    const long warps = (long)((M + rows - 1) / rows) * (K / 128);
    const long grid = (warps + QUANT_WARPS - 1) / QUANT_WARPS;
    if (grid <= 0)
        return cudaSuccess;
    if (grid > 0x7fffffffL)
        return cudaErrorInvalidValue;
    if (bf16_in)
        quantize_1x128_kernel<true><<<(unsigned)grid, QUANT_WARPS * 32, 0, stream>>>(x, q, sa, M, K, ld_sa);
    else
        quantize_1x128_kernel<false><<<(unsigned)grid, QUANT_WARPS * 32, 0, stream>>>(x, q, sa, M, K, ld_sa);
    return cudaGetLastError();
}

} // namespace fp8nt
