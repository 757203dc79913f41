// 1x128 activation quantiser: FP32 or BF16 [M, K] -> E4M3 bytes [M, K] and
// one FP32 scale per row per 128-wide K block, written column-major
// ([K/128][ld_sa]) as the GEMM reads them.  The DeepGEMM README (usage)
// leaves the cast and the transposition of the LHS scales to a kernel before
// the GEMM; the 1x128 granularity is the DeepSeek-V3 recipe.
//
// Per block: amax = max |x| (exact), s = max(amax, 1e-4) / 448 and
// q = E4M3(clamp(x / s, +-448)), both divisions IEEE round-to-nearest, the
// cast round-to-nearest-even.  HBM-bound: one warp per 32 rows x 128
// columns, each lane 16 bytes (FP32) or 8 bytes (BF16) of a row at a time,
// the next four rows' loads in flight while four rows are quantised;
// lane i keeps row i's scale, so the 32 scales of a block column go out as
// one coalesced 128-byte store.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace fp8nt {

namespace {

constexpr int QUANT_WARPS = 8; // warps per CTA
constexpr int QUANT_ROWS_IN_FLIGHT = 4;

// Two FP32 values -> two E4M3 bytes (round to nearest even, saturating),
// low byte = lo.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <bool BF16_IN>
__device__ __forceinline__ void load4(const void *x, long off, float (&v)[4])
{
    if constexpr (BF16_IN) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(x) + off));
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        v[0] = __low2float(lo);
        v[1] = __high2float(lo);
        v[2] = __low2float(hi);
        v[3] = __high2float(hi);
    } else {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + off));
        v[0] = f.x;
        v[1] = f.y;
        v[2] = f.z;
        v[3] = f.w;
    }
}

template <bool BF16_IN>
__global__ void __launch_bounds__(QUANT_WARPS * 32)
    quantize_1x128_kernel(const void *x, uint8_t *q, float *sa, int M, int K, long ld_sa)
{
    const int lane = threadIdx.x & 31;
    const long wid = (long)blockIdx.x * QUANT_WARPS + (threadIdx.x >> 5);
    const int nkb = K / 128;
    const long blocks = (long)((M + 31) / 32) * nkb;
    if (wid >= blocks)
        return;
    // consecutive warps take consecutive K blocks of the same 32 rows
    const int kb = (int)(wid % nkb);
    const int r0 = (int)(wid / nkb) * 32;
    const long col = (long)kb * 128 + lane * 4;
    float my_scale = 0.0f;
    // software pipeline: the next rows' loads are in flight while the
    // current rows are reduced, divided and stored
    float v[2][QUANT_ROWS_IN_FLIGHT][4];
    auto load_rows = [&](int i, float (&dst)[QUANT_ROWS_IN_FLIGHT][4]) {
#pragma unroll
        for (int j = 0; j < QUANT_ROWS_IN_FLIGHT; ++j) {
            const int row = r0 + i + j;
            if (row < M)
                load4<BF16_IN>(x, (long)row * K + col, dst[j]);
            else
                dst[j][0] = dst[j][1] = dst[j][2] = dst[j][3] = 0.0f;
        }
    };
    load_rows(0, v[0]);
#pragma unroll
    for (int i = 0; i < 32; i += QUANT_ROWS_IN_FLIGHT) {
        const int cur = (i / QUANT_ROWS_IN_FLIGHT) & 1;
        if (i + QUANT_ROWS_IN_FLIGHT < 32)
            load_rows(i + QUANT_ROWS_IN_FLIGHT, v[cur ^ 1]);
#pragma unroll
        for (int j = 0; j < QUANT_ROWS_IN_FLIGHT; ++j) {
            const float(&w)[4] = v[cur][j];
            float amax = fmaxf(fmaxf(fabsf(w[0]), fabsf(w[1])), fmaxf(fabsf(w[2]), fabsf(w[3])));
#pragma unroll
            for (int d = 16; d > 0; d >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
            const float s = __fdiv_rn(fmaxf(amax, 1e-4f), 448.0f);
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                y[e] = fminf(fmaxf(__fdiv_rn(w[e], s), -448.0f), 448.0f);
            const uint32_t packed = cvt_e4m3x2(y[0], y[1]) | (cvt_e4m3x2(y[2], y[3]) << 16);
            const int row = r0 + i + j;
            if (row < M)
                *reinterpret_cast<uint32_t *>(q + (long)row * K + col) = packed;
            if (lane == i + j)
                my_scale = s;
        }
    }
    if (r0 + lane < M)
        sa[(long)kb * ld_sa + r0 + lane] = my_scale;
}

} // namespace

cudaError_t launch_quantize_1x128(const void *x, bool bf16_in, uint8_t *q, float *sa, int M, int K,
                                  long ld_sa, cudaStream_t stream)
{
    const long warps = (long)((M + 31) / 32) * (K / 128);
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
