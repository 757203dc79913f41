// Persistent, warp-specialised FP8 NT GEMM with fine-grained scaling for
// sm_100a.
//
// What it computes (DeepGEMM README, introduction and usage):
//   D[m,n] = sum_kb P_kb[m,n] * sa[m,kb] * sb[n/128,kb],
//   P_kb = A[:, kb-block] . B[:, kb-block]^T  (FP8 x FP8, exact in FP32 here)
// with FP32 accumulation of the scaled partials (the README's two-level
// accumulation: tensor-core partial per 128-K block, promotion on CUDA cores)
// and BF16 output.
//
// Roles (384 threads, one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: A / B tiles into a multi-stage shared-memory
//               ring, the tile's LHS scales into a scale ring (TMA), the
//               tile's RHS scales into a per-tile slot (cp.async).  The
//               README's data-movement warpgroup, reduced to one warp.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer: one
//               128-K block per MMA group into one of two TMEM buffers, fresh
//               accumulation per block so each block's partial stays separable.
//   warps 4-11  promotion epilogue: tcgen05.ld of a block's partial, FMA with
//               sa*sb into FP32 registers, BF16 conversion and store at tile end.
// Warps 2-3 only help with set-up (masked tile counts).
//
// Tile shape: BLOCK_M = 128 * MW rows (MW = 2 issues two M=128 MMAs that share
// the B tile), BLOCK_N = BN columns, BN a multiple of 16 in [16, 256] so that
// non-power-of-two widths can fill the SMs (README, unaligned block sizes).
#pragma once

#include <cuda_bf16.h>

#include "params.h"
#include "ptx.cuh"

namespace fp8nt {

template <int MW, int BN>
struct KernelTraits {
    static_assert(MW == 1 || MW == 2, "MW is 1 or 2");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN must be a multiple of 16 in [16, 256]");
    static_assert(MW == 1 || BN <= 128, "two M halves need BN <= 128 (TMEM and registers)");
    static constexpr int BLOCK_M = MW * HALF_M;
    static constexpr int BUF_COLS = MW * BN;                 // TMEM columns per K-block buffer
    static constexpr int TMEM_NEED = 2 * BUF_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                   : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int COLS_PER_THREAD = (MW == 1) ? BN / 2 : BN;
    static constexpr uint32_t A_HALF_BYTES = HALF_M * BLOCK_K;
    static constexpr uint32_t B_BYTES = BN * BLOCK_K;
    static_assert(TMEM_NEED <= 512, "TMEM holds 512 columns");
    static_assert(COLS_PER_THREAD % 8 == 0, "epilogue works in 8-column chunks");
};

// Instruction descriptor of tcgen05.mma kind::f8f6f4: D FP32, A and B E4M3,
// both K-major, M = 128, N = BN, dense.
__host__ __device__ constexpr uint32_t make_idesc(int bn)
{
    return (1u << 4)                          // D format: F32
           | (0u << 7) | (0u << 10)           // A, B format: E4M3
           | (0u << 15) | (0u << 16)          // A, B K-major
           | ((uint32_t)(bn >> 3) << 17)      // N / 8
           | ((uint32_t)(HALF_M >> 4) << 24); // M / 16
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu)   // start address / 16
           | ((uint64_t)1u << 16)               // leading byte offset (unused when swizzled)
           | ((uint64_t)(1024u >> 4) << 32)     // stride byte offset: 8 rows x 128 B
           | ((uint64_t)1u << 46)               // descriptor version (sm_100)
           | ((uint64_t)2u << 61);              // layout: 128-byte swizzle
}

struct TileInfo {
    int valid;   // 0: nothing to compute (contiguous padding block, bad expert)
    int g;       // group (masked) / expert (contiguous) / 0 (dense)
    int m0;      // first row of the tile within its group
    int n0;      // first column
    int rows;    // rows of the tile that hold valid data (<= BLOCK_M)
    int a_row0;  // row coordinate of the tile in A's 2-D tensor map
    int b_row0;  // row coordinate in B's 2-D tensor map
    int sa_y0;   // row of sa's 2-D tensor map holding K block 0 of this group
    int sb_row0; // first sb row (128-column block) of the tile, group base included
    int sb_rows; // sb rows present from sb_row0 within the group (<= 3)
    int d_row0;  // row of D (all groups flattened) holding row m0
};

template <int MW, int BN>
__device__ __forceinline__ TileInfo get_tile(const Params &p, int t, const int *prefix)
{
    constexpr int BM = KernelTraits<MW, BN>::BLOCK_M;
    TileInfo ti;
    ti.valid = 1;
    int mb, nb;
    if (p.kind == KIND_MASKED) {
        // binary search for the group g with prefix[g] <= t < prefix[g + 1]
        int lo = 0, hi = p.num_groups - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (prefix[mid] <= t)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int g = lo;
        const int mm = prefix[p.num_groups + 1 + g];
        const int mblocks = (mm + BM - 1) / BM;
        const int local = t - prefix[g];
        mb = local % mblocks; // M fastest: tiles sharing a B block run side by side
        nb = local / mblocks;
        ti.g = g;
        ti.m0 = mb * BM;
        ti.rows = min(BM, mm - ti.m0);
        ti.a_row0 = g * p.M + ti.m0;
        ti.b_row0 = g * p.N + nb * BN;
        ti.sa_y0 = g * p.nkb;
        ti.d_row0 = g * p.M + ti.m0;
    } else {
        mb = t / p.n_blocks;
        nb = t - mb * p.n_blocks;
        ti.m0 = mb * BM;
        ti.rows = min(BM, p.M - ti.m0);
        ti.a_row0 = ti.m0;
        ti.sa_y0 = 0;
        ti.d_row0 = ti.m0;
        ti.g = 0;
        ti.b_row0 = nb * BN;
        if (p.kind == KIND_CONTIGUOUS) {
            const int e = __ldg(p.m_indices + ti.m0);
            if (e < 0 || e >= p.num_groups) {
                if (e >= p.num_groups)
                    atomicOr(p.status, DEVERR_BAD_INDEX);
                ti.valid = 0;
                ti.g = 0;
            } else {
                ti.g = e;
                ti.b_row0 = e * p.N + nb * BN;
            }
        }
    }
    ti.n0 = nb * BN;
    const int nb128 = ti.n0 >> 7;
    ti.sb_row0 = ti.g * p.nnb + nb128;
    ti.sb_rows = min(MAX_SB_BLOCKS, p.nnb - nb128);
    return ti;
}

// Bounded mbarrier wait.  Returns false if the CTA is aborting or the wait
// ran past the time limit (then it raises the abort flag and the status bit).
__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag,
                                       unsigned int *status, uint64_t timeout_ns, bool honour_abort)
{
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity))
                return true;
        if (honour_abort && *abort_flag)
            return false;
        if (global_timer_ns() - t0 > timeout_ns) {
            *abort_flag = 1u;
            atomicOr(status, DEVERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag,
                                         const Params &p)
{
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait(a, parity))
        return true;
    return wait_slow(a, parity, abort_flag, p.status, p.timeout_ns, true);
}

// Whole-warp wait: every lane waits (and so acquires the barrier's writes);
// the outcome is made warp-uniform so that no lane runs ahead alone when
// another lane gave up.
__device__ __forceinline__ bool wait_bar_warp(uint64_t *bar, uint32_t parity,
                                              volatile uint32_t *abort_flag, const Params &p)
{
    const bool ok = wait_bar(bar, parity, abort_flag, p);
    return __all_sync(0xffffffffu, ok) != 0;
}

// Wait used while draining at exit: ignores the abort flag, still bounded.
__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag,
                                           const Params &p)
{
    const uint32_t a = smem_addr(bar);
    if (!mbar_try_wait(a, parity))
        wait_slow(a, parity, abort_flag, p.status, p.timeout_ns, false);
}

// Columns [c0, c0 + W) of one TMEM group into registers (W = 32, 16 or 8).
template <int W>
__device__ __forceinline__ void tmem_ld_group(uint32_t taddr, float (&v)[32])
{
    if constexpr (W == 32)
        tmem_ld32(taddr, v);
    else if constexpr (W == 16)
        tmem_ld16(taddr, v);
    else
        tmem_ld8(taddr, v);
}

// A thread's NC columns are read from TMEM in groups: NC / 32 groups of 32,
// then a 16-column and / or an 8-column tail.
template <int NC>
struct Groups {
    static constexpr int n32 = NC / 32;
    static constexpr bool t16 = (NC % 32) >= 16;
    static constexpr bool t8 = (NC % 16) == 8;
    static constexpr int count = n32 + (t16 ? 1 : 0) + (t8 ? 1 : 0);
    __host__ __device__ static constexpr int width(int g) { return g < n32 ? 32 : (t16 && g == n32 ? 16 : 8); }
    __host__ __device__ static constexpr int offset(int g)
    {
        return g <= n32 ? 32 * g : 32 * n32 + (t16 ? 16 : 0);
    }
};

// acc[c0 + j] += v[j] * s for j in [0, W), two columns per instruction.
template <int NC, int W>
__device__ __forceinline__ void fma_group_uniform(float (&acc)[NC], int c0, const float (&v)[32],
                                                  uint64_t s2)
{
#pragma unroll
    for (int j = 0; j < W; j += 2)
        ffma2(acc[c0 + j], acc[c0 + j + 1], v[j], v[j + 1], s2);
}

// As above with the scale chosen per 8 columns: local columns before t use
// s_lo, the rest s_hi.  A thread owns at most 128 columns, so they span at
// most two 128-wide scale blocks.
template <int NC, int W>
__device__ __forceinline__ void fma_group_split(float (&acc)[NC], int c0, const float (&v)[32],
                                                float s_lo, float s_hi, int t)
{
#pragma unroll
    for (int j = 0; j < W; j += 8) {
        const uint64_t s2 = splat2(c0 + j < t ? s_lo : s_hi);
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            ffma2(acc[c0 + j + i], acc[c0 + j + i + 1], v[j + i], v[j + i + 1], s2);
    }
}

template <int NC, bool SPLIT, int G>
__device__ __forceinline__ void promote_from(float (&acc)[NC], uint32_t taddr, float (&buf)[2][32],
                                             float s_lo, float s_hi, uint64_t s2, int t)
{
    using Gs = Groups<NC>;
    if constexpr (G < Gs::count) {
        if constexpr (G + 1 < Gs::count)
            tmem_ld_group<Gs::width(G + 1)>(taddr + Gs::offset(G + 1), buf[(G + 1) & 1]);
        if constexpr (SPLIT)
            fma_group_split<NC, Gs::width(G)>(acc, Gs::offset(G), buf[G & 1], s_lo, s_hi, t);
        else
            fma_group_uniform<NC, Gs::width(G)>(acc, Gs::offset(G), buf[G & 1], s2);
        if constexpr (G + 1 < Gs::count)
            tmem_wait_ld(buf[(G + 1) & 1]);
        promote_from<NC, SPLIT, G + 1>(acc, taddr, buf, s_lo, s_hi, s2, t);
    }
}

// acc[c] += P[row, col0 + c] * scale(c), c in [0, NC): one K block's
// promotion.  The next TMEM group's load is in flight while the current
// group is multiplied in.  SPLIT: the columns straddle a scale-block boundary
// at local column t.
template <int NC, bool SPLIT>
__device__ __forceinline__ void promote(float (&acc)[NC], uint32_t taddr, float s_lo, float s_hi,
                                        int t)
{
    float buf[2][32];
    const uint64_t s2 = splat2(s_lo);
    tmem_ld_group<Groups<NC>::width(0)>(taddr, buf[0]);
    tmem_wait_ld(buf[0]);
    promote_from<NC, SPLIT, 0>(acc, taddr, buf, s_lo, s_hi, s2, t);
}

template <int MW, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_sa, const __grid_constant__ Params p)
{
    using T = KernelTraits<MW, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const SmemPlan &plan = p.plan;
    const int stages = p.stages;
    const int sf_stages = p.sf_stages;

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + plan.off_bars);
    uint64_t *empty = full + stages;
    uint64_t *sf_full = empty + stages;
    uint64_t *sf_empty = sf_full + sf_stages;
    uint64_t *tmem_full = sf_empty + sf_stages;
    uint64_t *tmem_empty = tmem_full + 2;
    uint64_t *sb_full = tmem_empty + 2;
    uint64_t *sb_empty = sb_full + 2;
    uint64_t *mma_done = sb_empty + 2;
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + plan.off_misc);
    volatile uint32_t *abort_flag = misc + 1;
    int *prefix = reinterpret_cast<int *>(smem + plan.off_prefix);
    float *sf_ring = reinterpret_cast<float *>(smem + plan.off_sf);
    float *sb_tile = reinterpret_cast<float *>(smem + plan.off_sb);
    const int pitch = (int)plan.sb_pitch;

    // ---------------------------------------------------------------- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < sf_stages; ++s) {
            mbar_init(&sf_full[s], 1);
            mbar_init(&sf_empty[s], NUM_EPI_WARPS);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], NUM_EPI_WARPS);
            mbar_init(&sb_full[b], 32);
            mbar_init(&sb_empty[b], NUM_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        misc[1] = 0u;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        tma_prefetch_desc(&tmap_sa);
    }
    if (warp == 1) {
        tmem_alloc(misc, T::TMEM_COLS);
        tmem_relinquish();
    }
    if (p.kind == KIND_MASKED && warp == 2) {
        // Tiles per group = ceil(masked_m / BLOCK_M) * n_blocks; prefix sums
        // in prefix[0..G], clamped masked_m in prefix[G+1 .. 2G].
        int carry = 0;
        for (int base = 0; base < p.num_groups; base += 32) {
            const int g = base + lane;
            int tiles = 0;
            if (g < p.num_groups) {
                int mm = __ldg(p.masked_m + g);
                if (mm < 0 || mm > p.M) {
                    atomicOr(p.status, DEVERR_BAD_INDEX);
                    mm = mm < 0 ? 0 : p.M;
                }
                prefix[p.num_groups + 1 + g] = mm;
                tiles = (mm + T::BLOCK_M - 1) / T::BLOCK_M * p.n_blocks;
            }
            int incl = tiles;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d)
                    incl += v;
            }
            if (g < p.num_groups)
                prefix[g] = carry + incl - tiles;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0)
            prefix[p.num_groups] = carry;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const int num_tiles = (p.kind == KIND_MASKED) ? prefix[p.num_groups] : p.num_tiles;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        regs_dec<REGS_PRODUCER>();
        uint32_t stage_it = 0, sf_it = 0, tile_it = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
            const TileInfo ti = get_tile<MW, BN>(p, t, prefix);
            if (!ti.valid)
                continue;
            const int slot = tile_it & 1;
            if (!wait_bar_warp(&sb_empty[slot], ((tile_it >> 1) & 1) ^ 1, abort_flag, p))
                break;
            float *dst = sb_tile + slot * MAX_SB_BLOCKS * pitch;
            for (int idx = lane; idx < MAX_SB_BLOCKS * p.nkb; idx += 32) {
                const int j = idx / p.nkb;
                const int kb = idx - j * p.nkb;
                if (j < ti.sb_rows)
                    cp_async_4(dst + j * pitch + kb, p.sb + (size_t)(ti.sb_row0 + j) * p.nkb + kb);
            }
            cp_async_mbar_arrive_noinc(&sb_full[slot]);
            if (lane == 0) {
                const int halves = (MW == 1) ? 1 : (ti.rows > HALF_M ? 2 : 1);
                const uint32_t ab_bytes = halves * T::A_HALF_BYTES + T::B_BYTES;
                for (int kb = 0; kb < p.nkb; ++kb) {
                    const int s = (int)(stage_it % (uint32_t)stages);
                    if (!wait_bar(&empty[s], ((stage_it / stages) & 1) ^ 1, abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    uint8_t *a_dst = smem + plan.off_stages + (uint32_t)s * plan.stage_bytes;
                    uint8_t *b_dst = a_dst + plan.a_bytes;
                    mbar_arrive_expect_tx(&full[s], ab_bytes);
                    for (int h = 0; h < halves; ++h)
                        tma_load_2d(a_dst + h * T::A_HALF_BYTES, &tmap_a, &full[s], kb * BLOCK_K,
                                    ti.a_row0 + h * HALF_M);
                    tma_load_2d(b_dst, &tmap_b, &full[s], kb * BLOCK_K, ti.b_row0);
                    ++stage_it;

                    const int f = (int)(sf_it % (uint32_t)sf_stages);
                    if (!wait_bar(&sf_empty[f], ((sf_it / sf_stages) & 1) ^ 1, abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sf_full[f], halves * HALF_M * 4);
                    for (int h = 0; h < halves; ++h)
                        tma_load_2d(sf_ring + f * MW * HALF_M + h * HALF_M, &tmap_sa, &sf_full[f],
                                    ti.m0 + h * HALF_M, ti.sa_y0 + kb);
                    ++sf_it;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            ++tile_it;
        }
        // Drain: every copy issued must land before the CTA exits.
        cp_async_wait_all();
        if (lane == 0) {
            const uint32_t n = stage_it < (uint32_t)stages ? stage_it : (uint32_t)stages;
            for (uint32_t i = stage_it - n; i < stage_it; ++i)
                wait_drain(&full[i % stages], (i / stages) & 1, abort_flag, p);
            const uint32_t nf = sf_it < (uint32_t)sf_stages ? sf_it : (uint32_t)sf_stages;
            for (uint32_t i = sf_it - nf; i < sf_it; ++i)
                wait_drain(&sf_full[i % sf_stages], (i / sf_stages) & 1, abort_flag, p);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        regs_dec<REGS_PRODUCER>();
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(BN);
            uint32_t stage_it = 0, kb_it = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
                const TileInfo ti = get_tile<MW, BN>(p, t, prefix);
                if (!ti.valid)
                    continue;
                const int halves = (MW == 1) ? 1 : (ti.rows > HALF_M ? 2 : 1);
                for (int kb = 0; kb < p.nkb; ++kb) {
                    const int s = (int)(stage_it % (uint32_t)stages);
                    if (!wait_bar(&full[s], (stage_it / stages) & 1, abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    const int buf = kb_it & 1;
                    if (!wait_bar(&tmem_empty[buf], ((kb_it >> 1) & 1) ^ 1, abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base =
                        smem_addr(smem + plan.off_stages + (uint32_t)s * plan.stage_bytes);
                    const uint32_t b_base = a_base + plan.a_bytes;
                    for (int h = 0; h < halves; ++h) {
                        const uint32_t d = tmem_base + (uint32_t)(buf * T::BUF_COLS + h * BN);
#pragma unroll
                        for (int k = 0; k < BLOCK_K / MMA_K; ++k)
                            mma_f8f6f4(d, make_sdesc(a_base + h * T::A_HALF_BYTES + k * MMA_K),
                                       make_sdesc(b_base + k * MMA_K), idesc, k > 0 ? 1u : 0u);
                    }
                    mma_commit(&empty[s]);
                    mma_commit(&tmem_full[buf]);
                    ++stage_it;
                    ++kb_it;
                }
            }
            // Drain: all MMAs complete before TMEM is released.
            mma_commit(mma_done);
            wait_drain(mma_done, 0, abort_flag, p);
        }
    } else if (warp < FIRST_EPI_WARP) {
        regs_dec<REGS_PRODUCER>(); // warps 2-3: idle until the end
    } else {
        // ------------------------------------------------------------ epilogue
        regs_inc<REGS_EPILOGUE>();
        constexpr int NC = T::COLS_PER_THREAD;
        const int ew = warp - FIRST_EPI_WARP;
        const int wg = ew >> 2;                 // epilogue warpgroup 0 / 1
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int col0 = (MW == 1) ? wg * NC : 0;
        const int half = (MW == 1) ? 0 : wg;
        const int row_in_tile = half * HALF_M + q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        uint32_t kb_it = 0, sf_it = 0, tile_it = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
            const TileInfo ti = get_tile<MW, BN>(p, t, prefix);
            if (!ti.valid)
                continue;
            const int slot = tile_it & 1;
            if (!wait_bar_warp(&sb_full[slot], (tile_it >> 1) & 1, abort_flag, p))
                break;
            const float *sbt = sb_tile + slot * MAX_SB_BLOCKS * pitch;
            const bool active = (MW == 1) || (half * HALF_M < ti.rows);
            const int cbase = ti.n0 + col0;
            // scale blocks of this thread's columns: lo = block of its first
            // column (relative to the tile's first block), t = local column
            // where the next block starts
            const int lo = (cbase >> 7) - (ti.n0 >> 7);
            const int t_split = ((cbase >> 7) + 1) * 128 - cbase;
            const bool split = t_split < NC;
            float acc[NC];
#pragma unroll
            for (int c = 0; c < NC; ++c)
                acc[c] = 0.0f;
            for (int kb = 0; kb < p.nkb; ++kb) {
                const int buf = kb_it & 1;
                if (!wait_bar_warp(&tmem_full[buf], (kb_it >> 1) & 1, abort_flag, p)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int f = (int)(sf_it % (uint32_t)sf_stages);
                if (!wait_bar_warp(&sf_full[f], (sf_it / sf_stages) & 1, abort_flag, p)) {
                    ok = false;
                    break;
                }
                const float sa_v = sf_ring[f * MW * HALF_M + row_in_tile];
                const float s_lo = sa_v * sbt[lo * pitch + kb];
                const uint32_t taddr =
                    tmem_base + lane_off + (uint32_t)(buf * T::BUF_COLS + half * BN + col0);
                if (active) {
                    if (split)
                        promote<NC, true>(acc, taddr, s_lo, sa_v * sbt[(lo + 1) * pitch + kb],
                                          t_split);
                    else
                        promote<NC, false>(acc, taddr, s_lo, s_lo, NC);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&tmem_empty[buf]);
                    mbar_arrive(&sf_empty[f]);
                }
                ++kb_it;
                ++sf_it;
            }
            if (!ok)
                break;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sb_empty[slot]);
            ++tile_it;

            // ---- store this thread's row segment as BF16
            bool row_ok = active && row_in_tile < ti.rows;
            if (row_ok && p.kind == KIND_CONTIGUOUS) {
                const int e = __ldg(p.m_indices + ti.d_row0 + row_in_tile);
                if (e != ti.g) {
                    row_ok = false;
                    if (e >= 0)
                        atomicOr(p.status, DEVERR_BAD_INDEX);
                }
            }
            if (row_ok) {
                uint16_t *drow = p.D + (size_t)(ti.d_row0 + row_in_tile) * p.N + cbase;
#pragma unroll
                for (int c = 0; c < NC; c += 8) {
                    if (cbase + c < p.N)
                        st_global_v4(drow + c, pack_bf16x2(acc[c], acc[c + 1]),
                                     pack_bf16x2(acc[c + 2], acc[c + 3]),
                                     pack_bf16x2(acc[c + 4], acc[c + 5]),
                                     pack_bf16x2(acc[c + 6], acc[c + 7]));
                }
            }
        }
    }

    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, T::TMEM_COLS);
    }
}

} // namespace fp8nt
