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
//   warp 0      TMA producer of the A tiles (one lane per 128-row half).
//   warp 2      TMA producer of the B tiles; at set-up it also counts the
//               masked form's tiles per group.  The two producers' copies of a
//               stage meet on one full barrier (two arrivals, each with its
//               byte count), so their issue latencies overlap.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer: one
//               128-K block per MMA group into a ring of TMEM buffers, fresh
//               accumulation per block so each block's partial stays
//               separable; one commit per K block frees the operand stage and
//               publishes the partial.
//   warp 3      scale producer: the tile's RHS scales (cp.async) and the LHS
//               scales of the CTA's rows, several K blocks per TMA box, into
//               two small rings the epilogue releases.
//   warps 4-11  promotion epilogue: tcgen05.ld of the blocks' partials, FMA
//               with sa*sb into FP32 registers, then BF16 into a shared
//               staging tile and asynchronous TMA stores.
// Variants: PAIR (a cluster of two CTAs computes a 256-row tile with
// cta_group::2 MMAs), SCALAR (per-tensor scaling: the whole K range
// accumulates in TMEM and the epilogue reads each tile once), and split-K
// over a thread-block cluster (runtime, dense only).
//
// Tile shape: BLOCK_M = 128 * MW rows (MW = 2 issues two M=128 MMAs that share
// the B tile), BLOCK_N = BN columns, BN a multiple of 16 in [16, 256] so that
// non-power-of-two widths can fill the SMs (README, unaligned block sizes).
#pragma once

#include <cuda_bf16.h>

#include "params.h"
#include "ptx.cuh"

namespace fp8nt {

template <int MW, int BN, bool PAIR = false, bool SCALAR = false>
struct KernelTraits {
    static_assert(MW == 1 || MW == 2, "MW is 1 or 2");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN must be a multiple of 16 in [16, 256]");
    static_assert(MW == 1 || BN <= 128, "two M halves need BN <= 128 (TMEM and registers)");
    static_assert(!PAIR || (MW == 1 && BN % 32 == 0), "a CTA pair splits B in halves of BN/2 rows");
    // rows of the tile a CTA (or, with PAIR, a CTA pair) computes
    static constexpr int BLOCK_M = PAIR ? 2 * HALF_M : MW * HALF_M;
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN; // rows of B each CTA loads
    // LHS scales reach shared memory in blocks of SA_GROUP K blocks x
    // SA_ROWS rows (the CTA's rows), SA_SLOT_BYTES per ring slot
    static constexpr int SA_ROWS = PAIR ? HALF_M : MW * HALF_M;
    static constexpr int SA_GROUP = (int)SA_SLOT_BYTES / (SA_ROWS * 4);
    // 32-column chunks of an epilogue thread's columns (output staging)
    static constexpr int OUT_CHUNKS = ((MW == 1 ? BN / 2 : BN) + 31) / 32;
    static constexpr int BUF_COLS = MW * BN;                 // TMEM columns per K-block buffer
    // ring of K-block partial buffers in TMEM: as many as fit, at most 16
    // (SCALAR: one whole-K accumulator per tile, two tiles in flight)
    static constexpr int NBUF = SCALAR ? 2
                              : (512 / BUF_COLS) < MAX_TMEM_BUFS ? (512 / BUF_COLS) : MAX_TMEM_BUFS;
    static_assert(!SCALAR || (MW == 1 && !PAIR), "per-tensor scaling uses one 128-row CTA per tile");
    static constexpr int TMEM_NEED = NBUF * BUF_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                   : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int COLS_PER_THREAD = (MW == 1) ? BN / 2 : BN;
    // a thread's whole partial fits one 64-register batch: the next K block's
    // partial can then be in flight while the current one is multiplied in
    static constexpr bool PREFETCH = COLS_PER_THREAD <= 64;
    // K blocks promoted per epilogue step: their partials (GROUP x
    // COLS_PER_THREAD <= 64 registers) are loaded with one wait and their
    // buffers released together, which amortises the per-block handshake.
    static constexpr int GROUP_BY_REGS = PREFETCH ? 64 / COLS_PER_THREAD : 1;
    static constexpr int GROUP = GROUP_BY_REGS < NBUF / 2 ? GROUP_BY_REGS : (NBUF / 2 > 0 ? NBUF / 2 : 1);
    static constexpr uint32_t A_HALF_BYTES = HALF_M * BLOCK_K;
    static constexpr uint32_t B_BYTES = B_ROWS * BLOCK_K;
    static_assert(NBUF >= 2 && NBUF <= MAX_TMEM_BUFS && TMEM_NEED <= 512, "TMEM holds 512 columns");
    static_assert(COLS_PER_THREAD % 8 == 0, "epilogue works in 8-column chunks");
};

// Instruction descriptor of tcgen05.mma kind::f8f6f4: D FP32, A and B E4M3,
// both K-major, M = 128 (256 for a CTA pair), N = BN, dense.
__host__ __device__ constexpr uint32_t make_idesc(int bn, int m = HALF_M)
{
    return (1u << 4)                          // D format: F32
           | (0u << 7) | (0u << 10)           // A, B format: E4M3
           | (0u << 15) | (0u << 16)          // A, B K-major
           | ((uint32_t)(bn >> 3) << 17)      // N / 8
           | ((uint32_t)(m >> 4) << 24);      // M / 16
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

// The same with a given stride between 8-row groups (bytes, a multiple of 16).
__device__ __forceinline__ uint64_t make_sdesc_sbo(uint32_t saddr, uint32_t sbo_bytes)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

struct TileInfo {
    int valid;   // 0: nothing to compute (contiguous padding block, bad expert)
    int g;       // group (masked) / expert (contiguous) / 0 (dense)
    int m0;      // first row of the tile within its group
    int n0;      // first column
    int rows;    // rows of the tile that hold valid data (<= BLOCK_M)
    int a_row0;  // row coordinate of the tile in A's 2-D tensor map
    int b_row0;  // row coordinate in B's 2-D tensor map
    int sa_y0;   // row of sa ([G*K/128][ld]) holding K block 0 of this group
    int sb_row0; // first sb row (128-column block) of the tile, group base included
    int sb_rows; // sb rows present from sb_row0 within the group (<= 3)
    int d_row0;  // row of D (all groups flattened) holding row m0
};

// Contiguous form: the expert of tile t's M block (m_indices of its first
// row), or 0 for the other forms and for t past the last tile.
template <int MW, int BN, bool PAIR>
__device__ __forceinline__ int expert_of_tile(const Params &p, int t, int num_tiles)
{
    if (p.kind != KIND_CONTIGUOUS || t >= num_tiles)
        return 0;
    constexpr int BM = KernelTraits<MW, BN, PAIR>::BLOCK_M;
    return __ldg(p.m_indices + (t / p.n_blocks) * BM);
}

// Tile t of this CTA's walk; `e` is the tile's expert for the contiguous form
// (expert_of_tile, read ahead by the caller).
template <int MW, int BN, bool PAIR>
__device__ __forceinline__ TileInfo get_tile(const Params &p, int t, const int *prefix, int pair_rank, int e)
{
    constexpr int BM = KernelTraits<MW, BN, PAIR>::BLOCK_M;
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
    if (PAIR) {
        // this CTA's 128 rows of the pair's 256, and its half of B
        const int off = pair_rank * HALF_M;
        ti.m0 += off;
        ti.a_row0 += off;
        ti.d_row0 += off;
        ti.rows = max(0, min(HALF_M, ti.rows - off));
        ti.b_row0 += pair_rank * (BN / 2);
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

// Issue tcgen05.ld for columns [C, N) of a thread's lane into v[C..N):
// 32-column loads, then a 16- and / or 8-column tail.  No wait.
template <int N, int C = 0>
__device__ __forceinline__ void tmem_issue_p(uint32_t taddr, float *v)
{
    if constexpr (C < N) {
        constexpr int W = (N - C >= 32) ? 32 : ((N - C >= 16) ? 16 : 8);
        if constexpr (W == 32)
            tmem_ld32(taddr + C, *reinterpret_cast<float(*)[32]>(v + C));
        else if constexpr (W == 16)
            tmem_ld16(taddr + C, *reinterpret_cast<float(*)[16]>(v + C));
        else
            tmem_ld8p(taddr + C, v + C);
        tmem_issue_p<N, C + W>(taddr, v);
    }
}

template <int N>
__device__ __forceinline__ void tmem_issue(uint32_t taddr, float (&v)[64])
{
    tmem_issue_p<N>(taddr, v);
}

// Wait for every outstanding tcgen05.ld of this thread; all 64 registers are
// tied to the wait so that none of them is read before it.
__device__ __forceinline__ void tmem_wait64(float (&v)[64])
{
    tmem_wait_ld(*reinterpret_cast<float(*)[32]>(&v[0]));
    reg_tie32(*reinterpret_cast<float(*)[32]>(&v[32]));
}

// acc[C0 + j] += v[j] * scale for j in [0, N), two columns per instruction.
// SPLIT: local columns before t use s_lo, the rest s_hi (chosen per 8
// columns; a thread owns at most 128 columns, so they span at most two
// 128-wide scale blocks).
template <int NC, int C0, int N, bool SPLIT>
__device__ __forceinline__ void fma_range(float (&acc)[NC], const float (&v)[64], float s_lo,
                                          float s_hi, int t)
{
    const uint64_t s2_lo = splat2(s_lo);
#pragma unroll
    for (int j = 0; j < N; j += 8) {
        const uint64_t s2 = SPLIT ? splat2(C0 + j < t ? s_lo : s_hi) : s2_lo;
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            ffma2(acc[C0 + j + i], acc[C0 + j + i + 1], v[j + i], v[j + i + 1], s2);
    }
}

// acc[c] += v[c] * scale(c) for all NC columns, v a pointer into a
// register array (compile-time offset after unrolling).
template <int NC, bool SPLIT>
__device__ __forceinline__ void fma_all_p(float (&acc)[NC], const float *v, float s_lo, float s_hi,
                                          int t)
{
    const uint64_t s2_lo = splat2(s_lo);
#pragma unroll
    for (int j = 0; j < NC; j += 8) {
        const uint64_t s2 = SPLIT ? splat2(j < t ? s_lo : s_hi) : s2_lo;
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            ffma2(acc[j + i], acc[j + i + 1], v[j + i], v[j + i + 1], s2);
    }
}

template <int NC, int C0, int N>
__device__ __forceinline__ void fma_range_any(float (&acc)[NC], const float (&v)[64], float s_lo,
                                              float s_hi, int t, bool split)
{
    if (split)
        fma_range<NC, C0, N, true>(acc, v, s_lo, s_hi, t);
    else
        fma_range<NC, C0, N, false>(acc, v, s_lo, s_hi, t);
}

template <int MW, int BN, bool PAIR, bool SCALAR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_sa,
                    const __grid_constant__ CUtensorMap tmap_d, const __grid_constant__ Params p)
{
    using T = KernelTraits<MW, BN, PAIR, SCALAR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const SmemPlan &plan = p.plan;
    const int stages = p.stages;

    // full[s]: stage s holds its operands (two arrivals: the A and the B
    // producer warp, each with its bytes); done[j]: the MMAs of K block j
    // (counted per CTA, j mod DONE_RING) have completed, which both frees
    // their operand stage and makes their TMEM partial readable;
    // tmem_empty[b]: the epilogue has read TMEM buffer b.
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + plan.off_bars);
    uint64_t *done = full + stages;
    uint64_t *tmem_empty = done + DONE_RING;
    uint64_t *sb_full = tmem_empty + MAX_TMEM_BUFS;
    uint64_t *sb_empty = sb_full + 2;
    uint64_t *sa_full = sb_empty + 2;  // LHS-scale ring (2 slots)
    uint64_t *sa_empty = sa_full + 2;
    uint64_t *mma_done = sa_empty + 2;
    uint64_t *tile_full = mma_done + 1; // per-tensor scaling: a tile's accumulator is complete (x2)
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + plan.off_misc);
    volatile uint32_t *abort_flag = misc + 1;
    int *prefix = reinterpret_cast<int *>(smem + plan.off_prefix);
    float *sb_tile = reinterpret_cast<float *>(smem + plan.off_sb);
    float *sa_ring = reinterpret_cast<float *>(smem + plan.off_sa);
    const int pitch = (int)plan.sb_pitch;

    // ---------------------------------------------------------------- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s)
            mbar_init(&full[s], 2);
        for (int j = 0; j < DONE_RING; ++j)
            mbar_init(&done[j], 1);
        for (int b = 0; b < T::NBUF; ++b) {
            // a pair's leader also counts the peer's epilogue warps
            mbar_init(&tmem_empty[b], PAIR ? 2 * NUM_EPI_WARPS : NUM_EPI_WARPS);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sb_full[b], 32);
            mbar_init(&sb_empty[b], NUM_EPI_WARPS);
            mbar_init(&sa_full[b], 1);
            mbar_init(&sa_empty[b], NUM_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        mbar_init(&tile_full[0], 1);
        mbar_init(&tile_full[1], 1);
        misc[1] = 0u;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        if (!SCALAR)
            tma_prefetch_desc(&tmap_sa);
        tma_prefetch_desc(&tmap_d);
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(misc, T::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(misc, T::TMEM_COLS);
            tmem_relinquish();
        }
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
    if constexpr (PAIR)
        cluster_sync(); // the peer may arrive on the leader's barriers from here on
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const int num_tiles = (p.kind == KIND_MASKED) ? prefix[p.num_groups] : p.num_tiles;
    // Split-K: the p.split CTAs of a cluster share one output tile, each
    // computing K blocks [kb_lo, kb_hi); otherwise CTAs are persistent over
    // tiles and cover all K blocks.
    const bool split_k = !PAIR && !SCALAR && p.split > 1;
    const int split_rank = split_k ? (int)cluster_ctarank() : 0;
    // a CTA pair walks the pair tiles together; rank 0 is the leader
    const int pair_rank = PAIR ? (int)cluster_ctarank() : 0;
    const bool leader = pair_rank == 0;
    const int t_first = split_k ? (int)blockIdx.x / p.split
                                : (PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x);
    const int t_stride = split_k ? num_tiles : (PAIR ? (int)gridDim.x / 2 : (int)gridDim.x);
    const int kb_lo = split_k ? min(p.nkb, split_rank * p.kb_chunk) : 0;
    const int kb_hi = split_k ? min(p.nkb, kb_lo + p.kb_chunk) : p.nkb;

    if (warp == 0 || warp == 2) {
        // ------------------------------------------------------------ producers
        // Warp 0 loads the A tile, warp 2 the B tile: two threads issue each
        // stage's copies, so that the issue latencies of the two overlap.
        regs_dec<REGS_PRODUCER>();
        const bool a_side = warp == 0;
        uint32_t it = 0, s = 0;
        bool ok = true;
        // the next tile's expert (contiguous form: a global read) is read
        // one tile ahead, so that it overlaps this tile
        int e_next = expert_of_tile<MW, BN, PAIR>(p, t_first, num_tiles);
        for (int t = t_first; ok && t < num_tiles; t += t_stride) {
            const TileInfo ti = get_tile<MW, BN, PAIR>(p, t, prefix, pair_rank, e_next);
            e_next = expert_of_tile<MW, BN, PAIR>(p, t + t_stride, num_tiles);
            if (!ti.valid)
                continue;
            // A: lanes 0..halves-1 copy the 128-row halves; B: lane 0
            const int halves = (MW == 1) ? 1 : (ti.rows > HALF_M ? 2 : 1);
            const uint32_t bytes = a_side ? halves * T::A_HALF_BYTES : T::B_BYTES;
            const bool copier = a_side ? lane < halves : lane == 0;
            const CUtensorMap *my_map = a_side ? &tmap_a : &tmap_b;
            const int my_row = a_side ? ti.a_row0 + lane * HALF_M : ti.b_row0;
            const uint32_t my_off = a_side ? (uint32_t)lane * T::A_HALF_BYTES : plan.a_bytes;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                int got = 1;
                if (lane == 0) {
                    // stage s was last used by K block it - stages
                    if (it >= (uint32_t)stages) {
                        const uint32_t j = it - (uint32_t)stages;
                        got = wait_bar(&done[j % DONE_RING], (j / DONE_RING) & 1, abort_flag, p) ? 1 : 0;
                    }
                    // a pair's leader expects both CTAs' bytes on its barrier
                    if (got && leader)
                        mbar_arrive_expect_tx(&full[s], PAIR ? 2 * bytes : bytes);
                }
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    ok = false;
                    break;
                }
                if (copier) {
                    uint8_t *dst = smem + plan.off_stages + s * plan.stage_bytes + my_off;
                    if constexpr (PAIR)
                        tma_load_2d_pair(dst, my_map, map_shared_rank(smem_addr(&full[s]), 0u),
                                         kb * BLOCK_K, my_row);
                    else
                        tma_load_2d(dst, my_map, &full[s], kb * BLOCK_K, my_row);
                }
                ++it;
                if (++s == (uint32_t)stages)
                    s = 0;
            }
        }
        // Drain: every copy issued must land before the CTA exits (the full
        // barriers count both producers' bytes, and a peer's copies are
        // counted on the leader's barriers).
        if (a_side && lane == 0 && leader) {
            const uint32_t n = it < (uint32_t)stages ? it : (uint32_t)stages;
            for (uint32_t i = it - n; i < it; ++i)
                wait_drain(&full[i % stages], (i / stages) & 1, abort_flag, p);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        regs_dec<REGS_PRODUCER>();
        if (lane == 0 && leader) { // a pair's MMAs are issued by the leader alone
            constexpr uint32_t idesc = make_idesc(BN, PAIR ? 2 * HALF_M : HALF_M);
            // descriptors of stage 0; a stage, an M half and a K step move
            // the start-address field (address / 16, 14 bits: no carry for
            // shared-memory addresses)
            const uint64_t a_desc0 = make_sdesc(smem_addr(smem + plan.off_stages));
            const uint64_t b_desc0 = make_sdesc(smem_addr(smem + plan.off_stages) + plan.a_bytes);
            const uint32_t stage_step = plan.stage_bytes >> 4;
            uint32_t kb_it = 0, s = 0, phase = 0;
            bool ok = true;
            if constexpr (SCALAR) {
                // Per-tensor scaling: the tile's whole K range accumulates in
                // TMEM buffer (tile mod 2); one commit per K block frees its
                // stage, one more at the last K block publishes the tile.
                uint32_t tile_it = 0;
                // the next tile's expert (contiguous form: a global read) is read
                // one tile ahead, so that it overlaps this tile
                int e_next = expert_of_tile<MW, BN, PAIR>(p, t_first, num_tiles);
                for (int t = t_first; ok && t < num_tiles; t += t_stride) {
                    const TileInfo ti = get_tile<MW, BN, PAIR>(p, t, prefix, pair_rank, e_next);
                    e_next = expert_of_tile<MW, BN, PAIR>(p, t + t_stride, num_tiles);
                    if (!ti.valid)
                        continue;
                    const uint32_t buf = tile_it & 1;
                    if (!wait_bar(&tmem_empty[buf], ((tile_it >> 1) & 1) ^ 1, abort_flag, p))
                        break;
                    const uint32_t d = tmem_base + buf * (uint32_t)BN;
                    for (int kb = kb_lo; kb < kb_hi; ++kb) {
                        if (!wait_bar(&full[s], phase, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t a_desc = a_desc0 + s * stage_step;
                        const uint64_t b_desc = b_desc0 + s * stage_step;
#pragma unroll
                        for (int k = 0; k < BLOCK_K / MMA_K; ++k)
                            mma_f8f6f4(d, a_desc + (uint64_t)((k * MMA_K) >> 4),
                                       b_desc + (uint64_t)((k * MMA_K) >> 4), idesc,
                                       (kb > kb_lo || k > 0) ? 1u : 0u);
                        mma_commit(&done[kb_it % DONE_RING]);
                        if (kb == kb_hi - 1)
                            mma_commit(&tile_full[buf]);
                        ++kb_it;
                        if (++s == (uint32_t)stages) {
                            s = 0;
                            phase ^= 1u;
                        }
                    }
                    ++tile_it;
                }
            }
            // the next tile's expert (contiguous form: a global read) is read
            // one tile ahead, so that it overlaps this tile
            int e_next = expert_of_tile<MW, BN, PAIR>(p, t_first, num_tiles);
            for (int t = t_first; !SCALAR && ok && t < num_tiles; t += t_stride) {
                const TileInfo ti = get_tile<MW, BN, PAIR>(p, t, prefix, pair_rank, e_next);
                e_next = expert_of_tile<MW, BN, PAIR>(p, t + t_stride, num_tiles);
                if (!ti.valid)
                    continue;
                const int halves = (MW == 1) ? 1 : (ti.rows > HALF_M ? 2 : 1);
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!wait_bar(&full[s], phase, abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    // The epilogue promotes K blocks in groups of GROUP (per
                    // tile, from K block 0) and releases a group's buffers
                    // together, each warp in order: at the first block of a
                    // group, waiting for the release of the group's last
                    // buffer covers the whole group.
                    const int gpos = (kb - kb_lo) % T::GROUP;
                    const int buf = (int)(kb_it % T::NBUF);
                    if (gpos == 0) {
                        const int cnt = min(T::GROUP, kb_hi - kb);
                        const uint32_t last = kb_it + (uint32_t)(cnt - 1);
                        if (!wait_bar(&tmem_empty[last % T::NBUF], ((last / T::NBUF) & 1) ^ 1,
                                      abort_flag, p)) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint64_t a_desc = a_desc0 + s * stage_step;
                    const uint64_t b_desc = b_desc0 + s * stage_step;
                    for (int h = 0; h < halves; ++h) {
                        const uint32_t d = tmem_base + (uint32_t)(buf * T::BUF_COLS + h * BN);
#pragma unroll
                        for (int k = 0; k < BLOCK_K / MMA_K; ++k) {
                            const uint64_t ad = a_desc + (uint64_t)((h * T::A_HALF_BYTES + k * MMA_K) >> 4);
                            const uint64_t bd = b_desc + (uint64_t)((k * MMA_K) >> 4);
                            if constexpr (PAIR)
                                mma_f8f6f4_pair(d, ad, bd, idesc, k > 0 ? 1u : 0u);
                            else
                                mma_f8f6f4(d, ad, bd, idesc, k > 0 ? 1u : 0u);
                        }
                    }
                    // one commit per K block frees its stage and publishes its
                    // partial (a pair's commit reaches both CTAs)
                    if constexpr (PAIR)
                        mma_commit_pair_mc(&done[kb_it % DONE_RING], 0x3);
                    else
                        mma_commit(&done[kb_it % DONE_RING]);
                    ++kb_it;
                    if (++s == (uint32_t)stages) {
                        s = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Drain: all MMAs complete before TMEM is released.
            if constexpr (PAIR)
                mma_commit_pair(mma_done);
            else
                mma_commit(mma_done);
            wait_drain(mma_done, 0, abort_flag, p);
        }
    } else if (warp == 3 && SCALAR) {
        regs_dec<REGS_PRODUCER>(); // per-tensor scaling: no scale tiles to load
    } else if (warp == 3) {
        // ------------------------------------------------------------ scales
        // Per tile, the RHS scales (<= 3 rows of K/128 floats, cp.async by
        // all lanes); per SA_GROUP K blocks, the LHS scales of the CTA's
        // rows (one TMA box of SA_GROUP x SA_ROWS floats, lane 0) into a
        // two-slot ring that the epilogue releases.
        regs_dec<REGS_PRODUCER>();
        uint32_t tile_it = 0, grp_it = 0;
        bool ok = true;
        // the next tile's expert (contiguous form: a global read) is read
        // one tile ahead, so that it overlaps this tile
        int e_next = expert_of_tile<MW, BN, PAIR>(p, t_first, num_tiles);
        for (int t = t_first; ok && t < num_tiles; t += t_stride) {
            const TileInfo ti = get_tile<MW, BN, PAIR>(p, t, prefix, pair_rank, e_next);
            e_next = expert_of_tile<MW, BN, PAIR>(p, t + t_stride, num_tiles);
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
            ++tile_it;
            for (int k0 = kb_lo; k0 < kb_hi; k0 += T::SA_GROUP) {
                const uint32_t gs = grp_it & 1;
                int got = 1;
                if (lane == 0) {
                    got = wait_bar(&sa_empty[gs], ((grp_it >> 1) & 1) ^ 1, abort_flag, p) ? 1 : 0;
                    if (got) {
                        mbar_arrive_expect_tx(&sa_full[gs], SA_SLOT_BYTES);
                        tma_load_2d(sa_ring + gs * (SA_SLOT_BYTES / 4), &tmap_sa, &sa_full[gs], ti.m0,
                                    ti.sa_y0 + k0);
                    }
                }
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
                ++grp_it;
            }
        }
        // Drain: the last copies must land before the CTA exits.
        cp_async_wait_all();
        if (lane == 0) {
            const uint32_t n = grp_it < 2u ? grp_it : 2u;
            for (uint32_t i = grp_it - n; i < grp_it; ++i)
                wait_drain(&sa_full[i & 1], (i >> 1) & 1, abort_flag, p);
        }
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
        uint32_t kb_it = 0, tile_it = 0, sa_it = 0;
        bool ok = true;
        // the next tile's expert (contiguous form: a global read) is read
        // one tile ahead, so that it overlaps this tile
        int e_next = expert_of_tile<MW, BN, PAIR>(p, t_first, num_tiles);
        for (int t = t_first; ok && t < num_tiles; t += t_stride) {
            const TileInfo ti = get_tile<MW, BN, PAIR>(p, t, prefix, pair_rank, e_next);
            e_next = expert_of_tile<MW, BN, PAIR>(p, t + t_stride, num_tiles);
            if (!ti.valid)
                continue;
            const bool active = (MW == 1) ? true : (half * HALF_M < ti.rows);
            const int cbase = ti.n0 + col0;
            // contiguous form: the expert of this thread's row, read now (a
            // global read) and checked when the tile is stored
            int row_expert = 0;
            if (p.kind == KIND_CONTIGUOUS && active && row_in_tile < ti.rows)
                row_expert = __ldg(p.m_indices + ti.d_row0 + row_in_tile);
            float acc[NC];
            if constexpr (SCALAR) {
                // Per-tensor scaling: read the tile's accumulator once, scale
                // it by scale_a * scale_b, hand the buffer back.
                const uint32_t buf = tile_it & 1;
                if (!wait_bar_warp(&tile_full[buf], (tile_it >> 1) & 1, abort_flag, p))
                    break;
                tc_fence_after();
                const float scale = __ldg(p.sa) * __ldg(p.sb);
                const uint32_t taddr = tmem_base + lane_off + buf * (uint32_t)BN + (uint32_t)col0;
                static_assert(NC % 32 == 0, "per-tensor tiles load 32-column chunks");
#pragma unroll
                for (int c = 0; c < NC; c += 32) {
                    float(&v)[32] = *reinterpret_cast<float(*)[32]>(&acc[c]);
                    tmem_ld32(taddr + c, v);
                    tmem_wait_ld(v);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] *= scale;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&tmem_empty[buf]);
                ++tile_it;
            } else {
            const int slot = tile_it & 1;
            if (!wait_bar_warp(&sb_full[slot], (tile_it >> 1) & 1, abort_flag, p))
                break;
            const float *sbt = sb_tile + slot * MAX_SB_BLOCKS * pitch;
            // scale blocks of this thread's columns: lo = block of its first
            // column (relative to the tile's first block), t_split = local
            // column where the next block starts
            const int lo = (cbase >> 7) - (ti.n0 >> 7);
            const int t_split = ((cbase >> 7) + 1) * 128 - cbase;
            const bool split = t_split < NC;
            // LHS scales of this thread's row come from the shared-memory
            // ring, SA_GROUP K blocks per slot; K blocks are consumed in
            // order, so a slot is awaited at its first K block and released
            // after its last (rows past M read the zero fill and are never
            // stored)
            // (returns false if the wait for a slot failed: the caller stops)
            auto scales = [&](int kb, float &s_lo, float &s_hi) {
                const int gpos = (kb - kb_lo) % T::SA_GROUP;
                const uint32_t gs = sa_it & 1;
                if (gpos == 0 && !wait_bar_warp(&sa_full[gs], (sa_it >> 1) & 1, abort_flag, p))
                    return false;
                const float sa_v = sa_ring[gs * (SA_SLOT_BYTES / 4) + gpos * T::SA_ROWS + row_in_tile];
                if (gpos == T::SA_GROUP - 1 || kb == kb_hi - 1) {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&sa_empty[gs]);
                    ++sa_it;
                }
                s_lo = sa_v * sbt[lo * pitch + kb];
                // the next scale block exists only where the columns cross into it
                s_hi = split ? sa_v * sbt[(lo + 1) * pitch + kb] : s_lo;
                return true;
            };
#pragma unroll
            for (int c = 0; c < NC; ++c)
                acc[c] = 0.0f;
            const uint32_t t_lane = tmem_base + lane_off + (uint32_t)(half * BN + col0);
            auto buf_addr = [&](uint32_t it) {
                return t_lane + (uint32_t)((int)(it % T::NBUF) * T::BUF_COLS);
            };
            // wait for K block `it`'s partial in TMEM
            auto wait_full = [&](uint32_t it) {
                const bool r = wait_bar_warp(&done[it % DONE_RING], (it / DONE_RING) & 1, abort_flag, p);
                tc_fence_after();
                return r;
            };
            // hand K blocks [it, it + cnt) back to the MMA issuer
            auto release = [&](uint32_t it, int cnt) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    for (int j = 0; j < cnt; ++j) {
                        uint64_t *bar = &tmem_empty[(it + j) % T::NBUF];
                        if (PAIR && !leader)
                            mbar_arrive_cluster(map_shared_rank(smem_addr(bar), 0u));
                        else
                            mbar_arrive(bar);
                    }
            };
            if constexpr (T::PREFETCH) {
                // Steps of up to GROUP K blocks: their partials are loaded
                // together (one wait) and multiplied in while the next step's
                // partials are in flight.
                constexpr int G = T::GROUP;
                float ra[64], rb[64];
                auto load_step = [&](uint32_t it0, int cnt, float (&v)[64]) {
                    // partials complete in issue order: the last one's
                    // barrier covers the step
                    if (!wait_full(it0 + cnt - 1))
                        return false;
                    if (active) {
#pragma unroll
                        for (int j = 0; j < G; ++j)
                            if (j < cnt)
                                tmem_issue_p<NC>(buf_addr(it0 + j), &v[j * NC]);
                    }
                    return true;
                };
                // cur holds K blocks [kb0, kb0 + cnt), loaded and waited
                auto step = [&](float (&cur)[64], float (&nxt)[64], int kb0) {
                    const int cnt = min(G, kb_hi - kb0);
                    release(kb_it, cnt);
                    const int nkb0 = kb0 + cnt;
                    const bool more = nkb0 < kb_hi;
                    if (more && !load_step(kb_it + cnt, min(G, kb_hi - nkb0), nxt))
                        return false;
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        if (j < cnt) {
                            float s_lo, s_hi;
                            if (!scales(kb0 + j, s_lo, s_hi)) {
                                if (more && active)
                                    tmem_wait64(nxt); // no load left in flight
                                return false;
                            }
                            if (active) {
                                if (split)
                                    fma_all_p<NC, true>(acc, &cur[j * NC], s_lo, s_hi, t_split);
                                else
                                    fma_all_p<NC, false>(acc, &cur[j * NC], s_lo, s_hi, t_split);
                            }
                        }
                    }
                    if (more && active)
                        tmem_wait64(nxt);
                    kb_it += cnt;
                    return true;
                };
                if (kb_lo >= kb_hi) {
                    // empty K range (split-K with more splits than blocks): zero partial
                } else if (!load_step(kb_it, min(G, kb_hi - kb_lo), ra)) {
                    ok = false;
                } else {
                    if (active)
                        tmem_wait64(ra);
                    for (int kb0 = kb_lo; kb0 < kb_hi; kb0 += 2 * G) {
                        if (!step(ra, rb, kb0)) {
                            ok = false;
                            break;
                        }
                        if (kb0 + G < kb_hi && !step(rb, ra, kb0 + G)) {
                            ok = false;
                            break;
                        }
                    }
                }
            } else {
                // Two batches of at most 64 columns per K block.
                constexpr int B0 = 64;
                constexpr int B1 = NC - 64;
                float r[64];
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!wait_full(kb_it)) {
                        ok = false;
                        break;
                    }
                    if (active)
                        tmem_issue<B0>(buf_addr(kb_it), r);
                    float s_lo, s_hi;
                    if (!scales(kb, s_lo, s_hi)) {
                        if (active)
                            tmem_wait64(r); // no load left in flight
                        ok = false;
                        break;
                    }
                    if (active) {
                        tmem_wait64(r);
                        fma_range_any<NC, 0, B0>(acc, r, s_lo, s_hi, t_split, split);
                        tmem_issue<B1>(buf_addr(kb_it) + B0, r);
                        tmem_wait64(r);
                    }
                    release(kb_it, 1);
                    if (active)
                        fma_range_any<NC, B0, B1>(acc, r, s_lo, s_hi, t_split, split);
                    ++kb_it;
                }
            }
            if (!ok)
                break;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sb_empty[slot]);
            ++tile_it;

            if (split_k) {
                // split-K: leave this CTA's FP32 partial in shared memory for
                // the cluster reduction below
                float *red = reinterpret_cast<float *>(smem + plan.off_red);
                float *rrow = red + row_in_tile * (BN + RED_PAD) + col0;
#pragma unroll
                for (int c = 0; c < NC; c += 4)
                    *reinterpret_cast<float4 *>(rrow + c) =
                        make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
                continue;
            }
            } // non-scalar promotion

            // ---- store the tile's rows as BF16
            bool row_ok = active && row_in_tile < ti.rows;
            if (row_ok && p.kind == KIND_CONTIGUOUS) {
                const int e = row_expert;
                if (e != ti.g) {
                    row_ok = false;
                    if (e >= 0)
                        atomicOr(p.status, DEVERR_BAD_INDEX);
                }
            }
            // Each warp owns 32 rows and NC columns.  It writes them as BF16
            // into its part of the tile's staging buffer, 32 columns (2 KB)
            // per chunk: 64-byte rows whose 16-byte pieces are XOR-swizzled
            // by (row / 2) % 4, the TMA 64-byte swizzle, which also spreads
            // the writes over all banks.  Full chunks go out as TMA stores
            // (asynchronous: the warp moves on to the next tile) when every
            // row of the warp is stored, or for the dense form, whose tensor
            // map clips the rows past M; other chunks use plain 16-byte
            // stores of whole 64-byte row segments.
            const uint32_t row_mask = __ballot_sync(0xffffffffu, row_ok);
            const bool use_tma = row_mask != 0u && (row_mask == 0xffffffffu || p.kind == KIND_DENSE);
            const int slots = (int)plan.out_slots; // 2 KB chunk slots of this warp
            const uint32_t stg_w = smem_addr(smem + plan.off_out) +
                                   (uint32_t)ew * (uint32_t)(slots * OUT_STAGE_BYTES);
            const int warp_row0 = ti.d_row0 + half * HALF_M + q * 32;
            const int rd_sub = lane >> 2;  // row within an 8-row group (read side)
            const int rd_piece = lane & 3; // 16-byte piece within a 64-byte row chunk
            auto stage_chunk = [&](int c, uint32_t stg) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (c + 8 * j < NC)
                        st_shared_v4(stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4),
                                     pack_bf16x2(acc[c + 8 * j], acc[c + 8 * j + 1]),
                                     pack_bf16x2(acc[c + 8 * j + 2], acc[c + 8 * j + 3]),
                                     pack_bf16x2(acc[c + 8 * j + 4], acc[c + 8 * j + 5]),
                                     pack_bf16x2(acc[c + 8 * j + 6], acc[c + 8 * j + 7]));
            };
            auto store_chunk_plain = [&](int c, uint32_t stg) {
                const int col = cbase + c + 8 * rd_piece;
                const bool col_ok = (c + 8 * rd_piece < NC) && col < p.N;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = i * 8 + rd_sub;
                    if (col_ok && ((row_mask >> r) & 1u)) {
                        const uint4 v = ld_shared_v4(stg + r * 64 + ((rd_piece ^ ((r >> 1) & 3)) << 4));
                        st_global_v4(p.D + (size_t)(warp_row0 + r) * p.N + col, v.x, v.y, v.z, v.w);
                    }
                }
            };
            if (slots >= T::OUT_CHUNKS) {
                // the whole row block is staged: the previous tile's TMA
                // stores must have read the buffer
                if (lane == 0)
                    bulk_wait_read_all();
                __syncwarp();
#pragma unroll
                for (int c = 0; c < NC; c += 32)
                    stage_chunk(c, stg_w + (uint32_t)(c / 32) * OUT_STAGE_BYTES);
                fence_proxy_async_smem();
                __syncwarp();
                bool issued = false;
                if (use_tma && p.d_store_3d) {
                    // every chunk is full: one 3-D box ([chunk][row][32 columns],
                    // the staging layout)
                    if (lane == 0)
                        tma_store_3d(&tmap_d, stg_w, 0, warp_row0, cbase >> 5);
                    issued = true;
                } else {
#pragma unroll
                    for (int c = 0; c < NC; c += 32) {
                        const uint32_t stg = stg_w + (uint32_t)(c / 32) * OUT_STAGE_BYTES;
                        if (use_tma && c + 32 <= NC) {
                            if (lane == 0)
                                tma_store_2d(&tmap_d, stg, cbase + c, warp_row0);
                            issued = true;
                        } else if (row_mask != 0u) {
                            store_chunk_plain(c, stg);
                        }
                    }
                }
                if (issued && lane == 0)
                    bulk_commit_group();
            } else {
                // fewer slots than chunks: the chunks stream through the
                // slots, a slot being rewritten only after the TMA store that
                // read it has finished reading (so more operand stages fit)
#pragma unroll
                for (int c = 0; c < NC; c += 32) {
                    const int k = c / 32;
                    const uint32_t stg = stg_w + (uint32_t)(k % slots) * OUT_STAGE_BYTES;
                    if (k % slots == 0) {
                        if (lane == 0)
                            bulk_wait_read_all();
                        __syncwarp();
                    }
                    stage_chunk(c, stg);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (use_tma && c + 32 <= NC) {
                        if (lane == 0) {
                            tma_store_2d(&tmap_d, stg, cbase + c, warp_row0);
                            bulk_commit_group();
                        }
                    } else if (row_mask != 0u) {
                        store_chunk_plain(c, stg);
                    }
                    __syncwarp(); // the plain path's reads finish before the slot is reused
                }
            }
        }
        // every TMA store has completed before the CTA exits
        if (lane == 0)
            bulk_wait_all();
    }

    __syncwarp();
    if (split_k) {
        // Every CTA of the cluster has its partial in shared memory; CTA r
        // sums rows [r, r + BLOCK_M / split) of all partials in rank order
        // (deterministic) through distributed shared memory and stores them.
        cluster_sync();
        const TileInfo ti = get_tile<MW, BN, PAIR>(p, t_first, prefix, pair_rank,
                                                   expert_of_tile<MW, BN, PAIR>(p, t_first, num_tiles));
        const int rows_per = T::BLOCK_M / p.split;
        const int r0 = split_rank * rows_per;
        constexpr int CHUNKS = BN / 8;
        const uint32_t red_local = smem_addr(smem + plan.off_red);
        for (int item = threadIdx.x; item < rows_per * CHUNKS; item += NUM_THREADS) {
            const int row = r0 + item / CHUNKS;
            const int c8 = (item % CHUNKS) * 8;
            if (!ti.valid || row >= ti.rows || ti.n0 + c8 >= p.N)
                continue;
            const uint32_t off = (uint32_t)(row * (BN + RED_PAD) + c8) * 4u;
            float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int q = 0; q < p.split; ++q) {
                const uint32_t remote = map_shared_rank(red_local + off, (uint32_t)q);
                const float4 lo4 = ld_shared_cluster_v4(remote);
                const float4 hi4 = ld_shared_cluster_v4(remote + 16);
                s[0] += lo4.x; s[1] += lo4.y; s[2] += lo4.z; s[3] += lo4.w;
                s[4] += hi4.x; s[5] += hi4.y; s[6] += hi4.z; s[7] += hi4.w;
            }
            st_global_v4(p.D + (size_t)(ti.d_row0 + row) * p.N + ti.n0 + c8, pack_bf16x2(s[0], s[1]),
                         pack_bf16x2(s[2], s[3]), pack_bf16x2(s[4], s[5]), pack_bf16x2(s[6], s[7]));
        }
        // no CTA may leave (or reuse its buffer) while a peer still reads it
        cluster_sync();
    }
    if constexpr (PAIR)
        cluster_sync(); // neither CTA leaves while its pair may still use its memory
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR)
            tmem_dealloc_pair(tmem_base, T::TMEM_COLS);
        else
            tmem_dealloc(tmem_base, T::TMEM_COLS);
    }
}

} // namespace fp8nt
