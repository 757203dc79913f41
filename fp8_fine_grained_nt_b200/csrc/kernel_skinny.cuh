// Dense FP8 NT GEMM with fine-grained scaling for calls with few rows of A
// (M <= 128: the decode-shaped calls of the DeepGEMM README's usage section,
// which are bandwidth-bound on the weights B), for sm_100a.
//
// It computes the same D[m,n] = sum_kb P_kb[m,n] * sa[m,kb] * sb[n/128,kb] as
// kernel.cuh, but transposed: a tile is 128 rows of B (128 columns of D), which
// take the MMA's 128-row operand, while the M rows of A, zero-padded to MN, take
// its N side.  Each K block's partial D^T[n, m] lands in TMEM with one B row per
// lane, so an epilogue thread owns one column n of D and all MN rows m; its
// RHS scale sb[n/128, kb] is one value per K block and its LHS scales are the
// MN values sa[., kb], read from shared memory as broadcasts.
//
// A tile's K range is split over the `split` CTAs of a thread-block cluster
// (each a contiguous range of K blocks).  Every CTA loads its whole range into
// a shared-memory ring at once (as deep as shared memory allows), one thread
// issues the MMAs of every K block into its own TMEM buffer (the ring of
// 512 / MN buffers usually holds the CTA's whole range, so the MMAs never wait
// for the epilogue), and four epilogue warps promote each partial into FP32
// registers as it completes.  At the end the CTAs' FP32 partial tiles meet in
// shared memory; each CTA sums a share of the output in rank order through
// distributed shared memory (deterministic) and stores it as BF16.
//
// Roles (256 threads, one CTA per SM):
//   warp 0      TMA producer of the B and A tiles (lane 0)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warp 2      loads the CTA's LHS and RHS scales into shared memory
//   warps 4-7   promotion epilogue (TMEM lane quarter = warp - 4)
#pragma once

#include "kernel.cuh"

namespace fp8nt {

template <int MN>
struct SkinnyTraits {
    static_assert(MN % 16 == 0 && MN >= 16 && MN <= SKINNY_MAX_M,
                  "MN (the padded rows of A) is a multiple of 16 in [16, 128]");
    static constexpr uint32_t B_BYTES = SKINNY_TILE_N * BLOCK_K; // 128 rows of B
    static constexpr uint32_t A_BYTES = MN * BLOCK_K;
    // TMEM ring of K-block partials (MN columns each)
    static constexpr int NBUF = (512 / MN) < MAX_TMEM_BUFS ? (512 / MN) : MAX_TMEM_BUFS;
    static constexpr int TMEM_NEED = NBUF * MN;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                   : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
    // a partial of up to 64 columns fits one register batch: the next K
    // block's partial is then in flight while the current one is promoted
    static constexpr bool PREFETCH = MN <= 64;
    static constexpr int CHUNK = MN <= 64 ? MN : 32; // columns per tcgen05.ld batch
};

// Ties 16 registers to this point of the instruction stream (no code).
__device__ __forceinline__ void reg_tie16(float *v)
{
    uint32_t *r = reinterpret_cast<uint32_t *>(v);
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

// Wait for this thread's outstanding tcgen05.ld and tie the N registers of v
// to the wait, so that no read of them is scheduled before it.
template <int N, int C = 0>
__device__ __forceinline__ void tmem_wait_tie(float *v)
{
    static_assert(N % 16 == 0, "loads come in 16-column multiples");
    if constexpr (C == 0) {
        if constexpr (N >= 32) {
            tmem_wait_ld(*reinterpret_cast<float(*)[32]>(v));
            tmem_wait_tie<N, 32>(v);
        } else {
            tmem_wait_ld(*reinterpret_cast<float(*)[16]>(v));
        }
    } else if constexpr (C < N) {
        if constexpr (N - C >= 32) {
            reg_tie32(*reinterpret_cast<float(*)[32]>(v + C));
            tmem_wait_tie<N, C + 32>(v);
        } else {
            reg_tie16(v + C);
            tmem_wait_tie<N, C + 16>(v);
        }
    }
}

// Two floats as one packed f32x2 operand.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ bool skinny_wait(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag,
                                            const SkinnyParams &p)
{
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait(a, parity))
        return true;
    return wait_slow(a, parity, abort_flag, p.status, p.timeout_ns, true);
}

__device__ __forceinline__ void skinny_drain(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag,
                                             const SkinnyParams &p)
{
    const uint32_t a = smem_addr(bar);
    if (!mbar_try_wait(a, parity))
        wait_slow(a, parity, abort_flag, p.status, p.timeout_ns, false);
}

// acc[C0 + j] += v[j] * sa[C0 + j] * sb for j in [0, N): the scale product is
// rounded once in FP32, then one FMA per element (two per instruction).
template <int MN, int C0, int N>
__device__ __forceinline__ void skinny_promote(float (&acc)[MN], const float *v, const float *sa_kb,
                                               float sbv)
{
    const float4 *sa4 = reinterpret_cast<const float4 *>(sa_kb + C0);
#pragma unroll
    for (int j = 0; j < N; j += 4) {
        const float4 s = sa4[j / 4]; // same address in every lane: a broadcast
        ffma2(acc[C0 + j], acc[C0 + j + 1], v[j], v[j + 1], pack_f32x2(s.x * sbv, s.y * sbv));
        ffma2(acc[C0 + j + 2], acc[C0 + j + 3], v[j + 2], v[j + 3], pack_f32x2(s.z * sbv, s.w * sbv));
    }
}

// Promotion of a partial wider than one register batch: chunks of CH columns,
// each loaded, waited for and multiplied in before the next is loaded.
template <int MN, int CH, int C = 0>
__device__ __forceinline__ void skinny_promote_chunks(float (&acc)[MN], float *v, uint32_t taddr,
                                                      const float *sa_kb, float sbv)
{
    if constexpr (C < MN) {
        tmem_issue_p<CH>(taddr + (uint32_t)C, v);
        tmem_wait_tie<CH>(v);
        skinny_promote<MN, C, CH>(acc, v, sa_kb, sbv);
        skinny_promote_chunks<MN, CH, C + CH>(acc, v, taddr, sa_kb, sbv);
    }
}

template <int MN>
__global__ void __launch_bounds__(SKINNY_THREADS, 1)
    fp8_gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmap_a,
                           const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ SkinnyParams p)
{
    using T = SkinnyTraits<MN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int stages = p.stages;

    // full[s]: stage s holds its B and A tiles; done[g % DONE_RING]: the MMAs
    // of this CTA's g-th K block (counted over all its tiles) have completed,
    // which frees the stage and publishes the partial; tmem_empty[b]: the
    // epilogue has read TMEM buffer b; scales_full: the tile's scales are in
    // shared memory (one phase per tile).
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bars);
    uint64_t *done = full + stages;
    uint64_t *tmem_empty = done + DONE_RING;
    uint64_t *scales_full = tmem_empty + MAX_TMEM_BUFS;
    uint64_t *mma_done = scales_full + 1;
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + p.off_misc);
    volatile uint32_t *abort_flag = misc + 1;
    float *sa_s = reinterpret_cast<float *>(smem + p.off_sa);
    float *sb_s = reinterpret_cast<float *>(smem + p.off_sb);

    // a cluster of `split` CTAs works on one tile at a time, CTA r on K blocks
    // [r * nkb / split, (r + 1) * nkb / split); clusters stride over the tiles
    const int rank = p.split > 1 ? (int)cluster_ctarank() : 0;
    const int kb_lo = (int)((long)rank * p.nkb / p.split);
    const int kb_hi = (int)((long)(rank + 1) * p.nkb / p.split);
    const int cnt = kb_hi - kb_lo;
    const uint32_t stage_tx = T::B_BYTES + T::A_BYTES;
    const int t_first = (int)blockIdx.y;
    const int t_stride = (int)gridDim.y;

    auto issue_load = [&](int s, int kb, int n0) {
        uint8_t *dst = smem + (uint32_t)s * p.stage_bytes;
        mbar_arrive_expect_tx(&full[s], stage_tx);
        tma_load_2d(dst, &tmap_b, &full[s], kb * BLOCK_K, n0);
        tma_load_2d(dst + T::B_BYTES, &tmap_a, &full[s], kb * BLOCK_K, 0);
    };

    // ---------------------------------------------------------------- set-up
    // Thread 0 initialises the barriers and issues the first tile's first
    // stages at once, before the CTA-wide barrier, so that the copies start as
    // early as possible; warp 1 allocates TMEM meanwhile.
    int first = 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s)
            mbar_init(&full[s], 1);
        for (int j = 0; j < DONE_RING; ++j)
            mbar_init(&done[j], 1);
        for (int b = 0; b < T::NBUF; ++b)
            mbar_init(&tmem_empty[b], 4);
        mbar_init(scales_full, 32);
        mbar_init(mma_done, 1);
        misc[1] = 0u;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmap_b);
        tma_prefetch_desc(&tmap_a);
        if (t_first < p.n_tiles) {
            first = cnt < stages ? cnt : stages;
            for (int i = 0; i < first; ++i)
                issue_load(i, kb_lo + i, t_first * SKINNY_TILE_N);
        }
    }
    if (warp == 1) {
        tmem_alloc(misc, T::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];

    uint32_t g0 = 0; // this CTA's K blocks of earlier tiles (ring position)
    int tile_it = 0;
    for (int tile = t_first; tile < p.n_tiles; tile += t_stride, g0 += (uint32_t)cnt, ++tile_it) {
        const int n0 = tile * SKINNY_TILE_N;
        if (warp == 0) {
            // -------------------------------------------------------- producer
            if (lane == 0) {
                uint32_t issued = g0 + (uint32_t)(tile_it == 0 ? first : 0);
                for (uint32_t g = issued; g < g0 + (uint32_t)cnt; ++g) {
                    const int s = (int)(g % (uint32_t)stages);
                    if (g >= (uint32_t)stages) {
                        // stage s was last used by K block g - stages
                        const uint32_t j = g - (uint32_t)stages;
                        if (!skinny_wait(&done[j % DONE_RING], (j / DONE_RING) & 1u, abort_flag, p))
                            break;
                    }
                    issue_load(s, kb_lo + (int)(g - g0), n0);
                    issued = g + 1;
                }
                // every copy issued must land before the ring is reused for
                // the partial tile or the CTA exits (normally the MMAs have
                // consumed them all)
                const uint32_t n = issued < (uint32_t)stages ? issued : (uint32_t)stages;
                for (uint32_t g = issued - n; g < issued; ++g)
                    skinny_drain(&full[g % stages], (g / stages) & 1u, abort_flag, p);
            }
        } else if (warp == 1) {
            // -------------------------------------------------------- MMA issuer
            if (lane == 0) {
                // D^T tile: the B tile is the MMA's A operand (M = 128), the A
                // tile its B operand (N = MN); both K-major, 128-byte swizzle.
                constexpr uint32_t idesc = make_idesc(MN, SKINNY_TILE_N);
                const uint64_t a_desc0 = make_sdesc(smem_addr(smem));
                const uint64_t b_desc0 = make_sdesc(smem_addr(smem) + T::B_BYTES);
                const uint32_t stage_step = p.stage_bytes >> 4;
                for (uint32_t g = g0; g < g0 + (uint32_t)cnt; ++g) {
                    const uint32_t s = g % (uint32_t)stages;
                    if (!skinny_wait(&full[s], (g / (uint32_t)stages) & 1u, abort_flag, p))
                        break;
                    const uint32_t buf = g % T::NBUF;
                    if (g >= (uint32_t)T::NBUF &&
                        !skinny_wait(&tmem_empty[buf], (g / T::NBUF - 1) & 1u, abort_flag, p))
                        break;
                    tc_fence_after();
                    const uint32_t d = tmem_base + buf * (uint32_t)MN;
                    const uint64_t ad = a_desc0 + (uint64_t)(s * stage_step);
                    const uint64_t bd = b_desc0 + (uint64_t)(s * stage_step);
#pragma unroll
                    for (int k = 0; k < BLOCK_K / MMA_K; ++k)
                        mma_f8f6f4(d, ad + (uint64_t)((k * MMA_K) >> 4), bd + (uint64_t)((k * MMA_K) >> 4),
                                   idesc, k > 0 ? 1u : 0u);
                    // frees the stage and publishes the partial
                    mma_commit(&done[g % DONE_RING]);
                }
            }
        } else if (warp == 2) {
            // -------------------------------------------------------- scales
            // LHS scales of rows m < M for the CTA's K blocks (zero for the
            // padding rows, whose partial columns are zero and never stored),
            // and the tile's RHS scale per K block.  The previous tile's have
            // been read (the end-of-tile barriers).
            for (int idx = lane; idx < cnt * MN; idx += 32) {
                const int i = idx / MN;
                const int m = idx - i * MN;
                sa_s[idx] = m < p.M ? __ldg(p.sa + (size_t)(kb_lo + i) * p.ld_sa + m) : 0.0f;
            }
            for (int i = lane; i < cnt; i += 32)
                sb_s[i] = __ldg(p.sb + (size_t)tile * p.nkb + kb_lo + i);
            mbar_arrive(scales_full);
        } else if (warp >= 4) {
            // -------------------------------------------------------- epilogue
            const int q = warp - 4;               // TMEM lane quarter
            const int row = q * 32 + lane;        // B row within the tile = column of D
            const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16);
            float acc[MN];
#pragma unroll
            for (int j = 0; j < MN; ++j)
                acc[j] = 0.0f;
            bool ok = true;
            auto wait_done = [&](uint32_t g) {
                const bool r = skinny_wait(&done[g % DONE_RING], (g / DONE_RING) & 1u, abort_flag, p);
                tc_fence_after();
                return __all_sync(0xffffffffu, r) != 0;
            };
            auto buf_addr = [&](uint32_t g) { return t_lane + (g % T::NBUF) * (uint32_t)MN; };
            // hand TMEM buffer of K block g back to the MMA issuer
            auto release = [&](uint32_t g) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&tmem_empty[g % T::NBUF]);
            };
            if (cnt > 0) {
                ok = __all_sync(0xffffffffu,
                                skinny_wait(scales_full, (uint32_t)tile_it & 1u, abort_flag, p)) != 0;
                if constexpr (T::PREFETCH) {
                    // cur holds K block i (loaded and waited): hand its buffer
                    // back, start loading K block i + 1 into nxt, promote cur
                    float va[MN], vb[MN];
                    auto step = [&](float (&cur)[MN], float (&nxt)[MN], int i) {
                        release(g0 + (uint32_t)i);
                        const bool more = i + 1 < cnt;
                        if (more) {
                            if (!wait_done(g0 + (uint32_t)i + 1))
                                return false;
                            tmem_issue_p<MN>(buf_addr(g0 + (uint32_t)i + 1), nxt);
                        }
                        skinny_promote<MN, 0, MN>(acc, cur, sa_s + i * MN, sb_s[i]);
                        if (more)
                            tmem_wait_tie<MN>(nxt);
                        return true;
                    };
                    if (ok && wait_done(g0)) {
                        tmem_issue_p<MN>(buf_addr(g0), va);
                        tmem_wait_tie<MN>(va);
                    } else {
                        ok = false;
                    }
                    for (int i = 0; ok && i < cnt; i += 2) {
                        if (!step(va, vb, i)) {
                            ok = false;
                            break;
                        }
                        if (i + 1 < cnt && !step(vb, va, i + 1)) {
                            ok = false;
                            break;
                        }
                    }
                } else {
                    float v[T::CHUNK];
                    for (int i = 0; ok && i < cnt; ++i) {
                        const uint32_t g = g0 + (uint32_t)i;
                        if (!wait_done(g)) {
                            ok = false;
                            break;
                        }
                        skinny_promote_chunks<MN, T::CHUNK>(acc, v, buf_addr(g), sa_s + i * MN, sb_s[i]);
                        release(g);
                    }
                }
            }
            // This CTA's FP32 partial tile, [MN][128] (m-major, so that the
            // reduction below reads 8 consecutive columns of D at once), in
            // the operand ring: every MMA of the tile has completed (its last
            // K block's barrier), so nothing reads the ring any more.
            if (ok) {
                float *red = reinterpret_cast<float *>(smem);
#pragma unroll
                for (int j = 0; j < MN; ++j)
                    red[j * SKINNY_TILE_N + row] = acc[j];
            }
        }
        __syncwarp();

        // ------------------------------------------------------------ reduce + store
        // Every CTA of the cluster holds its partial tile; CTA r sums a share
        // of the output items (one row m, 8 consecutive columns) over all
        // CTAs in rank order and stores them as BF16.
        if (p.split > 1)
            cluster_sync();
        else
            __syncthreads();
        {
            const int items = p.M * (SKINNY_TILE_N / 8);
            const int lo = (int)((long)rank * items / p.split);
            const int hi = (int)((long)(rank + 1) * items / p.split);
            const uint32_t red_local = smem_addr(smem);
            for (int it = lo + (int)threadIdx.x; it < hi; it += SKINNY_THREADS) {
                const int m = it >> 4;
                const int c8 = (it & 15) * 8;
                const int n = n0 + c8;
                if (n >= p.N)
                    continue;
                const uint32_t off = (uint32_t)(m * SKINNY_TILE_N + c8) * 4u;
                float sum[8];
                if (p.split > 1) {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        sum[e] = 0.0f;
                    for (int r = 0; r < p.split; ++r) {
                        const uint32_t remote = map_shared_rank(red_local + off, (uint32_t)r);
                        const float4 a = ld_shared_cluster_v4(remote);
                        const float4 b = ld_shared_cluster_v4(remote + 16);
                        sum[0] += a.x; sum[1] += a.y; sum[2] += a.z; sum[3] += a.w;
                        sum[4] += b.x; sum[5] += b.y; sum[6] += b.z; sum[7] += b.w;
                    }
                } else {
                    const float4 a = *reinterpret_cast<const float4 *>(smem + off);
                    const float4 b = *reinterpret_cast<const float4 *>(smem + off + 16);
                    sum[0] = a.x; sum[1] = a.y; sum[2] = a.z; sum[3] = a.w;
                    sum[4] = b.x; sum[5] = b.y; sum[6] = b.z; sum[7] = b.w;
                }
                st_global_v4(p.D + (size_t)m * p.N + n, pack_bf16x2(sum[0], sum[1]),
                             pack_bf16x2(sum[2], sum[3]), pack_bf16x2(sum[4], sum[5]),
                             pack_bf16x2(sum[6], sum[7]));
            }
        }
        // no CTA reuses its ring (next tile) or leaves while a peer still
        // reads its partial tile
        if (p.split > 1)
            cluster_sync();
        else
            __syncthreads();
    }

    if (warp == 1) {
        if (lane == 0) {
            // all MMAs complete before TMEM is released
            mma_commit(mma_done);
            skinny_drain(mma_done, 0, abort_flag, p);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, T::TMEM_COLS);
    }
}

} // namespace fp8nt
