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
// for the epilogue), and the epilogue warps promote each partial into FP32
// registers as it completes.  At the end each CTA owns a share of the output
// tile: every CTA sends the matching slices of its FP32 partial tile to their
// owners with bulk copies into the owners' shared memory (the copy engine
// moves them; completion is counted on the owner's barrier), and each owner
// sums the slices in rank order (deterministic) and stores them as BF16.
//
// Roles (one CTA per SM; 256 threads, 384 for MN = 128):
//   warp 0      TMA producer of the B tiles (lane 0)
//   warp 3      TMA producer of the A tiles (lane 0); the two copiers' issue
//               latencies overlap, each arriving on a stage's barrier with
//               its own bytes
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warp 2      copies the CTA's LHS and RHS scales into shared memory
//               (asynchronous copies, started at kernel entry)
//   warps 4..   promotion epilogue: one warpgroup (two for MN = 128, each
//               with half of the columns); TMEM lane quarter = warp % 4
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
    // epilogue warpgroups and the columns each thread owns (at most 64)
    static constexpr int EPI_WGS = MN > 64 ? 2 : 1;
    static constexpr int COLS = MN / EPI_WGS;
    static constexpr int THREADS = 128 + 128 * EPI_WGS;
    // with one warpgroup (256 threads, up to 255 registers each) the next K
    // block's partial is in flight while the current one is promoted; with
    // two (384 threads, 168 registers) one partial at a time
    static constexpr bool PREFETCH = EPI_WGS == 1;
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

// 16-byte asynchronous copy global -> shared that reads `src_bytes` (0..16)
// and zero-fills the rest of the 16 bytes.
__device__ __forceinline__ void cp_async_16_zfill(void *dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
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
template <int NC, int C0, int N>
__device__ __forceinline__ void skinny_promote(float (&acc)[NC], const float *v, const float *sa_cols,
                                               float sbv)
{
    const float4 *sa4 = reinterpret_cast<const float4 *>(sa_cols + C0);
#pragma unroll
    for (int j = 0; j < N; j += 4) {
        const float4 s = sa4[j / 4]; // same address in every lane: a broadcast
        ffma2(acc[C0 + j], acc[C0 + j + 1], v[j], v[j + 1], pack_f32x2(s.x * sbv, s.y * sbv));
        ffma2(acc[C0 + j + 2], acc[C0 + j + 3], v[j + 2], v[j + 3], pack_f32x2(s.z * sbv, s.w * sbv));
    }
}

// The scales of one tile for a CTA's K blocks, as asynchronous copies by one
// warp: sa[kb][m0 + m] for m < rows (zero-filled up to MN) and sb[nt][kb].
template <int MN>
__device__ __forceinline__ void skinny_copy_scales(const SkinnyParams &p, float *sa_s, float *sb_s,
                                                   int nt, int m0, int rows, int kb_lo, int cnt, int lane)
{
    constexpr int C4 = MN / 4; // 16-byte chunks per K block
    for (int idx = lane; idx < cnt * C4; idx += 32) {
        const int i = idx / C4;
        const int m = (idx - i * C4) * 4;
        const int avail = rows - m;
        const uint32_t bytes = avail >= 4 ? 16u : (avail > 0 ? 4u * (uint32_t)avail : 0u);
        // a chunk past the tile's rows reads nothing (a valid address is still
        // given; m0 is a multiple of MN, so every source chunk is 16-byte aligned)
        const float *src = p.sa + (size_t)(kb_lo + i) * p.ld_sa + m0 + (bytes ? m : 0);
        cp_async_16_zfill(sa_s + i * MN + m, src, bytes);
    }
    for (int i = lane; i < cnt; i += 32)
        cp_async_4(sb_s + i, p.sb + (size_t)nt * p.nkb + kb_lo + i);
}

template <int MN>
__global__ void __launch_bounds__(SkinnyTraits<MN>::THREADS, 1)
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
    uint64_t *recv_full = mma_done + 1; // split > 1: the tile's slices from every CTA arrived
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + p.off_misc);
    volatile uint32_t *abort_flag = misc + 1;
    float *sa_s = reinterpret_cast<float *>(smem + p.off_sa);
    float *sb_s = reinterpret_cast<float *>(smem + p.off_sb);

    // a cluster of `split` CTAs works on one tile at a time, CTA r on the K
    // blocks of stages [r * units / split, (r + 1) * units / split), a stage
    // being G = SKINNY_KB_PER_STAGE K blocks; clusters stride over the tiles
    constexpr int G = SKINNY_KB_PER_STAGE;
    const int rank = p.split > 1 ? (int)cluster_ctarank() : 0;
    const int units = (p.nkb + G - 1) / G;
    // (32-bit products: units < 2^24 and rank < 8)
    const int kb_lo = G * (int)((uint32_t)rank * (uint32_t)units / (uint32_t)p.split);
    const int kb_hi = min(p.nkb, G * (int)((uint32_t)(rank + 1) * (uint32_t)units / (uint32_t)p.split));
    const int cnt = max(0, kb_hi - kb_lo);
    const int ucnt = (cnt + G - 1) / G; // stages per tile
    const int t_first = (int)blockIdx.y;
    const int t_stride = (int)gridDim.y;
    // tile t: B rows [128 * (t / m_blocks), +128), A rows [MN * (t % m_blocks),
    // +MN) (the A blocks of one B block are neighbours: B is read from HBM
    // once and from L2 after); rows = A rows of the tile that exist
    auto tile_rows = [&](int t) { return min(MN, p.M - MN * (t % p.m_blocks)); };
    // the output items (one row m, 8 consecutive columns) of a tile that CTA
    // r of the cluster sums and stores: [r * items / split, (r + 1) * items / split)
    auto item_lo = [&](int items, int r) {
        return (int)((uint32_t)r * (uint32_t)items / (uint32_t)p.split); // items <= 2048, r <= 8
    };
    const uint32_t slot_bytes = skinny_recv_slot_items(min(MN, p.M), p.split) * 32u;
    auto my_bytes = [&](int t) {
        const int items = tile_rows(t) * (SKINNY_TILE_N / 8);
        return (uint32_t)(item_lo(items, rank + 1) - item_lo(items, rank)) * 32u;
    };

    // warp 0 copies B, warp 3 copies A into stage s (each with its bytes):
    // K blocks [kb, kb + G) (any past K are zero-filled and not used)
    const bool b_side = warp == 0;
    auto issue_load = [&](int s, int kb, int t) {
        uint8_t *dst = smem + (uint32_t)s * p.stage_bytes;
        if (b_side) {
            mbar_arrive_expect_tx(&full[s], G * T::B_BYTES);
            tma_load_4d(dst, &tmap_b, &full[s], 0, 0, kb, (t / p.m_blocks) * (SKINNY_TILE_N / 8));
        } else {
            mbar_arrive_expect_tx(&full[s], G * T::A_BYTES);
#pragma unroll
            for (int z = 0; z < G; ++z)
                tma_load_2d(dst + G * T::B_BYTES + z * T::A_BYTES, &tmap_a, &full[s], (kb + z) * BLOCK_K,
                            MN * (t % p.m_blocks));
        }
    };
    // the last K block (counted over this CTA's tiles) that stage use u holds
    auto last_kb_of_use = [&](uint32_t u) {
        const uint32_t t = u / (uint32_t)ucnt, j = u % (uint32_t)ucnt;
        const uint32_t end = (j + 1) * G < (uint32_t)cnt ? (j + 1) * G : (uint32_t)cnt;
        return t * (uint32_t)cnt + end - 1;
    };

    // ---------------------------------------------------------------- set-up
    // Thread 0 initialises the stage barriers and issues the first tile's
    // first stages at once, then the other barriers; warp 1 allocates TMEM and
    // warp 2 starts the first tile's scale copies meanwhile.  Launched with
    // programmatic dependent launch, this set-up overlaps the end of the
    // previous kernel: no thread touches global memory (the operands may be
    // that kernel's output, D its input) before the dependency wait.
    const int first = (t_first < p.tiles) ? (ucnt < stages ? ucnt : stages) : 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s)
            mbar_init(&full[s], 2);
        fence_mbarrier_init();
        tma_prefetch_desc(&tmap_b);
        tma_prefetch_desc(&tmap_a);
    }
    if (warp == 1) {
        tmem_alloc(misc, T::TMEM_COLS);
        tmem_relinquish();
    }
    grid_dependency_wait();
    if (warp == 0 || warp == 3) {
        named_barrier_sync(1, 64); // the stage barriers are initialised
        if (lane == 0)
            for (int i = 0; i < first; ++i)
                issue_load(i, kb_lo + G * i, t_first);
    }
    if (threadIdx.x == 0) {
        for (int j = 0; j < DONE_RING; ++j)
            mbar_init(&done[j], 1);
        for (int b = 0; b < T::NBUF; ++b)
            mbar_init(&tmem_empty[b], 4 * T::EPI_WGS);
        mbar_init(scales_full, 32);
        mbar_init(mma_done, 1);
        mbar_init(recv_full, 1);
        // the first tile's slices from the cluster: expected before any can arrive
        if (p.split > 1 && t_first < p.tiles)
            mbar_arrive_expect_tx(recv_full, (uint32_t)p.split * my_bytes(t_first));
        misc[1] = 0u;
        fence_mbarrier_init();
    }
    if (warp == 2 && t_first < p.tiles)
        skinny_copy_scales<MN>(p, sa_s, sb_s, t_first / p.m_blocks, MN * (t_first % p.m_blocks),
                               tile_rows(t_first), kb_lo, cnt, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    // the next kernel may start its own set-up on SMs this grid leaves free
    grid_launch_dependents();
    // the cluster's barriers are initialised before any CTA sends a slice
    // (the initialisation is ordered by fence.mbarrier_init; a releasing
    // arrive would also wait for this thread's earlier memory operations).
    // The cluster's CTAs start together, and every role's first wait (for
    // data, MMAs or scales) is longer than this barrier.
    if (p.split > 1) {
        cluster_arrive_relaxed();
        cluster_wait();
    }

    bool mma_done_committed = false; // (MMA issuer)
    bool cluster_wait_pending = false; // arrived on the closing cluster barrier
    uint32_t g0 = 0; // this CTA's K blocks of earlier tiles (ring position)
    uint32_t u0 = 0; // this CTA's stage uses of earlier tiles
    int tile_it = 0;
    for (int tile = t_first; tile < p.tiles;
         tile += t_stride, g0 += (uint32_t)cnt, u0 += (uint32_t)ucnt, ++tile_it) {
        const int n0 = (tile / p.m_blocks) * SKINNY_TILE_N;
        const int m0 = MN * (tile % p.m_blocks);
        const int rows = tile_rows(tile);
        if (warp == 0 || warp == 3) {
            // -------------------------------------------------------- producers
            if (lane == 0) {
                uint32_t issued = u0 + (uint32_t)(tile_it == 0 ? first : 0);
                for (uint32_t u = issued; u < u0 + (uint32_t)ucnt; ++u) {
                    const int s = (int)(u % (uint32_t)stages);
                    if (u >= (uint32_t)stages) {
                        // stage s was last used by stage use u - stages:
                        // free once its last K block's MMAs completed
                        const uint32_t j = last_kb_of_use(u - (uint32_t)stages);
                        if (!skinny_wait(&done[j % DONE_RING], (j / DONE_RING) & 1u, abort_flag, p))
                            break;
                    }
                    issue_load(s, kb_lo + G * (int)(u - u0), tile);
                    issued = u + 1;
                }
                // every copy issued must land before the ring is reused for
                // the partial tile or the CTA exits (normally the MMAs have
                // consumed them all)
                const uint32_t n = issued < (uint32_t)stages ? issued : (uint32_t)stages;
                for (uint32_t u = issued - n; u < issued; ++u)
                    skinny_drain(&full[u % stages], (u / stages) & 1u, abort_flag, p);
            }
        } else if (warp == 1) {
            // -------------------------------------------------------- MMA issuer
            if (lane == 0) {
                // D^T tile: the B tile is the MMA's A operand (M = 128), the A
                // tile its B operand (N = MN); both K-major, 128-byte swizzle.
                // K block z of a stage: B's 8-row groups are G KB apart
                // ([row group][K block][8 rows][128 B]), A's tile is whole.
                constexpr uint32_t idesc = make_idesc(MN, SKINNY_TILE_N);
                const uint64_t a_desc0 = make_sdesc_sbo(smem_addr(smem), G * 1024u);
                const uint64_t b_desc0 = make_sdesc(smem_addr(smem) + G * T::B_BYTES);
                const uint32_t stage_step = p.stage_bytes >> 4;
                uint32_t g = g0;
                bool ok = true;
                for (uint32_t u = u0; ok && u < u0 + (uint32_t)ucnt; ++u) {
                    const uint32_t s = u % (uint32_t)stages;
                    if (!skinny_wait(&full[s], (u / (uint32_t)stages) & 1u, abort_flag, p))
                        break;
                    const int kbs = min(G, cnt - G * (int)(u - u0)); // K blocks of this stage
                    for (int z = 0; z < kbs; ++z, ++g) {
                        const uint32_t buf = g % T::NBUF;
                        if (g >= (uint32_t)T::NBUF &&
                            !skinny_wait(&tmem_empty[buf], (g / T::NBUF - 1) & 1u, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem_base + buf * (uint32_t)MN;
                        const uint64_t ad = a_desc0 + (uint64_t)(s * stage_step + ((uint32_t)z * 1024u >> 4));
                        const uint64_t bd = b_desc0 + (uint64_t)(s * stage_step + ((uint32_t)z * T::A_BYTES >> 4));
#pragma unroll
                        for (int k = 0; k < BLOCK_K / MMA_K; ++k)
                            mma_f8f6f4(d, ad + (uint64_t)((k * MMA_K) >> 4), bd + (uint64_t)((k * MMA_K) >> 4),
                                       idesc, k > 0 ? 1u : 0u);
                        // publishes the partial (the stage's last one also frees it)
                        mma_commit(&done[g % DONE_RING]);
                    }
                }
                // after the CTA's last MMAs: the "all MMAs done" barrier,
                // awaited before TMEM is released at the end
                if (tile + t_stride >= p.tiles) {
                    mma_commit(mma_done);
                    mma_done_committed = true;
                }
            }
        } else if (warp == 2) {
            // -------------------------------------------------------- scales
            // the tile's scale copies (the first tile's were started at entry;
            // the previous tile's have been read: the end-of-tile barriers)
            if (tile_it > 0)
                skinny_copy_scales<MN>(p, sa_s, sb_s, tile / p.m_blocks, m0, rows, kb_lo, cnt, lane);
            cp_async_mbar_arrive_noinc(scales_full);
        } else if (warp >= 4) {
            // -------------------------------------------------------- epilogue
            constexpr int NC = T::COLS;
            const int q = warp & 3;                   // TMEM lane quarter
            const int col0 = ((warp - 4) >> 2) * NC;  // this warpgroup's columns
            const int row = q * 32 + lane;            // B row within the tile = column of D
            const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)col0;
            float acc[NC];
#pragma unroll
            for (int j = 0; j < NC; ++j)
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
                    float va[NC], vb[NC];
                    auto step = [&](float (&cur)[NC], float (&nxt)[NC], int i) {
                        release(g0 + (uint32_t)i);
                        const bool more = i + 1 < cnt;
                        if (more) {
                            if (!wait_done(g0 + (uint32_t)i + 1))
                                return false;
                            tmem_issue_p<NC>(buf_addr(g0 + (uint32_t)i + 1), nxt);
                        }
                        skinny_promote<NC, 0, NC>(acc, cur, sa_s + i * MN + col0, sb_s[i]);
                        if (more)
                            tmem_wait_tie<NC>(nxt);
                        return true;
                    };
                    if (ok && wait_done(g0)) {
                        tmem_issue_p<NC>(buf_addr(g0), va);
                        tmem_wait_tie<NC>(va);
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
                    // the whole partial loaded at once (one wait), its buffer
                    // handed back, then promoted (registers are fewer at 384
                    // threads: no next partial in flight)
                    float v[NC];
                    for (int i = 0; ok && i < cnt; ++i) {
                        const uint32_t g = g0 + (uint32_t)i;
                        if (!wait_done(g)) {
                            ok = false;
                            break;
                        }
                        tmem_issue_p<NC>(buf_addr(g), v);
                        tmem_wait_tie<NC>(v);
                        release(g);
                        skinny_promote<NC, 0, NC>(acc, v, sa_s + i * MN + col0, sb_s[i]);
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
                for (int j = 0; j < NC; ++j)
                    red[(col0 + j) * SKINNY_TILE_N + row] = acc[j];
                fence_proxy_async_smem(); // the bulk copies below read it
            }
        }
        __syncwarp();

        // ------------------------------------------------------------ reduce + store
        __syncthreads(); // the partial tile is complete
        const uint32_t red_local = smem_addr(smem);
        const int items = rows * (SKINNY_TILE_N / 8);
        const int lo = item_lo(items, rank), hi = item_lo(items, rank + 1);
        if (p.split > 1) {
            // Send slice r of this CTA's partial tile (items of CTA r) to CTA
            // r's receive area, slot `rank`; wait for the tile's slices from
            // every CTA, sum them in rank order, store.  The receive area is
            // this CTA's own shared memory outside the operand ring, free
            // since the previous tile's closing cluster barrier.
            if (threadIdx.x < p.split) {
                // lane r of warp 0 sends slice r (the copies are issued in parallel)
                const int r = (int)threadIdx.x;
                const int rlo = item_lo(items, r), rhi = item_lo(items, r + 1);
                const uint32_t recv_local = smem_addr(smem + p.off_recv) + (uint32_t)rank * slot_bytes;
                if (rhi > rlo)
                    bulk_copy_to_cluster(map_shared_rank(recv_local, (uint32_t)r),
                                         red_local + (uint32_t)rlo * 32u, (uint32_t)(rhi - rlo) * 32u,
                                         map_shared_rank(smem_addr(recv_full), (uint32_t)r));
            }
            const bool got = hi <= lo || skinny_wait(recv_full, (uint32_t)tile_it & 1u, abort_flag, p);
            const bool last = tile + t_stride >= p.tiles;
            if (last) {
                // Every slice sent to this CTA has landed.  Once every CTA
                // has said so, every copy that read this CTA's partial tile
                // has completed and the CTA may exit: the wait is left for
                // the very end, after the sums, the stores and the TMEM
                // release.  The barrier publishes no data (each copy's
                // completion was observed on its owner's mbarrier before the
                // owner arrives), so the arrive is relaxed.
                __syncwarp();
                cluster_arrive_relaxed();
                cluster_wait_pending = true;
            }
            const float *recv = reinterpret_cast<const float *>(smem + p.off_recv);
            for (int it = lo + (int)threadIdx.x; got && it < hi; it += T::THREADS) {
                const int m = it >> 4;
                const int c8 = (it & 15) * 8;
                const int n = n0 + c8;
                if (n >= p.N)
                    continue;
                // the slots' values summed in rank order (the loop unrolled
                // over the largest cluster, so that the reads are issued ahead)
                float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q = 0; q < SKINNY_MAX_SPLIT; ++q) {
                    if (q < p.split) {
                        const float *src = recv + (size_t)q * (slot_bytes / 4) + (size_t)(it - lo) * 8;
                        const float4 a = *reinterpret_cast<const float4 *>(src);
                        const float4 b = *reinterpret_cast<const float4 *>(src + 4);
                        sum[0] += a.x; sum[1] += a.y; sum[2] += a.z; sum[3] += a.w;
                        sum[4] += b.x; sum[5] += b.y; sum[6] += b.z; sum[7] += b.w;
                    }
                }
                st_global_v4(p.D + (size_t)(m0 + m) * (size_t)p.ld_d + n, pack_bf16x2(sum[0], sum[1]),
                             pack_bf16x2(sum[2], sum[3]), pack_bf16x2(sum[4], sum[5]),
                             pack_bf16x2(sum[6], sum[7]));
            }
            if (!last) {
                __syncthreads(); // every thread has read the receive area
                // the next tile's slices are expected before any can be sent
                if (threadIdx.x == 0) {
                    const uint32_t next_bytes = my_bytes(tile + t_stride);
                    if (next_bytes > 0)
                        mbar_arrive_expect_tx(recv_full, (uint32_t)p.split * next_bytes);
                }
                // every CTA has received all its slices and read them: the
                // rings and the receive areas can be reused
                cluster_sync();
            }
        } else {
            for (int it = lo + (int)threadIdx.x; it < hi; it += T::THREADS) {
                const int m = it >> 4;
                const int c8 = (it & 15) * 8;
                const int n = n0 + c8;
                if (n >= p.N)
                    continue;
                const uint32_t off = (uint32_t)(m * SKINNY_TILE_N + c8) * 4u;
                const float4 a = *reinterpret_cast<const float4 *>(smem + off);
                const float4 b = *reinterpret_cast<const float4 *>(smem + off + 16);
                st_global_v4(p.D + (size_t)(m0 + m) * (size_t)p.ld_d + n, pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                             pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
            }
            __syncthreads(); // the ring is reused by the next tile
        }
    }
    if (warp == 1) {
        if (lane == 0) {
            // all MMAs complete before TMEM is released
            if (!mma_done_committed)
                mma_commit(mma_done);
            skinny_drain(mma_done, 0, abort_flag, p);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, T::TMEM_COLS);
    }
    if (warp == 2)
        cp_async_wait_all(); // no scale copy outlives the CTA
    if (cluster_wait_pending)
        cluster_wait(); // no copy reads this CTA's shared memory any more
}

} // namespace fp8nt
