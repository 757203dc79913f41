// Kernel parameters and the shared-memory plan, shared by the host launcher
// and the kernel.
#pragma once

#include <stdint.h>

namespace fp8nt {

enum GemmKind : int { KIND_DENSE = 0, KIND_CONTIGUOUS = 1, KIND_MASKED = 2 };

constexpr int BLOCK_K = 128;          // one scale block of K = one 128-byte swizzle row
constexpr int HALF_M = 128;           // rows of one tcgen05 MMA (cta_group::1, M = 128)
constexpr int MMA_K = 32;             // K of one kind::f8f6f4 MMA
constexpr int NUM_THREADS = 384;      // 3 warpgroups
constexpr int FIRST_EPI_WARP = 4;     // warps 4..11 run the promotion epilogue
constexpr int NUM_EPI_WARPS = 8;
constexpr int MAX_SB_BLOCKS = 3;      // a BLOCK_N <= 256 tile spans at most 3 sb blocks
constexpr int MAX_MASKED_GROUPS = 1024;
constexpr int MAX_TMEM_BUFS = 16;      // K-block partial buffers in TMEM (ring)
constexpr int DONE_RING = 16;          // "K block done" barriers; >= stages and >= TMEM buffers
static_assert(DONE_RING >= MAX_TMEM_BUFS, "the done ring must cover every TMEM buffer");
constexpr uint32_t OUT_STAGE_BYTES = 2048; // output staging chunk: 32 rows x 32 BF16 columns
constexpr uint32_t SA_SLOT_BYTES = 4096;   // one slot of the LHS-scale ring (2 slots)
constexpr int RED_PAD = 4;             // FP32 padding per row of the split-K partial tile
constexpr int MAX_SPLIT = 8;           // split-K CTAs per cluster (portable cluster size)
constexpr int REGS_PRODUCER = 40;     // per-thread registers after setmaxnreg
constexpr int REGS_EPILOGUE = 232;
constexpr int REGS_AT_LAUNCH = 168;   // 65536 / 384 rounded down to a multiple of 8

static_assert(4 * 32 * REGS_PRODUCER + 8 * 32 * REGS_EPILOGUE <= NUM_THREADS * REGS_AT_LAUNCH,
              "register split exceeds the launch allocation");

// Device status bits (read back by dg_get_device_status).
constexpr uint32_t DEVERR_TIMEOUT = 1u;
constexpr uint32_t DEVERR_BAD_INDEX = 2u;

struct SmemPlan {
    uint32_t stage_bytes;   // A (MW x 16 KB) + B (BN x 128 B; BN/2 rows per CTA of a pair)
    uint32_t a_bytes;
    uint32_t off_stages;    // 1024-aligned
    uint32_t off_sb;        // RHS-scale tile slots: 2 x 3 x sb_pitch floats
    uint32_t sb_pitch;      // floats per sb row in smem (nkb rounded up to 4)
    uint32_t off_sa;        // LHS-scale ring: 2 x SA_SLOT_BYTES
    uint32_t off_out;       // output staging: out_slots 2 KB chunk slots per epilogue warp
    uint32_t out_slots;     // = the warp's chunk count (whole tile staged) or fewer (streamed)
    uint32_t off_red;       // split-K: this CTA's FP32 partial tile, rows padded by RED_PAD
    uint32_t off_prefix;    // masked: (G + 1) ints of per-group tile prefix sums
    uint32_t off_bars;      // all mbarriers
    uint32_t off_misc;      // tmem base address, abort flag
    uint32_t total;         // bytes, excluding the 1024 B alignment slack
};

struct Params {
    int kind;
    int M;          // dense: M; contiguous: M_sum; masked: M_max
    int N;
    int K;
    int num_groups; // 1 for dense
    int nkb;        // K / 128
    int nnb;        // ceil(N / 128)
    int m_blocks;   // dense / contiguous: ceil(M / BLOCK_M); masked: per-group maximum
    int n_blocks;   // ceil(N / BLOCK_N)
    int num_tiles;  // dense / contiguous; masked tiles are counted on the device
    int split;      // split-K CTAs per cluster (1 = off)
    int kb_chunk;   // K blocks per split-K CTA
    int stages;
    SmemPlan plan;
    const float *sa; // LHS scales, [G * K/128][ld_sa]
    int ld_sa;
    const float *sb;
    const int *m_indices;
    const int *masked_m;
    uint16_t *D;    // BF16 bits
    int d_store_3d; // 1: tmap_d is the 3-D [N/32][rows][32] view (one TMA store per warp)
    unsigned int *status; // device status word (DEVERR_* bits)
    uint64_t timeout_ns;  // limit on any single pipeline wait
};

__host__ __device__ inline uint32_t align_up_u32(uint32_t x, uint32_t a)
{
    return (x + a - 1) / a * a;
}

// Shared-memory layout for a (MW, BN) kernel with the given ring depths; a
// CTA of a pair holds half of the B tile.
__host__ __device__ inline SmemPlan make_smem_plan(int mw, int bn, int stages, int nkb,
                                                   int prefix_ints, bool split_k, bool pair = false,
                                                   int out_slots = 0)
{
    SmemPlan p;
    p.a_bytes = (uint32_t)mw * HALF_M * BLOCK_K;
    p.stage_bytes = p.a_bytes + (uint32_t)(pair ? bn / 2 : bn) * BLOCK_K;
    p.off_stages = 0;
    uint32_t off = p.stage_bytes * (uint32_t)stages;
    p.sb_pitch = align_up_u32((uint32_t)nkb, 4);
    p.off_sb = align_up_u32(off, 128);
    off = p.off_sb + 2u * MAX_SB_BLOCKS * p.sb_pitch * 4u;
    p.off_sa = align_up_u32(off, 128);
    off = p.off_sa + 2u * SA_SLOT_BYTES;
    p.off_out = align_up_u32(off, 1024);
    // (split-K CTAs reduce through distributed shared memory and store
    // directly: no output staging; out_slots <= 0 stages every chunk)
    const uint32_t out_chunks = split_k ? 0u : (uint32_t)((mw == 1 ? bn / 2 : bn) + 31) / 32;
    p.out_slots = (out_slots > 0 && (uint32_t)out_slots < out_chunks) ? (uint32_t)out_slots : out_chunks;
    off = p.off_out + NUM_EPI_WARPS * p.out_slots * OUT_STAGE_BYTES;
    p.off_red = align_up_u32(off, 128);
    if (split_k)
        off = p.off_red + (uint32_t)mw * HALF_M * (uint32_t)(bn + RED_PAD) * 4u;
    p.off_prefix = align_up_u32(off, 16);
    off = p.off_prefix + 4u * (uint32_t)prefix_ints;
    p.off_bars = align_up_u32(off, 8);
    // full per stage, the ring of "K block done" barriers, TMEM empty per
    // partial buffer, sb and sa full/empty x2, one "all MMAs done" barrier,
    // two "tile accumulated" barriers (per-tensor scaling)
    off = p.off_bars + 8u * (stages + DONE_RING + MAX_TMEM_BUFS + 8u + 1u + 2u);
    p.off_misc = align_up_u32(off, 16);
    p.total = p.off_misc + 16;
    return p;
}

// ---------------------------------------------------------------- skinny kernel
// Dense GEMM with few rows of A (M <= 128, decode-shaped calls), computed as
// D^T tiles: 128 rows of B per tile on the MMA's M side and the rows of A,
// zero-padded to MN, on its N side (kernel_skinny.cuh).

constexpr int SKINNY_TILE_N = 128;       // rows of B (columns of D) per tile
constexpr int SKINNY_MAX_SPLIT = 8;      // CTAs per cluster sharing a tile's K range
constexpr int SKINNY_MAX_M = 128;
// K blocks per operand stage: B arrives as one 4-D box holding these K blocks
// of each 8-row group, so every row's KB_PER_STAGE * 128 bytes are fetched
// together (longer contiguous reads from HBM than one K block at a time)
constexpr int SKINNY_KB_PER_STAGE = 2;

struct SkinnyParams {
    int M;          // rows of A and D
    int N;
    int K;
    int nkb;        // K / 128
    int n_tiles;    // ceil(N / 128): 128-row blocks of B
    int m_blocks;   // ceil(M / MN): blocks of MN rows of A
    int tiles;      // n_tiles * m_blocks (tile t: B block t / m_blocks, A block t % m_blocks)
    int split;      // CTAs of a cluster that share one tile, each a contiguous K range
                    // (whole stages of SKINNY_KB_PER_STAGE K blocks)
    int kb_max;     // K blocks of the largest share
    int stages;     // operand ring depth (each stage SKINNY_KB_PER_STAGE K blocks)
    uint32_t stage_bytes; // B: [16 row groups][KB_PER_STAGE][8 rows][128 B]; then A:
                          // [KB_PER_STAGE][MN rows][128 B]
    uint32_t region;      // operand ring, reused for the FP32 partial tile at the end
    uint32_t off_recv;    // split > 1: the output slices the cluster's CTAs send to this one
    uint32_t off_sa;      // LHS scales of the CTA's K range: kb_max x MN FP32
    uint32_t off_sb;      // RHS scales of the tile's 128-row block: kb_max FP32
    uint32_t off_bars;
    uint32_t off_misc;    // TMEM base address, abort flag
    uint32_t total;       // bytes, excluding the 1024 B alignment slack
    const float *sa;      // [K/128][ld_sa]
    int ld_sa;
    const float *sb;      // [ceil(N/128)][K/128]
    uint16_t *D;          // [M][ld_d] BF16 bits (the first N columns are written)
    long ld_d;            // row stride of D in elements (>= N, a multiple of 8)
    unsigned int *status;
    uint64_t timeout_ns;
};

// Barriers of the skinny kernel: full per stage, "K block done" ring, TMEM
// buffer released (ring), scales loaded, all MMAs done, partial slices
// received.
constexpr int SKINNY_NUM_BARS_FIXED = DONE_RING + MAX_TMEM_BUFS + 3;

// Bytes of the partial tile ([MN][128] FP32) and of the receive area for the
// slices of the output that the cluster's CTAs send to one CTA: split slots
// of ceil(items / split) items, an item being 8 FP32 values (items = 16 M).
__host__ __device__ inline uint32_t skinny_red_bytes(int mn) { return (uint32_t)mn * SKINNY_TILE_N * 4u; }
__host__ __device__ inline uint32_t skinny_recv_slot_items(int rows, int split)
{
    const uint32_t items = (uint32_t)rows * (SKINNY_TILE_N / 8);
    return (items + (uint32_t)split - 1) / (uint32_t)split;
}

__host__ __device__ inline void make_skinny_plan(SkinnyParams &p, int mn, int stages)
{
    p.stages = stages;
    p.stage_bytes = (uint32_t)SKINNY_KB_PER_STAGE * (SKINNY_TILE_N + mn) * BLOCK_K;
    const uint32_t ring = p.stage_bytes * (uint32_t)stages;
    const uint32_t red = skinny_red_bytes(mn);
    p.region = ring > red ? ring : red;
    p.off_recv = align_up_u32(p.region, 1024);
    const int rows = p.M < mn ? p.M : mn; // rows of the largest tile
    const uint32_t recv = p.split > 1 ? (uint32_t)p.split * skinny_recv_slot_items(rows, p.split) * 32u : 0u;
    p.off_sa = align_up_u32(p.off_recv + recv, 128);
    p.off_sb = p.off_sa + (uint32_t)p.kb_max * (uint32_t)mn * 4u;
    p.off_bars = align_up_u32(p.off_sb + (uint32_t)p.kb_max * 4u, 8);
    p.off_misc = align_up_u32(p.off_bars + 8u * (uint32_t)(stages + SKINNY_NUM_BARS_FIXED), 16);
    p.total = p.off_misc + 16;
}

} // namespace fp8nt
