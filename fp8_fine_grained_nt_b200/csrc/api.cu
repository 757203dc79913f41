// C-ABI entry points of libfp8nt.so (declared in include/fp8_nt.h): argument
// validation, tile-configuration choice, TMA descriptor encoding and launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <math.h>
#include <mutex>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "fp8_nt.h"
#include "launch.h"
#include "params.h"

using namespace fp8nt;

namespace {

// ------------------------------------------------------------------ kernels

struct Candidate {
    int mw;
    int bn;
    int pair;   // 1: a CTA pair computes a 256-row tile (tcgen05 cta_group::2)
    int scalar; // 1: per-tensor scaling (whole-K accumulation in TMEM)
    LaunchFn launch;
};

const Candidate kCandidates[] = {
#define FP8NT_KERNEL(mw, bn, pair, scalar)                                                       \
    {mw, bn, pair, scalar, launch_mw##mw##_bn##bn##_p##pair##_s##scalar},
#include "kernels.def"
#undef FP8NT_KERNEL
};
constexpr int kNumCandidates = sizeof(kCandidates) / sizeof(kCandidates[0]);

// Small-M dense kernels (D^T tiles of 128 rows of B x MN rows of A).
struct SkinnyCandidate {
    int mn;
    SkinnyLaunchFn launch;
    SkinnyCapacityFn capacity;
};

const SkinnyCandidate kSkinny[] = {
#define FP8NT_SKINNY(mn) {mn, launch_skinny_mn##mn, skinny_capacity_mn##mn},
#include "skinny.def"
#undef FP8NT_SKINNY
};
constexpr int kNumSkinny = sizeof(kSkinny) / sizeof(kSkinny[0]);
static_assert(kNumSkinny <= 8, "the device capacity cache holds 8 small-M kernels");

constexpr int kDefaultSms = 148;           // B200
constexpr int kDefaultMaxSmem = 232448;    // 227 KB opt-in per block on sm_100
constexpr int kMaxStages = 12;
static_assert(kMaxStages <= DONE_RING, "the done ring must cover every operand stage");
constexpr int kMinStages = 2;
constexpr int kMaxSplit = 8; // CTAs per split-K cluster (portable cluster size)
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull; // 2 s per pipeline wait

// ------------------------------------------------------------------ devices

// The device status word.  Host code must not take this symbol's address
// directly: its device address is fetched per device with
// cudaGetSymbolAddress and passed to the kernels.  The snapshot word receives
// the status word's value when dg_get_device_status clears it.
__device__ unsigned int g_status_word;
__device__ unsigned int g_status_snapshot;

__global__ void status_exchange_kernel(unsigned int *status, unsigned int *snapshot)
{
    *snapshot = atomicExch(status, 0u);
}

std::mutex g_status_mutex;

struct DeviceInfo {
    bool ready;
    int sm_count;
    int cc_major;
    int cc_minor;
    int max_smem;
    unsigned int *status;
    unsigned int *status_snapshot;
    // clusters of `split` small-M CTAs the device holds at once (0 = not yet
    // asked, -1 = the query failed), per kernel of kSkinny
    std::atomic<int> skinny_cap[8][SKINNY_MAX_SPLIT + 1];
};

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;
// Settings shared by every call (a caller may set them from any thread):
// the SM bound of set_num_sms and the test hook of dg_force_config, the
// latter packed into one word so that a call sees one consistent setting.
std::atomic<int> g_num_sms_limit{0};
std::atomic<uint32_t> g_forced{0};

// swap: 0 = automatic, 1 = never the small-M (swap-AB) kernel, 2 = always
// where it applies (dense calls with M <= 256).  tail: 0 = automatic (off),
// 1 = never move a dense call's last partial wave to the small-M kernel, 2 =
// wherever the layout allows it, 3 = where the estimate favours it.
std::atomic<int> g_forced_swap{0};
std::atomic<int> g_forced_tail{0};

struct Forced {
    int bm, bn, split, pair, swap, tail;
};

uint32_t pack_forced(int bm, int bn, int split, int pair)
{
    return (uint32_t)bm | ((uint32_t)bn << 10) | ((uint32_t)split << 20) | ((uint32_t)pair << 24);
}

Forced forced_config()
{
    const uint32_t w = g_forced.load(std::memory_order_relaxed);
    return Forced{(int)(w & 0x3FF), (int)((w >> 10) & 0x3FF), (int)((w >> 20) & 0xF),
                  (int)((w >> 24) & 0x3), g_forced_swap.load(std::memory_order_relaxed),
                  g_forced_tail.load(std::memory_order_relaxed)};
}

int device_info(DeviceInfo **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return DG_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_devices[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess)
            return DG_ERR_CUDA;
        if (d.cc_major != 10 || d.cc_minor != 0)
            return DG_ERR_UNSUPPORTED_ARCH;
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess)
            return DG_ERR_CUDA;
        d.status = static_cast<unsigned int *>(addr);
        if (cudaGetSymbolAddress(&addr, g_status_snapshot) != cudaSuccess)
            return DG_ERR_CUDA;
        d.status_snapshot = static_cast<unsigned int *>(addr);
        d.ready = true;
    }
    *out = &d;
    return DG_OK;
}

uint64_t wait_timeout_ns()
{
    // read once (thread-safe static initialisation)
    static const uint64_t timeout_ns = [] {
        const char *env = getenv("DG_WAIT_TIMEOUT_MS");
        const long ms = env ? atol(env) : 0;
        return ms > 0 ? (uint64_t)ms * 1000000ull : kDefaultTimeoutNs;
    }();
    return timeout_ns;
}

// ------------------------------------------------------------------ TMA

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D row-major tensor [rows][cols] of `elem` bytes per element, row pitch
// `pitch_elems`, box [box_rows][box_cols].
int make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType type, int elem,
                 uint64_t cols, uint64_t rows, uint64_t pitch_elems, uint32_t box_cols,
                 uint32_t box_rows, CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return DG_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch_elems * (uint64_t)elem};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// ------------------------------------------------------------------ config

int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }

struct Problem {
    int kind;
    int M;          // dense M / contiguous M_sum / masked M_max
    int N;
    int K;
    int groups;
    int expected_m; // masked only
};

// Relative cost of one K block of a tile, by tile shape, measured on B200
// (dense 4096x7168x2048, 256x7168x2048, masked and contiguous shapes; time
// per K block per wave, BLOCK_N = 256 with one 128-row CTA = 1.0).  It is
// nearly flat in BLOCK_N: a K block is bound by the per-K-block pipeline
// (operand ring latency, TMEM partial reads, promotion), not by MMA rate or
// L2 bandwidth, so wide tiles and few waves win.  Two 128-row halves in one
// CTA cost more per K block; narrow tiles (<= 64 columns per K block) less.
double kb_cost_factor(int mw, int bn, int halves)
{
    if (mw == 2 && halves == 2) {
        switch (bn) {
        case 64: return 1.05;
        case 96: return 1.18;
        case 112: return 1.26;
        case 128: return 1.18;
        default: return 1.2;
        }
    }
    switch (bn) {
    case 64: return 0.70;
    case 96: return 0.97;
    case 112: return 0.99;
    case 128: return 0.99;
    case 160: return 0.94;
    case 192: return 1.02;
    case 224: return 1.08;
    case 256: return 1.0;
    default: return bn < 64 ? 0.6 : 1.0;
    }
}

// Cycle estimate of a (MW, BN, split, pair) choice on `sms` SMs: whole
// waves of CTAs (a CTA pair takes two SMs), each working through its K
// blocks at ~1300 cycles x kb_cost_factor per K block, plus a per-tile cost
// (pipeline ramp, and the BF16 store, which grows with the tile's size);
// split-K adds the cluster reduction.
double estimate_cycles(const Problem &pb, int mw, int bn, int split, int pair, int stages, int sms,
                       int *tiles_out, double *wave_out = nullptr)
{
    (void)stages;
    const int bm = pair ? 256 : 128 * mw;
    const int nkb = pb.K / 128;
    long m_blocks;
    int rows_eff;
    if (pb.kind == DG_KIND_MASKED) {
        int em = pb.expected_m > 0 ? pb.expected_m : pb.M;
        em = em > pb.M ? pb.M : em;
        em = em < 1 ? 1 : em;
        m_blocks = (long)pb.groups * ceil_div(em, bm);
        rows_eff = em < bm ? em : bm;
    } else {
        m_blocks = ceil_div(pb.M, bm);
        rows_eff = pb.M < bm ? pb.M : bm;
    }
    const long n_blocks = ceil_div(pb.N, bn);
    const long tiles = m_blocks * n_blocks;
    const long ctas = tiles * split * (pair ? 2 : 1);
    const long waves = (ctas + sms - 1) / sms;
    const int halves = (mw == 2 && rows_eff > 128) ? 2 : 1;
    const int kb_per_cta = ceil_div(nkb, split);
    const int cta_rows = pair ? 128 : (rows_eff < 128 * mw ? rows_eff : 128 * mw);
    const double kb_cycles = pb.kind == DG_KIND_DENSE_PER_TENSOR
                                 ? 4.0 * (bn / 2 > 64 ? bn / 2 : 64) + 150.0
                                 : 1300.0 * kb_cost_factor(pair ? 1 : mw, bn, halves);
    double tile = kb_per_cta * kb_cycles + 1500.0 + 3500.0 * bn * cta_rows / (256.0 * 128.0);
    if (split > 1)
        tile += 800.0 + (double)bm * bn * 4.0 * split / 256.0 / split;
    if (tiles_out)
        *tiles_out = (int)(tiles > 0x7fffffff ? 0x7fffffff : tiles);
    if (wave_out)
        *wave_out = tile;
    return waves * tile;
}

int plan_for(const Problem &pb, int mw, int bn, int split, int pair, int max_smem, int *stages,
             SmemPlan *plan)
{
    const int nkb = pb.K / 128;
    const int prefix_ints = pb.kind == DG_KIND_MASKED ? 2 * pb.groups + 1 : 0;
    // Shared memory beyond the operand ring holds the output staging: the
    // whole BF16 tile (one bulk store per warp), or fewer 2 KB slots that
    // the output chunks stream through.  With per-block promotion the
    // epilogue bounds the kernel and a whole staged tile is faster than an
    // extra operand stage; with per-tensor scales the operand ring bounds it
    // and the extra stage wins (measured on B200: 4096x7168x2048 per-tensor
    // 60 -> 54 us with 4 stages and one slot; fine-grained 79 -> 84 us).
    const int chunks = ((mw == 1 ? bn / 2 : bn) + 31) / 32;
    const bool stages_first = pb.kind == DG_KIND_DENSE_PER_TENSOR;
    for (int pass = 0; pass < 2; ++pass) {
        for (int s = kMaxStages; s >= kMinStages; --s) {
            const int lo = (stages_first || pass == 1) ? 1 : chunks;
            for (int slots = chunks; slots >= lo; --slots) {
                SmemPlan p = make_smem_plan(mw, bn, s, nkb, prefix_ints, split > 1, pair != 0, slots);
                if ((int)p.total + 1024 <= max_smem) {
                    *stages = s;
                    *plan = p;
                    return DG_OK;
                }
            }
        }
    }
    return DG_ERR_UNSUPPORTED_SHAPE;
}

// Clusters of `split` CTAs that can be resident at once (conservative for a
// 148-SM part with one CTA per SM: clusters are placed within a GPC).
int max_resident_clusters(int split, int sms)
{
    if (split <= 1)
        return sms;
    if (split == 2)
        return sms / 2;
    return (sms / 4) * 4 / split - 1; // leave slack for GPCs with spare SMs
}

int choose(const Problem &pb, int sms, int max_smem, const Candidate **out_cand, dg_config *cfg,
           SmemPlan *plan)
{
    const Forced forced = forced_config();
    const Candidate *best = nullptr;
    int best_split = 1;
    double best_cost = 0;
    const int nkb = pb.K / 128;
    for (int i = 0; i < kNumCandidates; ++i) {
        const Candidate &c = kCandidates[i];
        const int c_bm = c.pair ? 256 : c.mw * 128;
        if (forced.bm && (c_bm != forced.bm || c.bn != forced.bn))
            continue;
        if (forced.pair && (forced.pair == 2) != (c.pair != 0))
            continue;
        // CTA pairs only on request: measured on B200 they were no faster
        // than one CTA per tile on the dense, masked and 256-row shapes
        if (c.pair && forced.pair != 2)
            continue;
        if (pb.kind == DG_KIND_CONTIGUOUS && c_bm != 128)
            continue; // a 256-row tile could straddle two 128-aligned experts
        if ((pb.kind == DG_KIND_DENSE_PER_TENSOR) != (c.scalar != 0))
            continue; // per-tensor and fine-grained scaling have their own kernels
        for (int split = 1; split <= kMaxSplit; split *= 2) {
            if (forced.split && split != forced.split)
                continue;
            if (c.pair && split > 1)
                continue;
            // 8-CTA clusters only on request: measured slower than 4 on the
            // decode shape (the 8-way reduction and cluster placement cost
            // more than the shorter K range saves)
            if (split > 4 && forced.split != split)
                continue;
            if (split > 1) {
                // split-K only for dense calls too small to fill the SMs
                if (pb.kind != DG_KIND_DENSE || nkb < 2 * split)
                    continue;
                const long tiles = (long)ceil_div(pb.M, c.mw * 128) * ceil_div(pb.N, c.bn);
                if (tiles * split > sms || tiles > max_resident_clusters(split, sms))
                    continue;
            }
            int st;
            SmemPlan p;
            if (plan_for(pb, c.mw, c.bn, split, c.pair, max_smem, &st, &p) != DG_OK)
                continue;
            // the split-K partial tile must not crowd out the operand ring
            if (split > 1 && (c.mw * c.bn > 128 || st < 4))
                continue;
            const double cost = estimate_cycles(pb, c.mw, c.bn, split, c.pair, st, sms, nullptr);
            // ties: wider tile first (fewer re-reads of A), then one M half,
            // then a single CTA, then no split
            const bool better =
                !best || cost < best_cost * (1 - 1e-9) ||
                (fabs(cost - best_cost) <= best_cost * 1e-9 &&
                 (c.bn > best->bn ||
                  (c.bn == best->bn &&
                   (c.mw < best->mw || (c.mw == best->mw && c.pair < best->pair)))));
            if (better) {
                best = &c;
                best_split = split;
                best_cost = cost;
            }
        }
    }
    if (!best)
        return DG_ERR_UNSUPPORTED_SHAPE;
    int st;
    plan_for(pb, best->mw, best->bn, best_split, best->pair, max_smem, &st, plan);
    const int bm = best->pair ? 256 : best->mw * 128;
    long tiles;
    if (pb.kind == DG_KIND_MASKED)
        tiles = (long)pb.groups * ceil_div(pb.M, bm) * ceil_div(pb.N, best->bn);
    else
        tiles = (long)ceil_div(pb.M, bm) * ceil_div(pb.N, best->bn);
    if (tiles > 0x7fffffffL)
        return DG_ERR_UNSUPPORTED_SHAPE;
    cfg->block_m = bm;
    cfg->block_n = best->bn;
    cfg->stages = st;
    cfg->num_tiles = (int)tiles;
    cfg->split = best_split;
    cfg->cta_pair = best->pair ? 2 : 1;
    cfg->swap_ab = 0;
    cfg->tail_tiles = 0;
    if (best_split > 1)
        cfg->grid = (int)tiles * best_split; // one tile per cluster
    else if (best->pair)
        cfg->grid = 2 * (int)(tiles < sms / 2 ? tiles : sms / 2); // persistent pairs
    else
        cfg->grid = (int)(tiles < sms ? tiles : sms);
    if (cfg->grid < 1)
        cfg->grid = 1;
    cfg->smem_bytes = (int)plan->total + 1024;
    const int buf_cols = best->mw * best->bn;
    const int nbuf = best->scalar ? 2 : (512 / buf_cols < MAX_TMEM_BUFS ? 512 / buf_cols : MAX_TMEM_BUFS);
    const int need = nbuf * buf_cols; // the kernel's ring of K-block partials
    cfg->tmem_cols = need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
    *out_cand = best;
    return DG_OK;
}

// ------------------------------------------------------------------ small M

// Dynamic shared memory of a small-M CTA is never below this, so that one CTA
// runs per SM (each allocates the SM's whole tensor memory) and the cluster
// capacity does not depend on K.
constexpr int kSkinnyMinSmem = 116 * 1024;

// Clusters of `split` CTAs (one per SM) that can run at once, when the device
// has not been asked: a cluster does not span a GPC, and B200's 148 SMs form
// 8 GPCs of at least 18 SMs; a lowered SM bound caps it too.
int cluster_capacity_model(int split, int sms)
{
    if (split <= 1)
        return sms;
    const int by_gpc = 8 * (18 / split);
    const int by_sms = sms / split;
    const int cap = by_gpc < by_sms ? by_gpc : by_sms;
    return cap > 0 ? cap : 1;
}

// Cycle estimate of a small-M choice: waves of clusters, each CTA streaming
// its share of K blocks at the slowest of (a) the four MMAs of a K block (at
// least ~64 cycles each for one issuing thread, ~75 at N = 128), (b) its share
// of the HBM bandwidth (~3300 B/clk at the boost clock) for 16 KB of B per K
// block, (c) what one CTA's operand ring keeps in flight: measured on B200
// (decode shape, 34 to 102 CTAs) a CTA takes in ~30 B/clk whatever the
// number of CTAs, so more CTAs stream faster until (b) binds; plus set-up
// and, with a cluster, the exchange of the partial tiles (~4000 cycles and
// more with the cluster's size: the partial tile's write, the bulk copies,
// the wait for the slowest CTA, the sums, the closing barrier; traced at
// ~4000-6000 cycles on the decode shape; 128x128x512 measured at 6.3 us per
// call in a graph on one CTA against 7.3 us on a cluster of 2 or 4).
double skinny_cycles(int M, int N, int K, int mn, int split, int cap)
{
    const long tiles = (long)ceil_div(N, SKINNY_TILE_N) * ceil_div(M, mn);
    const int nkb = K / 128;
    const long waves = (tiles + cap - 1) / cap;
    const long active = (tiles < cap ? tiles : cap) * (long)split;
    const int cnt = ceil_div(nkb, split);
    const double t_mma = 4.0 * (mn <= 64 ? 64.0 : 75.0);
    const double t_hbm = 128.0 * 128.0 * (double)active / 3300.0;
    const double t_tma = (128.0 + mn) * 128.0 / 30.0;
    double t_kb = t_mma > t_hbm ? t_mma : t_hbm;
    t_kb = t_kb > t_tma ? t_kb : t_tma;
    return (double)waves * (1200.0 + cnt * t_kb + (split > 1 ? 4000.0 + 150.0 * split : 300.0));
}

struct SkinnyChoice {
    const SkinnyCandidate *cand;
    int cand_index;
    SkinnyParams plan; // sizes, split, stages and shared-memory offsets
    int smem_bytes;
    double cycles;     // the estimate it was chosen by
};

// Shared-memory plan of a small-M kernel: as many operand stages as fit, up to
// the CTA's number of K blocks.
bool skinny_plan(const Problem &pb, int mn, int split, int max_smem, SkinnyParams *out)
{
    SkinnyParams p;
    memset(&p, 0, sizeof(p));
    p.M = pb.M;
    p.N = pb.N;
    p.K = pb.K;
    p.nkb = pb.K / 128;
    p.n_tiles = ceil_div(pb.N, SKINNY_TILE_N);
    p.m_blocks = ceil_div(pb.M, mn);
    p.tiles = p.n_tiles * p.m_blocks;
    p.split = split;
    const int units = ceil_div(p.nkb, SKINNY_KB_PER_STAGE);
    const int unit_max = ceil_div(units, split);
    p.kb_max = unit_max * SKINNY_KB_PER_STAGE;
    // stages (each KB_PER_STAGE K blocks) in flight stay within the ring of
    // "K block done" barriers
    const int st_cap = DONE_RING / SKINNY_KB_PER_STAGE;
    int st = unit_max < st_cap ? unit_max : st_cap;
    for (; st >= 1; --st) {
        make_skinny_plan(p, mn, st);
        if ((int)p.total + 1024 <= max_smem)
            break;
    }
    if (st < 1 || (st < 2 && unit_max > 1))
        return false;
    *out = p;
    return true;
}

// Capacity of the device (queried once per kernel and cluster size), or the
// GPC model when no device is given or the query fails.
int skinny_capacity(DeviceInfo *dev, int idx, int split, int sms)
{
    const int model = cluster_capacity_model(split, sms);
    if (!dev)
        return model;
    int c = dev->skinny_cap[idx][split].load(std::memory_order_relaxed);
    if (c == 0) {
        c = kSkinny[idx].capacity(split, kSkinnyMinSmem);
        dev->skinny_cap[idx][split].store(c > 0 ? c : -1, std::memory_order_relaxed);
    }
    if (c <= 0)
        return model;
    // a lowered SM bound (set_num_sms) caps the device's own figure
    const int by_sms = sms / split > 0 ? sms / split : 1;
    return c < by_sms ? c : by_sms;
}

// Small-M kernel for a dense call: the smallest MN >= M, and the cluster size
// (CTAs sharing a tile's K range) with the lowest estimate.
int choose_skinny(const Problem &pb, int sms, int max_smem, DeviceInfo *dev, SkinnyChoice *out)
{
    const Forced forced = forced_config();
    // the smallest MN >= M; for larger M the widest, over blocks of MN rows
    int idx = -1;
    for (int i = 0; i < kNumSkinny; ++i)
        if (kSkinny[i].mn >= pb.M && (idx < 0 || kSkinny[i].mn < kSkinny[idx].mn))
            idx = i;
    if (idx < 0)
        for (int i = 0; i < kNumSkinny; ++i)
            if (idx < 0 || kSkinny[i].mn > kSkinny[idx].mn)
                idx = i;
    const int nkb = pb.K / 128;
    double best = 0;
    bool found = false;
    for (int split = 1; split <= SKINNY_MAX_SPLIT; ++split) {
        if (forced.split ? split != forced.split : split > nkb)
            continue;
        SkinnyParams p;
        if (!skinny_plan(pb, kSkinny[idx].mn, split, max_smem, &p))
            continue;
        const int cap = skinny_capacity(dev, idx, split, sms);
        const double cost = skinny_cycles(pb.M, pb.N, pb.K, kSkinny[idx].mn, split, cap);
        if (!found || cost < best * (1 - 1e-9)) {
            found = true;
            best = cost;
            out->cycles = cost;
            out->cand = &kSkinny[idx];
            out->cand_index = idx;
            out->plan = p;
            const int need = (int)p.total + 1024;
            out->smem_bytes = need > kSkinnyMinSmem ? need : kSkinnyMinSmem;
        }
    }
    return found ? DG_OK : DG_ERR_UNSUPPORTED_SHAPE;
}

// Dense calls with M <= 256 take the small-M kernel (M > 128 in blocks of
// 128 rows: a 256-row call is two tiles per 128 columns of D, no split of K
// needed to fill the SMs), unless the test hooks turn it off or pin a tile
// shape or CTA pairs of the other kernels.
constexpr int kSkinnyMaxM = 256;

bool use_skinny(const Problem &pb)
{
    if (pb.kind != DG_KIND_DENSE || pb.M > kSkinnyMaxM)
        return false;
    if ((long)ceil_div(pb.N, SKINNY_TILE_N) * ceil_div(pb.M, SKINNY_MAX_M) > 65535)
        return false; // grid.y limit
    const Forced f = forced_config();
    if (f.swap != 0)
        return f.swap == 2;
    return f.bm == 0 && f.pair != 2;
}

void skinny_config(const SkinnyChoice &c, dg_config *cfg)
{
    memset(cfg, 0, sizeof(*cfg));
    cfg->block_m = c.cand->mn;
    cfg->block_n = SKINNY_TILE_N;
    cfg->stages = c.plan.stages;
    cfg->num_tiles = c.plan.tiles;
    cfg->grid = c.plan.tiles * c.plan.split;
    cfg->smem_bytes = c.smem_bytes;
    const int mn = c.cand->mn;
    const int nbuf = 512 / mn < MAX_TMEM_BUFS ? 512 / mn : MAX_TMEM_BUFS;
    const int need = nbuf * mn;
    cfg->tmem_cols = need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
    cfg->split = c.plan.split;
    cfg->cta_pair = 1;
    cfg->swap_ab = 1;
}

int effective_sms(const DeviceInfo *d)
{
    int n = d ? d->sm_count : kDefaultSms;
    const int limit = g_num_sms_limit.load(std::memory_order_relaxed);
    if (limit > 0 && limit < n)
        n = limit;
    return n;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(const void *A, const float *sa, const void *B, const float *sb, void *D, int M,
                 int N, int K, bool scalar_scales = false)
{
    if (M < 0 || N < 0 || K < 0)
        return DG_ERR_INVALID_ARGUMENT;
    if (K == 0 || K % 128 != 0 || N % 8 != 0)
        return DG_ERR_UNSUPPORTED_SHAPE;
    if (M == 0 || N == 0)
        return DG_OK;
    if (!A || !sa || !B || !sb || !D)
        return DG_ERR_INVALID_ARGUMENT;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D))
        return DG_ERR_MISALIGNED;
    // per-tensor scales are single FP32 values read as scalars: 4-byte
    // alignment; block scales are tensors read by TMA / vector copies: 16
    const uintptr_t scale_align = scalar_scales ? 3u : 15u;
    if ((reinterpret_cast<uintptr_t>(sa) & scale_align) || (reinterpret_cast<uintptr_t>(sb) & scale_align))
        return DG_ERR_MISALIGNED;
    return DG_OK;
}

// Operands of a dense call as the small-M kernel reads them: a whole call, or
// a block of one (rows [row0, M) and columns [col0, N) of D: A from row row0,
// B from row col0, the scales offset to match, D with the call's row stride).
struct DenseView {
    const void *A;
    const float *sa;
    long ld_sa;
    const void *B;
    const float *sb;
    void *D;
    long ld_d;
};

// Dense call with M <= 256 (or a block of one) through the small-M kernel.
int run_skinny(const Problem &pb, DeviceInfo *dev, int sms, const DenseView &v, cudaStream_t stream)
{
    SkinnyChoice ch;
    int st = choose_skinny(pb, sms, dev->max_smem, dev, &ch);
    if (st != DG_OK)
        return st;
    const void *A = v.A, *B = v.B;
    CUtensorMap tmap_a, tmap_b;
    // A: [M][K] bytes, box MN rows x 128 (rows past M are zero-filled)
    if ((st = make_tmap_2d(&tmap_a, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pb.K, pb.M, pb.K, 128,
                           (uint32_t)ch.cand->mn, CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
        return st;
    // B: [N][K] bytes viewed in 4-D as [N/8 row groups][K/128 K blocks][8 rows]
    // [128 bytes] (N % 8 == 0), box = 16 row groups x KB_PER_STAGE K blocks:
    // the tile's 128 rows of KB_PER_STAGE consecutive K blocks, laid out in
    // shared memory as [row group][K block][8 rows][128 B] (128-byte swizzle)
    {
        EncodeTiledFn fn = encode_fn();
        if (!fn)
            return DG_ERR_CUDA;
        cuuint64_t dims[4] = {128, 8, (cuuint64_t)(pb.K / 128), (cuuint64_t)(pb.N / 8)};
        cuuint64_t strides[3] = {(cuuint64_t)pb.K, 128, (cuuint64_t)pb.K * 8};
        cuuint32_t box[4] = {128, 8, SKINNY_KB_PER_STAGE, SKINNY_TILE_N / 8};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        if (fn(&tmap_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(B), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return DG_ERR_CUDA;
    }
    SkinnyParams p = ch.plan;
    p.sa = v.sa;
    p.ld_sa = (int)v.ld_sa;
    p.sb = v.sb;
    p.D = static_cast<uint16_t *>(v.D);
    p.ld_d = v.ld_d;
    p.status = dev->status;
    p.timeout_ns = wait_timeout_ns();
    // persistent clusters: no more than the SM bound (and the device) holds
    const int cap = skinny_capacity(dev, ch.cand_index, p.split, sms);
    const int by_sms = sms / p.split > 0 ? sms / p.split : 1;
    int clusters = p.tiles;
    if (clusters > cap)
        clusters = cap;
    if (clusters > by_sms)
        clusters = by_sms;
    SkinnyLaunchArgs args;
    args.tmap_a = &tmap_a;
    args.tmap_b = &tmap_b;
    args.params = &p;
    args.split = p.split;
    args.n_tiles = clusters;
    args.smem_bytes = ch.smem_bytes;
    args.stream = stream;
    return ch.cand->launch(args) == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

// The last wave of a dense call on the 128-row kernels, when only partly
// filled (tiles not a multiple of the persistent grid), runs a whole tile
// time on a few SMs while the rest idle.  Tiles are numbered with N fastest,
// so when that wave's tiles all lie in the last M block and start on a
// 128-column boundary (the granularity of sb), they form one block of D: the
// last M block's rows (at most 256) by the remaining columns.  That block is
// a small-M GEMM, which the small-M kernel spreads over the SMs with its K
// range split over clusters; it runs after the main kernel, which then
// computes whole waves only.  Measured on B200 it is no faster than the
// partial wave (dense 4096, 2048 and 8192 x 7168 x 2048: 81.2 / 50.9 / 143.3
// us without, 81.6 / 50.7 / 145.4 us with: a wave of a few tiles alone runs
// its K blocks faster than a full one), so it is taken only on request
// (dg_force_tail_split), where the small-M estimate plus the gap between two
// launches is below the wave it replaces or the request insists.
struct TailSplit {
    int main_tiles; // tiles left to the main kernel
    int row0;       // the block's first row and column in D
    int col0;
    Problem sub;    // the block as a dense problem
};

constexpr double kLaunchGapCycles = 4000.0; // ~2 us between dependent launches

bool plan_tail(const Problem &pb, const dg_config &cfg, int sms, int max_smem, DeviceInfo *dev,
               TailSplit *out)
{
    const Forced f = forced_config();
    if (pb.kind != DG_KIND_DENSE || cfg.split != 1 || cfg.cta_pair != 1 || cfg.swap_ab || f.tail == 0 ||
        f.tail == 1)
        return false;
    const long tiles = cfg.num_tiles, grid = cfg.grid;
    if (grid <= 0)
        return false;
    const long full = tiles / grid * grid;
    if (full == 0 || full == tiles)
        return false;
    const long m_blocks = ceil_div(pb.M, cfg.block_m), n_blocks = ceil_div(pb.N, cfg.block_n);
    const long last_row_first = (m_blocks - 1) * n_blocks; // first tile of the last M block
    if (full < last_row_first)
        return false;
    const long col0 = (full - last_row_first) * cfg.block_n;
    const long row0 = (m_blocks - 1) * cfg.block_m;
    if (col0 % 128 != 0 || col0 >= pb.N || pb.M - row0 > kSkinnyMaxM)
        return false;
    Problem sub{DG_KIND_DENSE, (int)(pb.M - row0), (int)(pb.N - col0), pb.K, 1, 0};
    if ((long)ceil_div(sub.N, SKINNY_TILE_N) * ceil_div(sub.M, SKINNY_MAX_M) > 65535)
        return false; // grid.y limit
    SkinnyChoice ch;
    if (choose_skinny(sub, sms, max_smem, dev, &ch) != DG_OK)
        return false;
    if (f.tail == 3) {
        double wave = 0;
        const int mw = cfg.block_m / 128;
        estimate_cycles(pb, mw, cfg.block_n, 1, 0, cfg.stages, sms, nullptr, &wave);
        if (ch.cycles + kLaunchGapCycles >= wave)
            return false;
    }
    out->main_tiles = (int)full;
    out->row0 = (int)row0;
    out->col0 = (int)col0;
    out->sub = sub;
    return true;
}

// Shared launch path for the three forms.
int run(const Problem &pb, const void *A, const float *sa, const void *B, const float *sb, void *D,
        const int *m_indices, const int *masked_m, cudaStream_t stream)
{
    DeviceInfo *dev = nullptr;
    int st = device_info(&dev);
    if (st != DG_OK)
        return st;
    const int sms = effective_sms(dev);
    if (use_skinny(pb)) {
        const DenseView v{A, sa, get_tma_aligned_size(pb.M, 4), B, sb, D, pb.N};
        return run_skinny(pb, dev, sms, v, stream);
    }
    const Candidate *cand = nullptr;
    dg_config cfg;
    SmemPlan plan;
    st = choose(pb, sms, dev->max_smem, &cand, &cfg, &plan);
    if (st != DG_OK)
        return st;
    TailSplit tail;
    const bool has_tail = plan_tail(pb, cfg, sms, dev->max_smem, dev, &tail);

    const int nkb = pb.K / 128;
    const int nnb = ceil_div(pb.N, 128);
    const int groups = (pb.kind == DG_KIND_DENSE || pb.kind == DG_KIND_DENSE_PER_TENSOR) ? 1 : pb.groups;
    const int ld_sa = get_tma_aligned_size(pb.M, 4);

    CUtensorMap tmap_a, tmap_b, tmap_sa, tmap_d;
    const long a_rows = pb.kind == DG_KIND_MASKED ? (long)groups * pb.M : pb.M;
    const long b_rows = (long)groups * pb.N;
    if ((st = make_tmap_2d(&tmap_a, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pb.K, a_rows, pb.K, 128,
                           128, CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
        return st;
    // a CTA of a pair loads half of the B tile
    const uint32_t b_box_rows = cand->pair ? cfg.block_n / 2 : cfg.block_n;
    if ((st = make_tmap_2d(&tmap_b, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pb.K, b_rows, pb.K, 128,
                           b_box_rows, CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK)
        return st;
    // LHS scales as a [sa_groups * K/128][ld_sa] FP32 matrix (only the
    // masked form has one scale block per group; the contiguous form's rows
    // are already concatenated); one box holds a CTA's rows for
    // SA_SLOT_BYTES / (rows * 4) consecutive K blocks
    const long sa_groups = pb.kind == DG_KIND_MASKED ? groups : 1;
    const uint32_t sa_box_rows = cand->pair ? 128u : (uint32_t)cfg.block_m;
    memset(&tmap_sa, 0, sizeof(tmap_sa)); // per-tensor scaling: not read by the kernel
    if (!cand->scalar &&
        (st = make_tmap_2d(&tmap_sa, sa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)ld_sa,
                           (uint64_t)sa_groups * nkb, (uint64_t)ld_sa, sa_box_rows,
                           SA_SLOT_BYTES / (sa_box_rows * 4u), CU_TENSOR_MAP_SWIZZLE_NONE)) != DG_OK)
        return st;
    // D as a [rows][N] BF16 matrix; the epilogue stores 32 x 32 boxes staged
    // with the 64-byte swizzle (elements past the tensor are not written)
    const long d_rows = pb.kind == DG_KIND_MASKED ? (long)groups * pb.M : pb.M;
    // When N and every epilogue thread's column span are multiples of 32,
    // D is viewed in 3-D as [N/32 column chunks][rows][32 columns] so that a
    // warp's whole staged row block (chunk-major, as staged) is one box.
    const int thread_cols = cand->mw == 1 ? cfg.block_n / 2 : cfg.block_n;
    bool d3 = cfg.split == 1 && pb.N % 32 == 0 && thread_cols % 32 == 0 &&
              (int)plan.out_slots * 32 >= thread_cols; // whole row block staged
    if (d3) {
        EncodeTiledFn fn = encode_fn();
        cuuint64_t dims[3] = {32, (cuuint64_t)d_rows, (cuuint64_t)(pb.N / 32)};
        cuuint64_t strides[2] = {(cuuint64_t)pb.N * 2, 64};
        cuuint32_t box[3] = {32, 32, (cuuint32_t)(thread_cols / 32)};
        cuuint32_t estr[3] = {1, 1, 1};
        d3 = fn && fn(&tmap_d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, D, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    if (!d3 && (st = make_tmap_2d(&tmap_d, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pb.N, d_rows,
                                  pb.N, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) != DG_OK)
        return st;

    Params p;
    memset(&p, 0, sizeof(p));
    p.kind = pb.kind == DG_KIND_DENSE_PER_TENSOR ? DG_KIND_DENSE : pb.kind;
    p.M = pb.M;
    p.N = pb.N;
    p.K = pb.K;
    p.num_groups = groups;
    p.nkb = nkb;
    p.nnb = nnb;
    p.m_blocks = ceil_div(pb.M, cfg.block_m);
    p.n_blocks = ceil_div(pb.N, cfg.block_n);
    p.num_tiles = has_tail ? tail.main_tiles : cfg.num_tiles;
    p.split = cfg.split;
    p.kb_chunk = ceil_div(nkb, cfg.split);
    p.stages = cfg.stages;
    p.plan = plan;
    p.sa = sa;
    p.ld_sa = ld_sa;
    p.sb = sb;
    p.m_indices = m_indices;
    p.masked_m = masked_m;
    p.D = static_cast<uint16_t *>(D);
    p.d_store_3d = d3 ? 1 : 0;
    p.status = dev->status;
    p.timeout_ns = wait_timeout_ns();

    LaunchArgs args;
    args.tmap_a = &tmap_a;
    args.tmap_b = &tmap_b;
    args.tmap_sa = &tmap_sa;
    args.tmap_d = &tmap_d;
    args.params = &p;
    args.grid = cfg.grid;
    args.cluster = cand->pair ? 2 : cfg.split;
    args.smem_bytes = cfg.smem_bytes;
    args.stream = stream;
    if (cand->launch(args) != cudaSuccess)
        return DG_ERR_CUDA;
    if (!has_tail)
        return DG_OK;
    const size_t r0 = (size_t)tail.row0, c0 = (size_t)tail.col0;
    const DenseView v{static_cast<const uint8_t *>(A) + r0 * (size_t)pb.K, sa + r0, ld_sa,
                      static_cast<const uint8_t *>(B) + c0 * (size_t)pb.K, sb + (c0 / 128) * (size_t)nkb,
                      static_cast<uint16_t *>(D) + r0 * (size_t)pb.N + c0, pb.N};
    return run_skinny(tail.sub, dev, sms, v, stream);
}

} // namespace

// ====================================================================== C ABI

extern "C" {

int gemm_fp8_fp8_bf16_nt(const void *A, const float *sa, const void *B, const float *sb, void *D,
                         int M, int N, int K, dg_stream_t stream)
{
    int st = check_common(A, sa, B, sb, D, M, N, K);
    if (st != DG_OK || M == 0 || N == 0)
        return st;
    Problem pb{DG_KIND_DENSE, M, N, K, 1, 0};
    return run(pb, A, sa, B, sb, D, nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int gemm_fp8_fp8_bf16_nt_per_tensor(const void *A, const float *scale_a, const void *B,
                                    const float *scale_b, void *D, int M, int N, int K,
                                    dg_stream_t stream)
{
    int st = check_common(A, scale_a, B, scale_b, D, M, N, K, true);
    if (st != DG_OK || M == 0 || N == 0)
        return st;
    Problem pb{DG_KIND_DENSE_PER_TENSOR, M, N, K, 1, 0};
    return run(pb, A, scale_a, B, scale_b, D, nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(const void *A, const float *sa, const void *B,
                                              const float *sb, void *D, const int *m_indices,
                                              int num_groups, int M_sum, int N, int K,
                                              dg_stream_t stream)
{
    if (num_groups <= 0)
        return DG_ERR_INVALID_ARGUMENT;
    int st = check_common(A, sa, B, sb, D, M_sum, N, K);
    if (st != DG_OK || M_sum == 0 || N == 0)
        return st;
    if (!m_indices)
        return DG_ERR_INVALID_ARGUMENT;
    if (!aligned16(m_indices))
        return DG_ERR_MISALIGNED;
    if (M_sum % get_m_alignment_for_contiguous_layout() != 0)
        return DG_ERR_UNSUPPORTED_SHAPE;
    if ((long)num_groups * N > 0x7fffffffL)
        return DG_ERR_UNSUPPORTED_SHAPE;
    Problem pb{DG_KIND_CONTIGUOUS, M_sum, N, K, num_groups, 0};
    return run(pb, A, sa, B, sb, D, m_indices, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int m_grouped_gemm_fp8_fp8_bf16_nt_masked(const void *A, const float *sa, const void *B,
                                          const float *sb, void *D, const int *masked_m, int G,
                                          int M_max, int N, int K, int expected_m,
                                          dg_stream_t stream)
{
    if (G <= 0 || expected_m < 0)
        return DG_ERR_INVALID_ARGUMENT;
    if (G > MAX_MASKED_GROUPS)
        return DG_ERR_UNSUPPORTED_SHAPE;
    int st = check_common(A, sa, B, sb, D, M_max, N, K);
    if (st != DG_OK || M_max == 0 || N == 0)
        return st;
    if (!masked_m)
        return DG_ERR_INVALID_ARGUMENT;
    if (!aligned16(masked_m))
        return DG_ERR_MISALIGNED;
    if ((long)G * M_max > 0x7fffffffL || (long)G * N > 0x7fffffffL)
        return DG_ERR_UNSUPPORTED_SHAPE;
    Problem pb{DG_KIND_MASKED, M_max, N, K, G, expected_m};
    return run(pb, A, sa, B, sb, D, nullptr, masked_m, reinterpret_cast<cudaStream_t>(stream));
}

int quantize_fp8_1x128(const void *x, int x_dtype, void *q, float *sa, int M, int K,
                       dg_stream_t stream)
{
    if (M < 0 || K < 0 || (x_dtype != DG_INPUT_F32 && x_dtype != DG_INPUT_BF16))
        return DG_ERR_INVALID_ARGUMENT;
    if (K == 0 || K % 128 != 0)
        return DG_ERR_UNSUPPORTED_SHAPE;
    if (M == 0)
        return DG_OK;
    if (!x || !q || !sa)
        return DG_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sa))
        return DG_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int st = device_info(&dev);
    if (st != DG_OK)
        return st;
    const long ld_sa = get_tma_aligned_size(M, 4);
    return launch_quantize_1x128(x, x_dtype == DG_INPUT_BF16, static_cast<uint8_t *>(q), sa, M, K,
                                 ld_sa, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DG_OK
               : DG_ERR_CUDA;
}

int dg_selftest_wait_timeout(int timeout_us, dg_stream_t stream)
{
    if (timeout_us <= 0 || timeout_us > 10000000)
        return DG_ERR_INVALID_ARGUMENT;
    DeviceInfo *dev = nullptr;
    int st = device_info(&dev);
    if (st != DG_OK)
        return st;
    return launch_wait_timeout_selftest(dev->status, (unsigned long long)timeout_us * 1000ull,
                                        reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DG_OK
               : DG_ERR_CUDA;
}

int get_m_alignment_for_contiguous_layout(void) { return 128; }

int get_tma_aligned_size(int x, int element_size)
{
    if (x < 0 || element_size <= 0 || 16 % element_size != 0)
        return -DG_ERR_INVALID_ARGUMENT;
    const int align = 16 / element_size;
    return (x + align - 1) / align * align;
}

int set_num_sms(int n)
{
    g_num_sms_limit.store(n > 0 ? n : 0, std::memory_order_relaxed);
    return DG_OK;
}

int get_num_sms(void)
{
    int count = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
        const int limit = g_num_sms_limit.load(std::memory_order_relaxed);
        if (limit > 0 && limit < count)
            return limit;
        return count;
    }
    cudaGetLastError(); // no device: clear the sticky-free error state
    return g_num_sms_limit.load(std::memory_order_relaxed);
}

const char *dg_status_string(int status)
{
    switch (status) {
    case DG_OK: return "ok";
    case DG_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DG_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case DG_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DG_ERR_UNSUPPORTED_ARCH: return "current device is not sm_100 (B200)";
    case DG_ERR_CUDA: return "CUDA call failed";
    case DG_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
    case DG_ERR_DEVICE_BAD_INDEX: return "masked_m or m_indices out of range";
    default: return "unknown status";
    }
}

int dg_get_device_status(dg_stream_t stream)
{
    DeviceInfo *dev = nullptr;
    int st = device_info(&dev);
    if (st != DG_OK)
        return st;
    // One thread swaps the status word for zero (so a bit set by a kernel on
    // another stream is either reported now or kept for the next call, never
    // lost) and leaves the old value in the snapshot word; host threads take
    // turns, so each reads its own snapshot.
    std::lock_guard<std::mutex> lock(g_status_mutex);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    status_exchange_kernel<<<1, 1, 0, s>>>(dev->status, dev->status_snapshot);
    if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return DG_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpy(&word, dev->status_snapshot, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return DG_ERR_CUDA;
    if (word & DEVERR_TIMEOUT)
        return DG_ERR_DEVICE_TIMEOUT;
    if (word & DEVERR_BAD_INDEX)
        return DG_ERR_DEVICE_BAD_INDEX;
    return DG_OK;
}

int dg_select_config(int kind, int M, int N, int K, int num_groups, int expected_m, int num_sms,
                     dg_config *out)
{
    if (!out || kind < 0 || kind > 3 || M <= 0 || N <= 0 || K <= 0 || num_groups <= 0)
        return DG_ERR_INVALID_ARGUMENT;
    if (K % 128 != 0 || N % 8 != 0)
        return DG_ERR_UNSUPPORTED_SHAPE;
    if (kind == DG_KIND_MASKED && num_groups > MAX_MASKED_GROUPS)
        return DG_ERR_UNSUPPORTED_SHAPE;
    const int limit = g_num_sms_limit.load(std::memory_order_relaxed);
    int sms = num_sms > 0 ? num_sms : (limit > 0 ? limit : kDefaultSms);
    const bool one_group = kind == DG_KIND_DENSE || kind == DG_KIND_DENSE_PER_TENSOR;
    Problem pb{kind, M, N, K, one_group ? 1 : num_groups, expected_m};
    if (use_skinny(pb)) {
        SkinnyChoice ch;
        const int st = choose_skinny(pb, sms, kDefaultMaxSmem, nullptr, &ch);
        if (st != DG_OK)
            return st;
        skinny_config(ch, out);
        const int cap = cluster_capacity_model(ch.plan.split, sms);
        const int by_sms = sms / ch.plan.split > 0 ? sms / ch.plan.split : 1;
        int clusters = ch.plan.tiles < cap ? ch.plan.tiles : cap;
        clusters = clusters < by_sms ? clusters : by_sms;
        out->grid = clusters * ch.plan.split;
        return DG_OK;
    }
    const Candidate *cand = nullptr;
    SmemPlan plan;
    const int st = choose(pb, sms, kDefaultMaxSmem, &cand, out, &plan);
    if (st != DG_OK)
        return st;
    out->swap_ab = 0;
    out->tail_tiles = 0;
    TailSplit tail;
    if (plan_tail(pb, *out, sms, kDefaultMaxSmem, nullptr, &tail))
        out->tail_tiles = out->num_tiles - tail.main_tiles;
    return DG_OK;
}

int dg_force_config(int block_m, int block_n, int split, int cta_pair)
{
    if (split < 0 || split > kMaxSplit)
        return DG_ERR_UNSUPPORTED_SHAPE;
    if (cta_pair < 0 || cta_pair > 2)
        return DG_ERR_UNSUPPORTED_SHAPE;
    if (block_m == 0 && block_n == 0) {
        g_forced.store(pack_forced(0, 0, split, cta_pair), std::memory_order_relaxed);
        return DG_OK;
    }
    for (int i = 0; i < kNumCandidates; ++i) {
        const Candidate &c = kCandidates[i];
        if ((c.pair ? 256 : c.mw * 128) == block_m && c.bn == block_n &&
            (cta_pair == 0 || (cta_pair == 2) == (c.pair != 0))) {
            g_forced.store(pack_forced(block_m, block_n, split, cta_pair), std::memory_order_relaxed);
            return DG_OK;
        }
    }
    return DG_ERR_UNSUPPORTED_SHAPE;
}

int dg_force_swap_ab(int mode)
{
    if (mode < 0 || mode > 2)
        return DG_ERR_INVALID_ARGUMENT;
    g_forced_swap.store(mode, std::memory_order_relaxed);
    return DG_OK;
}

int dg_force_tail_split(int mode)
{
    if (mode < 0 || mode > 3)
        return DG_ERR_INVALID_ARGUMENT;
    g_forced_tail.store(mode, std::memory_order_relaxed);
    return DG_OK;
}

} // extern "C"
