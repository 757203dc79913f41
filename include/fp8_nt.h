/*
 * fp8_nt.h — C ABI of libfp8nt.so: FP8 (E4M3) NT GEMM with fine-grained
 * scaling and BF16 output, for NVIDIA B200 (sm_100a).
 *
 * What is computed (DeepGEMM README, introduction: FP8 GEMMs "with
 * fine-grained scaling" as proposed in DeepSeek-V3; usage: NT format only):
 *
 *   D[m,n] = sum over 128-wide K blocks kb of
 *              ( sum_{k in kb} A[m,k] * B[n,k] ) * sa[m,kb] * sb[n/128,kb]
 *
 * accumulated in FP32 (each K block's tensor-core partial is promoted into an
 * FP32 accumulator with its scale product: the README's two-level
 * accumulation) and rounded to BF16 (round-to-nearest-even) on store.
 *
 * Common conventions for the three GEMM entry points
 * ---------------------------------------------------
 * Pointers.  Every pointer is CUDA device memory owned by the caller.  The
 *   library never allocates, frees or keeps a reference to it after the call
 *   returns; it reads A, sa, B, sb (and m_indices / masked_m) and writes D.
 *   Every pointer must be 16-byte aligned (except the two single-value
 *   scales of gemm_fp8_fp8_bf16_nt_per_tensor: 4-byte aligned).
 * Element types.  A and B hold E4M3 bytes (1 sign, 4 exponent bits with bias
 *   7, 3 mantissa bits; 0x7F/0xFF are NaN).  sa and sb are IEEE FP32.  D is
 *   BF16 (stored as uint16).
 * Layouts.  "NT": A is [M,K] row-major (K contiguous) and B is [N,K] row-major
 *   (K contiguous) (DeepGEMM README, usage).  sa is COLUMN-MAJOR and
 *   TMA-aligned: sa[kb * ld + m] with ld = get_tma_aligned_size(M, 4)
 *   (README, utility functions: get_tma_aligned_size,
 *   get_col_major_tma_aligned_tensor).  sb is row-major [ceil(N/128)][K/128].
 *   D is row-major [M,N] BF16.
 * Shape rules.  K % 128 == 0 (the scale block), N % 8 == 0 (16-byte rows of
 *   D), M >= 0.  A call with M == 0 (or all groups empty) does nothing.
 * Stream.  Work is enqueued on `stream` (a cudaStream_t / CUstream; NULL = the
 *   legacy default stream) and runs asynchronously.  No call synchronises,
 *   allocates or reads device memory on the host, so every call can be
 *   captured in a CUDA graph.
 * Errors.  Arguments the host can check are checked before anything is
 *   launched; the call then returns a nonzero dg_status and enqueues nothing.
 *   Errors the host cannot see (a masked_m or m_indices value out of range, a
 *   pipeline wait that timed out) are recorded in a device status word,
 *   read and cleared by dg_get_device_status().  The kernel never traps.
 */
#ifndef FP8_NT_H
#define FP8_NT_H

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dg_stream_t; /* same type as cudaStream_t */

typedef enum dg_status {
    DG_OK = 0,
    DG_ERR_INVALID_ARGUMENT = 1,  /* null pointer, negative size, bad count */
    DG_ERR_MISALIGNED = 2,        /* a pointer not 16-byte aligned */
    DG_ERR_UNSUPPORTED_SHAPE = 3, /* K % 128, N % 8, or a size over a limit */
    DG_ERR_UNSUPPORTED_ARCH = 4,  /* current device is not sm_100 */
    DG_ERR_CUDA = 5,              /* a CUDA runtime/driver call failed */
    DG_ERR_DEVICE_TIMEOUT = 6,    /* device: a pipeline wait ran out (kernel exited early) */
    DG_ERR_DEVICE_BAD_INDEX = 7   /* device: masked_m / m_indices out of range */
} dg_status;

/* Dense GEMM (DeepGEMM README, usage: deep_gemm.gemm_fp8_fp8_bf16_nt, the
 * basic non-grouped FP8 GEMM).
 *   A  [M,K] E4M3          sa [K/128][get_tma_aligned_size(M,4)] FP32
 *   B  [N,K] E4M3          sb [ceil(N/128)][K/128] FP32
 *   D  [M,N] BF16 (written in full) */
int gemm_fp8_fp8_bf16_nt(const void *A, const float *sa, const void *B, const float *sb,
                         void *D, int M, int N, int K, dg_stream_t stream);

/* Dense GEMM with per-tensor scaling (the tensor-wise FP8 recipe that the
 * FP8-training blog page contrasts with fine-grained scaling, section 4.2):
 *   D[m,n] = scale_a * scale_b * sum_k A[m,k] * B[n,k]
 * accumulated in FP32 over the whole K range in tensor memory (no per-block
 * promotion is needed when every block has the same scale) and rounded to
 * BF16 (RNE).  scale_a and scale_b point to ONE FP32 value each, in device
 * memory (read by the kernel, so a CUDA graph can update them), 4-byte
 * aligned (an element of a larger scales tensor is fine).  A, B, D and
 * the shape rules are as for gemm_fp8_fp8_bf16_nt. */
int gemm_fp8_fp8_bf16_nt_per_tensor(const void *A, const float *scale_a, const void *B,
                                    const float *scale_b, void *D, int M, int N, int K,
                                    dg_stream_t stream);

/* Contiguous m-grouped GEMM (DeepGEMM README, grouped GEMMs: tokens of all
 * experts concatenated into one tensor, each expert segment aligned to
 * get_m_alignment_for_contiguous_layout(); only the M axis is grouped, all
 * experts share N and K).
 *   A  [M_sum,K] E4M3       sa [K/128][M_sum] FP32 (M_sum is a multiple of the
 *                                                  alignment, so ld = M_sum)
 *   B  [num_groups,N,K]     sb [num_groups][ceil(N/128)][K/128]
 *   D  [M_sum,N] BF16
 *   m_indices [M_sum] int32 on the device: the expert of each row, or -1 on a
 *   padding row.  Each aligned block of rows takes the expert of its first
 *   row; all non-padding rows of a block must share it.  Rows marked -1 are
 *   not written; a block whose first row is -1 is skipped.  An expert index
 *   >= num_groups sets DG_ERR_DEVICE_BAD_INDEX and its block is skipped.
 *   M_sum % get_m_alignment_for_contiguous_layout() must be 0. */
int m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(const void *A, const float *sa, const void *B,
                                              const float *sb, void *D, const int *m_indices,
                                              int num_groups, int M_sum, int N, int K,
                                              dg_stream_t stream);

/* Masked m-grouped GEMM (DeepGEMM README, grouped GEMMs: for CUDA-graph
 * decode, when the host does not know how many tokens each expert got; the
 * kernel computes only the valid part given by a mask tensor).
 *   A  [G,M_max,K] E4M3      sa [G][K/128][get_tma_aligned_size(M_max,4)]
 *   B  [G,N,K]               sb [G][ceil(N/128)][K/128]
 *   D  [G,M_max,N] BF16
 *   masked_m [G] int32 on the device: rows 0..masked_m[g]-1 of group g are
 *   computed; rows at or beyond masked_m[g] are never written.  The host never
 *   reads masked_m.  A value outside [0, M_max] sets DG_ERR_DEVICE_BAD_INDEX
 *   and is clamped into range.
 *   expected_m: the caller's estimate of a typical masked_m (a hint for the
 *   tile choice only; 0 = assume M_max). */
int m_grouped_gemm_fp8_fp8_bf16_nt_masked(const void *A, const float *sa, const void *B,
                                          const float *sb, void *D, const int *masked_m, int G,
                                          int M_max, int N, int K, int expected_m,
                                          dg_stream_t stream);

/* 1x128 activation quantiser: the cast and LHS-scale transposition that the
 * DeepGEMM README (usage) leaves to a kernel before the GEMM; 1x128 tiles as
 * in the DeepSeek-V3 recipe cited above.  For each row m and 128-wide K block
 * kb of x [M,K] (row-major; FP32 or BF16 by x_dtype):
 *   s = max(max_k |x[m,k]|, 1e-4) / 448              (FP32, IEEE division)
 *   q[m,k] = E4M3(clamp(x[m,k] / s, -448, 448))      (IEEE division, then
 *                                                      round to nearest even)
 * q is [M,K] E4M3 bytes (row-major); s goes to sa[kb * ld + m] with
 * ld = get_tma_aligned_size(M, 4): the column-major layout every GEMM entry
 * point reads (columns M..ld-1 are not written).  x must be finite.
 * K % 128 == 0; pointers 16-byte aligned device memory owned by the caller;
 * M == 0 does nothing. */
enum { DG_INPUT_F32 = 0, DG_INPUT_BF16 = 1 };
int quantize_fp8_1x128(const void *x, int x_dtype, void *q, float *sa, int M, int K,
                       dg_stream_t stream);

/* Row alignment of each expert segment in the contiguous layout (DeepGEMM
 * README, utility functions: get_m_alignment_for_contiguous_layout).  128. */
int get_m_alignment_for_contiguous_layout(void);

/* Smallest count >= x whose size in bytes (x * element_size) is a multiple of
 * 16: the TMA-aligned leading dimension (DeepGEMM README, utility functions:
 * get_tma_aligned_size).  element_size must divide 16; returns
 * -DG_ERR_INVALID_ARGUMENT otherwise or if x < 0. */
int get_tma_aligned_size(int x, int element_size);

/* Upper bound on the SMs the kernels use (DeepGEMM README, utility
 * functions: set_num_sms / get_num_sms).  n <= 0 restores "all SMs of the
 * current device".  Returns DG_OK.  get_num_sms() returns the bound in force
 * (the device's SM count when unset and a device is present, else 0). */
int set_num_sms(int n);
int get_num_sms(void);

/* Self-test of the device-side error path (no counterpart in the pages): one
 * thread waits, with the bounded mbarrier wait every pipeline role uses, on a
 * barrier nothing arrives on.  After timeout_us microseconds (1..10^7) the
 * wait gives up and records DG_ERR_DEVICE_TIMEOUT in the device status word,
 * which dg_get_device_status() then returns; the kernel ends by itself and
 * the context stays usable.  Returns DG_OK once the kernel is enqueued. */
int dg_selftest_wait_timeout(int timeout_us, dg_stream_t stream);

/* Static description of a dg_status value. */
const char *dg_status_string(int status);

/* Reads and clears the device status word in one atomic exchange, enqueued
 * on `stream` (so it follows the work enqueued there), synchronises `stream`
 * and returns what it read: DG_OK, DG_ERR_DEVICE_TIMEOUT or
 * DG_ERR_DEVICE_BAD_INDEX; DG_ERR_CUDA if the launch or the synchronisation
 * failed.  A bit set meanwhile by a kernel on another stream is reported by
 * this call or by the next one, never dropped.  Host threads calling it take
 * turns. */
int dg_get_device_status(dg_stream_t stream);

/* Tile configuration chosen for a call (host logic; no GPU needed). */
typedef struct dg_config {
    int block_m;    /* rows per tile: 128, or 256 (two 128-row MMAs in one CTA,
                       or one 256-row MMA over a CTA pair) */
    int block_n;    /* columns per CTA tile: a multiple of 16 in [16, 256] */
    int stages;     /* depth of the shared-memory operand ring */
    int num_tiles;  /* tiles to compute (upper bound for the masked form) */
    int grid;       /* persistent CTAs launched */
    int smem_bytes; /* dynamic shared memory per CTA */
    int tmem_cols;  /* tensor-memory columns allocated per CTA */
    int split;      /* split-K: CTAs (one thread-block cluster) sharing a tile; 1 = none */
    int cta_pair;   /* 2: a cluster of two CTAs computes each 256-row tile with
                       tcgen05 cta_group::2 MMAs (each CTA loads its own 128 rows
                       of A and half of the B tile); 1: one CTA per tile */
    int swap_ab;    /* 1: the small-M dense kernel (M <= 256): each tile is
                       128 rows of B (block_n = 128 columns of D) against up to
                       block_m rows of A (zero-padded; M > 128 in blocks of 128
                       rows), computed as D^T with B in the MMA's 128-row slot;
                       split CTAs of a cluster share the tile's K range and
                       reduce through distributed shared memory.  0: the
                       kernels described above. */
    int tail_tiles; /* dense calls on the kernels above, when requested with
                       dg_force_tail_split: tiles of the last, partly filled
                       wave that form one block of D (the last M block from a
                       128-column boundary on) and are computed by the small-M
                       kernel after the main kernel, which then runs whole
                       waves (num_tiles - tail_tiles tiles); 0 = none */
} dg_config;

enum { DG_KIND_DENSE = 0, DG_KIND_CONTIGUOUS = 1, DG_KIND_MASKED = 2, DG_KIND_DENSE_PER_TENSOR = 3 };

/* The configuration a call of `kind` would use.  For DG_KIND_DENSE: M, N, K;
 * for DG_KIND_CONTIGUOUS: M = M_sum; for DG_KIND_MASKED: M = M_max and
 * expected_m as in the masked call.  num_sms <= 0 means the bound from
 * set_num_sms, else 148.  The selection is deterministic (DeepGEMM README, JIT
 * design: block sizes and pipeline stages chosen without auto-tuning) and
 * favours tile counts that fill the SMs, with non-power-of-two BLOCK_N where
 * that helps (README, unaligned block sizes).  Returns DG_OK or an argument
 * error. */
int dg_select_config(int kind, int M, int N, int K, int num_groups, int expected_m,
                     int num_sms, dg_config *out);

/* Test hook: pin block_m / block_n, the split-K factor and the CTA-pair mode
 * for later calls (0, 0 restores automatic tile choice; split 0 = automatic,
 * 1 = no split, 2..8 = that many CTAs per tile, used only where split-K
 * applies: 2, 4 or 8 for the kernels with 128- or 256-row tiles, any of 1..8
 * for the small-M kernel; cta_pair 0 = automatic, 1 = one CTA per tile,
 * 2 = CTA pairs).  block_m / block_n pin the tile of the kernels other than
 * the small-M one.  Returns DG_ERR_UNSUPPORTED_SHAPE if no kernel of that
 * shape is built, the split is outside 0..8, or cta_pair is not 0, 1 or 2. */
int dg_force_config(int block_m, int block_n, int split, int cta_pair);

/* Test hook: 0 = automatic (dense calls with M <= 256 use the small-M kernel
 * of dg_config.swap_ab), 1 = never use it, 2 = use it wherever it applies.
 * Returns DG_OK, or DG_ERR_INVALID_ARGUMENT for another mode. */
int dg_force_swap_ab(int mode);

/* Opt-in split of a dense call's last partial wave (dg_config.tail_tiles):
 * 0 = automatic, which is off (measured on B200 no faster than the partial
 * wave), 1 = never, 2 = wherever the block layout allows it, 3 = where the
 * block layout allows it and the cycle estimate favours it.  Returns DG_OK,
 * or DG_ERR_INVALID_ARGUMENT for another mode. */
int dg_force_tail_split(int mode);

#ifdef __cplusplus
}
#endif

#endif /* FP8_NT_H */
