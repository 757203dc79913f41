// Host-side launch interface between the C-ABI layer and the kernel
// instantiations (one launcher per tile shape listed in kernels.def).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "params.h"

namespace fp8nt {

struct LaunchArgs {
    const CUtensorMap *tmap_a;
    const CUtensorMap *tmap_b;
    const CUtensorMap *tmap_sa;
    const CUtensorMap *tmap_d;
    const Params *params;
    int grid;
    int cluster; // CTAs per cluster (split-K, or 2 for a CTA pair), 1 = no cluster
    int smem_bytes;
    cudaStream_t stream;
};

typedef cudaError_t (*LaunchFn)(const LaunchArgs &);

// Bounded-wait self-test (csrc/selftest.cu).
cudaError_t launch_wait_timeout_selftest(unsigned int *status, unsigned long long timeout_ns,
                                         cudaStream_t stream);

// 1x128 activation quantiser (csrc/quantize.cu).
cudaError_t launch_quantize_1x128(const void *x, bool bf16_in, uint8_t *q, float *sa, int M, int K,
                                  long ld_sa, cudaStream_t stream);

// Small-M dense kernel (csrc/kernel_skinny.cuh): grid (split, n_tiles), one
// cluster of `split` CTAs per 128-column tile of D.
struct SkinnyLaunchArgs {
    const CUtensorMap *tmap_a;
    const CUtensorMap *tmap_b;
    const SkinnyParams *params;
    int split;
    int n_tiles;
    int smem_bytes;
    cudaStream_t stream;
};

typedef cudaError_t (*SkinnyLaunchFn)(const SkinnyLaunchArgs &);
// Clusters of `split` CTAs with `smem_bytes` each that the current device can
// hold at once (cudaOccupancyMaxActiveClusters), or -1 if the query failed.
typedef int (*SkinnyCapacityFn)(int split, int smem_bytes);

#define FP8NT_SKINNY(mn)                                                                          \
    cudaError_t launch_skinny_mn##mn(const SkinnyLaunchArgs &);                                   \
    int skinny_capacity_mn##mn(int split, int smem_bytes);
#include "skinny.def"
#undef FP8NT_SKINNY

#define FP8NT_KERNEL(mw, bn, pair, scalar)                                                    \
    cudaError_t launch_mw##mw##_bn##bn##_p##pair##_s##scalar(const LaunchArgs &);
#include "kernels.def"
#undef FP8NT_KERNEL

} // namespace fp8nt
