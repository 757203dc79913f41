// One (MW, BN, PAIR, SCALAR) instantiation of the GEMM kernel and its
// launcher; the build compiles this file once per entry of kernels.def with
// -DFP8NT_MW, -DFP8NT_BN, -DFP8NT_PAIR and -DFP8NT_SCALAR.
#include <cuda_runtime.h>

#include <atomic>

#include "kernel.cuh"
#include "launch.h"

#ifndef FP8NT_MW
#error "FP8NT_MW must be defined"
#endif
#ifndef FP8NT_BN
#error "FP8NT_BN must be defined"
#endif
#ifndef FP8NT_PAIR
#error "FP8NT_PAIR must be defined"
#endif
#ifndef FP8NT_SCALAR
#error "FP8NT_SCALAR must be defined"
#endif

namespace fp8nt {

#define FP8NT_CAT_(a, b, c, d) launch_mw##a##_bn##b##_p##c##_s##d
#define FP8NT_NAME(a, b, c, d) FP8NT_CAT_(a, b, c, d)

cudaError_t FP8NT_NAME(FP8NT_MW, FP8NT_BN, FP8NT_PAIR, FP8NT_SCALAR)(const LaunchArgs &args)
{
    auto kernel = fp8_gemm_kernel<FP8NT_MW, FP8NT_BN, FP8NT_PAIR != 0, FP8NT_SCALAR != 0>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    // The dynamic shared-memory limit is raised once per device to the
    // largest size requested so far (a per-call attribute update costs host
    // time on every launch).
    static std::atomic<int> smem_limit[64];
    if (smem_limit[dev].load(std::memory_order_acquire) < args.smem_bytes) {
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               args.smem_bytes);
        if (err != cudaSuccess)
            return err;
        int seen = smem_limit[dev].load(std::memory_order_relaxed);
        while (seen < args.smem_bytes &&
               !smem_limit[dev].compare_exchange_weak(seen, args.smem_bytes)) {
        }
    }
    cudaLaunchConfig_t cfg = {};
    int grid = args.grid;
    if (FP8NT_PAIR && args.cluster == 2) {
        // persistent pairs: no more than can be resident at once (a GPC with
        // an odd number of free SMs holds one CTA fewer than a naive count)
        static std::atomic<int> max_pairs[64];
        if (max_pairs[dev].load(std::memory_order_relaxed) == 0) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3((unsigned)args.grid, 1, 1);
            q.blockDim = dim3(NUM_THREADS, 1, 1);
            q.dynamicSmemBytes = (size_t)args.smem_bytes;
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = 2;
            qa[0].val.clusterDim.y = 1;
            qa[0].val.clusterDim.z = 1;
            q.attrs = qa;
            q.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kernel, &q) != cudaSuccess || n < 1) {
                cudaGetLastError();
                n = 1 << 30; // unknown: keep the host's choice
            }
            max_pairs[dev] = n;
        }
        if (grid > 2 * max_pairs[dev])
            grid = 2 * max_pairs[dev];
    }
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)args.smem_bytes;
    cfg.stream = args.stream;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (args.cluster > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)args.cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kernel, *args.tmap_a, *args.tmap_b, *args.tmap_sa, *args.tmap_d,
                              *args.params);
}

} // namespace fp8nt
