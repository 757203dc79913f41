// One (MW, BN) instantiation of the GEMM kernel and its launcher; the build
// compiles this file once per entry of kernels.def with -DFP8NT_MW / -DFP8NT_BN.
#include <cuda_runtime.h>

#include "kernel.cuh"
#include "launch.h"

#ifndef FP8NT_MW
#error "FP8NT_MW must be defined"
#endif
#ifndef FP8NT_BN
#error "FP8NT_BN must be defined"
#endif

namespace fp8nt {

#define FP8NT_CAT_(a, b, c) launch_mw##a##_bn##b##c
#define FP8NT_NAME(a, b) FP8NT_CAT_(a, b, )

cudaError_t FP8NT_NAME(FP8NT_MW, FP8NT_BN)(const LaunchArgs &args)
{
    auto kernel = fp8_gemm_kernel<FP8NT_MW, FP8NT_BN>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           args.smem_bytes);
    if (err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)args.grid, 1, 1);
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
    return cudaLaunchKernelEx(&cfg, kernel, *args.tmap_a, *args.tmap_b, *args.params);
}

} // namespace fp8nt
