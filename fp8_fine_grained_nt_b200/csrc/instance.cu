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
    kernel<<<args.grid, NUM_THREADS, args.smem_bytes, args.stream>>>(*args.tmap_a, *args.tmap_b,
                                                                     *args.params);
    return cudaGetLastError();
}

} // namespace fp8nt
