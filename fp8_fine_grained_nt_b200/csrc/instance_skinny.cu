// One MN instantiation of the small-M dense kernel and its launcher; the build
// compiles this file once per entry of skinny.def with -DFP8NT_SKINNY_MN.
#include <cuda_runtime.h>

#include <atomic>

#include "kernel_skinny.cuh"
#include "launch.h"

#ifndef FP8NT_SKINNY_MN
#error "FP8NT_SKINNY_MN must be defined"
#endif

namespace fp8nt {

#define FP8NT_SK_CAT_(a, b) a##b
#define FP8NT_SK_NAME(a, b) FP8NT_SK_CAT_(a, b)

namespace {

// The dynamic shared-memory limit is raised once per device to the largest
// size requested so far (a per-call attribute update costs host time).
cudaError_t ensure_smem(int smem_bytes)
{
    auto kernel = fp8_gemm_skinny_kernel<FP8NT_SKINNY_MN>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    static std::atomic<int> smem_limit[64];
    if (smem_limit[dev].load(std::memory_order_acquire) < smem_bytes) {
        cudaError_t err =
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
        if (err != cudaSuccess)
            return err;
        int seen = smem_limit[dev].load(std::memory_order_relaxed);
        while (seen < smem_bytes && !smem_limit[dev].compare_exchange_weak(seen, smem_bytes)) {
        }
    }
    return cudaSuccess;
}

} // namespace

cudaError_t FP8NT_SK_NAME(launch_skinny_mn, FP8NT_SKINNY_MN)(const SkinnyLaunchArgs &args)
{
    cudaError_t err = ensure_smem(args.smem_bytes);
    if (err != cudaSuccess)
        return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)args.split, (unsigned)args.n_tiles, 1);
    cfg.blockDim = dim3(SkinnyTraits<FP8NT_SKINNY_MN>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)args.smem_bytes;
    cfg.stream = args.stream;
    cudaLaunchAttribute attr[2];
    cfg.attrs = attr;
    // programmatic dependent launch: the kernel's set-up may overlap the
    // previous kernel in the stream (it waits for that kernel before touching
    // global memory)
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (args.split > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)args.split;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, fp8_gemm_skinny_kernel<FP8NT_SKINNY_MN>, *args.tmap_a, *args.tmap_b,
                              *args.params);
}

int FP8NT_SK_NAME(skinny_capacity_mn, FP8NT_SKINNY_MN)(int split, int smem_bytes)
{
    if (ensure_smem(smem_bytes) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3((unsigned)(split > 0 ? split : 1), 1, 1);
    q.blockDim = dim3(SkinnyTraits<FP8NT_SKINNY_MN>::THREADS, 1, 1);
    q.dynamicSmemBytes = (size_t)smem_bytes;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = (unsigned)(split > 0 ? split : 1);
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fp8_gemm_skinny_kernel<FP8NT_SKINNY_MN>, &q) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return n;
}

} // namespace fp8nt
