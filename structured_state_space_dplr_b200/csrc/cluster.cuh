// cluster.cuh -- what the cluster kernels share: the two halves of the
// cluster barrier (device), and the host-side launch helpers that opt a
// kernel into its shared memory, count the co-resident CTAs or clusters and
// launch with a cluster dimension.
#pragma once
#include <atomic>
#include <cstddef>

#include <cuda_runtime.h>

namespace s4 {

// cluster barrier halves: release/acquire hand off shared-memory data between
// the CTAs; a relaxed arrive only says "I am done reading your memory" (every
// value read was consumed before the arrive issues)
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory"); }

// ------------------------------------------------------------ host helpers --
inline int device_sms(int dev) {
    static std::atomic<int> cache[64];
    int v = cache[dev & 63].load(std::memory_order_relaxed);
    if (v == 0) {
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        cache[dev & 63].store(v, std::memory_order_relaxed);
    }
    return v;
}

// Per-instantiation, per-device launch facts: smem opt-in done, how many
// clusters (or CTAs) are co-resident.
struct LaunchInfo {
    std::atomic<int> resident[64];
};

template <class Kern>
inline cudaError_t resident_units(Kern kern, LaunchInfo &info, int C, int T, size_t smem, int *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int v = info.resident[dev & 63].load(std::memory_order_relaxed);
    if (v == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (C > 8) {   // clusters beyond the portable size of 8 are opted into per kernel
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
        }
        if (C > 1) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = C; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(C * 1024); cfg.blockDim = dim3(T); cfg.dynamicSmemBytes = smem;
            cfg.attrs = at; cfg.numAttrs = 1;
            e = cudaOccupancyMaxActiveClusters(&v, (void *)kern, &cfg);
            if (e != cudaSuccess) return e;
        } else {
            int per_sm = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, T, smem);
            if (e != cudaSuccess) return e;
            v = per_sm * device_sms(dev);
        }
        if (v <= 0) return cudaErrorInvalidConfiguration;
        info.resident[dev & 63].store(v, std::memory_order_relaxed);
    }
    *out = v;
    return cudaSuccess;
}

template <class Kern, class... Args>
inline cudaError_t launch_clustered(Kern kern, int C, int nclusters, int T, size_t smem, cudaStream_t st,
                             Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.gridDim = dim3(C * nclusters);
    cfg.blockDim = dim3(T);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    if (C > 1) {
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = C; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace s4
