// decode_launch.cuh -- launcher of the decode kernel (one per token-tile width).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>

#include "decode_kernel.cuh"
#include "launch.cuh"

namespace fg8 {

// Launches fg8_decode_kernel<MT> on `grid` CTAs; cluster > 1 groups the CTAs
// in clusters of that many (the splits of one tile, reduced through DSMEM).
template <int MT>
cudaError_t launch_decode(const CUtensorMap& tmA, const CUtensorMap& tmB, const DecodeParams& p, int grid,
                          int cluster, size_t smem_bytes, cudaStream_t stream);

// How many clusters of `cluster` CTAs of fg8_decode_kernel<MT>, each with
// `smem_bytes` of dynamic shared memory, can be resident on the current device.
template <int MT>
cudaError_t decode_max_clusters(int cluster, size_t smem_bytes, int* out);

template <int MT>
cudaError_t prepare_decode_kernel() {
    static std::atomic<unsigned long long> attr_set{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (attr_set.load() & bit) return cudaSuccess;
    auto kernel = fg8_decode_kernel<MT>;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != REGS_LAUNCH) return cudaErrorInvalidDeviceFunction;   // register split safety
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynamicSmem);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
    return cudaSuccess;
}

template <int MT>
cudaError_t decode_max_clusters_impl(int cluster, size_t smem_bytes, int* out) {
    cudaError_t e = prepare_decode_kernel<MT>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cluster), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(out, fg8_decode_kernel<MT>, &cfg);
}

template <int MT>
cudaError_t launch_decode_impl(const CUtensorMap& tmA, const CUtensorMap& tmB, const DecodeParams& p, int grid,
                               int cluster, size_t smem_bytes, cudaStream_t stream) {
    cudaError_t e = prepare_decode_kernel<MT>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (pdl_enabled()) {
        attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
        ++cfg.numAttrs;
    }
    if (cluster > 1) {
        attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
        attr[cfg.numAttrs].val.clusterDim.x = static_cast<unsigned>(cluster);
        attr[cfg.numAttrs].val.clusterDim.y = 1;
        attr[cfg.numAttrs].val.clusterDim.z = 1;
        ++cfg.numAttrs;
    }
    return cudaLaunchKernelEx(&cfg, fg8_decode_kernel<MT>, tmA, tmB, p);
}

#define FG8_DEFINE_DECODE_LAUNCH(MT)                                                                          \
    template <>                                                                                               \
    cudaError_t launch_decode<MT>(const CUtensorMap& tmA, const CUtensorMap& tmB, const DecodeParams& p,      \
                                  int grid, int cluster, size_t smem_bytes, cudaStream_t stream) {            \
        return launch_decode_impl<MT>(tmA, tmB, p, grid, cluster, smem_bytes, stream);                        \
    }                                                                                                         \
    template <>                                                                                               \
    cudaError_t decode_max_clusters<MT>(int cluster, size_t smem_bytes, int* out) {                           \
        return decode_max_clusters_impl<MT>(cluster, smem_bytes, out);                                        \
    }

#define FG8_DECLARE_DECODE_LAUNCH(MT)                                                                         \
    template <>                                                                                               \
    cudaError_t launch_decode<MT>(const CUtensorMap& tmA, const CUtensorMap& tmB, const DecodeParams& p,      \
                                  int grid, int cluster, size_t smem_bytes, cudaStream_t stream);             \
    template <>                                                                                               \
    cudaError_t decode_max_clusters<MT>(int cluster, size_t smem_bytes, int* out);

#define FG8_FOR_EACH_MT(X) X(32) X(64) X(96) X(128) X(160) X(192) X(224) X(256)

}  // namespace fg8
