// launch.cuh -- the launchers each kernel instantiation exports to the host code.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>

#include "gemm_kernel.cuh"

namespace fg8 {

// Largest shared memory (static + dynamic) a CTA may use on sm_100 (227 KiB).
constexpr int kMaxDynamicSmem = 232448;
// Static shared memory of the GEMM kernel (the promotion warps' tile
// schedulers), reserved out of kMaxDynamicSmem when the stages are sized.
constexpr int kGemmStaticSmem = 1024;
static_assert(NUM_EPI_WARPS * sizeof(TileScheduler<true>) <= kGemmStaticSmem, "static shared memory");

// Programmatic dependent launch: a GEMM launched right after another kernel
// in the same stream may start its prologue (barrier set-up, TMEM allocation)
// while that kernel finishes; the kernels wait (griddepcontrol.wait) before
// touching global memory.  FG_PDL=0 turns it off.
inline bool pdl_enabled() {
    const char* env = std::getenv("FG_PDL");
    return !(env && std::atoi(env) == 0);
}

// Launches fg8_gemm_kernel<BN, PAIR> on `grid` CTAs (PAIR: clusters of two;
// otherwise clusters of `cluster` CTAs when cluster > 1, for the cluster
// split-K mode, whose grid the host has checked to be resident at once).
// On first use per device it checks the build's register count (the in-kernel
// register split is safe only at exactly REGS_LAUNCH) and raises the kernel's
// shared-memory limit.  Defined in gemm_inst.cu, one block width per object.
template <int BN, bool PAIR>
cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD, const GemmParams& p,
                        int grid, size_t smem_bytes, cudaStream_t stream, int cluster);

template <int BN, bool PAIR>
cudaError_t launch_gemm_impl(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,
                             const GemmParams& p, int grid, size_t smem_bytes, cudaStream_t stream, int cluster) {
    static std::atomic<unsigned long long> attr_set{0};
    static std::atomic<int> max_clusters[64];   // per device, 0 = not queried yet
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    auto kernel = fg8_gemm_kernel<BN, PAIR>;
    if (!(attr_set.load() & bit)) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != REGS_LAUNCH) return cudaErrorInvalidDeviceFunction;
        if (fa.sharedSizeBytes > static_cast<size_t>(kGemmStaticSmem)) return cudaErrorInvalidDeviceFunction;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxDynamicSmem - static_cast<int>(fa.sharedSizeBytes));
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit);
    }
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
    if (PAIR) {
        attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
        attr[cfg.numAttrs].val.clusterDim.x = 2;
        attr[cfg.numAttrs].val.clusterDim.y = 1;
        attr[cfg.numAttrs].val.clusterDim.z = 1;
        ++cfg.numAttrs;
        // A persistent grid must fit on the device at once: clusters that do not
        // would start only after others finish.  Query (once per device, at the
        // largest shared-memory size, which all launches stay within) how many
        // CTA pairs can be resident.
        int mc = max_clusters[dev & 63].load();
        if (mc == 0) {
            cudaLaunchConfig_t q = cfg;
            q.attrs = &attr[cfg.numAttrs - 1];   // the cluster dimension only
            q.numAttrs = 1;
            q.dynamicSmemBytes = kMaxDynamicSmem - kGemmStaticSmem;
            e = cudaOccupancyMaxActiveClusters(&mc, kernel, &q);
            if (e != cudaSuccess) return e;
            if (mc <= 0) return cudaErrorInvalidConfiguration;
            max_clusters[dev & 63].store(mc);
        }
        if (grid > 2 * mc) cfg.gridDim.x = static_cast<unsigned>(2 * mc);
    } else if (cluster > 1) {
        if (cluster > 8) return cudaErrorInvalidConfiguration;
        attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
        attr[cfg.numAttrs].val.clusterDim.x = static_cast<unsigned>(cluster);
        attr[cfg.numAttrs].val.clusterDim.y = 1;
        attr[cfg.numAttrs].val.clusterDim.z = 1;
        ++cfg.numAttrs;
        // The host sized the grid from gemm_max_split_clusters (whole grid resident).
        if (grid % cluster != 0) return cudaErrorInvalidConfiguration;
    }
    return cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmD, p);
}

// Largest number of clusters of `cluster` single CTAs of fg8_gemm_kernel<BN,
// false> that can be resident at once (cluster split-K sizing).
template <int BN>
cudaError_t gemm_max_split_clusters(int cluster, int* out);

template <int BN>
cudaError_t gemm_max_split_clusters_impl(int cluster, int* out) {
    auto kernel = fg8_gemm_kernel<BN, false>;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMaxDynamicSmem - static_cast<int>(fa.sharedSizeBytes));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cluster), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = kMaxDynamicSmem - kGemmStaticSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(out, kernel, &cfg);
}

#define FG8_DEFINE_LAUNCH_ONE(BN, PAIR)                                                                        \
    template <>                                                                                                \
    cudaError_t launch_gemm<BN, PAIR>(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,  \
                                      const GemmParams& p, int grid, size_t smem_bytes, cudaStream_t stream,   \
                                      int cluster) {                                                           \
        return launch_gemm_impl<BN, PAIR>(tmA, tmB, tmD, p, grid, smem_bytes, stream, cluster);                \
    }

#define FG8_DECLARE_LAUNCH_ONE(BN, PAIR)                                                                       \
    template <>                                                                                                \
    cudaError_t launch_gemm<BN, PAIR>(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmD,  \
                                      const GemmParams& p, int grid, size_t smem_bytes, cudaStream_t stream,   \
                                      int cluster);

// Block widths 16..256; CTA pairs from 32 (each CTA loads at least 16 B rows).
#define FG8_FOR_EACH_BN(X) \
    X(16) X(32) X(48) X(64) X(80) X(96) X(112) X(128) X(144) X(160) X(176) X(192) X(208) X(224) X(240) X(256)

}  // namespace fg8
