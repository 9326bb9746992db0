// launch.cuh -- the launcher each kernel instantiation exports to the host code.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>

#include "gemm_kernel.cuh"

namespace fg8 {

// Largest dynamic shared memory a CTA may request on sm_100 (227 KiB).
constexpr int kMaxDynamicSmem = 232448;

// Launches fg8_gemm_kernel<BN> (sets its shared-memory limit on first use per
// device).  Defined in the gemm_bn_*.cu instantiation files.
template <int BN>
cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p, int grid,
                        size_t smem_bytes, cudaStream_t stream);

template <int BN>
int gemm_stage_bytes() {
    return GemmShape<BN>::STAGE_BYTES;
}

#define FG8_DEFINE_LAUNCH(BN)                                                                                  \
    template <>                                                                                                \
    cudaError_t launch_gemm<BN>(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p, int grid, \
                                size_t smem_bytes, cudaStream_t stream) {                                      \
        static std::atomic<unsigned long long> attr_set{0};                                                    \
        int dev = 0;                                                                                           \
        cudaError_t e = cudaGetDevice(&dev);                                                                   \
        if (e != cudaSuccess) return e;                                                                        \
        const unsigned long long bit = 1ull << (dev & 63);                                                     \
        if (!(attr_set.load() & bit)) {                                                                        \
            /* The in-kernel register split is only safe at exactly REGS_LAUNCH. */                            \
            cudaFuncAttributes fa;                                                                             \
            e = cudaFuncGetAttributes(&fa, fg8_gemm_kernel<BN>);                                               \
            if (e != cudaSuccess) return e;                                                                    \
            if (fa.numRegs != REGS_LAUNCH) return cudaErrorInvalidDeviceFunction;                              \
            e = cudaFuncSetAttribute(fg8_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,         \
                                     kMaxDynamicSmem);                                                         \
            if (e != cudaSuccess) return e;                                                                    \
            attr_set.fetch_or(bit);                                                                            \
        }                                                                                                      \
        fg8_gemm_kernel<BN><<<grid, NUM_THREADS, smem_bytes, stream>>>(tmA, tmB, p);                           \
        return cudaGetLastError();                                                                             \
    }

#define FG8_DECLARE_LAUNCH(BN)                                                                                 \
    template <>                                                                                                \
    cudaError_t launch_gemm<BN>(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p, int grid, \
                                size_t smem_bytes, cudaStream_t stream);

#define FG8_FOR_EACH_BN(X) \
    X(16) X(32) X(48) X(64) X(80) X(96) X(112) X(128) X(144) X(160) X(176) X(192) X(208) X(224) X(240) X(256)

}  // namespace fg8
