// jit.h -- runtime specialisation of the tile GEMM kernel (jit.cu).
#pragma once

#include <cuda_runtime.h>

#include "fg8.h"
#include "gemm_kernel.cuh"

namespace fg8 {

// FG_JIT=1 in the environment (read at call time).
bool jit_enabled();

// Launches fg8_gemm_kernel<bn, pair> compiled at run time with p.KB as a
// compile-time constant (compiled once per specialisation and process, cached
// on disk across processes).  Returns FG_OK, or an error when NVRTC, the
// sources or the driver are unavailable; the caller then uses the
// ahead-of-time kernel.
fg_status jit_launch_gemm(int bn, bool pair, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                          const GemmParams& p, int grid, size_t smem, cudaStream_t stream);

}  // namespace fg8
