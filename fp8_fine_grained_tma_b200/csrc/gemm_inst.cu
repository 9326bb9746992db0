// gemm_inst.cu -- the GEMM kernels of one block width, selected by
// -DFG8_BN=<width>, so the sixteen block widths compile in parallel.
#include "launch.cuh"

#ifndef FG8_BN
#error "compile with -DFG8_BN=<16..256, multiple of 16>"
#endif

namespace fg8 {
template <>
cudaError_t gemm_max_split_clusters<FG8_BN>(int cluster, int* out) {
    return gemm_max_split_clusters_impl<FG8_BN>(cluster, out);
}
FG8_DEFINE_LAUNCH_ONE(FG8_BN, false)
#if FG8_BN >= 32
FG8_DEFINE_LAUNCH_ONE(FG8_BN, true)
#endif
}  // namespace fg8
