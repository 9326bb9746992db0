// gemm_inst.cu -- one instantiation of the GEMM kernel per build, selected by
// -DFG8_BN=<block width>, so the sixteen block widths compile in parallel.
#include "launch.cuh"

#ifndef FG8_BN
#error "compile with -DFG8_BN=<16..256, multiple of 16>"
#endif

namespace fg8 {
FG8_DEFINE_LAUNCH(FG8_BN)
}  // namespace fg8
