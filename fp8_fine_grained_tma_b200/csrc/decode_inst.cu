// decode_inst.cu -- the decode kernel of one token-tile width, selected by
// -DFG8_MT=<width>, so the widths compile in parallel.
#include "decode_launch.cuh"

#ifndef FG8_MT
#error "compile with -DFG8_MT=<32..256, multiple of 32>"
#endif

namespace fg8 {
FG8_DEFINE_DECODE_LAUNCH(FG8_MT)
}  // namespace fg8
