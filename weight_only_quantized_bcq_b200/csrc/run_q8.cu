// Instantiations of the LUT-GEMM kernel for 5 <= q <= 8 bit planes, walked in
// groups of four planes per pass over a unit.
#include "lutgemm_run.cuh"

namespace lutgemm {
RunKernel run_kernel_q8(int mode, bool has_offset, bool packed) { LUTGEMM_RUN_SELECT(4, true) }
}  // namespace lutgemm
