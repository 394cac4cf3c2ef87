// Instantiations of the LUT-GEMM kernel for q = 4 bit planes.
#include "lutgemm_run.cuh"

namespace lutgemm {
RunKernel run_kernel_q4(int mode, bool has_offset, bool packed) { LUTGEMM_RUN_SELECT(4, false) }
}  // namespace lutgemm
