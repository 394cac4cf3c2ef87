// Instantiations of the LUT-GEMM kernel for q = 1 bit planes.
#include "lutgemm_run.cuh"

namespace lutgemm {
RunKernel run_kernel_q1(int mode, bool has_offset, bool packed) { LUTGEMM_RUN_SELECT(1, false) }
}  // namespace lutgemm
