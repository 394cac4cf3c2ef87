// Instantiations of the LUT-GEMM kernel for q = 2 bit planes.
#include "lutgemm_run.cuh"

namespace lutgemm {
RunKernel run_kernel_q2(int mode, bool has_offset, bool packed) { LUTGEMM_RUN_SELECT(2, false) }
}  // namespace lutgemm
