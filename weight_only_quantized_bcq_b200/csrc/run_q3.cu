// Instantiations of the LUT-GEMM kernel for q = 3 bit planes.
#include "lutgemm_run.cuh"

namespace lutgemm {
RunKernel run_kernel_q3(int mode, bool has_offset, bool packed) { LUTGEMM_RUN_SELECT(3, false) }
}  // namespace lutgemm
