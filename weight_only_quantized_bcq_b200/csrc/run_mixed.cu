// Lookup kernels for mixed storage (up to four planes per block, stored and
// streamed in pairs; sparse fp16 outliers), one per group mode; unit-major
// scales and offsets are not used.
#include "lutgemm_run.cuh"

namespace lutgemm {

RunKernel run_kernel_mixed(int mode) {
  switch (mode) {
    case kG128: return lut_gemm_kernel<2, kG128, false, false, false, true>;
    case kG128x: return lut_gemm_kernel<2, kG128x, false, false, false, true>;
    case kG64: return lut_gemm_kernel<2, kG64, false, false, false, true>;
    case kG8: return lut_gemm_kernel<2, kG8, false, false, false, true>;
    default: return lut_gemm_kernel<2, kGAny, false, false, false, true>;
  }
}

}  // namespace lutgemm
