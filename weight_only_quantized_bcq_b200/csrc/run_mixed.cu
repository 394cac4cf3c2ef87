// Lookup kernels for mixed storage (up to four planes per block, stored and
// streamed in pairs; sparse fp16 outliers), one per group mode, with scales
// in [q][n/g][m] or, for one or two scales per piece, in the unit-major
// mixed layout; offsets are not used.
#include "lutgemm_run.cuh"

namespace lutgemm {

RunKernel run_kernel_mixed(int mode, bool packed) {
  switch (mode) {
    case kG128:
      return packed ? lut_gemm_kernel<2, kG128, false, false, true, true>
                    : lut_gemm_kernel<2, kG128, false, false, false, true>;
    case kG128x:
      return packed ? lut_gemm_kernel<2, kG128x, false, false, true, true>
                    : lut_gemm_kernel<2, kG128x, false, false, false, true>;
    case kG64:
      return packed ? lut_gemm_kernel<2, kG64, false, false, true, true>
                    : lut_gemm_kernel<2, kG64, false, false, false, true>;
    case kG8: return packed ? nullptr : lut_gemm_kernel<2, kG8, false, false, false, true>;
    default: return packed ? nullptr : lut_gemm_kernel<2, kGAny, false, false, false, true>;
  }
}

}  // namespace lutgemm
