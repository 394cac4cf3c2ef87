// Shared definitions of the sm_100a LUT-GEMM kernels.
//
// Terms (LUT-GEMM card, Elamur: Summary, Interesting ideas):
//   run    8 consecutive inputs; its 256 signed activation sums form one table
//          column ("lookup tables instead of multiplications").
//   slice  1024 inputs = 128 runs; one CTA holds the fp32 tables of one slice
//          of one batch column in shared memory (128 KB).
//   piece  128 inputs = 16 runs; the 16 bytes a lane reads per step and plane.
//   unit   32 output rows x one slice; one warp, one row per lane.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lutgemm {

constexpr int kSliceInputs = 1024;
constexpr int kRunsPerSlice = 128;
constexpr int kTileRows = 32;
constexpr int kBlockBytes = 4096;                   // one (slice, row tile, plane) block
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kHalfTableBytes = 256 * 64 * 4;       // 256 patterns x 64 run columns x fp32
constexpr int kTableBytes = 2 * kHalfTableBytes;    // both halves: 128 runs

// Shared-memory map, in absolute addresses of the CTA's shared window.  The
// tables start at 64 KB, so a table read address is a PRMT result (bytes 0-1:
// column and pattern, bytes 2-3: zero) plus a compile-time immediate.  The
// dynamic allocation starts at the window's base R0 (the reserved region,
// at most a few KB) and is sized to reach kSmemEnd; [R0, 64 KB) is unused.
constexpr uint32_t kTableBase = 0x10000;
constexpr uint32_t kMiscBase = kTableBase + kTableBytes;            // run sums for offsets
constexpr uint32_t kSmemEnd = kMiscBase + 2 * kRunsPerSlice * 4;
constexpr int kSmemBytes = (int)kSmemEnd;                          // dynamic bytes requested

// Register pipeline depth: a lane keeps NB steps of loads, NB - 1 in flight.
constexpr int pipeline_stages(int q) { return q <= 3 ? 4 : 2; }

// How the group size g maps onto the 128-input pieces a lane walks.
enum GroupMode : int {
  kG128 = 0,   // g == 128: one scale per piece
  kG128x = 1,  // g % 128 == 0, g > 128: one scale per piece, group found by division
  kG64 = 2,    // g == 64: two scales per piece
  kG8 = 3,     // g == 8: one scale per run
  kGAny = 4,   // other multiples of 8: one scale per run, group found by division
};

struct RunParams {
  const uint8_t* packed;   // packed bit planes (layout in include/lutgemm.h)
  const __half* alpha;     // [q][ng][m]
  const float* offset;     // [ng][m] or nullptr
  const __half* x;         // [batch][n]
  void* y;                 // [batch][m], fp32 or fp16
  float* part;             // [batch][ns][mt*32] split-K partial sums
  unsigned* cnt;           // [batch][mt] arrival counters (zero between calls)
  unsigned* status;        // sticky internal-error bits (1: shared window base above kTableBase)
  int m, n, batch, q, g;
  int ns, mt, ng;
  int y_f16;
  long long total_units;   // batch * ns * mt
};

using RunKernel = void (*)(RunParams);

RunKernel run_kernel_q1(int mode, bool has_offset);
RunKernel run_kernel_q2(int mode, bool has_offset);
RunKernel run_kernel_q3(int mode, bool has_offset);
RunKernel run_kernel_q4(int mode, bool has_offset);
RunKernel run_kernel_q8(int mode, bool has_offset);   // 5 <= q <= 8, planes in groups of four

}  // namespace lutgemm
