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
// window starts with the 1 KB region the driver reserves on sm_100, so the
// dynamic allocation begins at 0x400; the tables sit there, at a compile-time
// address, so a table read is a PRMT result (bytes 0-1: column and pattern,
// bytes 2-3: zero) plus an immediate.  After them: run sums for offsets, the
// mbarriers of the weight rings, and one ring of TMA stages per warp.
constexpr uint32_t kTableBase = 0x400;
constexpr uint32_t kMiscBase = kTableBase + kTableBytes;           // chunk / run sums (1 KB)
constexpr uint32_t kBarBase = kMiscBase + 1024;                    // 16 warps x <= 8 stages x 8 B
constexpr uint32_t kRingBase = kBarBase + 1024;                    // weight rings
constexpr uint32_t kSmemEnd = kTableBase + 227 * 1024;             // end of a 227 KB allocation
constexpr uint32_t kRingBytesPerWarp = (kSmemEnd - kRingBase) / kWarps / 512 * 512;
constexpr int kSmemBytes = (int)(kSmemEnd - kTableBase);           // dynamic bytes requested

// Planes one step of a unit carries; steps per TMA copy (two while a ring of
// two such copies fits a warp's share); TMA ring stages per warp (at most 8).
__host__ __device__ constexpr int step_planes(int q) { return q < 4 ? q : 4; }
__host__ __device__ constexpr int chunk_steps(int q) {
  return 2u * 2u * 512u * step_planes(q) <= kRingBytesPerWarp ? 2 : 1;
}
// Stages fit the warp's share, and at most one unit (8 steps) ahead.
__host__ __device__ constexpr int ring_stages(int q) {
  return (int)(kRingBytesPerWarp / (512u * step_planes(q) * chunk_steps(q))) < 8 / chunk_steps(q)
             ? (int)(kRingBytesPerWarp / (512u * step_planes(q) * chunk_steps(q)))
             : 8 / chunk_steps(q);
}

// Per-segment tile counters for dynamic tile assignment (segment-aligned
// mode); the last entry counts finished CTAs, so that the last one resets all.
constexpr int kMaxTileCounters = 1024;

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
  float* part;             // [batch][ns][mt*32] split-K partial sums (ns > 1)
  unsigned* tile_cnt;      // [segments] tile counters of segment-aligned mode (zero between calls)
  unsigned* status;        // sticky internal-error bits: 1 shared window base is not kTableBase,
                           // 2 a weight-ring wait timed out (results invalid)
  int m, n, batch, q, g;
  int ns, mt, ng;
  int y_f16;
  int seg_aligned;         // 1: CTAs grouped per segment; 0: unit list cut evenly
  int stall_test;          // test hook: each warp's first ring wait runs out (see LUTGEMM_TEST_STALL)
  long long total_units;   // batch * ns * mt
  // Mixed storage (lutgemm_run_mixed): per-block plane counts and sparse outliers.
  const uint32_t* block_off;  // [ns*mt + 1] exclusive prefix sums of the plane counts (4096-byte blocks)
  uint32_t packed_blocks;     // 4096-byte blocks in the packed buffer (bounds of block_off's values)
  const uint32_t* optr;       // [ns*m + 1] slice-major outlier pointers, or nullptr
  const uint32_t* oent;       // [nnz] outlier entries: (k - 1024 s) | fp16 << 16
  uint32_t nnz;
};

// Range [begin, end) of units of CTA c out of G: either a share of one
// segment's row tiles (segment-aligned), or a contiguous cut of the list.
__host__ __device__ inline void cta_range(long long c, long long G, long long segments, long long mt,
                                          bool aligned, long long* begin, long long* end) {
  if (aligned) {
    const long long z = c * segments / G;
    const long long c0 = (z * G + segments - 1) / segments, c1 = ((z + 1) * G + segments - 1) / segments;
    const long long k = c - c0, cz = c1 - c0;
    *begin = z * mt + k * mt / cz;
    *end = z * mt + (k + 1) * mt / cz;
  } else {
    *begin = c * segments * mt / G;
    *end = (c + 1) * segments * mt / G;
  }
}

// Slowest CTA of the contiguous cut, in unit-times: ceil(units / 16 warps)
// per segment touched plus a quarter for each table build.
inline double contiguous_worst(long long G, long long segments, long long mt) {
  double worst = 0.0;
  for (long long c = 0; c < G; ++c) {
    long long b, e;
    cta_range(c, G, segments, mt, false, &b, &e);
    double t = 0.0;
    while (b < e) {
      const long long seg_end = (b / mt + 1) * mt;
      const long long k = (e < seg_end ? e : seg_end) - b;
      t += (double)((k + kWarps - 1) / kWarps) + 0.25;
      b += k;
    }
    if (t > worst) worst = t;
  }
  return worst;
}

// Launch geometry.  Segment-aligned mode gives every segment the same number
// of CTAs, floor(grid / segments), whose warps share its tiles dynamically;
// the SMs left over start the next kernel of the stream early (programmatic
// launch).  It is chosen when its slowest group is no slower than the
// slowest CTA of the contiguous cut over the full grid.
inline void choose_launch(long long sms, long long segments, long long mt, long long* grid, int* aligned) {
  const long long units = segments * mt;
  const long long g = units < sms ? units : sms;
  *grid = g;
  *aligned = 0;
  if (segments > g || segments > kMaxTileCounters - 1) return;
  const long long cz = g / segments;
  const double t_aligned = (double)mt / (double)(cz * kWarps) + 0.25;
  if (t_aligned <= contiguous_worst(g, segments, mt)) {
    *grid = cz * segments;
    *aligned = 1;
  }
}

using RunKernel = void (*)(RunParams);

// y = sum over slices of the split-K partials (slice order), launched after
// the run kernel when ns > 1 (programmatic launch: it waits for the run).
cudaError_t launch_splitk_reduce(const RunParams& p, cudaStream_t stream);

// The fixed order in which the reduce kernel adds a row's slice partials: 2^L slice lanes, the
// smallest power of two (at most 32) that leaves each lane at most two
// slices; lane l adds slices l*per .. l*per + per - 1 (per = ceil(ns / 2^L))
// in order, in batches of 8 padded with +0, and the lane sums are added in
// lane order.
__host__ __device__ inline int reduce_lanes_log2(int ns) {
  int sl_log2 = 0;
  while (sl_log2 < 5 && ((ns + (1 << sl_log2) - 1) >> sl_log2) > 2) ++sl_log2;
  return sl_log2;
}

constexpr unsigned kStatusWindow = 1u;
constexpr unsigned kStatusTimeout = 2u;
constexpr unsigned kStatusFormat = 4u;   // a mixed-storage block or outlier entry out of range

// Kernel for q planes, group mode, offsets on/off and unit-major scales on/off
// (nullptr for unit-major scales with a mode that has several per piece).
RunKernel run_kernel_q1(int mode, bool has_offset, bool packed);
RunKernel run_kernel_q2(int mode, bool has_offset, bool packed);
RunKernel run_kernel_q3(int mode, bool has_offset, bool packed);
RunKernel run_kernel_q4(int mode, bool has_offset, bool packed);
RunKernel run_kernel_q8(int mode, bool has_offset, bool packed);   // 5 <= q <= 8, planes in groups of four
RunKernel run_kernel_mixed(int mode, bool packed);   // mixed storage: 1..4 planes per block, sparse outliers

}  // namespace lutgemm
