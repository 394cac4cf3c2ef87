// The LUT-GEMM kernel for sm_100a: y = sum_i alpha_i (B_i x) (+ offset * group sums of x)
// through per-run lookup tables, with no dequantisation of the weights.
//
// Method (LUT-GEMM card, Elamur: Summary; Interesting ideas, "Lookup tables
// instead of multiplications"): for a run of 8 activations the 256 signed sums
// T[p] = sum_t (2*bit_t(p) - 1) * x_t are computed once; a plane-row with sign
// byte p over that run contributes T[p], scaled by its group's alpha.
//
// Design on B200 (148 SMs, 228 KB shared memory per SM, 128 B/clk shared
// memory bandwidth per SM, HBM3e):
//   * One persistent 512-thread CTA per SM.  The work is the list of units
//     (batch column, slice, 32-row tile).  Either every (batch column, slice)
//     segment gets its own group of CTAs that share its tiles round-robin, or
//     the list is cut into one contiguous range per CTA, whichever the host
//     finds better balanced.  A CTA builds the 128 KB fp32 tables of a slice
//     once per segment it touches.
//   * A warp processes a unit, one output row per lane, in 8 steps.  Warp w
//     takes the CTA's tiles w, w+16, w+32, ... of a segment.
//   * Weights move by TMA: the q pieces of all 32 lanes of a step are q*512
//     contiguous bytes of the packed layout, and CH consecutive steps (CH = 2
//     for q <= 3) are fetched by one cp.async.bulk (L2 evict-first: the
//     weights are read once) into a per-warp ring of S
//     shared-memory stages (one mbarrier each), S copies ahead and across
//     unit boundaries; a warp's first copies of a segment are issued before
//     the table build.  Every wait is bounded in time; a timeout sets a
//     status bit instead of hanging.  At a stage's first step each lane reads
//     its 16-byte pieces of all the stage's steps (one LDS.128 each) and the
//     stage is refilled at once, so S copies stay in flight during compute.
//   * Table reads are conflict-free: at every step the 32 lanes read 32
//     distinct banks.  Lanes 0-15 and 16-31 walk the 8 pieces of the slice
//     four apart, and lane l reads the runs of its piece in the order
//     j xor (l mod 16), so (piece half, run) is a bijection onto banks.
//   * A table read is one PRMT that places the sign byte (pattern p, times
//     256) next to the lane's column byte, one LDS whose immediate carries the
//     table base, half and band, and one FADD.
//   * Per-group alpha (and offset) are applied once per piece (g = 128),
//     per half-piece (g = 64) or per run (other g); the per-piece values are
//     prefetched up to seven steps ahead in registers.  With scales in the
//     unit-major layout (g % 128 == 0), a lane's scales for a whole pass over
//     a tile are SP 16-byte loads, issued one pass ahead.
//   * Split-K: each unit stores its fp32 partial; a second, small kernel
//     (programmatically chained) sums the slices of every row in slice order
//     and writes y.  With a single slice the run kernel writes y itself.
#pragma once

#include <utility>

#include "lutgemm_common.cuh"

namespace lutgemm {
namespace detail {

template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt_i(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "n"(SEL));
  return d;
}

// Table read at shared-window address addr + IMM.
template <uint32_t IMM>
__device__ __forceinline__ float lds_at(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(IMM));
  return v;
}

__device__ __forceinline__ void sts_at(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint16_t ld_u16(const __half* ptr) {
  return __ldg(reinterpret_cast<const unsigned short*>(ptr));
}

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ uint32_t word_of(const uint4& v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred P;\n mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n selp.u32 %0, 1, 0, P;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of an mbarrier; give up after `limit_ns`
// nanoseconds (one second unless told otherwise).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns = 1000000000ull) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// L2 policy for the weight stream: every weight byte is read exactly once, so
// its lines are the first to go, and the scales, inputs and split-K partials
// keep their place in L2.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// One TMA bulk copy of `bytes` (a multiple of 16) from global memory into this
// CTA's shared memory, completing on mbarrier `bar`, with L2 policy `pol`.
// The proxy fence orders the warp's earlier generic reads of the stage before
// the copy overwrites it.
__device__ __forceinline__ void tma_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, uint64_t pol) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}

// PRMT selector for byte t of a stored word: result byte 0 <- column byte t of
// the offset register (source byte 4+t), byte 1 <- sign byte t of the word
// (source byte t, giving pattern*256), bytes 2-3 <- sign of the column byte,
// which is below 128, hence zero.
__host__ __device__ constexpr uint32_t table_sel(int t) {
  return (uint32_t)(((0x8 | (4 + t)) << 12) | ((0x8 | (4 + t)) << 8) | (t << 4) | (4 + t));
}

// Address immediate of step U: table base, half (U>>1)&1, band U&1.
template <int U>
__host__ __device__ constexpr uint32_t step_imm() {
  return kTableBase + (uint32_t)((U >> 1) & 1) * kHalfTableBytes + (uint32_t)(U & 1) * 128u;
}

// Four table reads of one stored word, into two accumulators.
template <uint32_t IMM>
__device__ __forceinline__ void lookup_word(uint32_t w, uint32_t cb, float& acc0, float& acc1) {
  acc0 += lds_at<IMM>(prmt_i<table_sel(0)>(w, cb));
  acc1 += lds_at<IMM>(prmt_i<table_sel(1)>(w, cb));
  acc0 += lds_at<IMM>(prmt_i<table_sel(2)>(w, cb));
  acc1 += lds_at<IMM>(prmt_i<table_sel(3)>(w, cb));
}

template <uint32_t IMM>
__device__ __forceinline__ void lookup_word_values(uint32_t w, uint32_t cb, float (&v)[4]) {
  v[0] = lds_at<IMM>(prmt_i<table_sel(0)>(w, cb));
  v[1] = lds_at<IMM>(prmt_i<table_sel(1)>(w, cb));
  v[2] = lds_at<IMM>(prmt_i<table_sel(2)>(w, cb));
  v[3] = lds_at<IMM>(prmt_i<table_sel(3)>(w, cb));
}

// Tables of one slice of batch column b, in fp32.
// Table column of run c (0..127 in the slice): half (c>>5)&1, column
// 32*((c>>4)&1) + 16*(c>>6) + (c&15) of 64; entry p at byte p*256 + 4*column.
// Thread mapping: warp w covers patterns [64*(w&3), +64) of runs with bits
// 5..4 = w>>2; lane l covers run bits 6 and 3..0, so the 32 lanes of a warp
// store to 32 distinct banks.  T[p] = (A + B) + (C + D) with A..D the signed
// pair sums of x0x1, x2x3, x4x5, x6x7 selected by bit pairs of p.
template <int RUN, bool HAS_OFF>
__device__ __forceinline__ void build_tables(const RunParams& p, int b, int s, float* chunk_sum,
                                             float* run_sum) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pq = warp & 3;
  const int c54 = warp >> 2;
  const int c = 64 * (lane >> 4) + 16 * c54 + (lane & 15);
  const int k0 = s * kSliceInputs + 8 * c;
  float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f, x4 = 0.f, x5 = 0.f, x6 = 0.f, x7 = 0.f;
  if (k0 < p.n) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)b * p.n + k0));
    const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    const float2 f45 = __half22float2(*reinterpret_cast<const __half2*>(&raw.z));
    const float2 f67 = __half22float2(*reinterpret_cast<const __half2*>(&raw.w));
    x0 = f01.x; x1 = f01.y; x2 = f23.x; x3 = f23.y;
    x4 = f45.x; x5 = f45.y; x6 = f67.x; x7 = f67.y;
  }
  // Index bit pair (lo, hi) -> (+-x_lo) + (+-x_hi), bit set meaning +.
  const float A[4] = {-x0 - x1, x0 - x1, x1 - x0, x0 + x1};
  const float B[4] = {-x2 - x3, x2 - x3, x3 - x2, x2 + x3};
  const float C[4] = {-x4 - x5, x4 - x5, x5 - x4, x4 + x5};
  const float D = pq == 0 ? -x6 - x7 : (pq == 1 ? x6 - x7 : (pq == 2 ? x7 - x6 : x6 + x7));
  const int colw = 32 * (c54 & 1) + 16 * (lane >> 4) + (lane & 15);
  const uint32_t base = kTableBase + (uint32_t)((c54 >> 1) * kHalfTableBytes + colw * 4 + pq * 64 * 256);
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {
    const float H = C[hh] + D;
#pragma unroll
    for (int v = 0; v < 16; ++v) sts_at(base + (uint32_t)((16 * hh + v) * 256), (A[v & 3] + B[v >> 2]) + H);
  }
  if (HAS_OFF && pq == 0) chunk_sum[c] = ((x0 + x1) + (x2 + x3)) + ((x4 + x5) + (x6 + x7));
  __syncthreads();
  if constexpr (RUN > 1 && HAS_OFF) {
    if (threadIdx.x < kRunsPerSlice / RUN) {
      float acc = 0.f;
#pragma unroll
      for (int r = 0; r < RUN; ++r) acc += chunk_sum[threadIdx.x * RUN + r];
      run_sum[threadIdx.x] = acc;
    }
    __syncthreads();
  }
}

// A one-plane pass of mixed-storage scales (8 * H halves, in the order
// (step, half)) moved into the two-plane order (step, plane, half) with
// plane 1 zero.  H = 1: half U goes to element 2U; H = 2: the word of step U
// goes to word 2U.
template <int H, int N>
__device__ __forceinline__ void spread_scales(uint4 (&sc)[N]) {
  static_assert(N == 1 || N == 2 * H, "a pass holds 2 * H words");
  if constexpr (N == 1) {
    return;                       // no unit-major scales: nothing to move
  } else if constexpr (H == 1) {
    uint32_t w[4] = {sc[0].x, sc[0].y, sc[0].z, sc[0].w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = (w[k >> 1] >> (16 * (k & 1))) & 0xffffu;
    sc[0] = make_uint4(o[0], o[1], o[2], o[3]);
    sc[1] = make_uint4(o[4], o[5], o[6], o[7]);
  } else {
    const uint32_t r[8] = {sc[0].x, sc[0].y, sc[0].z, sc[0].w, sc[1].x, sc[1].y, sc[1].z, sc[1].w};
#pragma unroll
    for (int v = 0; v < 4; ++v) sc[v] = make_uint4(r[2 * v], 0u, r[2 * v + 1], 0u);
  }
}

template <int... Is, class F>
__device__ __forceinline__ void static_for(std::integer_sequence<int, Is...>, F&& f) {
  (f.template operator()<Is>(), ...);
}

}  // namespace detail

// MIXED: mixed storage (lutgemm_run_mixed), with Q = 2.  Every (slice, row
// tile) block holds its own number of planes, 1..4, at the offset
// p.block_off gives, stored in pairs; a block is one pass per pair (one or
// two), each pass moving two planes per step like the q = 2 kernel.  Sparse
// fp16 outliers (slice-major CSR) are added to each row's sum.
template <int Q, int MODE, bool MULTI, bool HAS_OFF, bool PK, bool MIXED = false>
__global__ void __launch_bounds__(kThreads, 1) lut_gemm_kernel(const RunParams p) {
  using namespace detail;
  constexpr int SP = step_planes(MULTI ? 8 : Q);       // planes in one step (<= 4)
  constexpr int CH = chunk_steps(MULTI ? 8 : Q);       // steps per TMA copy
  constexpr int S = ring_stages(MULTI ? 8 : Q);        // TMA stages per warp
  constexpr uint32_t STEP_BYTES = 512u * SP;
  constexpr uint32_t STAGE_BYTES = STEP_BYTES * CH;
  static_assert(!MULTI || CH == 1, "plane groups are fetched one step at a time");
  static_assert(!MIXED || (Q == 2 && !MULTI && !HAS_OFF), "mixed storage: plane pairs, no offsets");
  constexpr uint32_t QB_MAX = MIXED ? 4u : (uint32_t)Q;   // planes of one mixed block
  static_assert(S >= 2 && S <= 7, "weight ring of 2..7 stages (barrier slot 7 is the test hook's)");
  constexpr int NPG = (MULTI || MIXED) ? 2 : 1;        // plane groups of a unit (at most)
  constexpr int GP = MIXED ? 2 : 4;                    // planes per plane group

  extern __shared__ __align__(16) unsigned char smem[];
  // Let the next kernel in the stream start on SMs as they free up; it waits
  // for this grid's completion before touching anything this grid writes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t r0 = (uint32_t)__cvta_generic_to_shared(smem);
  if (r0 != kTableBase) {  // uniform over the CTA: the map would not match the allocation
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) atomicOr(p.status, kStatusWindow);
    return;
  }
  float* const chunk_sum = reinterpret_cast<float*>(smem + (kMiscBase - kTableBase));
  float* const run_sum = chunk_sum + kRunsPerSlice;

  // Runs (8-input table columns) that share one alpha inside a piece.
  constexpr int RUN = (MODE == kG128 || MODE == kG128x) ? 16 : (MODE == kG64 ? 8 : 1);
  constexpr int APP = RUN >= 8 ? 16 / RUN : 1;      // prefetched scales per piece
  constexpr bool PRE_ALPHA = RUN >= 8;
  // Scales in the unit-major layout: p.alpha holds, for every (slice, row
  // tile, plane group, lane), the 8 x SP x HPK scales of that lane's pass
  // (HPK = 2 when g = 64: one per half of each piece).
  static_assert(!PK || RUN >= 8, "unit-major scales need one or two scales per piece");
  constexpr int HPK = RUN == 8 ? 2 : 1;
  // Register stages of prefetched scales: step j's are loaded NA-1 steps
  // ahead (7 with one scale per piece, 3 with two, to bound registers); the
  // scales come from HBM and their latency under full load is microseconds.
  // Mixed storage: 3 steps ahead, so that the next tile's block entry (read
  // when the tile becomes known, a tile ahead) has arrived first.
  constexpr int NA = (APP == 1 && !MIXED) ? 8 : 4;
  static_assert((8 * NPG) % NA == 0, "scale stages must tile the unit");
  // Step of a unit at which the next tile is first needed: the scale
  // prefetch reaches it NA-1 steps before the end, the ring refill S stages
  // before the end.  Three steps cover a tile-counter atomic comfortably.
  constexpr int NEED_A = PRE_ALPHA ? 8 * NPG - (NA - 1) : 8 * NPG;
  constexpr int NEED_R = ((8 / CH) * NPG - S) * CH;
  constexpr int NEED_P = PK ? 8 * (NPG - 1) : 8 * NPG;   // next tile's scales: start of its last pass
  constexpr int NEED_AR = NEED_A < NEED_R ? NEED_A : NEED_R;
  constexpr int NEED = NEED_AR < NEED_P ? NEED_AR : NEED_P;
  // Mixed storage grabs two tiles ahead: a tile's block entry is read as soon
  // as the tile is known, a whole tile before its copies are issued.
  constexpr bool AHEAD1 = NEED >= 3 && !MIXED;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t a = (uint32_t)lane >> 4;
  const uint32_t lam = (uint32_t)lane & 15;

  // colb[u2][k] byte t = 4 * (16*(u2 xor a) + ((4k + t) xor lam)): the lane's
  // column byte offset inside a 256-byte table row for stored byte 4k+t in
  // steps with U>>2 == u2.
  uint32_t colb[2][4];
#pragma unroll
  for (int u2 = 0; u2 < 2; ++u2) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t v = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        v |= (4u * (16u * ((uint32_t)u2 ^ a) + ((uint32_t)(4 * k + t) ^ lam))) << (8 * t);
      colb[u2][k] = v;
    }
  }

  // This warp's weight ring: S stages of STAGE_BYTES (CH steps), one mbarrier
  // each.  (st, ph) is the stage to consume next and its phase parity; both
  // run on across segments.  At a segment boundary every issued copy has been
  // consumed.
  const uint32_t ring = kRingBase + (uint32_t)warp * kRingBytesPerWarp;
  const uint32_t bars = kBarBase + (uint32_t)warp * 64u;
  // Slot 7 of the warp's barriers is never signalled: with the test hook
  // (p.stall_test) the warp's first ring wait is on it, runs out after 1 ms
  // and takes the timeout path.
  const uint32_t dead_bar = bars + 56u;
  if (lane == 0) {
#pragma unroll
    for (int st0 = 0; st0 < S; ++st0) mbar_init(bars + 8u * st0);
    if (p.stall_test) mbar_init(dead_bar);
  }
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncwarp();
  const uint64_t wpol = evict_first_policy();
  int st = 0;
  uint32_t ph = 0;
  bool failed = false;     // a ring wait timed out: stop streaming, keep taking the CTA barriers
  int outstanding = 0;     // copies issued and not yet consumed

  const int npg = MULTI ? (p.q + 3) >> 2 : 1;
  const int steps_per_unit = 8 * npg;
  const size_t plane_stride = (size_t)p.ng * (size_t)p.m;
  const uint32_t unit_bytes = (uint32_t)p.q * kBlockBytes;

  // Work of this CTA.  Segment-aligned: one segment z, whose row tiles its
  // cz CTAs share round-robin (CTA k takes tiles k, k+cz, ...), so that every
  // CTA's reads spread over the whole segment.  Otherwise: a contiguous range
  // [u_begin, u_end) of the unit list, visited segment by segment.
  // Index arithmetic is 32-bit where the host bounds allow it (batch * ns <
  // 2^31; segment-aligned mode has at most kMaxTileCounters - 1 segments and
  // one CTA per SM): 64-bit division is a long software sequence.
  const unsigned Z = (unsigned)p.batch * (unsigned)p.ns;
  long long u_begin = 0, u_end = 0;
  unsigned a_seg = 0, a_first = 0, a_stride = 1;
  if (p.seg_aligned) {
    // Segment z gets the CTAs c = z, z + Z, z + 2Z, ...: a group spread over
    // the whole grid rather than a block of neighbouring CTAs.
    const unsigned G = gridDim.x, c = blockIdx.x;
    a_seg = c % Z;
    a_first = c / Z;
    a_stride = (G - a_seg + Z - 1) / Z;
  } else {
    cta_range(blockIdx.x, gridDim.x, Z, p.mt, false, &u_begin, &u_end);
  }

  uint16_t ab[NA][Q][APP];
  uint4 sc_cur[PK ? SP * HPK : 1], sc_nxt[PK ? SP * HPK : 1];   // unit-major scales of this pass and the next
  float ob[NA][APP];
  uint4 wst[CH][SP];       // the pieces of the current ring stage

  auto group_size = [&](unsigned z) { return (gridDim.x - z + Z - 1) / Z; };

  for (int visit = 0;; ++visit) {
    // Segment-aligned mode visits the CTA's own segment once; the contiguous
    // mode visits the segments of its range in order.
    unsigned seg, tile_first = 0, tile_stride = 1, tile_count = 0;
    if (p.seg_aligned) {
      if (visit > 0) break;
      seg = a_seg;
      tile_first = a_first;
      tile_stride = a_stride;
      tile_count = a_first < (unsigned)p.mt ? ((unsigned)p.mt - 1 - a_first) / a_stride + 1 : 0;
    } else {
      if (u_begin >= u_end) break;
      const long long sg = u_begin / p.mt;
      const long long seg_end = min(u_end, (sg + 1) * p.mt);
      seg = (unsigned)sg;
      tile_first = (unsigned)(u_begin - sg * p.mt);
      tile_stride = 1;
      tile_count = (unsigned)(seg_end - u_begin);
      u_begin = seg_end;
    }
    const int b = (int)(seg / (unsigned)p.ns);
    const int s = (int)(seg - (unsigned)b * (unsigned)p.ns);
    const uint8_t* slice_base = p.packed + (size_t)s * p.mt * unit_bytes;
    // This warp's row tiles.  In the contiguous mode: indices warp, warp+16,
    // ... of the CTA's tiles (tile_first + index * tile_stride).  In
    // segment-aligned mode the G_z CTAs of a segment take two static tiles per
    // warp, covering tiles [0, 32 G_z); all further tiles come from the
    // segment's tile counter (lane 0 grabs), so the group's warps share out
    // the rest as they finish.  The last CTA to finish the kernel resets the
    // counters for the next call.
    const bool dyn = p.seg_aligned != 0;
    auto static_tile = [&](int k) -> int {
      const unsigned idx = (unsigned)warp + (unsigned)k * kWarps;
      return idx < tile_count ? (int)(tile_first + idx * tile_stride) : -1;
    };
    unsigned* const tile_ctr = p.tile_cnt + seg;
    const long long dyn_base = dyn ? 32ll * group_size(seg) : 0;
    int t_cur = failed ? -1 : static_tile(0);
    int t_nxt = static_tile(1);
    const bool busy = t_cur >= 0;
    constexpr int CPT = 8 / CH;                      // ring chunks per unit and plane group
    // Mixed storage: one pass per plane pair of the tile (npg_t, set per tile).
    int npg_t = npg;
    int chunks_per_unit = CPT * npg_t;

    // Mixed storage: (first 4096-byte block, planes) of row tile R_ of this
    // slice, from the block table.  An entry outside the packed buffer or
    // with no plane or more than Q planes is reported and its tile skipped
    // (planes = 0).  Uniform storage: (unused, Q).
    auto tile_info = [&](int R_) -> uint2 {
      if constexpr (MIXED) {
        const uint32_t* bo = p.block_off + (size_t)s * p.mt + R_;
        const uint32_t b0 = __ldg(bo), b1 = __ldg(bo + 1);
        const uint32_t qb = b1 - b0;
        if (b1 < b0 || qb < 1u || qb > QB_MAX || b1 > p.packed_blocks) {
          if (lane == 0) atomicOr(p.status, kStatusFormat);
          return make_uint2(0u, 0u);
        }
        return make_uint2(b0, qb);
      } else {
        return make_uint2(0u, (uint32_t)Q);
      }
    };

    // TMA copy of chunk c (steps c*CH .. c*CH+CH-1) of row tile R into ring
    // stage `stage` (lane 0 only).  The CH steps are contiguous.  A mixed
    // tile with no valid entry fetches nothing and completes its stage.
    auto issue = [&](int R_, uint2 ti, int c, int stage) {
      const int pg_ = c / CPT, U_ = (c - pg_ * CPT) * CH;
      if constexpr (MIXED) {
        if (ti.y == 0u) {
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bars + 8u * stage) : "memory");
          return;
        }
        // Pair pg_ of the block: e planes from byte 8192 * pg_, CH steps of e * 512.
        const uint32_t e = min(2u, ti.y - 2u * (uint32_t)pg_);
        const uint8_t* src = p.packed + (size_t)ti.x * kBlockBytes + (size_t)pg_ * 2 * kBlockBytes + (size_t)U_ * e * 512;
        tma_load(ring + (uint32_t)stage * STAGE_BYTES, src, 512u * e * CH, bars + 8u * stage, wpol);
      } else {
        const int planes = MULTI ? min(4, p.q - 4 * pg_) : Q;
        const uint8_t* src = slice_base + (size_t)R_ * unit_bytes + ((size_t)U_ * p.q + 4 * pg_) * 512;
        tma_load(ring + (uint32_t)stage * STAGE_BYTES, src, 512u * planes * CH, bars + 8u * stage, wpol);
      }
    };

    // Mixed storage: each lane's outlier range [o0, o1) in row tile R_ of
    // this slice (rows past m: empty), read a tile ahead of its use.
    auto outlier_range = [&](int R_) -> uint2 {
      uint2 r = make_uint2(0u, 0u);
      if constexpr (MIXED) {
        if (p.optr != nullptr && R_ >= 0 && R_ * kTileRows + lane < p.m) {
          const uint32_t* op = p.optr + (size_t)s * p.m + (size_t)R_ * kTileRows + lane;
          r = make_uint2(__ldg(op), __ldg(op + 1));
        }
      }
      return r;
    };

    // Per-piece scales (and offsets) of step j of row tile R into register
    // stage SLOT; `planes` of them (the tile's plane count in mixed storage).
    auto load_alpha = [&]<int SLOT>(int R_, int j, uint32_t planes) {
      if constexpr (PRE_ALPHA) {
        [[maybe_unused]] const int pg_ = j >> 3;
        const int U_ = j & 7;
        const int row = R_ * kTileRows + lane;
        const int P = U_ ^ (int)(4 * a);
#pragma unroll
        for (int r = 0; r < APP; ++r) {
          int G;
          if constexpr (MODE == kG128) G = 8 * s + P;
          else if constexpr (MODE == kG128x) G = (8 * s + P) / (p.g >> 7);
          else G = 16 * s + 2 * P + (r ^ (int)(lam >> 3));
          [[maybe_unused]] const bool ok = row < p.m && G < p.ng;
          [[maybe_unused]] const __half* ap = p.alpha + (size_t)G * p.m + row;
          if constexpr (!PK) {
#pragma unroll
            for (int i = 0; i < Q; ++i) {
              const int plane = pg_ * GP + i;
              const bool live = (!MULTI || (plane < p.q)) && (!MIXED || (uint32_t)plane < planes);
              ab[SLOT][i][r] = (ok && live) ? ld_u16(ap + (size_t)plane * plane_stride) : (uint16_t)0;
            }
          }
          if constexpr (HAS_OFF) ob[SLOT][r] = (ok && pg_ == 0) ? __ldg(p.offset + (size_t)G * p.m + row) : 0.f;
        }
      }
    };

    uint2 ti_cur = busy ? tile_info(t_cur) : make_uint2(0u, 0u);
    uint2 ti_nxt = t_nxt >= 0 ? tile_info(t_nxt) : make_uint2(0u, 0u);
    uint2 or_cur = busy ? outlier_range(t_cur) : make_uint2(0u, 0u);
    uint2 or_nxt = outlier_range(t_nxt);
    // The first S copies of the first tile go out before the tables are built.
    if (busy && lane == 0) {
      int st2 = st;
      for (int c = 0; c < S; ++c) {
        issue(t_cur, ti_cur, c, st2);
        st2 = st2 + 1 == S ? 0 : st2 + 1;
      }
    }
    if (busy) outstanding = S;
    // Programmatic dependent launch: everything above reads only the weights.
    // x, y and the workspace may belong to the previous kernel in the stream,
    // so wait for it to complete before the first touch (a no-op otherwise).
    if (visit == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();  // every warp is done with the previous segment's tables
    build_tables<RUN, HAS_OFF>(p, b, s, chunk_sum, run_sum);

    // Unit-major scales of pass pg_ of row tile R_ (SP * HPK 16-byte loads).
    // Mixed storage: the pass of pair pg_ of the tile's block (table entry
    // ti_.x) holds e planes, so a lane loads e * HPK of them; a one-plane pass
    // is spread to the two-plane order when it starts (spread_scales).
    auto load_scales = [&](int R_, uint2 ti_, int pg_, uint4 (&dst)[PK ? SP * HPK : 1]) {
      if constexpr (PK) {
        if constexpr (MIXED) {
          const uint32_t e = ti_.y > 2u * (uint32_t)pg_ ? min(2u, ti_.y - 2u * (uint32_t)pg_) : 0u;
          const uint4* src = reinterpret_cast<const uint4*>(p.alpha) +
                             ((size_t)ti_.x * 32 + (size_t)pg_ * 64 + (size_t)lane * e) * HPK;
#pragma unroll
          for (int v = 0; v < SP * HPK; ++v) dst[v] = (uint32_t)v < e * HPK ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(p.alpha) +
                             ((((size_t)s * p.mt + R_) * npg + pg_) * kTileRows + lane) * (SP * HPK);
#pragma unroll
          for (int e = 0; e < SP * HPK; ++e) dst[e] = __ldg(src + e);
        }
      }
    };

    if (busy) {
      load_scales(t_cur, ti_cur, 0, sc_cur);
      static_for(std::make_integer_sequence<int, NA - 1>{}, [&]<int D>() {
        load_alpha.template operator()<D>(t_cur, D, ti_cur.y);
      });
      int steps_per_unit_ = steps_per_unit;
      bool more = dyn;        // grabs may still succeed
      unsigned pend = 0;      // lane 0: raw count returned by the pending grab
      bool nxt_pending = false;

      for (int k = 0; !failed; ++k) {
        // Tile k is t_cur.  Tile k+1 is first needed NEED steps into tile k
        // (alpha prefetch or ring refill).  When that leaves time for the
        // atomic's round trip, tile k+1 is grabbed now and read at step NEED,
        // so a warp holds at most one tile that no other warp can take.
        // Otherwise tile k+1 is already known (t_nxt) and k+2 is grabbed now.
        bool grabbing;
        if constexpr (AHEAD1) {
          t_nxt = (dyn && k >= 1) ? -1 : static_tile(k + 1);
          grabbing = dyn && more && k >= 1;
          nxt_pending = grabbing;
        } else {
          grabbing = dyn && more && t_nxt >= 0;
        }
        if (grabbing && lane == 0) pend = atomicAdd(tile_ctr, 1u);
        if constexpr (MIXED) {
          npg_t = (int)((ti_cur.y + 1u) >> 1);
          steps_per_unit_ = 8 * npg_t;
          chunks_per_unit = CPT * npg_t;
        }
        const int R = t_cur;
        const int row = R * kTileRows + lane;
        float yacc = 0.f;
        // Mixed storage: this lane's row's outliers in this slice are the
        // entries [o0, o1), in input order.  The first six are pipelined over
        // the steps of the first pass (entry t read at step t, its x at step
        // t + 2, added at step t + 3), the rest follow the pass.  w * x is
        // exact in fp32, and the sum runs in entry order.
        uint32_t o0 = or_cur.x, o1 = or_cur.y;
        uint32_t oq[6] = {0u, 0u, 0u, 0u, 0u, 0u};   // entries, then (w bits << 16) | x bits
        float osum = 0.f;
        if constexpr (MIXED) {
          if (o1 < o0 || o1 > p.nnz) {
            atomicOr(p.status, kStatusFormat);
            o1 = o0;
          }
        }
        auto outlier_x = [&](uint32_t v) -> uint32_t {
          const uint32_t kin = v & 0xFFFFu, k = (uint32_t)s * kSliceInputs + kin;
          if (kin >= (uint32_t)kSliceInputs || k >= (uint32_t)p.n) {
            atomicOr(p.status, kStatusFormat);
            return 0u;
          }
          const uint32_t xb = __ldg(reinterpret_cast<const unsigned short*>(p.x) + (size_t)b * p.n + k);
          return (v & 0xFFFF0000u) | xb;
        };
        auto outlier_add = [&](uint32_t wx) {
          osum = fmaf(h2f((uint16_t)(wx >> 16)), h2f((uint16_t)(wx & 0xFFFFu)), osum);
        };
        // Mixed storage: the tile after next, settled at step 4 of the first
        // pass (its grab went out at the top of this tile), so that its
        // block-table entry and outlier range are read a whole tile before
        // its copies are issued.
        int t_aft = -1;
        bool aft_known = false;
        uint2 ti_aft = make_uint2(0u, 0u), or_aft = make_uint2(0u, 0u);
        for (int pg = 0; pg < npg_t && !failed; ++pg) {
          static_for(std::make_integer_sequence<int, 8>{}, [&]<int U>() {
            if (failed) return;
            const int j = pg * 8 + U;          // step within the unit
            if constexpr (AHEAD1) {
              if (j == NEED && nxt_pending) {
                int tile = -1;
                if (lane == 0) {
                  const long long t = dyn_base + pend;
                  tile = t < p.mt ? (int)t : -1;
                }
                t_nxt = __shfl_sync(0xffffffffu, tile, 0);
                more = t_nxt >= 0;
                nxt_pending = false;
              }
            }
            if constexpr (PK && U == 0) {
              // Scales of the next pass: this tile's next plane group, or the
              // next tile's first.
              if (pg + 1 < npg_t) load_scales(t_cur, ti_cur, pg + 1, sc_nxt);
              else if (t_nxt >= 0) load_scales(t_nxt, ti_nxt, 0, sc_nxt);
              // Mixed storage: a pass with one plane came as 8 * HPK scales;
              // place them where the two-plane order reads plane 0.
              if constexpr (MIXED) {
                if (ti_cur.y - 2u * (uint32_t)pg == 1u) spread_scales<HPK>(sc_cur);
              }
            }
            {
              const int ja = j + NA - 1;       // scales NA-1 steps ahead
              if (ja < steps_per_unit_) load_alpha.template operator()<(U + NA - 1) % NA>(t_cur, ja, ti_cur.y);
              else if (t_nxt >= 0)
                load_alpha.template operator()<(U + NA - 1) % NA>(t_nxt, ja - steps_per_unit_, ti_nxt.y);
            }
            if constexpr (MIXED) {
              if (pg == 0) {
                if constexpr (U <= 5) {
                  if (o0 + U < o1) oq[U] = __ldg(p.oent + o0 + U);
                }
                if constexpr (U >= 2 && U - 2 <= 5) {
                  if (o0 + (U - 2) < o1) oq[U - 2] = outlier_x(oq[U - 2]);
                }
                if constexpr (U >= 3 && U - 3 <= 5) {
                  if (o0 + (U - 3) < o1) outlier_add(oq[U - 3]);
                }
                if constexpr (U == 4) {
                  if (dyn) {
                    if (grabbing) {
                      int tile = -1;
                      if (lane == 0) {
                        const long long t = dyn_base + pend;
                        tile = t < p.mt ? (int)t : -1;
                      }
                      t_aft = __shfl_sync(0xffffffffu, tile, 0);
                      more = t_aft >= 0;
                    }
                  } else {
                    t_aft = static_tile(k + 2);
                  }
                  if (t_aft >= 0) {
                    ti_aft = tile_info(t_aft);
                    or_aft = outlier_range(t_aft);
                  }
                  aft_known = true;
                }
              }
            }

            // Pieces of a whole stage (CH steps) come out of the ring at its
            // first step; the stage is refilled (S copies ahead) right away, so
            // S full copies are in flight while the steps are computed.
            if constexpr (U % CH == 0) {
              const bool ok = __all_sync(0xffffffffu, p.stall_test ? mbar_wait(dead_bar, 0u, 1000000ull)
                                                                   : mbar_wait(bars + 8u * st, ph));
              if (!ok) {
                failed = true;
                if (lane == 0) atomicOr(p.status, kStatusTimeout);
                return;
              }
              const uint32_t src = ring + (uint32_t)st * STAGE_BYTES + (uint32_t)lane * 16u;
              // A mixed pass with one plane packs its steps 512 bytes apart.
              const uint32_t step_stride =
                  MIXED ? 512u * min(2u, ti_cur.y - 2u * (uint32_t)pg) : STEP_BYTES;
#pragma unroll
              for (int h = 0; h < CH; ++h)
#pragma unroll
                for (int i = 0; i < SP; ++i) {
                  const bool live =
                      (!MULTI || (pg * 4 + i < p.q)) && (!MIXED || (uint32_t)(pg * GP + i) < ti_cur.y);
                  wst[h][i] = live ? lds128(src + (uint32_t)h * step_stride + 512u * i) : make_uint4(0, 0, 0, 0);
                }
              __syncwarp();
              const int cn = j / CH + S;       // chunk to fetch into the freed stage
              if (cn < chunks_per_unit) {
                if (lane == 0) issue(t_cur, ti_cur, cn, st);
              } else if (t_nxt >= 0) {
                if (lane == 0) issue(t_nxt, ti_nxt, cn - chunks_per_unit, st);
              } else {
                --outstanding;
              }
              st = st + 1 == S ? 0 : st + 1;
              if (st == 0) ph ^= 1u;
            }
            const uint4 (&wv)[SP] = wst[U % CH];

            constexpr uint32_t IMM = step_imm<U>();
            constexpr int u2 = U >> 2;
            [[maybe_unused]] const int P = U ^ (int)(4 * a);
#pragma unroll
            for (int i = 0; i < Q; ++i) {
              if (MULTI && pg * 4 + i >= p.q) continue;
              if (MIXED && (uint32_t)(pg * GP + i) >= ti_cur.y) continue;
              const uint4 w4 = wv[i];
              if constexpr (RUN == 16) {
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) lookup_word<IMM>(word_of(w4, kk), colb[u2][kk], acc0, acc1);
                float al;
                if constexpr (PK) {
                  const int h = U * SP + i;       // half h of the lane's pass scales (unrolled: constant)
                  const uint32_t w2 = word_of(sc_cur[h / 8], (h / 2) % 4);
                  al = h2f((uint16_t)((h & 1) ? (w2 >> 16) : (w2 & 0xffffu)));
                } else {
                  al = h2f(ab[U % NA][i][0]);
                }
                yacc = fmaf(al, acc0 + acc1, yacc);
              } else if constexpr (RUN == 8) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                  float acc0 = 0.f, acc1 = 0.f;
                  lookup_word<IMM>(word_of(w4, 2 * r), colb[u2][2 * r], acc0, acc1);
                  lookup_word<IMM>(word_of(w4, 2 * r + 1), colb[u2][2 * r + 1], acc0, acc1);
                  float al;
                  if constexpr (PK) {
                    // Both halves of (step U, plane i) share one 32-bit word;
                    // run pair r of this lane is half r xor (lam >> 3).
                    const int wi = U * SP + i;   // unrolled: a constant
                    const uint32_t w2 = word_of(sc_cur[wi / 4], wi % 4);
                    al = h2f((uint16_t)(((uint32_t)r ^ (lam >> 3)) ? (w2 >> 16) : (w2 & 0xffffu)));
                  } else {
                    al = h2f(ab[U % NA][i][r]);
                  }
                  yacc = fmaf(al, acc0 + acc1, yacc);
                }
              } else {
                // One scale per run: group of run c is (1024 s + 8 c) / g.
                const __half* ap = p.alpha + (size_t)(pg * GP + i) * plane_stride + row;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  float v[4];
                  lookup_word_values<IMM>(word_of(w4, kk), colb[u2][kk], v);
#pragma unroll
                  for (int t = 0; t < 4; ++t) {
                    const int c = 16 * P + ((4 * kk + t) ^ (int)lam);
                    const int G = MODE == kG8 ? 128 * s + c : (s * kSliceInputs + 8 * c) / p.g;
                    const float al = (row < p.m && G < p.ng) ? h2f(ld_u16(ap + (size_t)G * p.m)) : 0.f;
                    yacc = fmaf(al, v[t], yacc);
                  }
                }
              }
            }
            // Offset of converted uniform weights: offset[G][row] * (sum of x over the run).
            if constexpr (HAS_OFF) {
              if (pg == 0) {
                if constexpr (RUN >= 8) {
#pragma unroll
                  for (int r = 0; r < APP; ++r) {
                    const int nat = RUN == 16 ? P : 2 * P + (r ^ (int)(lam >> 3));
                    yacc = fmaf(ob[U % NA][r], run_sum[nat], yacc);
                  }
                } else {
#pragma unroll
                  for (int jj = 0; jj < 16; ++jj) {
                    const int c = 16 * P + (jj ^ (int)lam);
                    const int G = MODE == kG8 ? 128 * s + c : (s * kSliceInputs + 8 * c) / p.g;
                    const float of = (row < p.m && G < p.ng) ? __ldg(p.offset + (size_t)G * p.m + row) : 0.f;
                    yacc = fmaf(of, chunk_sum[c], yacc);
                  }
                }
              }
            }
          });
          if constexpr (PK) {
#pragma unroll
            for (int e = 0; e < SP * HPK; ++e) sc_cur[e] = sc_nxt[e];
          }
          if constexpr (MIXED) {
            // Entries beyond the pipelined ones, after the first pass.
            if (pg == 0 && !failed) {
              if (o0 + 5u < o1) outlier_add(oq[5]);
              for (uint32_t e = o0 + 6u; e < o1; ++e) outlier_add(outlier_x(__ldg(p.oent + e)));
            }
          }
        }
        if (failed) break;
        // Mixed storage: the row's outliers, after its planes.
        if constexpr (MIXED) yacc += osum;
        // One slice: the row's sum is y.  Several: this slice's partial, summed
        // over slices by the split-K reduce kernel that follows.
        if (p.ns == 1) {
          if (row < p.m) {
            const size_t o = (size_t)b * p.m + row;
            if (p.y_f16) reinterpret_cast<__half*>(p.y)[o] = __float2half_rn(yacc);
            else reinterpret_cast<float*>(p.y)[o] = yacc;
          }
        } else {
          p.part[((size_t)((long long)b * p.ns + s) * p.mt + R) * kTileRows + lane] = yacc;
        }

        // Advance: tile k+2 comes from the grab (dynamic) or the static list.
        if (t_nxt < 0) break;
        if constexpr (AHEAD1) {
          t_cur = t_nxt;
          ti_cur = ti_nxt;
          or_cur = or_nxt;
          continue;
        }
        int t_after = -1;
        if (MIXED && aft_known) {
          t_after = t_aft;
        } else if (dyn) {
          if (grabbing) {
            int tile = -1;
            if (lane == 0) {
              const long long t = dyn_base + pend;
              tile = t < p.mt ? (int)t : -1;
            }
            t_after = __shfl_sync(0xffffffffu, tile, 0);
            more = t_after >= 0;
          }
        } else {
          t_after = static_tile(k + 2);
        }
        t_cur = t_nxt;
        t_nxt = t_after;
        ti_cur = ti_nxt;
        or_cur = or_nxt;
        if (MIXED && aft_known) {
          ti_nxt = ti_aft;
          or_nxt = or_aft;
        } else if (t_nxt >= 0) {
          ti_nxt = tile_info(t_nxt);
          or_nxt = outlier_range(t_nxt);
        }
      }
    }
  }

  // Segment-aligned mode: the last CTA to finish resets the tile counters.
  if (p.seg_aligned) {
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned* done = p.tile_cnt + (kMaxTileCounters - 1);
      __threadfence();
      if (atomicAdd(done, 1u) == gridDim.x - 1) {
        for (long long z = 0; z < Z; ++z) p.tile_cnt[z] = 0u;
        *done = 0u;
      }
    }
  }

  // After a timeout, let copies still in flight land before the CTA exits
  // (each wait bounded again).
  if (failed) {
    for (int k = 0; k < outstanding; ++k) {
      (void)mbar_wait(bars + 8u * st, ph);
      st = st + 1 == S ? 0 : st + 1;
      if (st == 0) ph ^= 1u;
    }
  }
}

// Kernel for (mode, offsets, unit-major scales); unit-major scales exist
// for the modes with one or two scales per piece (g % 128 == 0, g == 64).
#define LUTGEMM_RUN_SELECT_OFF(Qv, MULTIv, OFFv)                                   \
  switch (mode) {                                                                  \
    case kG128:                                                                    \
      return packed ? lut_gemm_kernel<Qv, kG128, MULTIv, OFFv, true>               \
                    : lut_gemm_kernel<Qv, kG128, MULTIv, OFFv, false>;             \
    case kG128x:                                                                   \
      return packed ? lut_gemm_kernel<Qv, kG128x, MULTIv, OFFv, true>              \
                    : lut_gemm_kernel<Qv, kG128x, MULTIv, OFFv, false>;            \
    case kG64:                                                                     \
      return packed ? lut_gemm_kernel<Qv, kG64, MULTIv, OFFv, true>                \
                    : lut_gemm_kernel<Qv, kG64, MULTIv, OFFv, false>;              \
    case kG8: return packed ? nullptr : lut_gemm_kernel<Qv, kG8, MULTIv, OFFv, false>;   \
    default: return packed ? nullptr : lut_gemm_kernel<Qv, kGAny, MULTIv, OFFv, false>;  \
  }

#define LUTGEMM_RUN_SELECT(Qv, MULTIv)                                             \
  if (has_offset) {                                                                \
    LUTGEMM_RUN_SELECT_OFF(Qv, MULTIv, true)                                       \
  } else {                                                                         \
    LUTGEMM_RUN_SELECT_OFF(Qv, MULTIv, false)                                      \
  }

}  // namespace lutgemm
