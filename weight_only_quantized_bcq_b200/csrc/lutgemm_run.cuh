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
//   * One persistent 512-thread CTA per SM.  The work is the linear list of
//     units (batch column, slice, 32-row tile), cut into one contiguous range
//     per CTA.  A range crosses at most a few (batch column, slice) segments;
//     the CTA rebuilds the 128 KB fp32 tables of a slice once per segment.
//   * A warp processes a unit, one output row per lane.  Per step U (8 steps
//     per unit) a lane reads one 16-byte piece per plane with a streaming
//     128-bit load; the packed layout makes each warp load 512 contiguous
//     bytes.  Loads run NB-1 steps ahead in registers, across unit
//     boundaries; a warp's first loads of a segment are issued before the
//     table build so that their latency overlaps it.
//   * Table reads are conflict-free: at every step the 32 lanes read 32
//     distinct banks.  Lanes 0-15 and 16-31 walk the 8 pieces of the slice
//     four apart, and lane l reads the runs of its piece in the order
//     j xor (l mod 16), so (piece half, run) is a bijection onto banks.
//   * A table read is one PRMT that places the sign byte (pattern p, times
//     256) next to the lane's column byte, one LDS whose immediate carries the
//     table base, half and band, and one FADD.
//   * Per-group alpha (and offset) are applied once per piece (g = 128),
//     per half-piece (g = 64) or per run (other g).
//   * Split-K: each unit stores its fp32 partial.  When a warp has finished
//     its units of a segment it fences once and bumps the arrival counters of
//     those row tiles (one lane per tile); the last arrival for a tile (no
//     waiting anywhere) sums the slices in fixed order, writes y and resets
//     the counter.
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

// 16 bytes of packed planes; each byte is read exactly once, so skip L1.
__device__ __forceinline__ uint4 ld_stream16(const uint8_t* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}

__device__ __forceinline__ uint16_t ld_u16(const __half* ptr) {
  return __ldg(reinterpret_cast<const unsigned short*>(ptr));
}

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ uint32_t word_of(const uint4& v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
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

template <int... Is, class F>
__device__ __forceinline__ void static_for(std::integer_sequence<int, Is...>, F&& f) {
  (f.template operator()<Is>(), ...);
}

}  // namespace detail

template <int Q, int MODE, bool MULTI, bool HAS_OFF, int NB>
__global__ void __launch_bounds__(kThreads, 1) lut_gemm_kernel(const RunParams p) {
  using namespace detail;
  static_assert(NB == 2 || NB == 4 || NB == 8, "pipeline stages must divide the 8 steps of a unit");
  extern __shared__ __align__(16) unsigned char smem[];
  const uint32_t r0 = (uint32_t)__cvta_generic_to_shared(smem);
  if (r0 > kTableBase) {  // uniform over the CTA: the tables would not fit the allocation
    if (threadIdx.x == 0) atomicOr(p.status, 1u);
    return;
  }
  float* const chunk_sum = reinterpret_cast<float*>(smem + (kMiscBase - r0));
  float* const run_sum = chunk_sum + kRunsPerSlice;

  // Runs (8-input table columns) that share one alpha inside a piece.
  constexpr int RUN = (MODE == kG128 || MODE == kG128x) ? 16 : (MODE == kG64 ? 8 : 1);
  constexpr int APP = RUN >= 8 ? 16 / RUN : 1;      // prefetched scales per piece
  constexpr bool PRE_ALPHA = RUN >= 8;

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

  const int npg = MULTI ? (p.q + 3) >> 2 : 1;
  const size_t plane_stride = (size_t)p.ng * (size_t)p.m;
  const uint32_t unit_bytes = (uint32_t)p.q * kBlockBytes;

  const long long total = p.total_units;
  const long long u_begin = (long long)blockIdx.x * total / gridDim.x;
  const long long u_end = (long long)(blockIdx.x + 1) * total / gridDim.x;

  uint4 wb[NB][Q];
  uint16_t ab[NB][Q][APP];
  float ob[NB][APP];

  for (long long u = u_begin; u < u_end;) {
    const long long seg = u / p.mt;
    const int b = (int)(seg / p.ns);
    const int s = (int)(seg - (long long)b * p.ns);
    const long long seg_first = seg * p.mt;
    const long long seg_end = min(u_end, seg_first + p.mt);
    const uint8_t* slice_base = p.packed + (size_t)s * p.mt * unit_bytes;
    const long long first_unit = u + warp;
    const bool busy = first_unit < seg_end;

    // Loads of one step into stage SLOT: the Q 16-byte pieces and, when
    // prefetched, the alpha (and offset) values the step will need.
    auto load_step = [&]<int SLOT>(int R_, int pg_, int U_) {
      const uint8_t* src = slice_base + ((size_t)R_ * p.q + (size_t)pg_ * 4) * kBlockBytes +
                           U_ * 512 + lane * 16;
#pragma unroll
      for (int i = 0; i < Q; ++i) {
        const bool live = !MULTI || (pg_ * 4 + i < p.q);
        if (live) wb[SLOT][i] = ld_stream16(src + (size_t)i * kBlockBytes);
      }
      if constexpr (PRE_ALPHA) {
        const int row = R_ * kTileRows + lane;
        const int P = U_ ^ (int)(4 * a);
#pragma unroll
        for (int r = 0; r < APP; ++r) {
          int G;
          if constexpr (MODE == kG128) G = 8 * s + P;
          else if constexpr (MODE == kG128x) G = (8 * s + P) / (p.g >> 7);
          else G = 16 * s + 2 * P + (r ^ (int)(lam >> 3));
          const bool ok = row < p.m && G < p.ng;
          const __half* ap = p.alpha + (size_t)G * p.m + row;
#pragma unroll
          for (int i = 0; i < Q; ++i) {
            const bool live = !MULTI || (pg_ * 4 + i < p.q);
            ab[SLOT][i][r] = (ok && live) ? ld_u16(ap + (size_t)(pg_ * 4 + i) * plane_stride) : (uint16_t)0;
          }
          if constexpr (HAS_OFF) ob[SLOT][r] = (ok && pg_ == 0) ? __ldg(p.offset + (size_t)G * p.m + row) : 0.f;
        }
      }
    };

    // The first NB-1 steps of this warp's first unit go out before the tables
    // are built; they do not touch shared memory.
    int R = busy ? (int)(first_unit - seg_first) : 0;
    if (busy)
      static_for(std::make_integer_sequence<int, NB - 1>{}, [&]<int D>() { load_step.template operator()<D>(R, 0, D); });
    __syncthreads();  // every warp is done with the previous segment's tables
    build_tables<RUN, HAS_OFF>(p, b, s, chunk_sum, run_sum);

    if (busy) {
      long long unit = first_unit;
      int pg = 0;
      float yacc = 0.f;
      while (true) {
        int next_pg = pg + 1;
        long long next_unit = unit;
        if (next_pg >= npg) {
          next_pg = 0;
          next_unit = unit + kWarps;
        }
        const bool has_next = next_unit < seg_end;
        const int next_R = has_next ? (int)(next_unit - seg_first) : 0;
        const int row = R * kTileRows + lane;

        static_for(std::make_integer_sequence<int, 8>{}, [&]<int U>() {
          constexpr int LU = U + NB - 1;          // step whose loads are issued now
          if constexpr (LU < 8) load_step.template operator()<LU % NB>(R, pg, LU);
          else if (has_next) load_step.template operator()<LU % NB>(next_R, next_pg, LU - 8);

          constexpr uint32_t IMM = step_imm<U>();
          constexpr int u2 = U >> 2;
          const int P = U ^ (int)(4 * a);
#pragma unroll
          for (int i = 0; i < Q; ++i) {
            if (MULTI && pg * 4 + i >= p.q) continue;
            const uint4 w4 = wb[U % NB][i];
            if constexpr (RUN == 16) {
              float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
              for (int k = 0; k < 4; ++k) lookup_word<IMM>(word_of(w4, k), colb[u2][k], acc0, acc1);
              yacc = fmaf(h2f(ab[U % NB][i][0]), acc0 + acc1, yacc);
            } else if constexpr (RUN == 8) {
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                float acc0 = 0.f, acc1 = 0.f;
                lookup_word<IMM>(word_of(w4, 2 * r), colb[u2][2 * r], acc0, acc1);
                lookup_word<IMM>(word_of(w4, 2 * r + 1), colb[u2][2 * r + 1], acc0, acc1);
                yacc = fmaf(h2f(ab[U % NB][i][r]), acc0 + acc1, yacc);
              }
            } else {
              // One scale per run: group of run c is (1024 s + 8 c) / g.
              const __half* ap = p.alpha + (size_t)(pg * 4 + i) * plane_stride + row;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                float v[4];
                lookup_word_values<IMM>(word_of(w4, k), colb[u2][k], v);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  const int c = 16 * P + ((4 * k + t) ^ (int)lam);
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
                  yacc = fmaf(ob[U % NB][r], run_sum[nat], yacc);
                }
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  const int c = 16 * P + (j ^ (int)lam);
                  const int G = MODE == kG8 ? 128 * s + c : (s * kSliceInputs + 8 * c) / p.g;
                  const float of = (row < p.m && G < p.ng) ? __ldg(p.offset + (size_t)G * p.m + row) : 0.f;
                  yacc = fmaf(of, chunk_sum[c], yacc);
                }
              }
            }
          }
        });

        if (pg == npg - 1) {
          // This slice's partial sum of the row tile; published below.
          p.part[((size_t)((long long)b * p.ns + s) * p.mt + R) * kTileRows + lane] = yacc;
          yacc = 0.f;
        }
        if (!has_next) break;
        unit = next_unit;
        R = next_R;
        pg = next_pg;
      }

      // Split-K arrival: one fence for all of this warp's partials, then one
      // lane per row tile bumps the tile's counter.  The last arrival sums the
      // slices in slice order, writes y and resets the counter.
      __threadfence();
      const int nunits = (int)((seg_end - 1 - first_unit) / kWarps) + 1;
      for (int k0 = 0; k0 < nunits; k0 += 32) {
        const int k = k0 + lane;
        int Rk = 0;
        unsigned prev = 0;
        if (k < nunits) {
          Rk = (int)(first_unit + (long long)k * kWarps - seg_first);
          prev = atomicAdd(p.cnt + (size_t)b * p.mt + Rk, 1u);
        }
        unsigned last = __ballot_sync(0xffffffffu, k < nunits && prev == (unsigned)(p.ns - 1));
        if (last) __threadfence();
        while (last) {
          const int src = __ffs(last) - 1;
          last &= last - 1;
          const int Rt = __shfl_sync(0xffffffffu, Rk, src);
          const float* col = p.part + ((size_t)b * p.ns * p.mt + Rt) * kTileRows + lane;
          float sum = 0.f;
          for (int s2 = 0; s2 < p.ns; ++s2) sum += __ldcg(col + (size_t)s2 * p.mt * kTileRows);
          const int row = Rt * kTileRows + lane;
          if (row < p.m) {
            const size_t o = (size_t)b * p.m + row;
            if (p.y_f16) reinterpret_cast<__half*>(p.y)[o] = __float2half_rn(sum);
            else reinterpret_cast<float*>(p.y)[o] = sum;
          }
          if (lane == 0) p.cnt[(size_t)b * p.mt + Rt] = 0u;
        }
      }
    }
    u = seg_end;
  }
}

#define LUTGEMM_RUN_SELECT_OFF(Qv, MULTIv, OFFv, NBv)                              \
  switch (mode) {                                                                  \
    case kG128: return lut_gemm_kernel<Qv, kG128, MULTIv, OFFv, NBv>;              \
    case kG128x: return lut_gemm_kernel<Qv, kG128x, MULTIv, OFFv, NBv>;            \
    case kG64: return lut_gemm_kernel<Qv, kG64, MULTIv, OFFv, NBv>;                \
    case kG8: return lut_gemm_kernel<Qv, kG8, MULTIv, OFFv, NBv>;                  \
    default: return lut_gemm_kernel<Qv, kGAny, MULTIv, OFFv, NBv>;                 \
  }

#define LUTGEMM_RUN_SELECT(Qv, MULTIv, NBv)                                        \
  if (has_offset) {                                                                \
    LUTGEMM_RUN_SELECT_OFF(Qv, MULTIv, true, NBv)                                  \
  } else {                                                                         \
    LUTGEMM_RUN_SELECT_OFF(Qv, MULTIv, false, NBv)                                 \
  }

}  // namespace lutgemm
