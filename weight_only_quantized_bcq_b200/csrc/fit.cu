// BCQ fitting on the GPU: FP16 weights -> q sign planes and group scales, the
// step that produces the weights the lookup kernel consumes.
//
// Source: LUT-GEMM card (Elamur), Summary (weights are stored in BCQ: q
// binary planes with group-wise scales) and its reference 48 ("Alternating
// multi-bit quantization"), which the pages cite without detail.  Per (row,
// group of g inputs):
//   1. greedy: r = w; for each plane i: beta_i = sign(r) (0 -> +1),
//      alpha_i = mean(beta_i * r), r -= alpha_i * beta_i;
//   2. `iters` rounds of a least-squares scale step (Cholesky of B^T B, whose
//      entries are exact integer counts; a pivot <= 1e-6 g keeps the previous
//      scales) and a nearest-code sign step (ties: the largest code, bit i of
//      a code meaning beta_i = +1);
//   3. scales rounded to fp16, then a last sign step with the rounded scales.
//
// With GRID (the variable grid: the planes plus one constant per group,
// w ~ off + sum_i alpha_i beta_i; BPDQ card: grids from bit-planes and scalar
// coefficients) the greedy pass starts from the group mean, the least-squares
// step adds a column of ones (its normal-matrix entries are again exact
// integer counts: sum_k beta_ik = 2 #(+1) - g, and g), the codes are
// off + sum_i +-alpha_i, and the constant is stored in fp32 (the offset type
// of lutgemm_run).
//
// A group is served by a segment of lpg lanes (the power of two at or above
// g/8, at most 32), so a warp serves 32/lpg groups at once (two at g = 128);
// a lane holds up to CPL chunks of 8 consecutive inputs (g <= 256 * CPL).  A chunk's signs are one mask with byte i = plane
// i (32 bits for q <= 4).  The 2^q code values sit in registers for q <= 4
// and in shared memory above; a code's mask bits are compile-time constants,
// so the nearest-code search carries them directly.  Sums are taken in a
// fixed order (per lane in input order, then a butterfly over the warp), so
// results are reproducible.
#include <type_traits>

#include "lutgemm.h"
#include "lutgemm_common.cuh"

namespace lutgemm {

namespace {

constexpr int kFitWarps = 8;
constexpr float kPivotRel = 1e-6f;

// Sum over an aligned segment of lpg lanes (every lane gets the segment's sum).
__device__ __forceinline__ float seg_sum(float v, int lpg) {
  for (int o = lpg >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int seg_sum_i(int v, int lpg) {
  for (int o = lpg >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Code c's sign bits spread to bit 8*i (plane i), element 0.
__host__ __device__ constexpr uint64_t spread_code(int c, int q) {
  uint64_t m = 0;
  for (int i = 0; i < q; ++i) m |= (uint64_t)((c >> i) & 1) << (8 * i);
  return m;
}

// Eight 0/1 bits -> eight int8 values +1 / -1 (two 32-bit words).
__device__ __forceinline__ uint2 bits_to_signs(uint32_t b) {
  const uint32_t lo = ((b & 0xFu) * 0x00204081u) & 0x01010101u;
  const uint32_t hi = (((b >> 4) & 0xFu) * 0x00204081u) & 0x01010101u;
  return make_uint2(0xFFFFFFFFu ^ (lo * 0xFEu), 0xFFFFFFFFu ^ (hi * 0xFEu));
}

template <int CPL, int Q, bool GRID>
__global__ void __launch_bounds__(kFitWarps * 32) fit_bcq_kernel(const __half* __restrict__ w, int m, int n, int g,
                                                               int lpg, int iters, int8_t* __restrict__ signs,
                                                               __half* __restrict__ alpha, float* __restrict__ offset,
                                                               float* __restrict__ err) {
  constexpr int D = Q + (GRID ? 1 : 0);   // least-squares unknowns: the planes' scales (+ the constant)
  using Mask = std::conditional_t<(Q <= 4), uint32_t, uint64_t>;
  constexpr int NC = 1 << Q;
  constexpr bool REG_CODES = Q <= 4;
  __shared__ float codebook[REG_CODES ? 1 : kFitWarps][REG_CODES ? 1 : NC];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int ng = n / g;
  const int chunks = g / 8;
  const int gpw = 32 / lpg;                  // groups per warp
  const int sl = lane & (lpg - 1);           // lane within its segment
  const long long groups = (long long)m * ng;
  const float inv_g = 1.0f / (float)g;

  // Warp-uniform loop; a segment whose group is past the end computes on
  // zeros and stores nothing.
  for (long long base = ((long long)blockIdx.x * kFitWarps + wid) * gpw; base < groups;
       base += (long long)gridDim.x * kFitWarps * gpw) {
    const long long grp = base + lane / lpg;
    const bool live = grp < groups;
    const int j = live ? (int)(grp / ng) : 0;
    const int G = live ? (int)(grp - (long long)j * ng) : 0;
    const __half* src = w + (size_t)j * n + (size_t)G * g;

    float x[CPL][8];
    Mask sg[CPL];
#pragma unroll
    for (int t = 0; t < CPL; ++t) {
      sg[t] = 0;
      const int c = sl + lpg * t;
      if (live && c < chunks) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src) + c);
        const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(h[e]);
          x[t][2 * e] = f.x;
          x[t][2 * e + 1] = f.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[t][e] = 0.f;
      }
    }

    // 1. Greedy planes on the residual (from the group mean on a grid).
    float a[Q];
    float off = 0.f;
    if constexpr (GRID) {
      float s = 0.f;
#pragma unroll
      for (int t = 0; t < CPL; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) s += x[t][e];
      off = seg_sum(s, lpg) * inv_g;
    }
    {
      float r[CPL][8];
#pragma unroll
      for (int t = 0; t < CPL; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) r[t][e] = x[t][e] - off;
#pragma unroll
      for (int i = 0; i < Q; ++i) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < CPL; ++t) {
          if (!live || sl + lpg * t >= chunks) continue;
          Mask bits = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            bits |= (Mask)(r[t][e] >= 0.f) << e;
            s += fabsf(r[t][e]);
          }
          sg[t] |= bits << (8 * i);
        }
        const float ai = seg_sum(s, lpg) * inv_g;
        a[i] = ai;
#pragma unroll
        for (int t = 0; t < CPL; ++t)
#pragma unroll
          for (int e = 0; e < 8; ++e) r[t][e] -= ((sg[t] >> (8 * i + e)) & 1) ? ai : -ai;
      }
    }

    // Nearest-code step for scales av; returns this lane's sum of squared
    // distances (the group error once the scales are final).
    auto sign_step = [&](const float (&av)[Q], float ov) -> float {
      float cb[REG_CODES ? NC : 1];
      if constexpr (REG_CODES) {
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          float v = ov;
#pragma unroll
          for (int i = 0; i < Q; ++i) v += ((c >> i) & 1) ? av[i] : -av[i];
          cb[c] = v;
        }
      } else {
        __syncwarp();
        for (int c = lane; c < NC; c += 32) {
          float v = ov;
#pragma unroll
          for (int i = 0; i < Q; ++i) v += ((c >> i) & 1) ? av[i] : -av[i];
          codebook[wid][c] = v;
        }
        __syncwarp();
      }
      float e2 = 0.f;
#pragma unroll
      for (int t = 0; t < CPL; ++t) {
        if (!live || sl + lpg * t >= chunks) continue;
        Mask mk = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xv = x[t][e];
          float best;
          Mask arg = 0;
          if constexpr (REG_CODES) {
            best = fabsf(xv - cb[0]);
#pragma unroll
            for (int c = 1; c < NC; ++c) {
              const float d = fabsf(xv - cb[c]);
              if (d <= best) {
                best = d;
                arg = (Mask)spread_code(c, Q);
              }
            }
          } else {
            best = fabsf(xv - codebook[wid][0]);
            int ac = 0;
            for (int c = 1; c < NC; ++c) {
              const float d = fabsf(xv - codebook[wid][c]);
              if (d <= best) {
                best = d;
                ac = c;
              }
            }
#pragma unroll
            for (int i = 0; i < Q; ++i) arg |= (Mask)((ac >> i) & 1) << (8 * i);
          }
          mk |= arg << e;
          e2 += best * best;
        }
        sg[t] = mk;
      }
      return e2;
    };

    // 2. Alternating rounds.
    for (int it = 0; it < iters; ++it) {
      // Normal equations: M_ik = g - 2 * #(inputs where planes i and k differ),
      // v_i = sum_k beta_ik * w_k; on a grid also M_iq = 2 #(beta_i = +1) - g,
      // M_qq = g and v_q = sum_k w_k.
      int diff[Q * (Q - 1) / 2 + 1];
      int plus[Q] = {};
      float v[D];
#pragma unroll
      for (int i = 0; i < Q; ++i) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < CPL; ++t) {
          if (!live || sl + lpg * t >= chunks) continue;
#pragma unroll
          for (int e = 0; e < 8; ++e) s += ((sg[t] >> (8 * i + e)) & 1) ? x[t][e] : -x[t][e];
        }
        v[i] = seg_sum(s, lpg);
#pragma unroll
        for (int k = 0; k < i; ++k) {
          int cnt = 0;
#pragma unroll
          for (int t = 0; t < CPL; ++t) {
            if (!live || sl + lpg * t >= chunks) continue;
            cnt += __popc((uint32_t)(((sg[t] >> (8 * i)) ^ (sg[t] >> (8 * k))) & 0xFFu));
          }
          diff[i * (i - 1) / 2 + k] = seg_sum_i(cnt, lpg);
        }
        if constexpr (GRID) {
          int cnt = 0;
#pragma unroll
          for (int t = 0; t < CPL; ++t) {
            if (!live || sl + lpg * t >= chunks) continue;
            cnt += __popc((uint32_t)((sg[t] >> (8 * i)) & 0xFFu));
          }
          plus[i] = seg_sum_i(cnt, lpg);
        }
      }
      if constexpr (GRID) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < CPL; ++t)
#pragma unroll
          for (int e = 0; e < 8; ++e) s += x[t][e];
        v[Q] = seg_sum(s, lpg);
      }
      // Entry (i, k) of the normal matrix, i >= k.
      auto mij = [&](int i, int k) -> float {
        if (i < Q) return (i == k) ? (float)g : (float)(g - 2 * diff[i * (i - 1) / 2 + k]);
        return (k < Q) ? (float)(2 * plus[k] - g) : (float)g;
      };
      // Cholesky of M (every lane, same arithmetic), then two triangular solves.
      float L[D][D];
      bool ok = true;
#pragma unroll
      for (int i = 0; i < D; ++i) {
#pragma unroll
        for (int k = 0; k <= i; ++k) {
          float acc = mij(i, k);
#pragma unroll
          for (int l = 0; l < k; ++l) acc -= L[i][l] * L[k][l];
          if (i == k) {
            ok = ok && acc > kPivotRel * (float)g;
            L[i][i] = sqrtf(fmaxf(acc, kPivotRel * (float)g));
          } else {
            L[i][k] = acc / L[k][k];
          }
        }
      }
      if (ok) {
        float y[D], sol[D];
#pragma unroll
        for (int i = 0; i < D; ++i) {
          float acc = v[i];
#pragma unroll
          for (int l = 0; l < i; ++l) acc -= L[i][l] * y[l];
          y[i] = acc / L[i][i];
        }
#pragma unroll
        for (int i = D - 1; i >= 0; --i) {
          float acc = y[i];
#pragma unroll
          for (int l = i + 1; l < D; ++l) acc -= L[l][i] * sol[l];
          sol[i] = acc / L[i][i];
        }
#pragma unroll
        for (int i = 0; i < Q; ++i) a[i] = sol[i];
        if constexpr (GRID) off = sol[Q];
      }
      (void)sign_step(a, off);
    }

    // 3. fp16 scales, last sign step with them (its distances give the error).
    float a16[Q];
#pragma unroll
    for (int i = 0; i < Q; ++i) a16[i] = __half2float(__float2half_rn(a[i]));
    const float e2 = seg_sum(sign_step(a16, off), lpg);
#pragma unroll
    for (int t = 0; t < CPL; ++t) {
      const int c = sl + lpg * t;
      if (!live || c >= chunks) continue;
#pragma unroll
      for (int i = 0; i < Q; ++i) {
        const uint2 sv = bits_to_signs((uint32_t)((sg[t] >> (8 * i)) & 0xFFu));
        *reinterpret_cast<uint2*>(signs + ((size_t)i * m + j) * n + (size_t)G * g + 8 * c) = sv;
      }
    }
    // Plane i's scale is written by lane i mod lpg of the segment.
#pragma unroll
    for (int i = 0; i < Q; ++i)
      if (live && (i & (lpg - 1)) == sl) alpha[((size_t)i * ng + G) * m + j] = __float2half_rn(a16[i]);
    if (live && err && sl == 0) err[(size_t)G * m + j] = e2;
    if constexpr (GRID)
      if (live && sl == 0) offset[(size_t)G * m + j] = off;
  }
}

}  // namespace

cudaError_t launch_fit_bcq(const __half* w, int q, int m, int n, int g, int iters, int8_t* signs, __half* alpha,
                           float* offset, float* err, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long groups = (long long)m * (n / g);
  // Above four planes the codes live in shared memory, one table per warp, so
  // such a warp serves one group.
  int lpg = 1;
  while (lpg < 32 && lpg < g / 8) lpg <<= 1;
  if (q > 4) lpg = 32;
  const long long warps = (groups + (32 / lpg) - 1) / (32 / lpg);
  long long blocks = (warps + kFitWarps - 1) / kFitWarps;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  const int cpl = (g + 255) / 256;
  const unsigned nb = (unsigned)blocks;
  const unsigned nt = kFitWarps * 32;
#define LUTGEMM_FIT_QG(CPLv, Qv)                                                                        \
  if (offset)                                                                                           \
    fit_bcq_kernel<CPLv, Qv, true><<<nb, nt, 0, stream>>>(w, m, n, g, lpg, iters, signs, alpha, offset, err); \
  else                                                                                                  \
    fit_bcq_kernel<CPLv, Qv, false><<<nb, nt, 0, stream>>>(w, m, n, g, lpg, iters, signs, alpha, offset, err);
#define LUTGEMM_FIT_Q(CPLv)                \
  switch (q) {                             \
    case 1: LUTGEMM_FIT_QG(CPLv, 1) break; \
    case 2: LUTGEMM_FIT_QG(CPLv, 2) break; \
    case 3: LUTGEMM_FIT_QG(CPLv, 3) break; \
    case 4: LUTGEMM_FIT_QG(CPLv, 4) break; \
    case 5: LUTGEMM_FIT_QG(CPLv, 5) break; \
    case 6: LUTGEMM_FIT_QG(CPLv, 6) break; \
    case 7: LUTGEMM_FIT_QG(CPLv, 7) break; \
    default: LUTGEMM_FIT_QG(CPLv, 8) break; \
  }
  if (cpl <= 1) {
    LUTGEMM_FIT_Q(1)
  } else if (cpl <= 2) {
    LUTGEMM_FIT_Q(2)
  } else {
    LUTGEMM_FIT_Q(4)
  }
#undef LUTGEMM_FIT_QG
#undef LUTGEMM_FIT_Q
  return cudaGetLastError();
}

}  // namespace lutgemm
