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
// One warp per (row, group); a lane holds up to CPL chunks of 8 consecutive
// inputs (g <= 256 * CPL).  Signs live in registers as one 64-bit mask per
// chunk (byte i = plane i).  Sums are taken in a fixed order (per lane in
// input order, then a butterfly over the warp), so results are reproducible.
#include "lutgemm.h"
#include "lutgemm_common.cuh"

namespace lutgemm {

namespace {

constexpr int kFitWarps = 8;
constexpr float kPivotRel = 1e-6f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Nearest code for value w among the 2^q codebook values vals[] (smem).
__device__ __forceinline__ int nearest(float w, const float* vals, int ncode) {
  float best = fabsf(w - vals[0]);
  int arg = 0;
  for (int c = 1; c < ncode; ++c) {
    const float d = fabsf(w - vals[c]);
    if (d <= best) {
      best = d;
      arg = c;
    }
  }
  return arg;
}

template <int CPL, int Q>
__global__ void __launch_bounds__(kFitWarps * 32) fit_bcq_kernel(const __half* __restrict__ w, int m, int n, int g,
                                                               int iters, int8_t* __restrict__ signs,
                                                               __half* __restrict__ alpha, float* __restrict__ err) {
  constexpr int q = Q;
  __shared__ float codebook[kFitWarps][256];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  float* vals = codebook[wid];
  const int ng = n / g;
  const int chunks = g / 8;
  const long long groups = (long long)m * ng;
  constexpr int ncode = 1 << Q;
  const float inv_g = 1.0f / (float)g;

  for (long long grp = (long long)blockIdx.x * kFitWarps + wid; grp < groups;
       grp += (long long)gridDim.x * kFitWarps) {
    const int j = (int)(grp / ng);
    const int G = (int)(grp - (long long)j * ng);
    const __half* src = w + (size_t)j * n + (size_t)G * g;

    float x[CPL][8];
    uint64_t sg[CPL];
#pragma unroll
    for (int t = 0; t < CPL; ++t) {
      sg[t] = 0;
      const int c = lane + 32 * t;
      if (c < chunks) {
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

    // 1. Greedy planes on the residual.
    float a[8];
    {
      float r[CPL][8];
#pragma unroll
      for (int t = 0; t < CPL; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) r[t][e] = x[t][e];
#pragma unroll
      for (int i = 0; i < q; ++i) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < CPL; ++t) {
          if (lane + 32 * t >= chunks) continue;
          uint32_t bits = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const bool pos = r[t][e] >= 0.f;
            bits |= (uint32_t)pos << e;
            s += fabsf(r[t][e]);
          }
          sg[t] |= (uint64_t)bits << (8 * i);
        }
        const float ai = warp_sum(s) * inv_g;
        a[i] = ai;
#pragma unroll
        for (int t = 0; t < CPL; ++t)
#pragma unroll
          for (int e = 0; e < 8; ++e) r[t][e] -= ((sg[t] >> (8 * i + e)) & 1) ? ai : -ai;
      }
    }

    auto fill_codebook = [&](const float* av) {
      __syncwarp();
      for (int c = lane; c < ncode; c += 32) {
        float v = 0.f;
#pragma unroll
        for (int i = 0; i < q; ++i) v += ((c >> i) & 1) ? av[i] : -av[i];
        vals[c] = v;
      }
      __syncwarp();
    };
    auto sign_step = [&]() {
#pragma unroll
      for (int t = 0; t < CPL; ++t) {
        if (lane + 32 * t >= chunks) continue;
        uint64_t m8 = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint64_t c = (uint64_t)nearest(x[t][e], vals, ncode);
          // spread code bit i to bit 8*i + e
#pragma unroll
          for (int i = 0; i < q; ++i) m8 |= ((c >> i) & 1ull) << (8 * i + e);
        }
        sg[t] = m8;
      }
    };

    // 2. Alternating rounds.
    for (int it = 0; it < iters; ++it) {
      // Normal equations: M_ik = g - 2 * #(inputs where planes i and k differ),
      // v_i = sum_k beta_ik * w_k.
      int diff[36];
      float v[8];
#pragma unroll
      for (int i = 0; i < q; ++i) {
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < CPL; ++t) {
          if (lane + 32 * t >= chunks) continue;
#pragma unroll
          for (int e = 0; e < 8; ++e) s += ((sg[t] >> (8 * i + e)) & 1) ? x[t][e] : -x[t][e];
        }
        v[i] = warp_sum(s);
#pragma unroll
        for (int k = 0; k < i; ++k) {
          int cnt = 0;
#pragma unroll
          for (int t = 0; t < CPL; ++t) {
            if (lane + 32 * t >= chunks) continue;
            cnt += __popc((uint32_t)(((sg[t] >> (8 * i)) ^ (sg[t] >> (8 * k))) & 0xFFull));
          }
          diff[i * (i - 1) / 2 + k] = warp_sum_i(cnt);
        }
      }
      // Cholesky of M (every lane, same arithmetic), then two triangular solves.
      float L[8][8];
      bool ok = true;
#pragma unroll
      for (int i = 0; i < q; ++i) {
#pragma unroll
        for (int k = 0; k <= i; ++k) {
          float acc = (i == k) ? (float)g : (float)(g - 2 * diff[i * (i - 1) / 2 + k]);
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
        float y[8];
#pragma unroll
        for (int i = 0; i < q; ++i) {
          float acc = v[i];
#pragma unroll
          for (int l = 0; l < i; ++l) acc -= L[i][l] * y[l];
          y[i] = acc / L[i][i];
        }
#pragma unroll
        for (int i = q - 1; i >= 0; --i) {
          float acc = y[i];
#pragma unroll
          for (int l = i + 1; l < q; ++l) acc -= L[l][i] * a[l];
          a[i] = acc / L[i][i];
        }
      }
      fill_codebook(a);
      sign_step();
    }

    // 3. fp16 scales, last sign step with them, outputs.
    float a16[8];
#pragma unroll
    for (int i = 0; i < q; ++i) a16[i] = __half2float(__float2half_rn(a[i]));
    fill_codebook(a16);
    sign_step();
    float e2 = 0.f;
#pragma unroll
    for (int t = 0; t < CPL; ++t) {
      const int c = lane + 32 * t;
      if (c >= chunks) continue;
#pragma unroll
      for (int i = 0; i < q; ++i) {
        const uint32_t bits = (uint32_t)((sg[t] >> (8 * i)) & 0xFFull);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          lo |= (uint32_t)(uint8_t)(((bits >> e) & 1) ? 1 : -1) << (8 * e);
          hi |= (uint32_t)(uint8_t)(((bits >> (e + 4)) & 1) ? 1 : -1) << (8 * e);
        }
        *reinterpret_cast<uint2*>(signs + ((size_t)i * m + j) * n + (size_t)G * g + 8 * c) = make_uint2(lo, hi);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float vv = 0.f;
#pragma unroll
        for (int i = 0; i < q; ++i) vv += ((sg[t] >> (8 * i + e)) & 1) ? a16[i] : -a16[i];
        const float d = x[t][e] - vv;
        e2 += d * d;
      }
    }
    e2 = warp_sum(e2);
    if (lane < q) {
      float mine = a16[0];
#pragma unroll
      for (int i = 1; i < q; ++i)
        if (lane == i) mine = a16[i];
      alpha[((size_t)lane * ng + G) * m + j] = __float2half_rn(mine);
    }
    if (err && lane == 0) err[(size_t)G * m + j] = e2;
  }
}

}  // namespace

cudaError_t launch_fit_bcq(const __half* w, int q, int m, int n, int g, int iters, int8_t* signs, __half* alpha,
                           float* err, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long groups = (long long)m * (n / g);
  long long blocks = (groups + kFitWarps - 1) / kFitWarps;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  const int cpl = (g + 255) / 256;
  const unsigned nb = (unsigned)blocks;
  const unsigned nt = kFitWarps * 32;
#define LUTGEMM_FIT_Q(CPLv)                                                                        \
  switch (q) {                                                                                     \
    case 1: fit_bcq_kernel<CPLv, 1><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
    case 2: fit_bcq_kernel<CPLv, 2><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
    case 3: fit_bcq_kernel<CPLv, 3><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
    case 4: fit_bcq_kernel<CPLv, 4><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
    case 5: fit_bcq_kernel<CPLv, 5><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
    case 6: fit_bcq_kernel<CPLv, 6><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
    case 7: fit_bcq_kernel<CPLv, 7><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
    default: fit_bcq_kernel<CPLv, 8><<<nb, nt, 0, stream>>>(w, m, n, g, iters, signs, alpha, err); break; \
  }
  if (cpl <= 1) {
    LUTGEMM_FIT_Q(1)
  } else if (cpl <= 2) {
    LUTGEMM_FIT_Q(2)
  } else {
    LUTGEMM_FIT_Q(4)
  }
#undef LUTGEMM_FIT_Q
  return cudaGetLastError();
}

}  // namespace lutgemm
