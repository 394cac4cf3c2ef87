// Set-up kernels: pack +-1 planes into the tiled bit-plane layout, and rewrite
// uniform q-bit weights as BCQ planes, scales and group offsets.
//
// Sources: LUT-GEMM card (Elamur), Summary and Interesting ideas ("Lookup
// tables instead of multiplications": weights are binary +-1 vectors with
// scales; "One format for many schemes": uniform quantisation is a special
// case of BCQ).  The layout is defined in include/lutgemm.h.
//
// One thread writes one 16-byte lane piece: chunk (s, R, U, i), lane l.
// Byte j of the piece holds inputs 1024 s + 128 P + 8 c .. +7 of row 32R + l
// with P = U xor 4*(l/16), c = j xor (l%16).  The 8 source bytes of a byte are
// contiguous, so each is one 8-byte load.
#include "lutgemm_common.cuh"
#include "lutgemm.h"

namespace lutgemm {

namespace {

__device__ __forceinline__ int piece_of(int U, int l) { return U ^ (4 * (l >> 4)); }
__device__ __forceinline__ int run_of(int j, int l) { return j ^ (l & 15); }

// Eight int8 signs -> sign byte (bit t set iff sign t > 0); flags values other than +-1.
__device__ __forceinline__ uint32_t sign_byte(uint2 v, bool& bad) {
  uint32_t byte = 0;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const uint32_t w = t < 4 ? v.x : v.y;
    const int8_t sv = (int8_t)((w >> (8 * (t & 3))) & 0xFFu);
    bad |= (sv != 1) && (sv != -1);
    byte |= (uint32_t)(sv > 0) << t;
  }
  return byte;
}

__global__ void pack_signs_kernel(const int8_t* __restrict__ signs, int q, int m, int n, int mt,
                                  long long nthreads, uint8_t* __restrict__ packed, int32_t* flags) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nthreads) return;
  const long long chunk = tid >> 5;          // (((s*mt + R)*8 + U)*q + i)
  const int l = (int)(tid & 31);
  const int i = (int)(chunk % q);
  const long long sRU = chunk / q;
  const int U = (int)(sRU & 7);
  const long long sR = sRU >> 3;
  const int R = (int)(sR % mt);
  const int s = (int)(sR / mt);
  const int r = R * kTileRows + l;
  const int P = piece_of(U, l);
  uint32_t words[4] = {0u, 0u, 0u, 0u};
  bool bad = false;
  if (r < m) {
    const int8_t* rowp = signs + ((size_t)i * m + r) * (size_t)n;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int k0 = s * kSliceInputs + 128 * P + 8 * run_of(j, l);
      if (k0 < n) {
        const uint2 v = *reinterpret_cast<const uint2*>(rowp + k0);
        words[j >> 2] |= sign_byte(v, bad) << (8 * (j & 3));
      }
    }
  }
  *reinterpret_cast<uint4*>(packed + chunk * 512 + l * 16) = make_uint4(words[0], words[1], words[2], words[3]);
  if (bad && flags) atomicOr(flags, LUTGEMM_FLAG_BAD_SIGN);
}

// Mixed storage: block (s, R) holds q_b = block_off[u+1] - block_off[u]
// planes (u = s*mt + R) from byte 4096 * block_off[u], in pairs: pair h
// (planes 2h and 2h+1, or 2h alone when q_b = 2h+1; e planes) from byte
// 8192 * h of the block, its chunk (U, i') at (U * e + i') * 512, with the
// byte map of the uniform layout.  One
// thread per (block, U, plane i < q_max, lane); threads of planes the block
// does not store return.  A table entry that would write past the buffer is
// flagged and its block left unwritten.
__global__ void pack_signs_mixed_kernel(const int8_t* __restrict__ signs, const uint32_t* __restrict__ block_off,
                                        int q_max, int m, int n, int mt, long long nthreads, size_t packed_bytes,
                                        uint8_t* __restrict__ packed, int32_t* flags) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nthreads) return;
  const long long chunk = tid >> 5;          // ((s*mt + R)*8 + U)*q_max + i
  const int l = (int)(tid & 31);
  const int i = (int)(chunk % q_max);
  const long long sRU = chunk / q_max;
  const int U = (int)(sRU & 7);
  const long long u = sRU >> 3;
  const int R = (int)(u % mt);
  const int s = (int)(u / mt);
  const uint32_t b0 = block_off[u], b1 = block_off[u + 1];
  const uint32_t qb = b1 - b0;
  if (b1 < b0 || qb < 1u || qb > (uint32_t)q_max || (size_t)b1 * kBlockBytes > packed_bytes) {
    if (flags && i == 0 && U == 0 && l == 0) atomicOr(flags, LUTGEMM_FLAG_BAD_BLOCK);
    return;
  }
  if ((uint32_t)i >= qb) return;
  const int r = R * kTileRows + l;
  const int P = piece_of(U, l);
  uint32_t words[4] = {0u, 0u, 0u, 0u};
  bool bad = false;
  if (r < m) {
    const int8_t* rowp = signs + ((size_t)i * m + r) * (size_t)n;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int k0 = s * kSliceInputs + 128 * P + 8 * run_of(j, l);
      if (k0 < n) {
        const uint2 v = *reinterpret_cast<const uint2*>(rowp + k0);
        words[j >> 2] |= sign_byte(v, bad) << (8 * (j & 3));
      }
    }
  }
  const uint32_t h = (uint32_t)i >> 1, e = min(2u, qb - 2u * h);
  const size_t dst = (size_t)b0 * kBlockBytes + (size_t)h * 2 * kBlockBytes + ((size_t)U * e + (i & 1)) * 512 +
                     (size_t)l * 16;
  *reinterpret_cast<uint4*>(packed + dst) = make_uint4(words[0], words[1], words[2], words[3]);
  if (bad && flags) atomicOr(flags, LUTGEMM_FLAG_BAD_SIGN);
}

// Plane i of a uniform code is bit i of the code (0-based, least significant first).
__global__ void pack_codes_kernel(const uint8_t* __restrict__ codes, int q, int m, int n, int mt,
                                  long long nthreads, uint8_t* __restrict__ packed, int32_t* flags) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nthreads) return;
  const long long sRU = tid >> 5;            // ((s*mt + R)*8 + U)
  const int l = (int)(tid & 31);
  const int U = (int)(sRU & 7);
  const long long sR = sRU >> 3;
  const int R = (int)(sR % mt);
  const int s = (int)(sR / mt);
  const int r = R * kTileRows + l;
  const int P = piece_of(U, l);
  uint32_t words[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) words[i][k] = 0u;
  bool bad = false;
  const uint32_t top_mask = q >= 8 ? 0u : (0xFFu << q) & 0xFFu;
  if (r < m) {
    const uint8_t* rowp = codes + (size_t)r * n;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int k0 = s * kSliceInputs + 128 * P + 8 * run_of(j, l);
      if (k0 < n) {
        const uint2 v = *reinterpret_cast<const uint2*>(rowp + k0);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint32_t code = ((t < 4 ? v.x : v.y) >> (8 * (t & 3))) & 0xFFu;
          bad |= (code & top_mask) != 0u;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            words[i][j >> 2] |= ((code >> i) & 1u) << (8 * (j & 3) + t);
        }
      }
    }
  }
  for (int i = 0; i < q; ++i) {
    *reinterpret_cast<uint4*>(packed + (sRU * q + i) * 512 + l * 16) =
        make_uint4(words[i][0], words[i][1], words[i][2], words[i][3]);
  }
  if (bad && flags) atomicOr(flags, LUTGEMM_FLAG_BAD_CODE);
}

// alpha_i = RNE_fp16(s * 2^(i-1)); offset = s * ((2^q - 1)/2 - z), exact in fp32.
__global__ void uniform_scales_kernel(const __half* __restrict__ scale, const uint8_t* __restrict__ zero,
                                      int q, long long count, size_t plane_stride,
                                      __half* __restrict__ alpha, float* __restrict__ offset,
                                      int32_t* flags) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= count) return;
  const float sf = __half2float(scale[e]);
  const int top = 1 << q;
  const int z = zero[e];
  if (z >= top && flags) atomicOr(flags, LUTGEMM_FLAG_BAD_ZERO);
  const int zz = z & (top - 1);
  for (int i = 0; i < q; ++i) alpha[(size_t)i * plane_stride + e] = __float2half_rn(ldexpf(sf, i - 1));
  offset[e] = sf * ((float)(top - 1) * 0.5f - (float)zz);
}

// Unit-major scales: one thread per (slice, row tile, plane group, lane)
// writes that lane's 8 x SP scales (SP 16-byte stores).  Element (U, e) is
// alpha[4*pg + e][(1024*s + 128*P) / g][32*R + l], P = U xor 4*(l/16), or 0
// for a plane, row or piece out of range.
__global__ void pack_scales_kernel(const __half* __restrict__ alpha, int q, int m, int n, int g, int mt,
                                   int npg, int sp, int halves, long long nthreads, uint4* __restrict__ out) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nthreads) return;
  const int l = (int)(tid & 31);
  const long long sRp = tid >> 5;            // ((s*mt + R)*npg + pg)
  const int pg = (int)(sRp % npg);
  const long long sR = sRp / npg;
  const int R = (int)(sR % mt);
  const int s = (int)(sR / mt);
  const int row = R * kTileRows + l;
  const int ng = n / g;
  uint32_t words[32];
#pragma unroll
  for (int w = 0; w < 32; ++w) words[w] = 0u;
#pragma unroll
  for (int U = 0; U < 8; ++U) {
    const int P = U ^ (4 * (l >> 4));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k0 = s * kSliceInputs + 128 * P + 64 * h;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * pg + e;
        if (h < halves && e < sp && i < q && row < m && k0 < n) {
          const uint32_t v = __ldg(reinterpret_cast<const unsigned short*>(alpha) +
                                   ((size_t)i * ng + k0 / g) * (size_t)m + row);
          const int idx = (U * sp + e) * halves + h;
          words[idx >> 1] |= v << (16 * (idx & 1));
        }
      }
    }
  }
  uint4* dst = out + (size_t)tid * sp * halves;
  for (int v = 0; v < sp * halves; ++v)
    dst[v] = make_uint4(words[4 * v], words[4 * v + 1], words[4 * v + 2], words[4 * v + 3]);
}

}  // namespace

cudaError_t launch_pack_scales(const __half* alpha, int q, int m, int n, int g, uint16_t* scales,
                               cudaStream_t stream) {
  const int mt = (m + kTileRows - 1) / kTileRows;
  const int ns = (n + kSliceInputs - 1) / kSliceInputs;
  const int npg = (q + 3) / 4;
  const int sp = q < 4 ? q : 4;
  const int halves = g == 64 ? 2 : 1;
  const long long nthreads = (long long)ns * mt * npg * 32;
  const int block = 256;
  pack_scales_kernel<<<(unsigned)((nthreads + block - 1) / block), block, 0, stream>>>(
      alpha, q, m, n, g, mt, npg, sp, halves, nthreads, reinterpret_cast<uint4*>(scales));
  return cudaGetLastError();
}

cudaError_t launch_pack_signs(const int8_t* signs, int q, int m, int n, uint8_t* packed, int32_t* flags,
                              cudaStream_t stream) {
  const int mt = (m + kTileRows - 1) / kTileRows;
  const int ns = (n + kSliceInputs - 1) / kSliceInputs;
  const long long nthreads = (long long)ns * mt * q * 256;
  const int block = 256;
  const long long grid = (nthreads + block - 1) / block;
  pack_signs_kernel<<<(unsigned)grid, block, 0, stream>>>(signs, q, m, n, mt, nthreads, packed, flags);
  return cudaGetLastError();
}

cudaError_t launch_pack_signs_mixed(const int8_t* signs, const uint32_t* block_off, int q_max, int m, int n,
                                    uint8_t* packed, size_t packed_bytes, int32_t* flags, cudaStream_t stream) {
  const int mt = (m + kTileRows - 1) / kTileRows;
  const int ns = (n + kSliceInputs - 1) / kSliceInputs;
  const long long nthreads = (long long)ns * mt * q_max * 256;
  const int block = 256;
  const long long grid = (nthreads + block - 1) / block;
  pack_signs_mixed_kernel<<<(unsigned)grid, block, 0, stream>>>(signs, block_off, q_max, m, n, mt, nthreads,
                                                                packed_bytes, packed, flags);
  return cudaGetLastError();
}

// Unit-major scales of mixed storage: one thread per (block, pair, lane)
// writes the lane's pass, e * H 16-byte words from element
// table[u] * 256 * H + pair * 512 * H + lane * 8 * e * H (layout in
// include/lutgemm.h).  Threads of pairs a block does not store return; a
// table entry past the buffer is flagged and not written.
__global__ void pack_scales_mixed_kernel(const __half* __restrict__ alpha, const uint32_t* __restrict__ block_off,
                                         int q_max, int m, int n, int g, int mt, int halves, long long nthreads,
                                         size_t out_elems, uint16_t* __restrict__ out, int32_t* flags) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nthreads) return;
  const int l = (int)(tid & 31);
  const int h = (int)((tid >> 5) & 1);
  const long long u = tid >> 6;
  const int R = (int)(u % mt);
  const int s = (int)(u / mt);
  const uint32_t b0 = block_off[u], b1 = block_off[u + 1];
  const uint32_t qb = b1 - b0;
  if (b1 < b0 || qb < 1u || qb > (uint32_t)q_max || (size_t)b1 * 256 * halves > out_elems) {
    if (flags && h == 0 && l == 0) atomicOr(flags, LUTGEMM_FLAG_BAD_BLOCK);
    return;
  }
  if (2u * (uint32_t)h >= qb) return;
  const uint32_t e_h = min(2u, qb - 2u * (uint32_t)h);
  const int row = R * kTileRows + l;
  const int ng = n / g;
  uint32_t words[16];
#pragma unroll
  for (int w = 0; w < 16; ++w) words[w] = 0u;
  for (int U = 0; U < 8; ++U) {
    const int P = U ^ (4 * (l >> 4));
    for (int hh = 0; hh < halves; ++hh) {
      const int k0 = s * kSliceInputs + 128 * P + 64 * hh;
      for (uint32_t e = 0; e < e_h; ++e) {
        if (row < m && k0 < n) {
          const uint32_t v = __ldg(reinterpret_cast<const unsigned short*>(alpha) +
                                   ((size_t)(2 * h + e) * ng + k0 / g) * (size_t)m + row);
          const int idx = (int)((U * e_h + e) * halves + hh);
          words[idx >> 1] |= v << (16 * (idx & 1));
        }
      }
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)b0 * 256 * halves + (size_t)h * 512 * halves +
                                        (size_t)l * 8 * e_h * halves);
  for (uint32_t v = 0; v < e_h * halves; ++v)
    dst[v] = make_uint4(words[4 * v], words[4 * v + 1], words[4 * v + 2], words[4 * v + 3]);
}

cudaError_t launch_pack_scales_mixed(const __half* alpha, const uint32_t* block_off, int q_max, int m, int n, int g,
                                     uint16_t* scales, size_t scales_bytes, int32_t* flags, cudaStream_t stream) {
  const int mt = (m + kTileRows - 1) / kTileRows;
  const int ns = (n + kSliceInputs - 1) / kSliceInputs;
  const int halves = g == 64 ? 2 : 1;
  const long long nthreads = (long long)ns * mt * 64;
  const int block = 256;
  pack_scales_mixed_kernel<<<(unsigned)((nthreads + block - 1) / block), block, 0, stream>>>(
      alpha, block_off, q_max, m, n, g, mt, halves, nthreads, scales_bytes / 2, scales, flags);
  return cudaGetLastError();
}

cudaError_t launch_uniform_to_bcq(const uint8_t* codes, const __half* scale, const uint8_t* zero, int q,
                                  int m, int n, int g, uint8_t* packed, __half* alpha, float* offset,
                                  int32_t* flags, cudaStream_t stream) {
  const int mt = (m + kTileRows - 1) / kTileRows;
  const int ns = (n + kSliceInputs - 1) / kSliceInputs;
  const long long nthreads = (long long)ns * mt * 256;
  const int block = 256;
  pack_codes_kernel<<<(unsigned)((nthreads + block - 1) / block), block, 0, stream>>>(
      codes, q, m, n, mt, nthreads, packed, flags);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const long long count = (long long)(n / g) * m;
  uniform_scales_kernel<<<(unsigned)((count + block - 1) / block), block, 0, stream>>>(
      scale, zero, q, count, (size_t)count, alpha, offset, flags);
  return cudaGetLastError();
}

}  // namespace lutgemm
