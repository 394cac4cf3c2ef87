// Split-K reduction of the LUT-GEMM: y[b][r] = sum over slices s (in order
// s = 0, 1, ...) of the fp32 partials part[b][s][r], so repeated calls give
// identical bits.  One thread sums four rows with 16-byte loads, eight slices
// in flight.  Launched right after the run kernel with programmatic
// dependent launch: it waits for the run to complete before reading.
#include "lutgemm_common.cuh"

namespace lutgemm {

namespace {

__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ part, void* y, int m, int mt,
                                                           int ns, int batch, int y_f16) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long quads = (long long)mt * (kTileRows / 4);
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)batch * quads) return;
  const int b = (int)(idx / quads);
  const long long rq = idx - (long long)b * quads;
  const float4* src = reinterpret_cast<const float4*>(part) + (size_t)b * ns * quads + rq;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int s = 0;
  for (; s + 8 <= ns; s += 8) {
    float4 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __ldcg(src + (size_t)(s + e) * quads);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc.x += v[e].x;
      acc.y += v[e].y;
      acc.z += v[e].z;
      acc.w += v[e].w;
    }
  }
  for (; s < ns; ++s) {
    const float4 v = __ldcg(src + (size_t)s * quads);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  const float r[4] = {acc.x, acc.y, acc.z, acc.w};
  const long long row0 = rq * 4;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (row0 + e < m) {
      const size_t o = (size_t)b * m + (size_t)(row0 + e);
      if (y_f16) reinterpret_cast<__half*>(y)[o] = __float2half_rn(r[e]);
      else reinterpret_cast<float*>(y)[o] = r[e];
    }
  }
}

}  // namespace

cudaError_t launch_splitk_reduce(const RunParams& p, cudaStream_t stream) {
  const long long threads = (long long)p.batch * p.mt * (kTileRows / 4);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((threads + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, (const float*)p.part, p.y, p.m, p.mt, p.ns,
                                       p.batch, p.y_f16);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace lutgemm
