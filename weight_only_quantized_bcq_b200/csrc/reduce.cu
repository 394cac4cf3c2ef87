// Split-K reduction of the LUT-GEMM: y[b][r] = sum over slices of the fp32
// partials part[b][s][r], in a fixed order, so repeated calls give identical
// bits.  A block covers 256/SL row quads (four rows, one 16-byte load); its
// SL slice lanes per quad each sum a contiguous run of slices in slice order,
// all loads of a thread in flight at once, and lane 0 then adds the SL lane
// sums in lane order.  Launched right after the run kernel with programmatic
// dependent launch: it waits for the run to complete before reading.
#include "lutgemm_common.cuh"

namespace lutgemm {

namespace {

constexpr int kReduceThreads = 256;
constexpr int kMaxLaneSlices = 8;   // loads of one thread kept in flight together

__global__ void __launch_bounds__(kReduceThreads) splitk_reduce_kernel(const float* __restrict__ part, void* y,
                                                                      int m, int mt, int ns, int batch,
                                                                      int sl_log2, int y_f16) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float4 lane_sum[kReduceThreads];
  const int SL = 1 << sl_log2;
  const int qpb = kReduceThreads >> sl_log2;               // quads per block
  const long long quads = (long long)mt * (kTileRows / 4);
  const long long blocks_per_col = (quads + qpb - 1) / qpb;
  const int b = (int)(blockIdx.x / blocks_per_col);
  const long long rq = (blockIdx.x - (long long)b * blocks_per_col) * qpb + (threadIdx.x >> sl_log2);
  const int sl = threadIdx.x & (SL - 1);
  const int per = (ns + SL - 1) >> sl_log2;                // slices per lane
  const int s0 = sl * per, s1 = min(ns, s0 + per);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (rq < quads) {
    const float4* src = reinterpret_cast<const float4*>(part) + (size_t)b * ns * quads + rq;
    for (int s = s0; s < s1; s += kMaxLaneSlices) {
      float4 v[kMaxLaneSlices];
#pragma unroll
      for (int e = 0; e < kMaxLaneSlices; ++e)
        v[e] = s + e < s1 ? __ldcg(src + (size_t)(s + e) * quads) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int e = 0; e < kMaxLaneSlices; ++e) {
        acc.x += v[e].x;
        acc.y += v[e].y;
        acc.z += v[e].z;
        acc.w += v[e].w;
      }
    }
  }
  lane_sum[threadIdx.x] = acc;
  __syncthreads();
  if (sl != 0 || rq >= quads) return;
  float4 t = lane_sum[threadIdx.x];
  for (int k = 1; k < SL; ++k) {
    const float4 u = lane_sum[threadIdx.x + k];
    t.x += u.x;
    t.y += u.y;
    t.z += u.z;
    t.w += u.w;
  }
  const float r[4] = {t.x, t.y, t.z, t.w};
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
  // Slice lanes per quad: the smallest power of two that leaves each lane at
  // most two slices, up to 32 lanes.
  const int sl_log2 = reduce_lanes_log2(p.ns);
  const int qpb = kReduceThreads >> sl_log2;
  const long long quads = (long long)p.mt * (kTileRows / 4);
  const long long blocks = (long long)p.batch * ((quads + qpb - 1) / qpb);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kReduceThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, (const float*)p.part, p.y, p.m, p.mt, p.ns,
                                       p.batch, sl_log2, p.y_f16);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace lutgemm
