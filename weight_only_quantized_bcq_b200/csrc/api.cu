// C ABI of the LUT-GEMM library: argument validation, workspace sizing and
// kernel launches on the caller's stream.  Declarations and the contract of
// every call are in include/lutgemm.h.
#include <algorithm>
#include <cmath>
#include <mutex>
#include <set>
#include <utility>

#include "lutgemm.h"
#include "lutgemm_common.cuh"

namespace lutgemm {
cudaError_t launch_pack_signs(const int8_t* signs, int q, int m, int n, uint8_t* packed, int32_t* flags,
                              cudaStream_t stream);
cudaError_t launch_uniform_to_bcq(const uint8_t* codes, const __half* scale, const uint8_t* zero, int q,
                                  int m, int n, int g, uint8_t* packed, __half* alpha, float* offset,
                                  int32_t* flags, cudaStream_t stream);
cudaError_t launch_pack_scales(const __half* alpha, int q, int m, int n, int g, uint16_t* scales,
                               cudaStream_t stream);
cudaError_t launch_pack_signs_mixed(const int8_t* signs, const uint32_t* block_off, int q_max, int m, int n,
                                    uint8_t* packed, size_t packed_bytes, int32_t* flags, cudaStream_t stream);
cudaError_t launch_pack_scales_mixed(const __half* alpha, const uint32_t* block_off, int q_max, int m, int n, int g,
                                     uint16_t* scales, size_t scales_bytes, int32_t* flags, cudaStream_t stream);
cudaError_t launch_tc_gemm(const uint8_t* packed, const __half* alpha, const float* offset, const __half* x, void* y,
                           float* part, int nsplit, int m, int n, int batch, int q, int g, int y_f16, unsigned* status,
                           cudaStream_t stream);
cudaError_t launch_fit_bcq(const __half* w, int q, int m, int n, int g, int iters, int8_t* signs, __half* alpha,
                           float* offset,
                           float* err, cudaStream_t stream);

// The tensor-core plan: how many K splits to run it with, or 0 when the
// lookup kernel is expected to be faster.  A cost model fitted to B200
// measurements of both paths (OPT-175B and LLaMA-70B linears, batch 8-32,
// isolated back-to-back launches):
//   tensor cores: waves x (K blocks per split x c + 14k) + 15k cycles, with
//     waves = ceil(ceil(m/128) * ceil(batch/BN) * splits / SMs) and
//     c = q/3 x 1600 / 1870 / 2450 cycles per 128-input block at BN = 32 /
//     64 / 128 (the A-tile stores and expansion scale with the planes); a split
//     run adds the fp32 partials' reduce (launch + bytes at HBM speed);
//   lookups: q m n batch / 8 table reads at e(q) = 0.39 + 0.092 q of one
//     32-read wavefront per clock per SM (0.57 at q = 2, 0.67 at q = 3:
//     per-unit costs are shared by the planes), + 20k cycles.
// It picks the faster path (and split count) for the 12 measured (shape,
// batch >= 8) cases and the batch-256 layer: FC2- and out-proj-like matrices
// (few 128-row blocks, long K) take 3 splits, QKV and FC1 none, LLaMA-70B at
// batch 8 the lookups.  Splits are whole 1024-input slices, at most 8 (and
// max_split), and never empty.
int tc_plan_for(int m, int n, int batch, int q, int max_split, int sm_count) {
  if (m < 1 || n < 128 || batch < 8 || q < 1 || max_split < 1 || sm_count < 1) return 0;
  const double sms = sm_count;
  const int bn = batch <= 32 ? 32 : (batch <= 64 ? 64 : 128);
  const double block_cycles = (bn == 32 ? 1600.0 : (bn == 64 ? 1870.0 : 2450.0)) * q / 3.0;
  const double ctas = (double)((m + 127) / 128) * (double)((batch + bn - 1) / bn);
  const int s_all = (n + 1023) / 1024;
  const int nkb = n / 128;
  const double mt32 = (double)((m + 31) / 32) * 32.0;
  double best = 0.0, unsplit = 0.0;
  int best_s = 0;
  for (int sp = 1; sp <= max_split && sp <= s_all && sp <= 8; ++sp) {
    const int spz = (s_all + sp - 1) / sp;
    if ((s_all + spz - 1) / spz != sp) continue;          // would leave a split empty
    const double kb = (double)(8 * spz < nkb ? 8 * spz : nkb);
    double t = std::ceil(ctas * sp / sms) * (kb * block_cycles + 14000.0) + 15000.0;
    if (sp > 1) t += 4000.0 + ((double)batch * mt32 * sp * 4.0 + (double)batch * m * 4.0) / 6.4e12 * 1.965e9;
    if (sp == 1) unsplit = t;
    if (best_s == 0 || t < best) {
      best = t;
      best_s = sp;
    }
  }
  // A split must be expected to save at least 5 % (near ties measured slower).
  if (best_s > 1 && best > 0.95 * unsplit) {
    best = unsplit;
    best_s = 1;
  }
  const double e_lut = std::min(0.39 + 0.092 * q, 0.85);
  const double t_lut = (double)q * m * n * batch / 8.0 / (sms * 32.0) / e_lut + 20000.0;
  return best_s > 0 && best < t_lut ? best_s : 0;
}

// The plan on the current device (its SM count read once per device).
int tc_plan(int m, int n, int batch, int q, int max_split) {
  static int sms_cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (sms_cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 0;
    sms_cache[dev] = v;
  }
  return tc_plan_for(m, n, batch, q, max_split, sms_cache[dev]);
}

}  // namespace lutgemm

namespace {

using namespace lutgemm;

constexpr int kVersion = 10000;  // 1.0.0

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool valid_matrix(int q, int m, int n) { return q >= 1 && q <= 8 && m >= 1 && n >= 8 && n % 8 == 0; }

bool valid_groups(int n, int g) { return g >= 8 && g % 8 == 0 && n % g == 0; }

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Per-device state that is set once: SM count and the shared-memory opt-in of
// every kernel launched on that device.
std::mutex g_mutex;
std::set<std::pair<const void*, int>> g_smem_done;
int g_sm_count[64] = {0};

cudaError_t device_setup(RunKernel kernel, int* sm_count) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_sm_count[dev] == 0) {
    int v = 0, reserved = 0, optin = 0;
    err = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err != cudaSuccess) return err;
    // The tables sit at a fixed window address right after the reserved region.
    if ((unsigned)reserved != kTableBase || optin < kSmemBytes) return cudaErrorInvalidConfiguration;
    g_sm_count[dev] = v;
  }
  *sm_count = g_sm_count[dev];
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  if (g_smem_done.find(key) == g_smem_done.end()) {
    // Static shared memory would move the dynamic window off kTableBase.
    cudaFuncAttributes fa;
    err = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kernel));
    if (err != cudaSuccess) return err;
    if (fa.sharedSizeBytes != 0) return cudaErrorInvalidConfiguration;
    err = cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    g_smem_done.insert(key);
  }
  return cudaSuccess;
}

int group_mode(int g) {
  if (g == 128) return kG128;
  if (g % 128 == 0) return kG128x;
  if (g == 64) return kG64;
  if (g == 8) return kG8;
  return kGAny;
}

RunKernel select_kernel(int q, int mode, bool has_offset, bool packed) {
  switch (q) {
    case 1: return run_kernel_q1(mode, has_offset, packed);
    case 2: return run_kernel_q2(mode, has_offset, packed);
    case 3: return run_kernel_q3(mode, has_offset, packed);
    case 4: return run_kernel_q4(mode, has_offset, packed);
    default: return run_kernel_q8(mode, has_offset, packed);
  }
}

// Workspace: [status word (256 B) | tile counters (4 KB) | split-K partials].
// The status word sits at the start whatever the shape, so that
// lutgemm_workspace_status can find it from the pointer alone.
size_t part_bytes(int m, int n, int batch) {
  return (size_t)batch * ceil_div(n, kSliceInputs) * ceil_div(m, kTileRows) * kTileRows * sizeof(float);
}

constexpr size_t kStatusBytes = 256;
constexpr size_t kTileCounterBytes = kMaxTileCounters * sizeof(unsigned);
constexpr size_t kPartOffset = kStatusBytes + kTileCounterBytes;

// Fill the workspace pointers and geometry of `p` and enqueue the lookup
// kernel (and the split-K reduce when there are several slices).
int launch_lookup(RunParams& p, RunKernel kernel, void* workspace, cudaStream_t stream) {
  char* ws = reinterpret_cast<char*>(workspace);
  p.ns = ceil_div(p.n, kSliceInputs);
  p.mt = ceil_div(p.m, kTileRows);
  p.ng = p.n / p.g;
  p.total_units = (long long)p.batch * p.ns * p.mt;
  p.part = reinterpret_cast<float*>(ws + kPartOffset);
  p.tile_cnt = reinterpret_cast<unsigned*>(ws + kStatusBytes);
  p.status = reinterpret_cast<unsigned*>(ws);
  if (kernel == nullptr) return LUTGEMM_ERR_VALUE;
  int sm_count = 0;
  if (device_setup(kernel, &sm_count) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  long long grid = 0;
  choose_launch(sm_count, (long long)p.batch * p.ns, p.mt, &grid, &p.seg_aligned);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, p) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return LUTGEMM_ERR_CUDA;
  if (p.ns > 1 && launch_splitk_reduce(p, stream) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  return LUTGEMM_OK;
}

}  // namespace

extern "C" {

int lutgemm_version(void) { return kVersion; }

const char* lutgemm_status_string(int status) {
  switch (status) {
    case LUTGEMM_OK: return "success";
    case LUTGEMM_ERR_NULL: return "a required pointer is NULL";
    case LUTGEMM_ERR_SHAPE: return "invalid shape (need m,n,batch >= 1, 1 <= q <= 8, n%8 == 0, g%8 == 0, n%g == 0)";
    case LUTGEMM_ERR_ALIGN: return "a pointer is not aligned as the call requires";
    case LUTGEMM_ERR_WORKSPACE: return "workspace is smaller than lutgemm_workspace_size()";
    case LUTGEMM_ERR_VALUE: return "an argument value is out of range";
    case LUTGEMM_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    default: return "unknown status";
  }
}

size_t lutgemm_packed_bytes(int q, int m, int n) {
  if (!valid_matrix(q, m, n)) return 0;
  return (size_t)ceil_div(n, kSliceInputs) * ceil_div(m, kTileRows) * q * kBlockBytes;
}

size_t lutgemm_scales_bytes(int q, int m, int n, int g) {
  if (!valid_matrix(q, m, n) || !valid_groups(n, g) || !(g % 128 == 0 || g == 64)) return 0;
  const size_t sp = q < 4 ? (size_t)q : 4u;
  const size_t halves = g == 64 ? 2u : 1u;
  return (size_t)ceil_div(n, kSliceInputs) * ceil_div(m, kTileRows) * ceil_div(q, 4) * 512u * sp * halves;
}

int lutgemm_run_tc(int m, int n, int batch, int q, int g, const uint8_t* packed, const uint16_t* alpha,
                   const float* offset, const uint16_t* x, void* y, unsigned flags, void* stream) {
  if (!packed || !alpha || !x || !y) return LUTGEMM_ERR_NULL;
  if (!valid_matrix(q, m, n) || !valid_groups(n, g) || batch < 1 || g % 64 != 0 || n % 128 != 0)
    return LUTGEMM_ERR_SHAPE;
  if ((flags & ~LUTGEMM_Y_F16) != 0u) return LUTGEMM_ERR_VALUE;
  const bool y_f16 = (flags & LUTGEMM_Y_F16) != 0u;
  if (!aligned(packed, 16) || !aligned(alpha, 2) || !aligned(offset, 4) || !aligned(x, 16) ||
      !aligned(y, y_f16 ? 2 : 4))
    return LUTGEMM_ERR_ALIGN;
  const cudaError_t e = launch_tc_gemm(packed, reinterpret_cast<const __half*>(alpha), offset,
                                       reinterpret_cast<const __half*>(x), y, nullptr, 1, m, n, batch, q, g,
                                       y_f16 ? 1 : 0, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_fit_bcq(const uint16_t* w, int q, int m, int n, int g, int iters, int8_t* signs, uint16_t* alpha,
                    float* err, void* stream) {
  if (!w || !signs || !alpha) return LUTGEMM_ERR_NULL;
  if (!valid_matrix(q, m, n) || !valid_groups(n, g) || g > 1024) return LUTGEMM_ERR_SHAPE;
  if (iters < 0 || iters > 64) return LUTGEMM_ERR_VALUE;
  if (!aligned(w, 16) || !aligned(signs, 8) || !aligned(alpha, 2) || !aligned(err, 4)) return LUTGEMM_ERR_ALIGN;
  const cudaError_t e = launch_fit_bcq(reinterpret_cast<const __half*>(w), q, m, n, g, iters, signs,
                                       reinterpret_cast<__half*>(alpha), nullptr, err,
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_fit_bcq_grid(const uint16_t* w, int q, int m, int n, int g, int iters, int8_t* signs, uint16_t* alpha,
                         float* offset, float* err, void* stream) {
  if (!w || !signs || !alpha || !offset) return LUTGEMM_ERR_NULL;
  if (!valid_matrix(q, m, n) || !valid_groups(n, g) || g > 1024) return LUTGEMM_ERR_SHAPE;
  if (iters < 0 || iters > 64) return LUTGEMM_ERR_VALUE;
  if (!aligned(w, 16) || !aligned(signs, 8) || !aligned(alpha, 2) || !aligned(offset, 4) || !aligned(err, 4))
    return LUTGEMM_ERR_ALIGN;
  const cudaError_t e = launch_fit_bcq(reinterpret_cast<const __half*>(w), q, m, n, g, iters, signs,
                                       reinterpret_cast<__half*>(alpha), offset, err,
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_pack_scales(const uint16_t* alpha, int q, int m, int n, int g, uint16_t* scales, void* stream) {
  if (!alpha || !scales) return LUTGEMM_ERR_NULL;
  if (!valid_matrix(q, m, n) || !valid_groups(n, g) || !(g % 128 == 0 || g == 64)) return LUTGEMM_ERR_SHAPE;
  if (!aligned(alpha, 2) || !aligned(scales, 16)) return LUTGEMM_ERR_ALIGN;
  const cudaError_t err = launch_pack_scales(reinterpret_cast<const __half*>(alpha), q, m, n, g, scales,
                                             reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_tc_plan(int m, int n, int batch, int q, int max_split, int sm_count) {
  return lutgemm::tc_plan_for(m, n, batch, q, max_split, sm_count);
}

int lutgemm_launch_plan(int m, int n, int batch, int sm_count, int* grid, int* seg_aligned, int* dynamic_tiles) {
  if (!grid || !seg_aligned || !dynamic_tiles) return LUTGEMM_ERR_NULL;
  if (m < 1 || n < 8 || n % 8 != 0 || batch < 1 || sm_count < 1) return LUTGEMM_ERR_SHAPE;
  if ((long long)batch * ceil_div(n, kSliceInputs) >= (1ll << 31)) return LUTGEMM_ERR_SHAPE;
  const long long segments = (long long)batch * ceil_div(n, kSliceInputs);
  const long long mt = ceil_div(m, kTileRows);
  long long g = 0;
  int aligned_mode = 0;
  choose_launch(sm_count, segments, mt, &g, &aligned_mode);
  *grid = (int)g;
  *seg_aligned = aligned_mode;
  long long dyn = 0;
  if (aligned_mode) {
    // Segment z has (grid - z + segments - 1) / segments CTAs (the kernel's
    // group_size); their warps take two static tiles each, 32 per CTA.
    for (long long z = 0; z < segments; ++z) {
      const long long cz = (g - z + segments - 1) / segments;
      dyn += mt > 32 * cz ? mt - 32 * cz : 0;
    }
  }
  *dynamic_tiles = dyn > 0x7fffffffLL ? 0x7fffffff : (int)dyn;
  return LUTGEMM_OK;
}

int lutgemm_workspace_status(void* workspace, size_t workspace_bytes, uint32_t* status, int clear, void* stream) {
  if (!workspace || !status) return LUTGEMM_ERR_NULL;
  if (!aligned(workspace, 16)) return LUTGEMM_ERR_ALIGN;
  if (workspace_bytes < kPartOffset) return LUTGEMM_ERR_WORKSPACE;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  *status = v;
  if (clear && v != 0u && cudaMemsetAsync(workspace, 0, sizeof(v), st) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  return LUTGEMM_OK;
}

size_t lutgemm_workspace_size(int m, int n, int batch, int q, int g) {
  if (!valid_matrix(q, m, n) || !valid_groups(n, g) || batch < 1) return 0;
  return kPartOffset + round_up(part_bytes(m, n, batch), 256);
}

int lutgemm_pack_bcq(const int8_t* signs, int q, int m, int n, uint8_t* packed, int32_t* status_flags,
                     void* stream) {
  if (!signs || !packed) return LUTGEMM_ERR_NULL;
  if (!valid_matrix(q, m, n)) return LUTGEMM_ERR_SHAPE;
  if (!aligned(signs, 8) || !aligned(packed, 16) || !aligned(status_flags, 4)) return LUTGEMM_ERR_ALIGN;
  const cudaError_t err =
      launch_pack_signs(signs, q, m, n, packed, status_flags, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_uniform_to_bcq(const uint8_t* codes, const uint16_t* scale, const uint8_t* zero, int q, int m,
                           int n, int g, uint8_t* packed, uint16_t* alpha, float* offset,
                           int32_t* status_flags, void* stream) {
  if (!codes || !scale || !zero || !packed || !alpha || !offset) return LUTGEMM_ERR_NULL;
  if (!valid_matrix(q, m, n) || !valid_groups(n, g)) return LUTGEMM_ERR_SHAPE;
  if (!aligned(codes, 8) || !aligned(scale, 2) || !aligned(packed, 16) || !aligned(alpha, 2) ||
      !aligned(offset, 4) || !aligned(status_flags, 4))
    return LUTGEMM_ERR_ALIGN;
  const cudaError_t err = launch_uniform_to_bcq(
      codes, reinterpret_cast<const __half*>(scale), zero, q, m, n, g, packed,
      reinterpret_cast<__half*>(alpha), offset, status_flags, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_run(int m, int n, int batch, int q, int g, const uint8_t* packed, const uint16_t* alpha,
                const float* offset, const uint16_t* x, void* y, unsigned flags, void* workspace,
                size_t workspace_bytes, void* stream) {
  if (!packed || !alpha || !x || !y || !workspace) return LUTGEMM_ERR_NULL;
  if (!valid_matrix(q, m, n) || !valid_groups(n, g) || batch < 1) return LUTGEMM_ERR_SHAPE;
  if ((long long)batch * ceil_div(n, kSliceInputs) >= (1ll << 31)) return LUTGEMM_ERR_SHAPE;
  if ((flags & ~(LUTGEMM_Y_F16 | LUTGEMM_SCALES_PACKED | LUTGEMM_ALLOW_TENSOR_CORES | LUTGEMM_TEST_STALL)) != 0u)
    return LUTGEMM_ERR_VALUE;
  const bool stall = (flags & LUTGEMM_TEST_STALL) != 0u;
  const bool y_f16 = (flags & LUTGEMM_Y_F16) != 0u;
  const bool scales_packed = (flags & LUTGEMM_SCALES_PACKED) != 0u;
  if (scales_packed && !(g % 128 == 0 || g == 64)) return LUTGEMM_ERR_VALUE;
  if (!aligned(packed, 16) || !aligned(alpha, scales_packed ? 16 : 2) || !aligned(offset, 4) ||
      !aligned(x, 16) || !aligned(y, y_f16 ? 2 : 4) || !aligned(workspace, 16))
    return LUTGEMM_ERR_ALIGN;
  if (workspace_bytes < lutgemm_workspace_size(m, n, batch, q, g)) return LUTGEMM_ERR_WORKSPACE;
  char* ws = reinterpret_cast<char*>(workspace);
  unsigned* const status = reinterpret_cast<unsigned*>(ws);
  // The tensor-core path, where it takes the operands and its cost model
  // says it is the faster one (never below batch 8); split K adds its fp32
  // partials with the split-K reduce, in split order.
  if ((flags & LUTGEMM_ALLOW_TENSOR_CORES) != 0u && !stall && batch >= 8 && !scales_packed && n % 128 == 0 &&
      g % 64 == 0) {
    const int nsplit = tc_plan(m, n, batch, q, ceil_div(n, kSliceInputs));
    if (nsplit > 0) {
      float* part = nsplit > 1 ? reinterpret_cast<float*>(ws + kPartOffset) : nullptr;
      cudaError_t e = launch_tc_gemm(packed, reinterpret_cast<const __half*>(alpha), offset,
                                     reinterpret_cast<const __half*>(x), y, part, nsplit, m, n, batch, q, g,
                                     y_f16 ? 1 : 0, status, reinterpret_cast<cudaStream_t>(stream));
      if (e == cudaSuccess && nsplit > 1) {
        RunParams r = {};
        r.part = part;
        r.y = y;
        r.m = m;
        r.n = n;
        r.batch = batch;
        r.q = q;
        r.g = g;
        r.ns = nsplit;
        r.mt = ceil_div(m, kTileRows);
        r.y_f16 = y_f16 ? 1 : 0;
        e = launch_splitk_reduce(r, reinterpret_cast<cudaStream_t>(stream));
      }
      return e == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
    }
  }

  RunParams p = {};
  p.packed = packed;
  p.alpha = reinterpret_cast<const __half*>(alpha);
  p.offset = offset;
  p.x = reinterpret_cast<const __half*>(x);
  p.y = y;
  p.m = m;
  p.n = n;
  p.batch = batch;
  p.q = q;
  p.g = g;
  p.y_f16 = y_f16 ? 1 : 0;
  p.stall_test = stall ? 1 : 0;
  return launch_lookup(p, select_kernel(q, group_mode(g), offset != nullptr, scales_packed), workspace,
                       reinterpret_cast<cudaStream_t>(stream));
}

int lutgemm_mixed_offsets(const uint8_t* block_planes, int q_max, int m, int n, uint32_t* offsets) {
  if (!block_planes || !offsets) return LUTGEMM_ERR_NULL;
  if (q_max < 1 || q_max > 4 || m < 1 || n < 8 || n % 8 != 0) return LUTGEMM_ERR_SHAPE;
  const long long blocks = (long long)ceil_div(n, kSliceInputs) * ceil_div(m, kTileRows);
  unsigned long long acc = 0;
  for (long long u = 0; u < blocks; ++u)
    if (block_planes[u] < 1 || block_planes[u] > q_max) return LUTGEMM_ERR_VALUE;
  for (long long u = 0; u < blocks; ++u) {
    offsets[u] = (uint32_t)acc;
    acc += block_planes[u];
  }
  if (acc > 0xFFFFFFFFull) return LUTGEMM_ERR_SHAPE;
  offsets[blocks] = (uint32_t)acc;
  return LUTGEMM_OK;
}

int lutgemm_pack_outliers(const int32_t* row_ptr, const int32_t* col, const uint16_t* val, int m, int n, int nnz,
                          uint32_t* optr, uint32_t* oent) {
  if (!row_ptr || !optr || (nnz > 0 && (!col || !val || !oent))) return LUTGEMM_ERR_NULL;
  if (m < 1 || n < 8 || n % 8 != 0 || nnz < 0) return LUTGEMM_ERR_SHAPE;
  if (row_ptr[0] != 0 || row_ptr[m] != nnz) return LUTGEMM_ERR_VALUE;
  for (int r = 0; r < m; ++r) {
    if (row_ptr[r + 1] < row_ptr[r]) return LUTGEMM_ERR_VALUE;
    for (int e = row_ptr[r]; e < row_ptr[r + 1]; ++e)
      if (col[e] < 0 || col[e] >= n || (e > row_ptr[r] && col[e] <= col[e - 1])) return LUTGEMM_ERR_VALUE;
  }
  const int ns = ceil_div(n, kSliceInputs);
  // Within a row the entries are sorted by input, so each row's entries of
  // slice s are one run; a cursor per row walks them slice by slice.
  uint32_t out = 0;
  optr[0] = 0;
  for (int s_ = 0; s_ < ns; ++s_) {
    for (int r = 0; r < m; ++r) {
      int e = row_ptr[r];
      while (e < row_ptr[r + 1] && col[e] < s_ * kSliceInputs) ++e;
      for (; e < row_ptr[r + 1] && col[e] < (s_ + 1) * kSliceInputs; ++e)
        oent[out++] = (uint32_t)(col[e] - s_ * kSliceInputs) | ((uint32_t)val[e] << 16);
      optr[(size_t)s_ * m + r + 1] = out;
    }
  }
  return LUTGEMM_OK;
}

int lutgemm_pack_bcq_mixed(const int8_t* signs, const uint32_t* block_off, int q_max, int m, int n,
                           uint8_t* packed, size_t packed_bytes, int32_t* status_flags, void* stream) {
  if (!signs || !block_off || !packed) return LUTGEMM_ERR_NULL;
  if (q_max < 1 || q_max > 4 || !valid_matrix(q_max, m, n)) return LUTGEMM_ERR_SHAPE;
  if (!aligned(signs, 8) || !aligned(block_off, 4) || !aligned(packed, 16) || !aligned(status_flags, 4))
    return LUTGEMM_ERR_ALIGN;
  if (packed_bytes % kBlockBytes != 0 ||
      packed_bytes < (size_t)ceil_div(n, kSliceInputs) * ceil_div(m, kTileRows) * kBlockBytes)
    return LUTGEMM_ERR_VALUE;
  const cudaError_t err = launch_pack_signs_mixed(signs, block_off, q_max, m, n, packed, packed_bytes, status_flags,
                                                  reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_pack_scales_mixed(const uint16_t* alpha, const uint32_t* block_off, int q_max, int m, int n, int g,
                              uint16_t* scales, size_t scales_bytes, int32_t* status_flags, void* stream) {
  if (!alpha || !block_off || !scales) return LUTGEMM_ERR_NULL;
  if (q_max < 1 || q_max > 4 || !valid_matrix(q_max, m, n) || !valid_groups(n, g) || !(g % 128 == 0 || g == 64))
    return LUTGEMM_ERR_SHAPE;
  if (!aligned(alpha, 2) || !aligned(block_off, 4) || !aligned(scales, 16) || !aligned(status_flags, 4))
    return LUTGEMM_ERR_ALIGN;
  const size_t per_plane = g == 64 ? 1024u : 512u;
  if (scales_bytes % per_plane != 0 ||
      scales_bytes < (size_t)ceil_div(n, kSliceInputs) * ceil_div(m, kTileRows) * per_plane)
    return LUTGEMM_ERR_VALUE;
  const cudaError_t err = launch_pack_scales_mixed(reinterpret_cast<const __half*>(alpha), block_off, q_max, m, n, g,
                                                   scales, scales_bytes, status_flags,
                                                   reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
}

int lutgemm_run_mixed(int m, int n, int batch, int q_max, int g, const uint8_t* packed, size_t packed_bytes,
                      const uint32_t* block_off, const uint16_t* alpha, const uint32_t* optr, const uint32_t* oent,
                      int nnz, const uint16_t* x, void* y, unsigned flags, void* workspace, size_t workspace_bytes,
                      void* stream) {
  if (!packed || !block_off || !alpha || !x || !y || !workspace) return LUTGEMM_ERR_NULL;
  if (nnz > 0 && (optr == nullptr || oent == nullptr)) return LUTGEMM_ERR_NULL;
  if (q_max < 1 || q_max > 4 || !valid_matrix(q_max, m, n) || !valid_groups(n, g) || batch < 1 || nnz < 0)
    return LUTGEMM_ERR_SHAPE;
  if ((long long)batch * ceil_div(n, kSliceInputs) >= (1ll << 31)) return LUTGEMM_ERR_SHAPE;
  if ((flags & ~(LUTGEMM_Y_F16 | LUTGEMM_SCALES_PACKED | LUTGEMM_TEST_STALL)) != 0u) return LUTGEMM_ERR_VALUE;
  const bool y_f16 = (flags & LUTGEMM_Y_F16) != 0u;
  const bool scales_packed = (flags & LUTGEMM_SCALES_PACKED) != 0u;
  if (scales_packed && !(g % 128 == 0 || g == 64)) return LUTGEMM_ERR_VALUE;
  if (packed_bytes % kBlockBytes != 0 || packed_bytes / kBlockBytes > 0xFFFFFFFFull) return LUTGEMM_ERR_VALUE;
  if (!aligned(packed, 16) || !aligned(block_off, 4) || !aligned(alpha, scales_packed ? 16 : 2) || !aligned(optr, 4) ||
      !aligned(oent, 4) || !aligned(x, 16) || !aligned(y, y_f16 ? 2 : 4) || !aligned(workspace, 16))
    return LUTGEMM_ERR_ALIGN;
  if (workspace_bytes < lutgemm_workspace_size(m, n, batch, q_max, g)) return LUTGEMM_ERR_WORKSPACE;
  RunParams p = {};
  p.packed = packed;
  p.alpha = reinterpret_cast<const __half*>(alpha);
  p.offset = nullptr;
  p.x = reinterpret_cast<const __half*>(x);
  p.y = y;
  p.m = m;
  p.n = n;
  p.batch = batch;
  p.q = q_max;
  p.g = g;
  p.y_f16 = y_f16 ? 1 : 0;
  p.stall_test = (flags & LUTGEMM_TEST_STALL) != 0u ? 1 : 0;
  p.block_off = block_off;
  p.packed_blocks = (uint32_t)(packed_bytes / kBlockBytes);
  p.optr = nnz > 0 ? optr : nullptr;
  p.oent = nnz > 0 ? oent : nullptr;
  p.nnz = (uint32_t)nnz;
  return launch_lookup(p, run_kernel_mixed(group_mode(g), scales_packed), workspace,
                       reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
