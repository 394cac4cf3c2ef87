// lutgemm_run_noalloc: the LUT-GEMM product for callers that cannot allocate
// device memory.  Some callers own no allocator of their own: a serving
// runtime that hands all device memory to its own pool up front, a plugin or
// FFI host that gives a kernel nothing but its input and output tensors, or a
// latency-critical path where an allocation (and its possible failure) is not
// acceptable.  They cannot provide the split-K workspace that lutgemm_run
// needs, so this entry point takes its scratch from a fixed-size array in the
// library's own device memory instead and allocates nothing.
//
// The scratch is a file-scope __device__ array: every GPU on which the library
// is loaded holds its LUTGEMM_NOALLOC_SCRATCH_BYTES until the process exits.
// Layout (fixed, independent of the problem size):
//   [0, 256)              status word (sticky error bits, read and cleared
//                         with lutgemm_library_status)
//   [256, +4 KB)          per-segment tile counters, zero between calls
//   [.., end)             split-K partial sums, written before they are read
// The counters sit at a fixed place so that they are never overlaid by
// another call's partial sums; the kernel resets every counter it uses, and
// the first call on a device zeroes them once.  Every call shares the array,
// so calls that overlap on the GPU (other streams, other host threads) race
// and must be serialised by the caller.
#include <mutex>
#include <set>
#include <utility>

#include "lutgemm.h"
#include "lutgemm_common.cuh"

namespace lutgemm {
cudaError_t launch_tc_gemm(const uint8_t* packed, const __half* alpha, const float* offset, const __half* x, void* y,
                           float* part, int nsplit, int m, int n, int batch, int q, int g, int y_f16, unsigned* status,
                           cudaStream_t stream);
cudaError_t tc_status_address(unsigned** out);
int tc_plan(int m, int n, int batch, int q, int max_split);
}  // namespace lutgemm

namespace {

using namespace lutgemm;

constexpr size_t kScratchBytes = LUTGEMM_NOALLOC_SCRATCH_BYTES;
constexpr size_t kStatusOff = 0;
constexpr size_t kTileCounterOff = 256;
constexpr size_t kPartOff = kTileCounterOff + kMaxTileCounters * sizeof(unsigned);

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct DeviceScratch {
  bool ready = false;
  unsigned char* base = nullptr;  // device address of g_scratch on this device
  int sm_count = 0;
};

std::mutex g_mutex;
DeviceScratch g_dev[64];
std::set<std::pair<const void*, int>> g_smem_done;

int ceil_div(int a, int b) { return (a + b - 1) / b; }
const __half* alpha_ptr_h(const uint16_t* a) { return reinterpret_cast<const __half*>(a); }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

RunKernel pick_kernel(int q, int g, bool has_offset, bool packed) {
  const int mode = g == 128 ? kG128 : (g % 128 == 0 ? kG128x : (g == 64 ? kG64 : (g == 8 ? kG8 : kGAny)));
  switch (q) {
    case 1: return run_kernel_q1(mode, has_offset, packed);
    case 2: return run_kernel_q2(mode, has_offset, packed);
    case 3: return run_kernel_q3(mode, has_offset, packed);
    case 4: return run_kernel_q4(mode, has_offset, packed);
    default: return run_kernel_q8(mode, has_offset, packed);
  }
}

// Once per device, with that device current: look up the scratch array's
// device address (the host-side name g_scratch is not a device address) and
// zero its status word and counters on the caller's stream, ordered before
// the first launch that uses them.
cudaError_t scratch_setup(cudaStream_t stream, DeviceScratch* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceScratch& d = g_dev[dev];
  if (!d.ready) {
    void* ptr = nullptr;
    err = cudaGetSymbolAddress(&ptr, g_scratch);
    if (err != cudaSuccess) return err;
    int sms = 0;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    err = cudaMemsetAsync(ptr, 0, kPartOff, stream);
    if (err != cudaSuccess) return err;
    d.base = static_cast<unsigned char*>(ptr);
    d.sm_count = sms;
    d.ready = true;
  }
  *out = d;
  return cudaSuccess;
}

// Once per kernel and device: the shared-memory window check and opt-in.
cudaError_t kernel_setup(RunKernel kernel) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_mutex);
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  if (g_smem_done.find(key) != g_smem_done.end()) return cudaSuccess;
  int reserved = 0, optin = 0;
  if ((err = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess)
    return err;
  if ((err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return err;
  // The tables sit at a fixed window address right after the reserved region,
  // and static shared memory would move the dynamic window off it.
  if ((unsigned)reserved != kTableBase || optin < kSmemBytes) return cudaErrorInvalidConfiguration;
  cudaFuncAttributes fa;
  err = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kernel));
  if (err != cudaSuccess) return err;
  if (fa.sharedSizeBytes != 0) return cudaErrorInvalidConfiguration;
  err = cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes);
  if (err != cudaSuccess) return err;
  g_smem_done.insert(key);
  return cudaSuccess;
}

}  // namespace

extern "C" int lutgemm_run_noalloc(int m, int n, int batch, int q, int g, const uint8_t* packed,
                                   const uint16_t* alpha, const float* offset, const uint16_t* x, void* y,
                                   unsigned flags, void* stream) {
  if (!packed || !alpha || !x || !y) return LUTGEMM_ERR_NULL;
  if (q < 1 || q > 8 || m < 1 || n < 8 || n % 8 != 0 || g < 8 || g % 8 != 0 || n % g != 0 || batch < 1)
    return LUTGEMM_ERR_SHAPE;
  if ((long long)batch * ceil_div(n, kSliceInputs) >= (1ll << 31)) return LUTGEMM_ERR_SHAPE;
  if ((flags & ~(LUTGEMM_Y_F16 | LUTGEMM_SCALES_PACKED | LUTGEMM_ALLOW_TENSOR_CORES | LUTGEMM_TEST_STALL)) != 0u)
    return LUTGEMM_ERR_VALUE;
  const bool y_f16 = (flags & LUTGEMM_Y_F16) != 0u;
  const bool scales_packed = (flags & LUTGEMM_SCALES_PACKED) != 0u;
  const bool stall = (flags & LUTGEMM_TEST_STALL) != 0u;
  if (scales_packed && !(g % 128 == 0 || g == 64)) return LUTGEMM_ERR_VALUE;
  if (!aligned(packed, 16) || !aligned(alpha, scales_packed ? 16 : 2) || !aligned(offset, 4) ||
      !aligned(x, 16) || !aligned(y, y_f16 ? 2 : 4))
    return LUTGEMM_ERR_ALIGN;
  const int ns = ceil_div(n, kSliceInputs);
  const int mt = ceil_div(m, kTileRows);
  // Split-K partials exist only with several slices; one slice writes y directly.
  const size_t partials = ns > 1 ? (size_t)batch * ns * mt * kTileRows * sizeof(float) : 0;
  const bool fits = partials <= kScratchBytes - kPartOff;
  // The tensor-core path with one K split needs no scratch.  It runs where
  // lutgemm_run would pick it, and also where the lookup kernel's partials
  // would not fit the scratch.
  const bool tc_ok = (flags & LUTGEMM_ALLOW_TENSOR_CORES) != 0u && !stall && batch >= 8 && !scales_packed &&
                     n % 128 == 0 && g % 64 == 0;
  const bool use_tc = tc_ok && (tc_plan(m, n, batch, q, 1) > 0 || !fits);
  if (!use_tc && !fits) return LUTGEMM_ERR_WORKSPACE;

  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DeviceScratch d;
  if (scratch_setup(st, &d) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  unsigned* const status = reinterpret_cast<unsigned*>(d.base + kStatusOff);
  if (use_tc) {
    const cudaError_t e = launch_tc_gemm(packed, alpha_ptr_h(alpha), offset, reinterpret_cast<const __half*>(x), y,
                                         nullptr, 1, m, n, batch, q, g, y_f16 ? 1 : 0, status, st);
    return e == cudaSuccess ? LUTGEMM_OK : LUTGEMM_ERR_CUDA;
  }

  const RunKernel kernel = pick_kernel(q, g, offset != nullptr, scales_packed);
  if (kernel == nullptr) return LUTGEMM_ERR_VALUE;
  if (kernel_setup(kernel) != cudaSuccess) return LUTGEMM_ERR_CUDA;

  RunParams p = {};
  p.packed = packed;
  p.alpha = reinterpret_cast<const __half*>(alpha);
  p.offset = offset;
  p.x = reinterpret_cast<const __half*>(x);
  p.y = y;
  p.part = reinterpret_cast<float*>(d.base + kPartOff);
  p.tile_cnt = reinterpret_cast<unsigned*>(d.base + kTileCounterOff);
  p.status = status;
  p.m = m;
  p.n = n;
  p.batch = batch;
  p.q = q;
  p.g = g;
  p.ns = ns;
  p.mt = mt;
  p.ng = n / g;
  p.y_f16 = y_f16 ? 1 : 0;
  p.stall_test = stall ? 1 : 0;
  p.total_units = (long long)batch * ns * mt;
  long long grid = 0;
  choose_launch(d.sm_count, (long long)batch * ns, mt, &grid, &p.seg_aligned);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, p) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return LUTGEMM_ERR_CUDA;
  if (p.ns > 1 && launch_splitk_reduce(p, st) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  return LUTGEMM_OK;
}

// The status words of the calls that run without a caller workspace, on the
// current device: the no-alloc scratch's and the tensor-core path's own.
extern "C" int lutgemm_library_status(uint32_t* status, int clear, void* stream) {
  if (!status) return LUTGEMM_ERR_NULL;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DeviceScratch d;
  if (scratch_setup(st, &d) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  unsigned* tc = nullptr;
  if (tc_status_address(&tc) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  unsigned* const words[2] = {reinterpret_cast<unsigned*>(d.base + kStatusOff), tc};
  unsigned v[2] = {0u, 0u};
  for (int k = 0; k < 2; ++k)
    if (cudaMemcpyAsync(&v[k], words[k], sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return LUTGEMM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  *status = v[0] | v[1];
  if (clear) {
    for (int k = 0; k < 2; ++k)
      if (v[k] != 0u && cudaMemsetAsync(words[k], 0, sizeof(unsigned), st) != cudaSuccess) return LUTGEMM_ERR_CUDA;
  }
  return LUTGEMM_OK;
}
