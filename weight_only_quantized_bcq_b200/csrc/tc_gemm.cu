// Large-batch BCQ product on the tensor cores (tcgen05), for batches where the
// lookup kernel's per-column table reads dominate.
//
// Same result as the lookup path: y[b][r] = sum_i sum_k alpha_i[r][G(k)] *
// beta_i[r][k] * x[b][k] (LUT-GEMM card, Summary: weights stored as q binary
// planes with group-wise scales).  Each plane is fed to the tensor cores as
// its exact fp16 values +-alpha_i (an fp16 times a sign is exact), so no
// dequantised weight is ever rounded; the planes accumulate into one fp32
// tensor-memory accumulator.  Needs g % 128 == 0 (one scale per plane and
// 128-input piece) and no uniform offsets.
//
// CTA tile: 128 rows (MMA M) x BN batch columns (MMA N) over K blocks of 128
// inputs (one piece of the packed layout).  Warps 0-7 expand a plane's bits
// for the tile into a 128 x 128 fp16 A tile in shared memory (128-byte
// swizzled, K-major: the canonical UMMA layout; warps w and w+4 take the two
// 64-input halves of rows 32(w mod 4)..+31); warp 12 loads the x tile by TMA
// (same swizzle), issues the 8 tcgen05.mma (K = 16 each) per plane and
// commits them to mbarriers that free the buffers.  Three A buffers and two
// x buffers form the pipeline.
//
// Accumulation: the tensor cores add into their fp32 accumulator with
// truncation, so an error of up to an ulp per MMA step would build up over
// the q * n / 16 steps of a long row.  Each K block therefore accumulates in
// a fresh tensor-memory buffer (two, ping-pong), and warps 8-11 add it into
// fp32 running sums (round to nearest) as soon as its MMAs complete; warp
// 8+w owns accumulator lanes 32w..32w+31 = tile rows, keeps the running sums
// in a third tensor-memory buffer and writes them to y.
// Every mbarrier wait is bounded (1 s); a timeout sets status bit 2, the CTA
// stops issuing work, waits (bounded) for its tensor-core work in flight and
// frees its tensor memory before exiting.
#include <cuda.h>

#include "lutgemm.h"
#include "lutgemm_common.cuh"

namespace lutgemm {

namespace {

constexpr int kTcDequantThreads = 256;                 // warps 0-7
constexpr int kTcFlushThreads = 128;                   // warps 8-11
constexpr int kTcThreads = kTcDequantThreads + kTcFlushThreads + 32;   // + warp 12: TMA and MMA
constexpr int kTcAStages = 3;
constexpr int kTcBM = 128;
constexpr int kTcBK = 128;
constexpr uint32_t kTcATile = kTcBM * kTcBK * 2;      // 32 KB
constexpr uint64_t kWaitNs = 1000000000ull;

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred P;\n mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n selp.u32 %0, 1, 0, P;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
  if (bar_try(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  while (!bar_try(bar, parity))
    if (now_ns() - t0 > kWaitNs) return false;
  return true;
}

__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(addr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (start address and offsets in 16-byte units).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const uint8_t* __restrict__ packed,
                   const __half* __restrict__ alpha, void* y, int m, int n, int batch, int q, int g, int mt,
                   int y_f16, unsigned* status) {
  constexpr uint32_t kBTile = (uint32_t)BN * kTcBK * 2;   // x tile: BN rows x 128 inputs
  // Instruction descriptor: fp32 accumulator, fp16 A and B, both K-major, N = BN, M = 128.
  constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kTcBM >> 4) << 24);

  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  const uint32_t raw = (uint32_t)__cvta_generic_to_shared(tc_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sA = base;                                  // kTcAStages x 32 KB
  const uint32_t sB = base + kTcAStages * kTcATile;          // 2 x kBTile
  const uint32_t bars = sB + 2 * kBTile;                     // 15 mbarriers
  const uint32_t fullA = bars, emptyA = bars + 24, fullB = bars + 48, emptyB = bars + 64, done = bars + 80;
  const uint32_t accFull = bars + 88, accFree = bars + 104;
  const uint32_t tmem_slot = bars + 120;
  const uint32_t flag_slot = bars + 124;                     // CTA failure flag (shared)
  // Tensor memory: two accumulator buffers and the running sums, BN columns each.
  constexpr uint32_t kTmemCols =
      3 * BN <= 32 ? 32 : (3 * BN <= 64 ? 64 : (3 * BN <= 128 ? 128 : (3 * BN <= 256 ? 256 : 512)));
  static_assert(3 * BN <= 512, "three BN-column buffers must fit tensor memory");

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int rb = blockIdx.x;                                 // 128-row block
  const int b0 = blockIdx.y * BN;                            // first batch column
  const int nkb = n / kTcBK;
  const int ng = n / g;

  if (tid == 0) {
    for (int s = 0; s < kTcAStages; ++s) {
      bar_init(fullA + 8 * s, kTcDequantThreads);
      bar_init(emptyA + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      bar_init(fullB + 8 * s, 1);
      bar_init(emptyB + 8 * s, 1);
    }
    bar_init(done, 1);
    for (int s = 0; s < 2; ++s) {
      bar_init(accFull + 8 * s, 1);
      bar_init(accFree + 8 * s, kTcFlushThreads);
    }
    asm volatile("st.shared.u32 [%0], 0;" ::"r"(flag_slot) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(tmem_slot) : "memory");

  auto fail = [&]() {
    asm volatile("st.shared.u32 [%0], 1;" ::"r"(flag_slot) : "memory");
    atomicOr(status, kStatusTimeout);
  };
  auto failed = [&]() {
    uint32_t f;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(f) : "r"(flag_slot) : "memory");
    return f != 0;
  };

  if (warp < 8) {
    // ---- Dequant warps: plane tiles of +-alpha in the swizzled K-major layout.
    const int wq = warp & 3;                                 // rows 32wq..32wq+31 of the tile
    const int hsel = warp >> 2;                              // K half: runs 8 hsel .. 8 hsel + 7
    const int R = rb * 4 + wq;                               // 32-row tile of this warp
    const int row = R * kTileRows + lane;                    // weight row of this thread
    const int lrow = wq * 32 + lane;                         // row within the 128-row tile
    const uint32_t rowoff = (uint32_t)(lrow >> 3) * 1024u + (uint32_t)(lrow & 7) * 128u;
    const uint32_t sw = (uint32_t)(lrow & 7);
    const int half_sel = lane >> 4;
    const int lam = lane & 15;
    // The plane bits and scale of plane step ai = kb * q + i are loaded kPf
    // steps ahead, so their global-memory latency overlaps the expansion of
    // the steps before.
    constexpr int kPf = 3;
    const int nsteps = nkb * q;
    auto load_step = [&](int ai, uint4& bits, uint32_t& ah) {
      bits = make_uint4(0, 0, 0, 0);
      ah = 0;
      if (ai < nsteps && R < mt) {
        const int kb = ai / q, i = ai - kb * q;
        const int s = kb >> 3, P = kb & 7;
        const int U = P ^ (4 * half_sel);
        const int G = (s * kSliceInputs + 128 * P) / g;
        bits = __ldg(reinterpret_cast<const uint4*>(packed + ((((size_t)s * mt + R) * 8 + U) * q + i) * 512 +
                                                    (size_t)lane * 16));
        if (row < m) ah = __ldg(reinterpret_cast<const unsigned short*>(alpha) + ((size_t)i * ng + G) * m + row);
      }
    };
    uint4 pb[kPf];
    uint32_t pa[kPf];
#pragma unroll
    for (int d = 0; d < kPf; ++d) load_step(d, pb[d], pa[d]);
    for (int ai = 0; ai < nsteps && !failed(); ++ai) {
      const int st = ai % kTcAStages;
      const uint4 bits = pb[0];
      const uint32_t ah = pa[0];
#pragma unroll
      for (int d = 0; d + 1 < kPf; ++d) {
        pb[d] = pb[d + 1];
        pa[d] = pa[d + 1];
      }
      load_step(ai + kPf, pb[kPf - 1], pa[kPf - 1]);
      if (ai >= kTcAStages && !bar_wait(emptyA + 8 * st, (uint32_t)(((ai - kTcAStages) / kTcAStages) & 1))) {
        fail();
        break;
      }
      const uint32_t pos = ah, neg = ah ^ 0x8000u;
      const uint32_t dst = sA + (uint32_t)st * kTcATile + rowoff;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {                      // run c = 8 hsel + cc: inputs 8c..8c+7 of the piece
        const int c = 8 * hsel + cc;
        const int j = c ^ lam;                               // byte of the lane's piece holding run c
        const uint32_t word = j < 4 ? bits.x : (j < 8 ? bits.y : (j < 12 ? bits.z : bits.w));
        const uint32_t b = (word >> (8 * (j & 3))) & 0xFFu;
        uint32_t v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t lo = ((b >> (2 * e)) & 1u) ? pos : neg;
          const uint32_t hi = ((b >> (2 * e + 1)) & 1u) ? pos : neg;
          v[e] = lo | (hi << 16);
        }
        const uint32_t a = dst + (uint32_t)hsel * (kTcATile / 2) + (((uint32_t)cc ^ sw) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v[0]), "r"(v[1]), "r"(v[2]),
                     "r"(v[3])
                     : "memory");
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      bar_arrive(fullA + 8 * st);
    }
  } else if (warp == 12 && lane == 0) {
    // ---- Control thread: x tiles by TMA, MMAs, commits.
    auto load_x = [&](int kb) {
      const int st = kb & 1;
      const uint32_t bar = fullB + 8 * st;
      const uint32_t dst = sB + (uint32_t)st * kBTile;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kBTile) : "memory");
#pragma unroll
      for (int h = 0; h < 2; ++h)
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
                dst + (uint32_t)h * (kBTile / 2)),
            "l"(&xmap), "r"(kb * kTcBK + 64 * h), "r"(b0), "r"(bar)
            : "memory");
    };
    load_x(0);
    bool ok = true;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int sb = kb & 1;
      // Refill the other x buffer (last used by kb - 1) with kb + 1.
      if (kb + 1 < nkb) {
        if (kb >= 1 && !bar_wait(emptyB + 8 * ((kb + 1) & 1), (uint32_t)(((kb - 1) >> 1) & 1))) {
          ok = false;
          break;
        }
        load_x(kb + 1);
      }
      if (!bar_wait(fullB + 8 * sb, (uint32_t)((kb >> 1) & 1))) {
        ok = false;
        break;
      }
      // The accumulator buffer of this K block is free once warps 4-7 have
      // added in what it held for K block kb - 2.
      const uint32_t acc_tm = tmem + (uint32_t)(kb & 1) * BN;
      if (kb >= 2 && !bar_wait(accFree + 8 * (kb & 1), (uint32_t)(((kb - 2) >> 1) & 1))) {
        ok = false;
        break;
      }
      for (int i = 0; i < q; ++i) {
        const int ai = kb * q + i, st = ai % kTcAStages;
        if (!bar_wait(fullA + 8 * st, (uint32_t)((ai / kTcAStages) & 1))) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = sA + (uint32_t)st * kTcATile;
        const uint32_t bb0 = sB + (uint32_t)sb * kBTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t da = smem_desc(a0 + (uint32_t)(kk >> 2) * (kTcATile / 2) + (uint32_t)(kk & 3) * 32u);
          const uint64_t db = smem_desc(bb0 + (uint32_t)(kk >> 2) * (kBTile / 2) + (uint32_t)(kk & 3) * 32u);
          const uint32_t acc = (i | kk) != 0 ? 1u : 0u;     // each K block starts a fresh sum
          asm volatile(
              "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
              " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(acc_tm),
              "l"(da), "l"(db), "r"(kIdesc), "r"(acc)
              : "memory");
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         emptyA + 8 * st)
                     : "memory");
        if (i == q - 1) {
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           emptyB + 8 * sb)
                       : "memory");
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           accFull + 8 * (kb & 1))
                       : "memory");
        }
      }
    }
    if (!ok) fail();
    // Completion of everything issued (also after a failure, before tensor memory is freed).
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(done)
                 : "memory");
  }

  // ---- Warps 8-11: add each K block's accumulator into the running sums
  // (tensor memory, fp32 adds with round to nearest), then write y.
  bool wrote = true;
  if (warp >= 8 && warp < 12) {
    const int wq = warp - 8;                                 // accumulator lanes 32wq..32wq+31
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t run_tm = lane_base + 2u * BN;
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      ok = ok && __all_sync(0xffffffffu, bar_wait(accFull + 8 * (kb & 1), (uint32_t)((kb >> 1) & 1)));
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t acc_tm = lane_base + (uint32_t)(kb & 1) * BN;
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t a[32], r[32];
        tmem_ld32(acc_tm + (uint32_t)c0, a);
        if (kb > 0) tmem_ld32(run_tm + (uint32_t)c0, r);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
          r[jj] = kb > 0 ? __float_as_uint(__uint_as_float(r[jj]) + __uint_as_float(a[jj])) : a[jj];
        tmem_st32(run_tm + (uint32_t)c0, r);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      bar_arrive(accFree + 8 * (kb & 1));
    }
    wrote = ok;
    if (!ok && lane == 0) fail();
    const int row = (rb * 4 + wq) * kTileRows + lane;
    if (ok) {
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(run_tm + (uint32_t)c0, r);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (row < m) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int b = b0 + c0 + jj;
            if (b < batch) {
              const size_t o = (size_t)b * m + row;
              const float f = __uint_as_float(r[jj]);
              if (y_f16) reinterpret_cast<__half*>(y)[o] = __float2half_rn(f);
              else reinterpret_cast<float*>(y)[o] = f;
            }
          }
        }
      }
    }
  }
  (void)wrote;
  // Everything issued has completed before tensor memory is freed.
  const bool all_done = __all_sync(0xffffffffu, bar_wait(done, 0));
  if (!all_done && lane == 0) atomicOr(status, kStatusTimeout);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // Tensor memory is freed only once the accumulator has no work in flight.
    if (all_done)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                   : "memory");
  }
}

// Sticky status word of the tensor-core path (bit 2: a wait timed out).
__device__ unsigned g_tc_status;

template <int BN>
size_t tc_smem_bytes() {
  return 1024 + kTcAStages * (size_t)kTcATile + 2 * (size_t)BN * kTcBK * 2 + 128;
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

template <int BN>
cudaError_t launch_bn(const uint8_t* packed, const __half* alpha, const __half* x, void* y, int m, int n,
                      int batch, int q, int g, int y_f16, unsigned* status, cudaStream_t stream) {
  EncodeTiled enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)batch};
  const cuuint64_t strides[1] = {(cuuint64_t)n * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)BN};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(x), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = tc_smem_bytes<BN>();
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_done[64] = {false};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    e = cudaFuncSetAttribute(tc_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  if (status == nullptr) {
    void* sp = nullptr;
    e = cudaGetSymbolAddress(&sp, g_tc_status);
    if (e != cudaSuccess) return e;
    status = static_cast<unsigned*>(sp);
  }
  const int mt = (m + kTileRows - 1) / kTileRows;
  dim3 grid((unsigned)((m + kTcBM - 1) / kTcBM), (unsigned)((batch + BN - 1) / BN));
  tc_gemm_kernel<BN><<<grid, kTcThreads, smem, stream>>>(map, packed, alpha, y, m, n, batch, q, g, mt, y_f16, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm(const uint8_t* packed, const __half* alpha, const __half* x, void* y, int m, int n,
                           int batch, int q, int g, int y_f16, unsigned* status, cudaStream_t stream) {
  if (batch <= 32) return launch_bn<32>(packed, alpha, x, y, m, n, batch, q, g, y_f16, status, stream);
  if (batch <= 64) return launch_bn<64>(packed, alpha, x, y, m, n, batch, q, g, y_f16, status, stream);
  return launch_bn<128>(packed, alpha, x, y, m, n, batch, q, g, y_f16, status, stream);
}

}  // namespace lutgemm
