// Large-batch BCQ product on the tensor cores (tcgen05), for batches where the
// lookup kernel's per-column table reads dominate.
//
// Same result as the lookup path: y[b][r] = sum_i sum_k alpha_i[r][G(k)] *
// beta_i[r][k] * x[b][k] (LUT-GEMM card, Summary: weights stored as q binary
// planes with group-wise scales).  Each plane is fed to the tensor cores as
// its exact fp16 values +-alpha_i (an fp16 times a sign is exact), so no
// dequantised weight is ever rounded; the planes accumulate into one fp32
// tensor-memory accumulator.  Needs g % 64 == 0: a 64-input half of a
// 128-input K block then lies in one scale group.  Group offsets (uniform
// weights rewritten as BCQ) are added per K block in fp32 by the accumulate
// warps.
//
// CTA tile: 128 rows (MMA M) x BN batch columns (MMA N) over K blocks of 128
// inputs (one piece of the packed layout).  Warp roles:
//   warp 21 (producer): streams the operands into a shared-memory ring of
//     units.  A unit is the K-block pair (P, P ^ 4) of one 1024-input slice:
//     those two blocks read the same two chunk groups of the packed layout
//     (lanes 0-15 of a row tile hold piece P in chunk P, lanes 16-31 in
//     chunk P ^ 4), so one copy per chunk group serves both.  Each unit
//     holds the two x tiles (128-byte swizzle, K-major), the 8 chunk groups
//     of the tile's 4 row tiles and the scale rows of the tile (per K block
//     and plane one row, or one per 64-input half when g = 64), fetched by
//     4-6 TMA tensor copies: one per x tile (both 64-input halves), one per
//     chunk group (all planes of the 4 row tiles), one per K block and scale
//     group (all planes).
//   warps 0-15 (dequant, two groups of 8 taking alternate plane steps):
//     expand a plane's bits for the tile into a 128 x 128 fp16 A tile in
//     tensor memory (row r in lane r, inputs 2c and 2c+1 in column c: the
//     layout the tensor cores read an A operand from); in a group, warp w
//     takes rows 32(w mod 4)..+31 (the lanes it may access) and the
//     64-input half (w / 4) mod 2.  A never touches shared memory.  A warp
//     visits only its group's steps; a unit slot is released by the MMA
//     warp's commit alone (that commit follows its waits for every step of
//     the unit, and each step's barrier is arrived after the reads).
//   warp 20 (MMA): the converged warp runs the loop and one elected lane
//     issues the 8 tcgen05.mma (K = 16 each, A from tensor memory, B from
//     shared memory) per plane and the commits that free A stages, units
//     and accumulators.
//   warps 16-19 (accumulate): see below.
// Split K (grid z, whole 1024-input slices per split) writes fp32 partials
// that the split-K reduce of the lookup path adds in split order.
//
// Accumulation: the tensor cores add into their fp32 accumulator with
// truncation, so an error of up to an ulp per MMA step would build up over
// the q * n / 16 steps of a long row.  Each K block therefore accumulates in
// fresh tensor-memory buffers (two per K block at BN = 64, even and odd K
// steps, so consecutive MMAs are independent; one at BN = 32 and 128;
// ping-pong between K blocks),
// and warps 16-19 add them into fp32 running sums (round to nearest) as soon
// as the block's MMAs complete; warp 16+w owns accumulator lanes
// 32w..32w+31 = tile rows, keeps the running sums (in registers at BN = 32,
// in tensor memory above) and writes them to y.
// Every mbarrier wait is bounded (1 s); a timeout sets status bit 2, the CTA
// stops issuing work, waits (bounded) for its tensor-core work in flight and
// frees its tensor memory before exiting.
#include <cuda.h>

#include "lutgemm.h"
#include "lutgemm_common.cuh"

namespace lutgemm {

namespace {

constexpr int kTcDequantWarps = 16;                    // warps 0-15
constexpr int kTcFlushWarp0 = kTcDequantWarps;          // warps 16-19
constexpr int kTcMmaWarp = kTcFlushWarp0 + 4;           // warp 20
constexpr int kTcProdWarp = kTcMmaWarp + 1;             // warp 21
constexpr int kTcThreads = (kTcProdWarp + 1) * 32;
constexpr int kTcBM = 128;
constexpr int kTcBK = 128;
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

// The same, backing off between polls: for warps whose polling would take
// issue slots from the warps doing the work.
__device__ __forceinline__ bool bar_wait_sleep(uint32_t bar, uint32_t parity) {
  if (bar_try(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  while (!bar_try(bar, parity)) {
    __nanosleep(20);
    if (now_ns() - t0 > kWaitNs) return false;
  }
  return true;
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

// 8 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld8(uint32_t addr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(addr)
               : "memory");
}

// 16 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(addr)
      : "memory");
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

// Orders the computation of v before the following volatile asm statements
// (an empty statement that takes the 32 values as operands).
__device__ __forceinline__ void pin32(const uint32_t (&v)[32]) {
  asm volatile("" ::"r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
               "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
               "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
               "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]));
}

// tcgen05.commit from one elected lane of a converged warp: the mbarrier
// arrives once all tensor-core work this thread issued before has completed.
__device__ __forceinline__ void commit_one(uint32_t bar) {
  asm volatile(
      "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}" ::"r"(bar)
      : "memory");
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (start address and offsets in 16-byte units).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Units of the K loop in processing order: slice s, low piece P (0..3), and
// whether piece P + 4 exists in the slice.
struct UnitIter {
  int n, ns, s, P, np;
  // Slices s_begin .. s_end - 1 (the CTA's share of K).
  __device__ __forceinline__ void init(int n_, int s_begin, int s_end) {
    n = n_;
    ns = s_end;
    s = s_begin;
    P = 0;
    np = s < ns ? pieces(s) : 0;
  }
  __device__ __forceinline__ int pieces(int sl) const {
    const int r = (n - kSliceInputs * sl) / kTcBK;
    return r < 8 ? r : 8;
  }
  __device__ __forceinline__ bool valid() const { return s < ns; }
  __device__ __forceinline__ int count() const { return P + 4 < np ? 2 : 1; }   // K blocks in the unit
  __device__ __forceinline__ int kb(int which) const { return 8 * s + P + 4 * which; }
  __device__ __forceinline__ void next() {
    if (++P >= 4 || P >= np) {
      P = 0;
      if (++s < ns) np = pieces(s);
    }
  }
};

// Position in a ring of n slots: the slot and the parity of the pass over
// the ring (the mbarrier phase of the slot's current use).  Advanced one use
// at a time, so no division by a run-time ring size is needed.
struct RingPos {
  int n, slot;
  uint32_t phase;
  __device__ __forceinline__ void init(int n_) {
    n = n_;
    slot = 0;
    phase = 0;
  }
  __device__ __forceinline__ void next() {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

struct TcLayout {
  uint32_t slot_bytes;     // one unit: x tiles, chunk groups, scale rows (multiple of 1024)
  uint32_t bits_off;       // 8 chunk groups of q * 512 bytes: (half, row tile) = 4 h + wq
  uint32_t alpha_off;      // 2 x 2 x q scale rows of 128 fp16: (which, K half, plane)
  int nu;                  // ring depth in units
  int alpha_bulk;          // scale rows by bulk copy (16-byte aligned rows) or by lane loads
};

template <int BN, bool HAS_OFF>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap amap, const uint8_t* __restrict__ packed,
                   const __half* __restrict__ alpha, const float* __restrict__ offset, void* y, float* part,
                   int spz, int m, int n, int batch, int q, int g, int mt, int y_f16, unsigned* status, TcLayout L) {
  constexpr uint32_t kBTile = (uint32_t)BN * kTcBK * 2;   // x tile: BN rows x 128 inputs
  // Instruction descriptor: fp32 accumulator, fp16 A and B, both K-major, N = BN, M = 128.
  constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kTcBM >> 4) << 24);
  // Accumulator sets per K block.  At BN = 64 two sets (even and odd K steps
  // of every plane, summed when the K block is flushed) keep consecutive MMAs
  // independent.  At BN = 32 the 24 dependent MMAs of a K block into one set
  // issue at the same rate (measured), and one set leaves a seventh A stage
  // and halves the flush; at BN = 128 an MMA takes longer than the
  // dependency, and tensor memory holds one set only.
  constexpr int kSets = BN == 64 ? 2 : 1;
  // At BN = 32 the accumulate warps keep the running sums in registers (32
  // per thread); wider tiles keep them in tensor memory.
  constexpr bool kRunRegs = BN <= 32;
  // Tensor memory (all 512 columns): per K block (two, ping-pong) kSets
  // accumulators of BN columns, the running sums at 2 kSets BN, then kSA A
  // stages of 64 columns (128 rows x 128 fp16 inputs, two per column) from
  // column kACol0.
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kRunCol = 2u * kSets * BN;
  constexpr int kACol0 = ((2 * kSets + (kRunRegs ? 0 : 1)) * BN + 63) / 64 * 64;
  constexpr int kSA = (512 - kACol0) / 64 < 7 ? (512 - kACol0) / 64 : 7;
  static_assert(kSA >= 2, "at least two A stages must fit tensor memory");

  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  const uint32_t raw = (uint32_t)__cvta_generic_to_shared(tc_smem_raw);
  const uint32_t ring = (raw + 1023u) & ~1023u;
  const uint32_t bars = ring + (uint32_t)L.nu * L.slot_bytes;
  // mbarriers: 8 unit slots, 8 A stages, 2 accumulator buffers each.
  const uint32_t fullU = bars, emptyU = bars + 64, fullA = bars + 128, emptyA = bars + 192;
  const uint32_t accFull = bars + 256, accFree = bars + 272, done = bars + 288;
  const uint32_t tmem_slot = bars + 296;
  const uint32_t flag_slot = bars + 300;                     // CTA failure flag (shared)

  const int tid = threadIdx.x;
  // Broadcast from lane 0 so that the compiler knows the warp index, and all
  // that derives from it, is warp-uniform.
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
  const int lane = tid & 31;
  const int rb = blockIdx.x;                                 // 128-row block
  const int b0 = blockIdx.y * BN;                            // first batch column
  // Split K (grid z): slices z * spz .. of the input, written as fp32
  // partials part[b][z][32 mt] for the split-K reduce when part != nullptr.
  const int s_begin = (int)blockIdx.z * spz;
  const int s_all = (n + kSliceInputs - 1) / kSliceInputs;
  const int s_end = s_begin + spz < s_all ? s_begin + spz : s_all;
  const int nkb = (n / kTcBK < 8 * s_end ? n / kTcBK : 8 * s_end) - 8 * s_begin;   // K blocks of this split
  const int ng = n / g;
  // Scale group of K half h of K block kb (one per block when g % 128 == 0).
  const int halves_per_g = g / 64;
  const int apb = g % kTcBK == 0 ? 1 : 2;                   // distinct scale rows per K block and plane

  if (tid == 0) {
    for (int s = 0; s < L.nu; ++s) {
      bar_init(fullU + 8 * s, 1);
      // The MMA commit (+ the accumulate warps, which read the x tiles for the
      // offset term).  The commit follows the MMA warp's waits for every plane
      // step of the unit, each arrived after the dequant warps' reads of the
      // unit's bits and scales, so no dequant warp needs to arrive here.
      bar_init(emptyU + 8 * s, 1 + (HAS_OFF ? 4 : 0));
    }
    for (int s = 0; s < kSA; ++s) {
      bar_init(fullA + 8 * s, kTcDequantWarps / 2);       // one group of dequant warps per step
      bar_init(emptyA + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      bar_init(accFull + 8 * s, 1);
      bar_init(accFree + 8 * s, 128);
    }
    bar_init(done, 1);
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

  if (warp < kTcDequantWarps) {
    // ---- Dequant warps: plane tiles of +-alpha, written to tensor memory.
    // Two groups of 8 warps take alternate plane steps, so each warp has two
    // step periods for its part of a step and consecutive A stages are filled
    // by different warps.
    const int grp = warp >> 3;                               // plane steps ai with ai mod 2 == grp
    const int wq = warp & 3;                                 // tile rows (= TMEM lanes) 32wq..32wq+31
    const int hsel = (warp >> 2) & 1;                        // K half: runs 8 hsel .. 8 hsel + 7
    const int row = (rb * 4 + wq) * kTileRows + lane;        // weight row of this thread
    const int half_sel = lane >> 4;
    // The lane's 16-byte piece holds run c in byte c ^ (lane mod 16): runs
    // 8 hsel .. 8 hsel + 7 sit in its 8-byte half hsel ^ (bit 3 of the lane),
    // byte cc ^ (lane mod 8) for run 8 hsel + cc.  Two byte permutations per
    // step put them in run order.
    const int h8 = hsel ^ ((lane >> 3) & 1);
    uint32_t sel0 = 0, sel1 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      sel0 |= ((uint32_t)k ^ (uint32_t)(lane & 7)) << (4 * k);
      sel1 |= ((uint32_t)(k + 4) ^ (uint32_t)(lane & 7)) << (4 * k);
    }
    const uint32_t row_mask = row < m ? 0xFFFFFFFFu : 0u;   // rows past m get a zero scale
    const uint32_t a_tm = tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)kACol0 + (uint32_t)(32 * hsel);
    const uint32_t bits_lane = L.bits_off + (uint32_t)(wq * q * 512 + lane * 16 + h8 * 8);
    const uint32_t alpha_lane = L.alpha_off + (uint32_t)((wq * 32 + lane) * 2);
    // The group's plane steps are ai = grp, grp + 2, ...; the warp visits
    // only those, carrying the unit, the K block in the unit (w), the plane
    // (i) and the A stage along, and waits for a unit only when its next step
    // lies there.
    UnitIter it;
    it.init(n, s_begin, s_end);
    RingPos ur, ar;                                          // unit slot, A stage
    ur.init(L.nu);
    ar.init(kSA);
    int ai = 0, w = 0, i = 0;
    bool need_unit = true;                                   // the unit changed since the last wait
    // Moves the step position d plane steps on.
    auto advance = [&](int d) {
      ai += d;
      for (int k = 0; k < d; ++k) ar.next();
      i += d;
      while (i >= q && it.valid()) {
        i -= q;
        if (++w >= it.count()) {
          w = 0;
          it.next();
          ur.next();
          need_unit = true;
        }
      }
    };
    advance(grp);
    uint32_t slot = 0;
    bool go = true;
    // The stage whose store is still in flight (-1: none).  With enough A
    // stages (kDefer) a step's store is completed and its stage handed to the
    // MMA warp only after the warp has expanded its next step, so the store's
    // latency overlaps that work (FC1 at batch 32: 275 -> 268 us); with two
    // or three stages, holding a stage longer costs more than it hides.
    constexpr bool kDefer = kSA >= 4;
    int pend = -1;
    auto hand_over = [&]() {
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) bar_arrive(fullA + 8 * pend);
      pend = -1;
    };
    while (it.valid() && go) {
      if (need_unit) {
        // A store still in flight is handed over before waiting for a new
        // unit: the slot's refill may need the MMAs of that very step.
        if (pend >= 0) hand_over();
        slot = ring + (uint32_t)ur.slot * L.slot_bytes;
        if (!__all_sync(0xffffffffu, bar_wait_sleep(fullU + 8 * ur.slot, ur.phase))) {
          if (lane == 0) fail();
          break;
        }
        if (__any_sync(0xffffffffu, failed())) break;
        need_unit = false;
      }
      const int st = ar.slot;
      const uint32_t bsrc = slot + bits_lane + (uint32_t)(((half_sel ^ w) * 4 * q + i) * 512);
      const uint32_t asrc = slot + alpha_lane + (uint32_t)(((w * 2 + (apb == 2 ? hsel : 0)) * q + i) * 256);
      uint32_t b0w, b1w, ah;
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b0w), "=r"(b1w) : "r"(bsrc) : "memory");
      asm volatile("ld.shared.u16 %0, [%1];" : "=r"(ah) : "r"(asrc) : "memory");
      const uint32_t w0 = __byte_perm(b0w, b1w, sel0);       // runs 0..3 of the half, in order
      const uint32_t w1 = __byte_perm(b0w, b1w, sel1);       // runs 4..7
      // Element pair (2e, 2e+1) of a run byte rb8: the product rb8 *
      // (2^(15-2e) + 2^(30-2e)) puts bit 2e at bit 15 and bit 2e+1 at bit 31
      // (the two fp16 sign bits), with no carries between the two copies.  A
      // clear bit (beta = -1) sets the sign of +alpha.
      const uint32_t a2 = (ah | (ah << 16)) & row_mask;
      uint32_t v[32];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint32_t rb8 = __byte_perm(cc < 4 ? w0 : w1, 0u, 0x4440u | (uint32_t)(cc & 3));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t t = rb8 * ((1u << (15 - 2 * e)) + (1u << (30 - 2 * e)));
          v[4 * cc + e] = a2 ^ (~t & 0x80008000u);
        }
      }
      if (pend >= 0) {
        pin32(v);
        hand_over();
      }
      // The stage's previous use (one pass back) must have been consumed.
      if (ai >= kSA && !__all_sync(0xffffffffu, bar_wait_sleep(emptyA + 8 * st, ar.phase ^ 1u))) {
        if (lane == 0) fail();
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      tmem_st32(a_tm + (uint32_t)(st * 64), v);
      pend = st;
      if constexpr (!kDefer) hand_over();
      advance(2);
    }
    if (pend >= 0) hand_over();
    // No store of this warp is in flight when tensor memory is released.
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  } else if (warp == kTcProdWarp) {
    // ---- Producer: one unit of x tiles, chunk groups and scale rows per ring slot.
    UnitIter it;
    it.init(n, s_begin, s_end);
    RingPos ur;
    ur.init(L.nu);
    for (int u = 0; it.valid(); it.next(), ++u, ur.next()) {
      const int sl = ur.slot;
      const uint32_t slot = ring + (uint32_t)sl * L.slot_bytes;
      const uint32_t bar = fullU + 8 * sl;
      // The slot's previous use (one pass back) must have been released.
      if (u >= L.nu && !__all_sync(0xffffffffu, bar_wait_sleep(emptyU + 8 * sl, ur.phase ^ 1u))) {
        if (lane == 0) fail();
        break;
      }
      if (__any_sync(0xffffffffu, failed())) break;
      const int cnt = it.count();
      {
        // The whole warp computes the copies; one elected lane issues each.
        // Per K block one x tile (both 64-input halves); per chunk group
        // (P, P ^ 4) the q planes of the 4 row tiles; per K block and scale
        // group the q planes' scale rows.  Rows and row tiles past m are
        // filled with zeros and counted.
        uint32_t bytes = (uint32_t)cnt * kBTile + 8u * (uint32_t)q * 512u;
        if (L.alpha_bulk) bytes += (uint32_t)(cnt * apb * q * kTcBM * 2);
        asm volatile(
            "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
            " @e mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n}" ::"r"(bar),
            "r"(bytes)
            : "memory");
        for (int w = 0; w < cnt; ++w)
          asm volatile(
              "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
              " @e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
              "[%5];\n}" ::"r"(slot + (uint32_t)w * kBTile),
              "l"(&xmap), "r"(0), "r"(b0), "r"(2 * it.kb(w)), "r"(bar)
              : "memory");
#pragma unroll
        for (int h = 0; h < 2; ++h)
          asm volatile(
              "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
              " @e cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
              "[%1, {%2, %3, %4, %5, %6}], [%7];\n}" ::"r"(slot + L.bits_off + (uint32_t)(h * 4 * q * 512)),
              "l"(&bmap), "r"(0), "r"(0), "r"(it.P ^ (4 * h)), "r"(rb * 4), "r"(it.s), "r"(bar)
              : "memory");
        if (L.alpha_bulk) {
          for (int w = 0; w < cnt; ++w)
            for (int h = 0; h < apb; ++h) {
              const int G = (2 * it.kb(w) + h) / halves_per_g;
              asm volatile(
                  "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
                  " @e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
                  "[%1, {%2, %3, %4}], [%5];\n}" ::"r"(slot + L.alpha_off + (uint32_t)((w * 2 + h) * q * 256)),
                  "l"(&amap), "r"(rb * kTcBM), "r"(G), "r"(0), "r"(bar)
                  : "memory");
            }
        }
      }
      if (!L.alpha_bulk) {
        // Scale rows by plain loads: lane l covers rows 4l..4l+3 of the tile.
        for (int w = 0; w < cnt; ++w)
          for (int h = 0; h < apb; ++h) {
            const int G = (2 * it.kb(w) + h) / halves_per_g;
            for (int i = 0; i < q; ++i) {
              const unsigned short* src = reinterpret_cast<const unsigned short*>(alpha) + ((size_t)i * ng + G) * m;
              uint32_t v[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int r = rb * kTcBM + 4 * lane + k;
                v[k] = r < m ? (uint32_t)__ldg(src + r) : 0u;
              }
              asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(
                               slot + L.alpha_off + (uint32_t)(((w * 2 + h) * q + i) * 256 + lane * 8)),
                           "r"(v[0] | (v[1] << 16)), "r"(v[2] | (v[3] << 16))
                           : "memory");
            }
          }
      }
      __syncwarp();
      if (lane == 0) bar_arrive(bar);
    }
  } else if (warp == kTcMmaWarp) {
    // ---- MMA warp: per plane step, 8 MMAs into the K block's accumulator
    // buffers.  The whole warp runs the loop (its values stay warp-uniform,
    // as the MMA operands must be); one elected lane issues each MMA and
    // commit.
    UnitIter it;
    it.init(n, s_begin, s_end);
    int j = 0;                                               // K block (processing order)
    RingPos ur, ar;                                          // unit slot, A stage
    ur.init(L.nu);
    ar.init(kSA);
    bool ok = true;
    for (; it.valid() && ok; it.next(), ur.next()) {
      const int sl = ur.slot;
      const uint32_t slot = ring + (uint32_t)sl * L.slot_bytes;
      if (!__all_sync(0xffffffffu, bar_wait(fullU + 8 * sl, ur.phase))) {
        ok = false;
        break;
      }
      const int cnt = it.count();
      for (int w = 0; w < cnt && ok; ++w, ++j) {
        // The accumulator buffers of this K block are free once warps 16-19
        // have added in what they held for K block j - 2.
        const uint32_t acc_tm = tmem + (uint32_t)(j & 1) * kSets * BN;
        if (j >= 2 && !__all_sync(0xffffffffu, bar_wait(accFree + 8 * (j & 1), (uint32_t)(((j - 2) >> 1) & 1)))) {
          ok = false;
          break;
        }
        const uint64_t db0 = smem_desc(slot + (uint32_t)w * kBTile);
        for (int i = 0; i < q; ++i, ar.next()) {
          const int st = ar.slot;
          if (!__all_sync(0xffffffffu, bar_wait(fullA + 8 * st, ar.phase))) {
            ok = false;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t a0 = tmem + (uint32_t)kACol0 + (uint32_t)(st * 64);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // B: K step kk is 32 bytes into the 128-byte swizzle row, in the
            // first or second 64-input half of the x tile (descriptor start
            // address in 16-byte units).
            const uint64_t db = db0 + (uint64_t)(((kk >> 2) * (kBTile / 2) + (kk & 3) * 32) >> 4);
            // Each K block starts fresh sums; K step kk goes to set kk mod kSets.
            const uint32_t acc = (i | (kk / kSets)) != 0 ? 1u : 0u;
            asm volatile(
                "{\n .reg .pred p, e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
                " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(
                    acc_tm + (uint32_t)(kk % kSets) * BN),
                "r"(a0 + 8u * (uint32_t)kk), "l"(db), "r"(kIdesc), "r"(acc)
                : "memory");
          }
          commit_one(emptyA + 8 * st);
        }
        if (ok) commit_one(accFull + 8 * (j & 1));
      }
      // The unit's x tiles are free once its MMAs have completed.
      commit_one(emptyU + 8 * sl);
    }
    if (!ok && lane == 0) fail();
    // Completion of everything issued (also after a failure, before tensor memory is freed).
    commit_one(done);
  }

  // ---- Warps 16-19: add each K block's accumulator into the running sums
  // (fp32 adds with round to nearest; registers at BN = 32, tensor memory
  // above), then write y.  With offsets (uniform weights rewritten as BCQ)
  // each K block also adds off[G][r] * S_b, where S_b is the sum of the
  // block's 128 inputs of batch column b, summed in fp32 by every accumulate
  // warp from the x tile in shared memory (lane l holds the columns l, l + 32,
  // ...; a row of the 128-byte swizzled tile is one 128-byte line whose
  // 16-byte pieces are only permuted, so their sum is the row's sum).
  if (warp >= kTcFlushWarp0 && warp < kTcFlushWarp0 + 4) {
    const int wq = warp - kTcFlushWarp0;                     // accumulator lanes 32wq..32wq+31
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t run_tm = lane_base + kRunCol;
    const int row = (rb * 4 + wq) * kTileRows + lane;
    constexpr int kCols = BN / 32;                           // x columns summed by each lane
    auto store_y = [&](int c0, const uint32_t (&r)[32]) {
      if (row >= m) return;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const int b = b0 + c0 + jj;
        if (b < batch) {
          const float f = __uint_as_float(r[jj]);
          if (part != nullptr) {
            part[((size_t)b * gridDim.z + blockIdx.z) * ((size_t)mt * kTileRows) + row] = f;
          } else {
            const size_t o = (size_t)b * m + row;
            if (y_f16) reinterpret_cast<__half*>(y)[o] = __float2half_rn(f);
            else reinterpret_cast<float*>(y)[o] = f;
          }
        }
      }
    };
    // Sums of each 64-input half of this K block for the lane's x columns,
    // and the row's offsets of the halves' groups.
    auto offset_terms = [&](uint32_t xtile, int kb, float (&sx)[2][kCols], float (&offr)[2]) {
#pragma unroll
      for (int k = 0; k < kCols; ++k) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float acc = 0.f;
          const uint32_t line = xtile + (uint32_t)h * (kBTile / 2) + (uint32_t)(lane + 32 * k) * 128u;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t w0, w1, w2, w3;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                         : "r"(line + 16u * c)
                         : "memory");
            const uint32_t wv[4] = {w0, w1, w2, w3};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[e]));
              acc += f.x;
              acc += f.y;
            }
          }
          sx[h][k] = acc;
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
        offr[h] = row < m ? __ldg(offset + (size_t)((2 * kb + h) / halves_per_g) * m + row) : 0.f;
    };
    bool ok = true;
    uint32_t run[kRunRegs ? 32 : 1];
#pragma unroll
    for (int jj = 0; jj < (kRunRegs ? 32 : 1); ++jj) run[jj] = 0u;
    // K block j (processing order): wait for its MMAs, add its accumulators
    // (and the offset term) into the running sums, free the buffers.
    auto add_block = [&](int j, const float (&sx)[2][kCols], const float (&offr)[2]) -> bool {
      if (!__all_sync(0xffffffffu, bar_wait_sleep(accFull + 8 * (j & 1), (uint32_t)((j >> 1) & 1)))) return false;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t acc_tm = lane_base + (uint32_t)(j & 1) * kSets * BN;
      if constexpr (kRunRegs) {
        // 16-column pieces (two round trips per block); 8 with the offset
        // term, whose values need the registers.
        constexpr int kPiece = HAS_OFF ? 8 : 16;
#pragma unroll
        for (int c0 = 0; c0 < 32; c0 += kPiece) {
          uint32_t a[kPiece], b[kPiece];
          if constexpr (kPiece == 16) {
            tmem_ld16(acc_tm + (uint32_t)c0, a);
            if constexpr (kSets == 2) tmem_ld16(acc_tm + (uint32_t)(BN + c0), b);
          } else {
            tmem_ld8(acc_tm + (uint32_t)c0, a);
            if constexpr (kSets == 2) tmem_ld8(acc_tm + (uint32_t)(BN + c0), b);
          }
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int jj = 0; jj < kPiece; ++jj) {
            const float f = kSets == 2 ? __uint_as_float(a[jj]) + __uint_as_float(b[jj]) : __uint_as_float(a[jj]);
            float r = __uint_as_float(run[c0 + jj]) + f;       // the sums start at +0
            if constexpr (HAS_OFF) {
              r = fmaf(offr[0], __shfl_sync(0xffffffffu, sx[0][0], c0 + jj), r);
              r = fmaf(offr[1], __shfl_sync(0xffffffffu, sx[1][0], c0 + jj), r);
            }
            run[c0 + jj] = __float_as_uint(r);
          }
        }
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t a[32], r[32];
          tmem_ld32(acc_tm + (uint32_t)c0, a);
          if (kSets == 2) {
            tmem_ld32(acc_tm + (uint32_t)(BN + c0), r);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) a[jj] = __float_as_uint(__uint_as_float(a[jj]) + __uint_as_float(r[jj]));
          }
          if (j > 0) tmem_ld32(run_tm + (uint32_t)c0, r);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            float v = j > 0 ? __uint_as_float(r[jj]) + __uint_as_float(a[jj]) : __uint_as_float(a[jj]);
            if constexpr (HAS_OFF) {
              v = fmaf(offr[0], __shfl_sync(0xffffffffu, sx[0][c0 / 32], jj), v);
              v = fmaf(offr[1], __shfl_sync(0xffffffffu, sx[1][c0 / 32], jj), v);
            }
            r[jj] = __float_as_uint(v);
          }
          tmem_st32(run_tm + (uint32_t)c0, r);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      bar_arrive(accFree + 8 * (j & 1));
      return true;
    };
    if constexpr (HAS_OFF) {
      UnitIter it;
      it.init(n, s_begin, s_end);
      int j = 0;
      RingPos ur;
      ur.init(L.nu);
      for (; it.valid() && ok; it.next(), ur.next()) {
        const int sl = ur.slot;
        const uint32_t slot = ring + (uint32_t)sl * L.slot_bytes;
        ok = __all_sync(0xffffffffu, bar_wait_sleep(fullU + 8 * sl, ur.phase));
        if (!ok) break;
        const int cnt = it.count();
        for (int w = 0; w < cnt && ok; ++w, ++j) {
          float sx[2][kCols];
          float offr[2];
          offset_terms(slot + (uint32_t)w * kBTile, it.kb(w), sx, offr);
          ok = add_block(j, sx, offr);
        }
        // This warp has read the unit's x tiles.
        __syncwarp();
        if (lane == 0) bar_arrive(emptyU + 8 * sl);
      }
    } else {
      const float none[2][kCols] = {};
      const float zero2[2] = {0.f, 0.f};
      for (int j = 0; j < nkb && ok; ++j) ok = add_block(j, none, zero2);
    }
    if (ok) {
      if constexpr (kRunRegs) {
        store_y(0, run);
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(run_tm + (uint32_t)c0, r);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          store_y(c0, r);
        }
      }
    }
    if (!ok && lane == 0) fail();
  }
  // Everything issued has completed before tensor memory is freed.
  const bool all_done = __all_sync(0xffffffffu, bar_wait_sleep(done, 0));
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

// Shared memory: a ring of unit slots (x tiles, chunk groups, scale rows)
// plus the mbarriers, as deep as fits (2 to 4 units).
template <int BN>
TcLayout tc_layout(int q, bool alpha_bulk) {
  TcLayout L;
  const uint32_t xt = 2u * BN * kTcBK * 2;
  L.bits_off = xt;
  L.alpha_off = xt + 8u * (uint32_t)q * 512u;
  L.slot_bytes = (L.alpha_off + 4u * (uint32_t)q * 256u + 1023u) & ~1023u;
  const uint32_t budget = 227u * 1024u - 1024u - 512u;
  const int fit = (int)(budget / L.slot_bytes);
  L.nu = fit < 4 ? fit : 4;
  L.alpha_bulk = alpha_bulk ? 1 : 0;
  return L;
}

inline size_t tc_smem_bytes(const TcLayout& L) { return 1024 + (size_t)L.nu * L.slot_bytes + 512; }

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

template <int BN, bool HAS_OFF>
cudaError_t launch_bn(const uint8_t* packed, const __half* alpha, const float* offset, const __half* x, void* y,
                      float* part, int nsplit, int m, int n, int batch, int q, int g, int y_f16, unsigned* status,
                      cudaStream_t stream) {
  EncodeTiled enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // x as [n/64][batch][64] fp16: one box is the two 64-input halves of a K
  // block for BN batch rows (128-byte swizzle, K-major).
  CUtensorMap map;
  {
    const cuuint64_t dims[3] = {64, (cuuint64_t)batch, (cuuint64_t)n / 64};
    const cuuint64_t strides[2] = {(cuuint64_t)n * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)BN, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<__half*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // The packed planes as [slice][row tile][chunk group U][plane][256] uint16
  // (512-byte pieces): one box is the q pieces of the 4 row tiles of a
  // 128-row block for one chunk group; row tiles past m are zero-filled.
  CUtensorMap bmap;
  {
    const cuuint64_t mt = (cuuint64_t)((m + kTileRows - 1) / kTileRows);
    const cuuint64_t dims[5] = {256, (cuuint64_t)q, 8, mt, (cuuint64_t)((n + kSliceInputs - 1) / kSliceInputs)};
    const cuuint64_t strides[4] = {512, (cuuint64_t)q * 512, (cuuint64_t)q * 4096, mt * q * 4096};
    const cuuint32_t box[5] = {256, (cuuint32_t)q, 1, 4, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (enc(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 5, const_cast<uint8_t*>(packed), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // Scale rows by tensor copy when every row of the [q][n/g][m] scales starts
  // on a 16-byte boundary (one box: 128 rows of one group, all q planes,
  // rows past m zero-filled); otherwise the producer warp loads them.
  const bool alpha_bulk = m % 8 == 0 && (reinterpret_cast<uintptr_t>(alpha) % 16) == 0;
  CUtensorMap amap = map;
  if (alpha_bulk) {
    const cuuint64_t dims[3] = {(cuuint64_t)m, (cuuint64_t)(n / g), (cuuint64_t)q};
    const cuuint64_t strides[2] = {(cuuint64_t)m * 2, (cuuint64_t)(n / g) * (cuuint64_t)m * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kTcBM, 1, (cuuint32_t)q};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<__half*>(alpha), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const TcLayout L = tc_layout<BN>(q, alpha_bulk);
  if (L.nu < 2) return cudaErrorInvalidValue;
  const size_t smem = tc_smem_bytes(L);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int attr_bytes[64] = {0};
  if (attr_bytes[dev] < (int)smem) {
    e = cudaFuncSetAttribute(tc_gemm_kernel<BN, HAS_OFF>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_bytes[dev] = (int)smem;
  }
  if (status == nullptr) {
    void* sp = nullptr;
    e = cudaGetSymbolAddress(&sp, g_tc_status);
    if (e != cudaSuccess) return e;
    status = static_cast<unsigned*>(sp);
  }
  const int mt = (m + kTileRows - 1) / kTileRows;
  // Splits of whole slices; the caller passes a count with no empty split.
  const int s_all = (n + kSliceInputs - 1) / kSliceInputs;
  if (part == nullptr) nsplit = 1;
  const int spz = (s_all + nsplit - 1) / nsplit;
  if (nsplit < 1 || (s_all + spz - 1) / spz != nsplit) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((m + kTcBM - 1) / kTcBM), (unsigned)((batch + BN - 1) / BN), (unsigned)nsplit);
  tc_gemm_kernel<BN, HAS_OFF><<<grid, kTcThreads, smem, stream>>>(map, bmap, amap, packed, alpha, offset, y, part,
                                                                   spz, m, n, batch, q, g, mt, y_f16, status, L);
  return cudaGetLastError();
}

}  // namespace

// Device address of the tensor-core path's own status word on the current
// device (used when the caller gives none).
cudaError_t tc_status_address(unsigned** out) {
  void* sp = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&sp, g_tc_status);
  if (e != cudaSuccess) return e;
  *out = static_cast<unsigned*>(sp);
  return cudaSuccess;
}

cudaError_t launch_tc_gemm(const uint8_t* packed, const __half* alpha, const float* offset, const __half* x, void* y,
                           float* part, int nsplit, int m, int n, int batch, int q, int g, int y_f16, unsigned* status,
                           cudaStream_t stream) {
#define LUTGEMM_TC_LAUNCH(BNv, OFFv) \
  launch_bn<BNv, OFFv>(packed, alpha, offset, x, y, part, nsplit, m, n, batch, q, g, y_f16, status, stream)
  if (offset != nullptr) {
    if (batch <= 32) return LUTGEMM_TC_LAUNCH(32, true);
    if (batch <= 64) return LUTGEMM_TC_LAUNCH(64, true);
    return LUTGEMM_TC_LAUNCH(128, true);
  }
  if (batch <= 32) return LUTGEMM_TC_LAUNCH(32, false);
  if (batch <= 64) return LUTGEMM_TC_LAUNCH(64, false);
  return LUTGEMM_TC_LAUNCH(128, false);
#undef LUTGEMM_TC_LAUNCH
}

}  // namespace lutgemm
