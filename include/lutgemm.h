/*
 * lutgemm.h -- C ABI of a B200 (sm_100a) LUT-GEMM library for weights stored
 * in binary-coding quantisation (BCQ).
 *
 * What the library computes (source: "LUT-GEMM -- paper by Park et al. (2022),
 * ICLR 2024", Elamur card, sections Summary and Interesting ideas; pith.science
 * card of the same paper, abstract):
 *
 *   A BCQ weight matrix W (m outputs x n inputs) is a sum of q binary planes,
 *   each scaled per group of g consecutive inputs:
 *       W[j,k] = sum_{i<q} alpha[i][k/g][j] * beta[i][j][k] (+ offset[k/g][j]),
 *   beta in {-1,+1}.  The product y = W x is formed without dequantising W:
 *   for every run of 8 activations the 256 possible signed sums are put in a
 *   table once, and each plane-row reads the entry indexed by its 8 sign bits
 *   ("Lookup tables instead of multiplications").  Uniform quantisation is
 *   rewritten as BCQ plus a per-group offset, so one kernel serves both
 *   (Summary; "One format for many schemes").  q and g are independent
 *   parameters ("Group size as a separate hyper-parameter").
 *
 * Conventions shared by every call
 *   - Every buffer is caller-owned and caller-allocated.  The library
 *     allocates nothing and keeps no state between calls, except that the
 *     workspace of lutgemm_run must be zero-filled once before its first use;
 *     its tile counters are left zero by every call, and its status word
 *     keeps its bits until lutgemm_workspace_status clears them.
 *   - "dev" pointers are CUDA device pointers on the current device; fp16
 *     values are passed as their raw 16-bit patterns (uint16_t).
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All device work is enqueued on it and is asynchronous.
 *   - Arguments are validated before anything is enqueued: a status other
 *     than LUTGEMM_OK means no work was enqueued (LUTGEMM_ERR_CUDA: the launch
 *     itself failed, as reported by cudaGetLastError).
 *   - A status returned by a call describes the enqueueing only: the kernels
 *     run later.  A kernel that fails while it runs (a bounded wait inside
 *     it ran out, or its shared-memory window is not where its tables are
 *     placed) does not hang or fault: it ORs a LUTGEMM_STATUS_* bit into a
 *     sticky status word and its outputs are not valid.  The word of a
 *     lutgemm_run call is the first 4 bytes of its workspace
 *     (lutgemm_workspace_status reads it); lutgemm_run_tc and
 *     lutgemm_run_noalloc use words held by the library
 *     (lutgemm_library_status reads them).  A caller that must know that
 *     y is valid reads the word after the calls it covers.
 *   - Values that can only be checked on the device (a sign that is not +-1,
 *     a code or zero-point >= 2^q) are reported through an optional
 *     device int32 *status_flags: the kernel ORs LUTGEMM_FLAG_* bits into it.
 *     Read it after synchronising the stream; pass NULL to skip reporting.
 *
 * Packed bit-plane layout (produced by lutgemm_pack_bcq and
 * lutgemm_uniform_to_bcq, consumed by lutgemm_run).  The pages do not fix a
 * layout; this one lets each GPU lane read 16 contiguous bytes per step and
 * makes the table reads of a warp fall in 32 distinct shared-memory banks.
 *   n_s = ceil(n/1024) slices of 1024 inputs, m_t = ceil(m/32) row tiles.
 *   The buffer holds n_s * m_t * 8 * q chunks of 512 bytes; chunk
 *   (s, R, U, i) (U < 8, plane i < q) starts at byte
 *   (((s * m_t + R) * 8 + U) * q + i) * 512.
 *   In chunk (s, R, U, i), byte l*16 + j  (l < 32, j < 16) holds the 8 sign
 *   bits of row r = 32*R + l, plane i, inputs k = 1024*s + 128*P + 8*c + t
 *   for t = 0..7 (bit t, least significant first), where
 *   P = U xor (4 * (l / 16)) and c = j xor (l % 16).
 *   A bit is 1 iff beta = +1.  Bits of rows r >= m or inputs k >= n are 0.
 *   The q * 4096 bytes of one (slice, row tile) are contiguous, and so are
 *   the q * 512 bytes a warp reads per step.
 *
 * Unit-major scale layout (produced by lutgemm_pack_scales, consumed by
 * lutgemm_run with LUTGEMM_SCALES_PACKED; for g % 128 == 0, where every
 * 128-input piece has one scale per plane, H = 1, and for g == 64, where it
 * has two, one per 64-input half, H = 2).  The pages fix no layout; this one
 * gives each lane the scales of a whole (slice, row tile) in 16*SP*H
 * contiguous bytes, so they arrive in a few 16-byte loads one tile ahead.
 *   SP = min(q, 4) planes per step, n_pg = ceil(q/4) plane groups.
 *   Element (s, R, pg, l, U, e, h) (pg < n_pg, l < 32, U < 8, e < SP, h < H)
 *   is the fp16 at element index
 *   (((((s * m_t + R) * n_pg + pg) * 32 + l) * 8 + U) * SP + e) * H + h
 *   and holds alpha[4*pg + e][G][32*R + l] with
 *   G = (1024*s + 128*P + 64*h) / g, P = U xor (4 * (l / 16)) (the piece
 *   lane l reads at step U).  It is 0 when 4*pg + e >= q, 32*R + l >= m or
 *   1024*s + 128*P + 64*h >= n.  Size: n_s * m_t * n_pg * 512 * SP * H bytes
 *   (equal to the [q][n/g][m] array when g is 128 or 64, m % 32 == 0 and
 *   n % 1024 == 0).
 *
 * Other layouts (row-major, innermost last):
 *   signs  int8   [q][m][n]     each -1 or +1
 *   codes  uint8  [m][n]        uniform codes in [0, 2^q)
 *   scale  fp16   [n/g][m]      uniform scale s
 *   zero   uint8  [n/g][m]      uniform integer zero-point z in [0, 2^q)
 *   alpha  fp16   [q][n/g][m]   group-wise plane scales
 *   offset fp32   [n/g][m]      group offsets of converted uniform weights
 *   x      fp16   [batch][n]
 *   y      fp32 (or fp16 with LUTGEMM_Y_F16) [batch][m]
 */
#ifndef LUTGEMM_H
#define LUTGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every int-valued call. */
#define LUTGEMM_OK             0
#define LUTGEMM_ERR_NULL       1  /* a required pointer is NULL */
#define LUTGEMM_ERR_SHAPE      2  /* m, n, batch < 1; q not in [1,8]; n%8, g%8 or n%g != 0 */
#define LUTGEMM_ERR_ALIGN      3  /* a pointer is not aligned as its call requires */
#define LUTGEMM_ERR_WORKSPACE  4  /* workspace smaller than lutgemm_workspace_size() */
#define LUTGEMM_ERR_VALUE      5  /* a host-checkable value is out of range */
#define LUTGEMM_ERR_CUDA       6  /* a CUDA runtime call or launch failed */

/* Bits OR-ed into *status_flags by device-side value checks. */
#define LUTGEMM_FLAG_BAD_SIGN  1  /* lutgemm_pack_bcq: a sign was neither -1 nor +1 */
#define LUTGEMM_FLAG_BAD_CODE  2  /* lutgemm_uniform_to_bcq: a code >= 2^q */
#define LUTGEMM_FLAG_BAD_ZERO  4  /* lutgemm_uniform_to_bcq: a zero-point >= 2^q */
#define LUTGEMM_FLAG_BAD_BLOCK 8  /* lutgemm_pack_bcq_mixed: a block-table entry out of range (block not written) */

/* Bits of the sticky status word a kernel sets when it fails while it runs
 * (read with lutgemm_workspace_status / lutgemm_library_status).  Any bit
 * set means the outputs of the calls since the word was last cleared are
 * not valid. */
#define LUTGEMM_STATUS_WINDOW  1u /* the lookup kernel's shared-memory window does not start where its
                                     tables are placed: nothing was computed */
#define LUTGEMM_STATUS_TIMEOUT 2u /* a bounded wait on a copy or an MMA ran out (1 s): the kernel stopped */
#define LUTGEMM_STATUS_FORMAT  4u /* lutgemm_run_mixed: a block-table entry or an outlier entry was out of
                                     range; the rows it touches are not valid */

/* Flags of lutgemm_run. */
#define LUTGEMM_Y_F16          1u /* write y as fp16 (round to nearest even of the fp32 sum) */
#define LUTGEMM_SCALES_PACKED  2u /* alpha is in the unit-major scale layout (g % 128 == 0 or g == 64) */
#define LUTGEMM_ALLOW_TENSOR_CORES 4u /* lutgemm_run may compute on the tensor cores (see there) */
/* Test hook of lutgemm_run and lutgemm_run_noalloc, for checking error
 * reporting: every warp of the lookup kernel makes its first weight wait on
 * a barrier that nothing signals, gives up after 1 ms, lets its copies in
 * flight land and stops, so the call sets LUTGEMM_STATUS_TIMEOUT and y is
 * not valid.  The tensor-core path is not taken with this flag.  Not for
 * production use. */
#define LUTGEMM_TEST_STALL     0x80000000u

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
int lutgemm_version(void);

/* Static English text for a status code (never NULL). */
const char* lutgemm_status_string(int status);

/* Bytes of the packed bit-plane buffer for (q, m, n):
 * ceil(n/1024) * ceil(m/32) * q * 4096.  Returns 0 for invalid shapes.
 * Pure host function. */
size_t lutgemm_packed_bytes(int q, int m, int n);

/* Bytes of the unit-major scale buffer for (q, m, n, g):
 * ceil(n/1024) * ceil(m/32) * ceil(q/4) * 512 * min(q, 4) * H, H = 2 for
 * g == 64 and 1 otherwise.  Returns 0 for invalid shapes and unless
 * g % 128 == 0 or g == 64.  Pure host function. */
size_t lutgemm_scales_bytes(int q, int m, int n, int g);

/* Bytes of the lutgemm_run workspace: [status word, 256 B | per-segment tile
 * counters, 4 KB | split-K partial sums, batch * ceil(n/1024) *
 * ceil(m/32) * 128 B rounded up to 256 B].  Returns 0 for invalid shapes.
 * Pure host function. */
size_t lutgemm_workspace_size(int m, int n, int batch, int q, int g);

/* Read the sticky status word of a lutgemm_run workspace: waits for the work
 * enqueued on `stream` so far (cudaStreamSynchronize), stores the word's
 * LUTGEMM_STATUS_* bits in *status (host) and, when clear != 0 and a bit is
 * set, enqueues its reset to 0 on `stream`.  0 means every lutgemm_run on
 * this workspace since the last clear ran to the end.  Synchronous: not for
 * use inside a stream capture.
 *   workspace        dev, 16-byte aligned, as given to lutgemm_run
 *   workspace_bytes  at least 256 + 4096
 * Returns LUTGEMM_OK, ERR_NULL, ERR_ALIGN, ERR_WORKSPACE or ERR_CUDA. */
int lutgemm_workspace_status(void* workspace, size_t workspace_bytes, uint32_t* status, int clear, void* stream);

/* The same for the status words the library holds on the current device,
 * OR-ed together: the one of lutgemm_run_noalloc (in its scratch array) and
 * the one lutgemm_run_tc uses.  The first call on a device does the set-up
 * lutgemm_run_noalloc describes.  Synchronous, like lutgemm_workspace_status.
 * Returns LUTGEMM_OK, ERR_NULL or ERR_CUDA. */
int lutgemm_library_status(uint32_t* status, int clear, void* stream);

/* How lutgemm_run spreads the lookup kernel over `sm_count` SMs: the same
 * choice the call makes (pure host function).  Outputs (host):
 *   *grid           CTAs launched (one persistent 512-thread CTA per SM)
 *   *seg_aligned    1 when every (batch column, slice) segment gets its own
 *                   group of CTAs, whose warps take two row tiles each and
 *                   the rest of the segment's tiles from a per-segment tile
 *                   counter; 0 when the list of (batch column, slice, row
 *                   tile) units is cut into one contiguous range per CTA
 *   *dynamic_tiles  row tiles taken through the counters, summed over the
 *                   segments (0 when *seg_aligned is 0)
 * m, batch, sm_count >= 1, n >= 8, n % 8 == 0.
 * Returns LUTGEMM_OK, ERR_NULL or ERR_SHAPE. */
int lutgemm_launch_plan(int m, int n, int batch, int sm_count, int* grid, int* seg_aligned, int* dynamic_tiles);

/* The tensor-core plan lutgemm_run uses with LUTGEMM_ALLOW_TENSOR_CORES: the
 * number of K splits it runs tc_gemm with (whole 1024-input slices, at most
 * 8 and max_split), or 0 when its cost model expects the lookup kernel to
 * be faster (always 0 below batch 8).  The model is fitted to B200
 * measurements of both paths: tensor cores ~ waves x (K blocks per split x
 * q/3 x 1600 / 1870 / 2450 cycles at 32 / 64 / 128 batch columns per tile +
 * 14k) + 15k (+ the reduce when split); lookups ~ q m n batch / 8 table reads
 * at 0.39 + 0.092 q of a 32-read wavefront per clock per SM + 20k.  lutgemm_run passes
 * ceil(n / 1024) and the device's SM count.  A pure host function (whether
 * the operands suit the tensor-core path -- n % 128, g % 64, scale layout --
 * is checked by lutgemm_run, not here). */
int lutgemm_tc_plan(int m, int n, int batch, int q, int max_split, int sm_count);

/* Pack q planes of +-1 signs into the packed bit-plane layout above.
 * Defines the BCQ binary planes of the LUT-GEMM card (Summary; Interesting
 * ideas: weights are binary +-1 vectors with scales).
 *   signs        dev int8 [q][m][n], 8-byte aligned, each -1 or +1
 *   q, m, n      1 <= q <= 8, m >= 1, n >= 8, n % 8 == 0
 *   packed       dev, lutgemm_packed_bytes(q,m,n) bytes, 16-byte aligned;
 *                every byte is written (padding bits 0)
 *   status_flags dev int32 or NULL; LUTGEMM_FLAG_BAD_SIGN is OR-ed in if a
 *                sign is neither -1 nor +1 (its bit is then written as
 *                1 iff the value is > 0)
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN or ERR_CUDA. */
int lutgemm_pack_bcq(const int8_t* signs, int q, int m, int n,
                     uint8_t* packed, int32_t* status_flags, void* stream);

/* Rewrite a uniform q-bit weight w = s * (c - z) as BCQ plus a group offset
 * (LUT-GEMM card, Summary and "One format for many schemes": uniform
 * quantisation is a special case of BCQ; the pages give no formula).  With
 * c = sum_i 2^i b_i and beta_i = 2 b_i - 1:
 *     plane i = bit i of c,   alpha_i = s * 2^(i-1),
 *     offset  = s * ((2^q - 1)/2 - z),
 * so sum_i alpha_i beta_i + offset = s * (c - z).  alpha_i is rounded to
 * fp16 (nearest even; exact unless s/2 is an fp16 subnormal with its last bit
 * set); offset is exact in fp32.
 *   codes        dev uint8 [m][n], 8-byte aligned, each < 2^q
 *   scale        dev fp16 [n/g][m]
 *   zero         dev uint8 [n/g][m], each < 2^q
 *   q, m, n, g   1 <= q <= 8, m >= 1, n % 8 == 0, g % 8 == 0, n % g == 0
 *   packed       dev, lutgemm_packed_bytes(q,m,n) bytes, 16-byte aligned
 *   alpha        dev fp16 [q][n/g][m] (output)
 *   offset       dev fp32 [n/g][m] (output), 4-byte aligned
 *   status_flags dev int32 or NULL; LUTGEMM_FLAG_BAD_CODE / _BAD_ZERO are
 *                OR-ed in for out-of-range codes / zero-points (the values
 *                are then used modulo 2^q)
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN or ERR_CUDA. */
int lutgemm_uniform_to_bcq(const uint8_t* codes, const uint16_t* scale,
                           const uint8_t* zero, int q, int m, int n, int g,
                           uint8_t* packed, uint16_t* alpha, float* offset,
                           int32_t* status_flags, void* stream);

/* Fit q sign planes and group-wise fp16 scales to dense fp16 weights: BCQ
 * quantisation, the step that produces the weights lutgemm_run consumes
 * (LUT-GEMM card, Summary: weights stored in BCQ; the pages cite the
 * alternating multi-bit method, reference 48, without detail).  Per (row,
 * group of g inputs): greedy signs of the residual with scales mean|r|, then
 * `iters` rounds of a least-squares scale step (a plane set that is linearly
 * dependent on the group keeps its scales) and a nearest-code sign step
 * (ties go to the largest code c, where bit i of c set means beta_i = +1);
 * scales are rounded to fp16 and the signs refitted to the rounded scales.  Arithmetic is fp32 in a fixed order (results are
 * reproducible).
 *   w          dev fp16 [m][n], 16-byte aligned
 *   q, m, n, g 1 <= q <= 8, m >= 1, n % 8 == 0, g % 8 == 0, n % g == 0,
 *              g <= 1024
 *   iters      0..64 alternating rounds (0: greedy only)
 *   signs      dev int8 [q][m][n], 8-byte aligned (output, each -1 or +1;
 *              the input of lutgemm_pack_bcq)
 *   alpha      dev fp16 [q][n/g][m], 2-byte aligned (output)
 *   err        dev fp32 [n/g][m], 4-byte aligned, or NULL (output: squared
 *              error of each group with the stored signs and scales)
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE (also for g > 1024), ERR_VALUE
 * (iters out of range), ERR_ALIGN or ERR_CUDA. */
int lutgemm_fit_bcq(const uint16_t* w, int q, int m, int n, int g, int iters,
                    int8_t* signs, uint16_t* alpha, float* err, void* stream);

/* The same fit on a variable grid: the planes plus one constant per (row,
 * group), w ~ offset + sum_i alpha_i beta_i, a grid of 2^q points built from
 * bit-planes and scalar coefficients (BPDQ card; the pages give no more than
 * that line).  The greedy pass starts from the group mean; the least-squares
 * step solves for the scales and the constant together (a plane set that is
 * linearly dependent on the group and the constant keeps its values); the
 * sign step takes the nearest grid point.  The result is the format
 * lutgemm_run consumes with an offset: pack the signs with lutgemm_pack_bcq
 * and pass alpha and offset.
 *   w, q, m, n, g, iters, signs, alpha, err   as lutgemm_fit_bcq
 *   offset     dev fp32 [n/g][m], 4-byte aligned (output; not rounded to fp16)
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE (also for g > 1024), ERR_VALUE
 * (iters out of range), ERR_ALIGN or ERR_CUDA. */
int lutgemm_fit_bcq_grid(const uint16_t* w, int q, int m, int n, int g, int iters,
                         int8_t* signs, uint16_t* alpha, float* offset, float* err,
                         void* stream);

/* Reorder group-wise plane scales into the unit-major scale layout above
 * (a data movement only: every output is one input value or 0).  The scales
 * are those of the BCQ format (LUT-GEMM card, Summary: q binary planes, each
 * with a scale per group of g inputs).
 *   alpha        dev fp16 [q][n/g][m], 2-byte aligned
 *   q, m, n, g   1 <= q <= 8, m >= 1, n % 8 == 0, g % 128 == 0 or g == 64,
 *                n % g == 0
 *   scales       dev, lutgemm_scales_bytes(q,m,n,g) bytes, 16-byte aligned
 *                (output, fully written)
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE (also for other g),
 * ERR_ALIGN or ERR_CUDA. */
int lutgemm_pack_scales(const uint16_t* alpha, int q, int m, int n, int g,
                        uint16_t* scales, void* stream);

/* y = W x for a BCQ weight, through per-8-activation lookup tables, with no
 * dequantisation (LUT-GEMM card, Summary and "Lookup tables instead of
 * multiplications"; pith.science abstract).  For each batch column b and each
 * slice of 1024 inputs, tables T[c][p] = sum_{t<8} (2*bit_t(p) - 1) * x[b][8c+t]
 * are built in fp32 in shared memory; each plane-row adds T[c][byte] over the
 * runs of a group, scales the sum by alpha (and adds offset * sum of the
 * group's x for converted uniform weights), and the per-slice partial sums
 * are reduced in a fixed order, so repeated calls give identical bits.
 *   m, n, batch, q, g  m >= 1, batch >= 1, 1 <= q <= 8, n % 8 == 0,
 *                      g % 8 == 0, n % g == 0, batch * ceil(n/1024) < 2^31
 *   packed     dev, packed layout above, 16-byte aligned
 *   alpha      dev fp16 [q][n/g][m], 2-byte aligned; with
 *              LUTGEMM_SCALES_PACKED the lutgemm_pack_scales output instead
 *              (16-byte aligned; g % 128 == 0 or g == 64), which gives the same bits
 *   offset     dev fp32 [n/g][m] or NULL (pure BCQ), 4-byte aligned
 *   x          dev fp16 [batch][n], 16-byte aligned
 *   y          dev [batch][m] fp32 (4-byte aligned) or, with LUTGEMM_Y_F16,
 *              fp16 (2-byte aligned); fully overwritten.  For n > 1024 the
 *   call enqueues two kernels: the lookup kernel writes per-slice partial
 *   sums to the workspace and a reduce kernel adds them in slice order.
 *   flags      OR of LUTGEMM_Y_F16, LUTGEMM_SCALES_PACKED and
 *              LUTGEMM_ALLOW_TENSOR_CORES; other bits, or
 *              LUTGEMM_SCALES_PACKED with another g, give ERR_VALUE.
 *              With LUTGEMM_ALLOW_TENSOR_CORES the call computes the product
 *              on the tensor cores as lutgemm_run_tc does (same result within
 *              the same tolerance, not the same bits) when that path takes
 *              the operands (batch >= 8, scales in [q][n/g][m],
 *              n % 128 == 0, g % 64 == 0) and the cost model of
 *              lutgemm_tc_plan expects it to be faster (tall matrices: many
 *              128-row blocks to spread over the SMs, or large batches).
 *              When that model splits K, each split writes fp32 partial sums
 *              to the workspace's partial-sum area and the split-K reduce
 *              adds them in split order (deterministic); the workspace's
 *              counters are not touched.  Otherwise the flag changes
 *              nothing.
 *   workspace  dev, >= lutgemm_workspace_size(m,n,batch,q,g) bytes,
 *              16-byte aligned, zero-filled before its first use; its
 *              counters are left zero by every call, its status word keeps
 *              its bits until lutgemm_workspace_status clears them.  Calls that share a
 *              workspace must not overlap on the device.
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_WORKSPACE or
 * ERR_CUDA. */
int lutgemm_run(int m, int n, int batch, int q, int g,
                const uint8_t* packed, const uint16_t* alpha,
                const float* offset, const uint16_t* x, void* y,
                unsigned flags, void* workspace, size_t workspace_bytes,
                void* stream);

/* y = W x for a BCQ weight on the tensor cores: the large-batch path, where
 * the lookup kernel's per-column table reads dominate (one table per batch
 * column).  Same operands and result as lutgemm_run.
 * Each plane enters the tensor cores as its exact fp16 values +-alpha (a
 * scale times a sign), so no rounded dequantised weight is formed; the planes
 * accumulate in fp32 (tcgen05.mma, tensor memory; each 128-input block's sum
 * is added into round-to-nearest fp32 running sums).  Tiles: 128 rows x 32,
 * 64 or 128 batch columns x 128 inputs; one K split (lutgemm_run with
 * LUTGEMM_ALLOW_TENSOR_CORES may split K).  The pages' kernel is the lookup
 * one; this path is for prompt-sized batches, where the method is
 * compute-bound (LUT-GEMM card, Summary and Key points: generation is
 * memory-bound, large batches are not).
 *   m, n, batch, q, g  as lutgemm_run, and n % 128 == 0, g % 64 == 0
 *   packed, alpha, offset, x, y  as lutgemm_run ([q][n/g][m] scales; offset
 *              NULL for pure BCQ, else fp32 [n/g][m], 4-byte aligned: each
 *              128-input block adds offset * (the block's input sum) in fp32)
 *   flags      0 or LUTGEMM_Y_F16
 * Needs no workspace.  Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE, ERR_VALUE,
 * ERR_ALIGN or ERR_CUDA. */
int lutgemm_run_tc(int m, int n, int batch, int q, int g,
                   const uint8_t* packed, const uint16_t* alpha,
                   const float* offset, const uint16_t* x, void* y,
                   unsigned flags, void* stream);

/* ---------------------------------------------------------------------------
 * Mixed storage: 2-, 4- and 16-bit weights in one matrix (OpenAlex record
 * "Fast and Efficient 2-bit LLM Inference on GPU: 2/4/16-bit in a Weight
 * Matrix with Asynchronous Dequantization", abstract: weights are quantised
 * by groups, wide-range groups need more bits, and sparse outliers are kept
 * in 16 bits; the record gives no format).  This library's format:
 *   - a precision block is 32 rows x 1024 inputs (row tile R, slice s, the
 *     unit the lookup kernel streams); block (s, R) stores q_b planes,
 *     1 <= q_b <= q_max <= 4 (for example 2 for most blocks, 4 for blocks
 *     with a wide range);
 *   - W[j,k] = sum_{i < q_b} alpha[i][k/g][j] * beta[i][j][k] + S[j,k],
 *     S a sparse fp16 matrix (the outliers), added to the BCQ value;
 *   - block_planes  uint8 [n_s][m_t]: q_b of block (s, R);
 *   - block table   uint32 [n_s*m_t + 1]: the exclusive prefix sum of q_b
 *     in (s, R) order, in 4096-byte units (lutgemm_mixed_offsets); the last
 *     entry is the total, and the packed buffer holds 4096 * total bytes;
 *   - packed planes: block (s, R) occupies q_b * 4096 bytes from byte
 *     4096 * table[s*m_t + R], its planes in pairs: pair h holds planes 2h
 *     and 2h+1 (2h alone when q_b = 2h+1), e_h planes, from byte 8192 * h of
 *     the block, and chunk (U, i') (U < 8, plane 2h + i') of the pair sits
 *     at (U * e_h + i') * 512 from there, with the byte map of the uniform
 *     layout (so blocks of at most two planes are laid out as
 *     lutgemm_pack_bcq lays them out; the kernel streams a block one pair,
 *     that is one pass, at a time);
 *   - alpha fp16 [q_max][n/g][m]: entries of planes a block does not store
 *     are never read;
 *   - outliers, as the caller gives them: row CSR, row_ptr int32 [m+1],
 *     col int32 [nnz] strictly increasing within a row, val fp16 [nnz];
 *     as the kernel reads them (lutgemm_pack_outliers): slice-major CSR,
 *     optr uint32 [n_s*m + 1] with the entries of (slice s, row r) at
 *     [optr[s*m + r], optr[s*m + r + 1]) sorted by input, each entry a
 *     uint32 (k - 1024 s) | (fp16 bits << 16).
 * ------------------------------------------------------------------------- */

/* The block table of a mixed matrix, on the host (pure host function).
 *   block_planes  host uint8 [ceil(n/1024)][ceil(m/32)], each in [1, q_max]
 *   q_max         1..4;  m >= 1, n >= 8, n % 8 == 0
 *   offsets       host uint32 [ceil(n/1024)*ceil(m/32) + 1] (output)
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE (also when the total exceeds
 * 2^32 - 1 blocks) or ERR_VALUE (a plane count out of range). */
int lutgemm_mixed_offsets(const uint8_t* block_planes, int q_max, int m, int n, uint32_t* offsets);

/* Pack the planes of a mixed matrix: block (s, R) stores planes 0..q_b-1.
 *   signs         dev int8 [q_max][m][n], 8-byte aligned; the signs of planes
 *                 a block does not store are not read
 *   block_off     dev uint32 block table (lutgemm_mixed_offsets), 4-byte aligned
 *   packed        dev, packed_bytes = 4096 * (the table's last entry),
 *                 16-byte aligned; every stored byte is written
 *   status_flags  dev int32 or NULL: LUTGEMM_FLAG_BAD_SIGN as for
 *                 lutgemm_pack_bcq; LUTGEMM_FLAG_BAD_BLOCK for a table entry
 *                 with no plane, more than q_max planes or past packed_bytes
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_VALUE (packed_bytes
 * not a multiple of 4096 or below one plane per block) or ERR_CUDA. */
int lutgemm_pack_bcq_mixed(const int8_t* signs, const uint32_t* block_off, int q_max, int m, int n,
                           uint8_t* packed, size_t packed_bytes, int32_t* status_flags, void* stream);

/* Row-CSR outliers -> the slice-major layout the kernel reads (pure host
 * function; all pointers host).  optr: uint32 [ceil(n/1024)*m + 1];
 * oent: uint32 [nnz].  Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE or ERR_VALUE
 * (row_ptr not from 0 to nnz and non-decreasing, a column outside [0, n), or
 * columns not strictly increasing within a row). */
int lutgemm_pack_outliers(const int32_t* row_ptr, const int32_t* col, const uint16_t* val, int m, int n, int nnz,
                          uint32_t* optr, uint32_t* oent);

/* Unit-major scales of a mixed matrix (for g % 128 == 0, H = 1, or g == 64,
 * H = 2): the scales of the planes each block stores, in the order the
 * lookup kernel's lanes read them, so that a lane's scales for a pass arrive
 * in a few 16-byte loads a pass ahead.  Block (s, R) with table entry t
 * starts at element t * 256 * H; its pair h (planes 2h and 2h+1, or 2h
 * alone; e_h planes) at + h * 512 * H; lane l's pass at + l * 8 * e_h * H;
 * element (U * e_h + e) * H + hh of it holds alpha[2h + e][G][32R + l],
 * G = (1024 s + 128 P + 64 hh) / g, P = U xor (4 * (l / 16)); 0 for rows
 * >= m or inputs >= n.  Size: 512 * H * (the table's last entry) bytes.
 *   alpha         dev fp16 [q_max][n/g][m], 2-byte aligned
 *   block_off     dev uint32 block table, 4-byte aligned
 *   scales        dev, scales_bytes = 512 * H * (table's last entry),
 *                 16-byte aligned (output; every element of a stored plane
 *                 is written)
 *   status_flags  dev int32 or NULL: LUTGEMM_FLAG_BAD_BLOCK for a table
 *                 entry out of range (that block is not written)
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE (also for other g), ERR_ALIGN,
 * ERR_VALUE (scales_bytes not a multiple of 512 * H or below one plane per
 * block) or ERR_CUDA. */
int lutgemm_pack_scales_mixed(const uint16_t* alpha, const uint32_t* block_off, int q_max, int m, int n, int g,
                              uint16_t* scales, size_t scales_bytes, int32_t* status_flags, void* stream);

/* y = W x for a mixed matrix, by the lookup kernel: the same tables, with
 * each block's own plane count, and each row's outliers added after its
 * planes (w * x in fp32, in entry order), so repeated calls give identical
 * bits.  Operands as described above; x, y, flags (LUTGEMM_Y_F16,
 * LUTGEMM_SCALES_PACKED: alpha is the lutgemm_pack_scales_mixed output,
 * 16-byte aligned, g % 128 == 0 or g == 64, which gives the same bits; or the
 * test hook LUTGEMM_TEST_STALL) and workspace (lutgemm_workspace_size with
 * q = q_max) as lutgemm_run.  optr and oent may be NULL when nnz == 0.
 * The kernel checks every block-table and outlier entry it uses against
 * packed_bytes, q_max, nnz and n; one out of range sets
 * LUTGEMM_STATUS_FORMAT in the workspace's status word instead of reading
 * outside the buffers.
 * Returns LUTGEMM_OK, ERR_NULL, ERR_SHAPE (also q_max outside 1..4),
 * ERR_VALUE, ERR_ALIGN, ERR_WORKSPACE or ERR_CUDA. */
int lutgemm_run_mixed(int m, int n, int batch, int q_max, int g, const uint8_t* packed, size_t packed_bytes,
                      const uint32_t* block_off, const uint16_t* alpha, const uint32_t* optr, const uint32_t* oent,
                      int nnz, const uint16_t* x, void* y, unsigned flags, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Bytes of the device scratch array used by lutgemm_run_noalloc (16 MiB). */
#define LUTGEMM_NOALLOC_SCRATCH_BYTES (16u << 20)

/* lutgemm_run for callers that cannot allocate device memory.  The paper has
 * no counterpart to this call; it exists for callers that own no device
 * allocator: a serving runtime that gave all device memory to its own pool up
 * front, a plugin or FFI host that hands a kernel only its input and output
 * tensors, or a latency-critical path where an allocation and its possible
 * failure are not acceptable.  Such callers cannot supply lutgemm_run's
 * workspace, so this call takes its split-K scratch from a fixed
 * LUTGEMM_NOALLOC_SCRATCH_BYTES array in the library's own device memory
 * (held on every GPU that loads the library until the process exits) and
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   Arguments, layouts and results are those of lutgemm_run, without the
 *   workspace.  Returns LUTGEMM_ERR_WORKSPACE when the problem needs more
 *   scratch than the array holds: more than 16 MiB - 4 KiB - 256 B of
 *   split-K partial sums (batch * ceil(n/1024) * ceil(m/32) * 128 bytes
 *   when n > 1024; with one slice none are needed).  With
 *   LUTGEMM_ALLOW_TENSOR_CORES a problem the tensor-core path takes runs
 *   there with one K split, which needs no scratch, when lutgemm_run would
 *   take that path or when the partials would not fit.  Other statuses as
 *   for lutgemm_run.
 *   The first call on a device does a one-time set-up on that device (looks
 *   up the array's device address and zeroes its counters on `stream`); make
 *   that first call before any stream capture.  Every call shares the one
 *   array, so calls that overlap on the GPU race: serialise them. */
int lutgemm_run_noalloc(int m, int n, int batch, int q, int g,
                        const uint8_t* packed, const uint16_t* alpha,
                        const float* offset, const uint16_t* x, void* y,
                        unsigned flags, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LUTGEMM_H */
