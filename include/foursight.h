/*
 * foursight.h — C ABI of the SpliceGEMM hot path for NVIDIA B200 (sm_100a).
 *
 * The operations follow FourSight (arXiv 2611.04887, "FourSight: Stable FP4 RL
 * Post-Training via Sequence Filtering and Sparse Channel Compensation"):
 *   - a W4A4 NVFP4 linear layer Y = X W^T in which a small protected set S of
 *     input channels (64 by default) stays in BF16 (§4.2 Eq. 5, §5.1);
 *   - running channel moments and per-step top-s reselection (§5.2);
 *   - the TIM-aware dual-gate sequence filter with advantage masking (§4.1 Eq. 3-4).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is a DEVICE pointer owned by the caller unless its
 *   comment says "host".  The library never keeps a pointer past the call.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream).  Apart from fs_plan_create, fs_plan_destroy, fs_plan_check and
 *   fs_stats_check, no call allocates, frees or synchronises, so a sequence of
 *   calls can be captured into a CUDA graph.
 * - Argument errors are found on the host before anything is launched and are
 *   returned as FS_ERR_INVALID_ARGUMENT (bad pointer, size, alignment) or
 *   FS_ERR_UNSUPPORTED (a legal shape this build has no kernel for); nothing
 *   is written in that case.  A launch failure returns FS_ERR_CUDA.
 *   fs_last_error() gives a readable detail string for the calling thread.
 * - Conditions only the device can see are recorded in a caller-visible word and
 *   reported by the *_check calls: FS_ERR_RANGE (a statistics input out of range)
 *   and FS_ERR_TIMEOUT (a bounded wait inside a kernel gave up; the kernel
 *   returned early and its output is undefined).
 * - dtype codes: FS_DTYPE_BF16 (row-major bf16), FS_DTYPE_F32 (row-major fp32).
 * - Leading dimensions (ldx, ldw, ldy) are in elements and must make every row
 *   start on a 16-byte boundary; base pointers must be 16-byte aligned (the packed
 *   operands of fs_splice_gemm are read by TMA, whose tensor maps need exactly that).
 *
 * Packed NVFP4 operand layout (written by fs_quantize_splice / fs_prepare_weights,
 * read by fs_splice_gemm):
 *   q    [R][K/2] bytes: E2M1 codes, two per byte, the even-K element in the low
 *        nibble; protected lanes hold code 0.
 *   sf   UE4M3 block scales (one per 16 elements along K) in the MMA-ready tiled
 *        layout: 512-byte atoms of 128 rows x 4 blocks, atoms running first along K
 *        then along rows; inside an atom row r sits at byte (r%32)*16 + ((r%128)/32)*4
 *        and its 4 blocks are consecutive bytes.  Size: roundup(R,128) * roundup(K/16,4)
 *        bytes; padding bytes are written as 0.
 *   side [R][Pp] bf16 with Pp = roundup(p,16): the protected columns in ascending
 *        channel order (X_S for activations, W'_S = BF16(W_S/alpha) for weights),
 *        columns p..Pp-1 zero.
 * fs_side_cols(p) returns Pp; fs_sf_bytes(R, K) returns the sf size.
 */
#ifndef FOURSIGHT_H
#define FOURSIGHT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fs_status {
  FS_OK = 0,
  FS_ERR_INVALID_ARGUMENT = 1,
  FS_ERR_UNSUPPORTED = 2,
  FS_ERR_CUDA = 3,
  FS_ERR_RANGE = 4,
  FS_ERR_TIMEOUT = 5
} fs_status;

enum { FS_DTYPE_BF16 = 0, FS_DTYPE_F32 = 1 };

/* Option bits (the `opts` arguments). */
enum {
  FS_RESIDUAL = 1u << 0,   /* residual-correction form: block scales and gains are taken with the
                              protected lanes present, then only their codes are zeroed (the
                              "auxiliary residual" prior art FourSight contrasts with, §1, §7.1) */
  FS_KEY_M2 = 1u << 1,     /* select by second moment E[x^2] instead of variance (§9.3 Prop. 2) */
  FS_GAIN_EXACT = 1u << 2, /* encode gain fl32(2688/amax) instead of the power-of-two gain */
  FS_OUT_BF16 = 1u << 3,   /* fs_splice_gemm writes bf16 Y instead of fp32 */
  FS_PATH_TENSOR = 1u << 4, /* plan option: always use the tcgen05 tensor-core kernel */
  FS_PATH_DECODE = 1u << 5, /* plan option: always use the weight-streaming decode kernel (M <= 16);
                              fs_splice_gemm_grouped: experts of at most 16 rows on it */
  FS_COMPACT_K = 1u << 7,   /* fs_quantize_splice / fs_prepare_weights: compacted-K operand (below) */
  FS_FAULT_NO_COPIES = 1u << 6 /* plan (and fs_splice_gemm_noalloc) option for tests of failure detection:
                              the GEMM kernels' producers issue no copies and every bounded wait is
                              limited to 20 ms, so each launch gives up its waits, takes its abort path
                              (no copy in flight, TMEM released) and reports FS_ERR_TIMEOUT through
                              fs_plan_check; the output is left undefined.  Never set in production. */
};

/* Readable name of a status code (static storage). */
const char* fs_status_string(fs_status s);
/* Detail of the last non-FS_OK status returned on the calling host thread ("" if none). */
const char* fs_last_error(void);
/* Library version string (static storage). */
const char* fs_version(void);

/* Pp = roundup(p, 16): the column count of the packed side buffers. */
int32_t fs_side_cols(int32_t p);
/* Kc = roundup(K - p, 256): the columns of a compacted-K NVFP4 operand (FS_COMPACT_K).  In that
 * form the protected channels are REMOVED from the NVFP4 operand rather than zeroed in place: its
 * columns are the K - p unprotected channels in ascending order followed by zero columns, so the
 * 16-element blocks (and their scales) are re-formed over the unprotected channels.  Gains, side
 * buffers and alpha are those of the split form.  A SpliceGEMM of compacted operands runs with a
 * plan of K = Kc; it saves whole 256-wide k-tiles of NVFP4 work once p reaches 256.  The
 * residual form cannot be compacted (FS_ERR_INVALID_ARGUMENT). */
int32_t fs_compact_cols(int32_t K, int32_t p);
/* Bytes of the tiled scale array for R rows and K channels. */
int64_t fs_sf_bytes(int64_t R, int32_t K);

/* ------------------------------------------------------------------------------------------
 * Running channel moments — FourSight §5.2 "System Implementation": a forward hook uniformly
 * subsamples token rows, before masking, and accumulates running channel moments in a GPU buffer.
 *
 * Adds rows 0, row_stride, 2*row_stride, ... of X [M][K] (row-major, leading dimension ldx,
 * dtype FS_DTYPE_BF16 or FS_DTYPE_F32) to the state of ONE input group:
 *   n     [1] int64   += number of rows taken
 *   s1    [K] int64   += sum rint(x * 2^16)          (exact integer fixed point)
 *   s2    [K] int64   += sum rint(x^2 * 2^14)        (x^2 formed exactly)
 *   amax  [K] uint32  = bits of max(|x|) as float32
 *   flags [1] uint32  |= 1 if some |x| >= 2^15 or x is not finite (read by fs_stats_check);
 *                      such an element adds nothing to the sums or the maximum
 * Integer sums make the state independent of the reduction order.  The state must be
 * zeroed before the first call (e.g. cudaMemsetAsync or fs_select_topk with reset=1).
 * Requirements: K % 8 == 0, M >= 0, row_stride >= 1; the state must hold fewer than 2^19
 * rows of values near the range limit for s2 not to overflow.
 * ---------------------------------------------------------------------------------------- */
fs_status fs_channel_stats(const void* X, int32_t dtype, int64_t M, int32_t K, int64_t ldx,
                           int32_t row_stride, int64_t* n, int64_t* s1, int64_t* s2,
                           uint32_t* amax, uint32_t* flags, void* stream);

/* Synchronises `stream` and returns FS_ERR_RANGE if any of the nprob flag words is non-zero. */
fs_status fs_stats_check(const uint32_t* flags, int32_t nprob, void* stream);

/* ------------------------------------------------------------------------------------------
 * Protected-channel reselection — FourSight §5.2: after each optimizer step the protected set is
 * reselected as the top-s channels by the variance gathered in the previous step; §9.3 Prop. 2 /
 * Cor. 1 for the key; §6.1 for s = 64.
 *
 * Batched over nprob problems that share K; state arrays are stacked: n [nprob], s1/s2/amax
 * [nprob][K], flags [nprob].  For each problem:
 *   key_j = m2 - m1*m1 (or m2 with FS_KEY_M2), m1 = s1/65536/n, m2 = s2/16384/n in float64
 *           (key 0 when n == 0);
 *   P     [nprob][p] int32: the p channels with the largest key (ties: lower index first),
 *         written in ascending channel order;
 *   mask  [nprob][ceil(K/32)] uint32: bit j%32 of word j/32 set for every j in P;
 *   gA    [nprob] float: next-step activation encode gain from max amax over channels not in P
 *         (over all channels with FS_RESIDUAL): the largest power of two g with amax*g <= 2688
 *         (exponent clamped to [-126,127]; 1 when amax == 0), or fl32(2688/amax) with FS_GAIN_EXACT.
 * reset != 0 zeroes the state after it has been read (start of the next window).
 * Requirements: 0 <= p <= K <= 16384, p <= 256.  Runs one cluster of 8 CTAs per problem.
 * ---------------------------------------------------------------------------------------- */
fs_status fs_select_topk(int32_t nprob, int32_t K, int64_t* n, int64_t* s1, int64_t* s2,
                         uint32_t* amax, uint32_t* flags, int32_t p, uint32_t opts,
                         int32_t* P, uint32_t* mask, float* gA, int32_t reset, void* stream);

/* ------------------------------------------------------------------------------------------
 * Weight pre-split — FourSight §5.1 "Data preparation": after each policy update W is split into
 * an NVFP4 pack of W_{~S} and a pre-scaled BF16 pack W'_S = BF16(W_S / alpha) (Eq. 5), fixed for
 * one rollout step.
 *
 * W [N][K] (leading dimension ldw, dtype bf16 or fp32); mask as written by fs_select_topk
 * (ceil(K/32) words; may be NULL when p == 0); gA: device float, the activation gain of this
 * projection's input.  Writes
 *   wq  [N][K/2], sfw (tiled, fs_sf_bytes(N,K)), ws [N][Pp] bf16 (the packed layout above);
 *   gW  [1] float: the weight encode gain from max |W| over unprotected columns (all columns with
 *       FS_RESIDUAL), same rule as gA;
 *   alpha [1] float: fl32(1 / fl32(gA*gW)).
 * Protected lanes are zeroed before the block scales are computed (split form) unless
 * FS_RESIDUAL; with FS_COMPACT_K they are removed (wq [N][Kc/2], sfw fs_sf_bytes(N,Kc)).  Block quantisation: t = fl32(fl32(a_b*g)/6), sf = UE4M3 round-to-nearest-even
 * (saturating at 448), v = fl32(fl32(w*g)/sf), code = E2M1 round-to-nearest-even (saturating at
 * 6, sign kept; sf == 0 gives code 0 with the sign of w).
 * Requirements: K % 64 == 0, 0 <= p <= min(K, 256), N >= 1.
 * ---------------------------------------------------------------------------------------- */
fs_status fs_prepare_weights(const void* W, int32_t dtype, int32_t N, int32_t K, int64_t ldw,
                             const uint32_t* mask, int32_t p, uint32_t opts, const float* gA,
                             uint8_t* wq, uint8_t* sfw, uint16_t* ws, float* gW, float* alpha,
                             void* stream);

/* ------------------------------------------------------------------------------------------
 * Activation preparation — FourSight §5.1 "Data preparation": one pass over X that zeroes the
 * protected lanes with a register bitmask (Mask S->0), quantises the rest to NVFP4 (FP4 Quant)
 * and copies the protected columns to a compact BF16 side buffer X_S (Extract X_S).
 *
 * X [M][K] (ldx, bf16 or fp32); mask/p as for fs_prepare_weights; gA: device float (frozen gain).
 * Writes xq [M][K/2], sfx (tiled, fs_sf_bytes(M,K)), xs [M][Pp] bf16 (bf16 of X_S, rounded to
 * nearest even for fp32 input).  Same block rule as fs_prepare_weights.  With FS_COMPACT_K in
 * opts the NVFP4 operand is compacted (see fs_compact_cols): xq [M][Kc/2], sfx fs_sf_bytes(M,Kc).
 * Requirements: K % 64 == 0, M >= 0, 0 <= p <= min(K, 256).
 * ---------------------------------------------------------------------------------------- */
fs_status fs_quantize_splice(const void* X, int32_t dtype, int64_t M, int32_t K, int64_t ldx,
                             const uint32_t* mask, int32_t p, const float* gA, uint32_t opts,
                             uint8_t* xq, uint8_t* sfx, uint16_t* xs, void* stream);

/* Activation preparation and channel statistics in ONE pass over X — FourSight §5.2 (the forward
 * hook accumulates running channel moments of the token rows BEFORE masking) together with §5.1
 * "Data preparation".  Equivalent, bit for bit, to
 *     fs_channel_stats(X, dtype, M, K, ldx, row_stride, n, s1, s2, amax, flags)
 *     fs_quantize_splice(X, dtype, M, K, ldx, mask, p, gA, opts, xq, sfx, xs)
 * but X is read once.  The moments go into the state that the NEXT reselection reads, while mask,
 * p and gA are the CURRENT protected set and gain (the paper's order: reselect after each step from
 * the moments gathered during it).  Arguments, layouts and requirements as for the two calls;
 * dtype must be FS_DTYPE_BF16 (FS_ERR_UNSUPPORTED for fp32 input). */
fs_status fs_quantize_splice_stats(const void* X, int32_t dtype, int64_t M, int32_t K, int64_t ldx,
                                   const uint32_t* mask, int32_t p, const float* gA, uint32_t opts,
                                   uint8_t* xq, uint8_t* sfx, uint16_t* xs, int32_t row_stride, int64_t* n,
                                   int64_t* s1, int64_t* s2, uint32_t* amax, uint32_t* flags, void* stream);

/* Grouped (mixture-of-experts) form: E experts, expert e owning rows
 * [row_offsets[e], row_offsets[e+1]) of X (row_offsets: device int64 [E+1], row_offsets[0] == 0,
 * non-decreasing, row_offsets[E] <= max_rows).  Each expert has its own mask [E][ceil(K/32)] and
 * gain gA [E]; all share p; E <= 256.  Expert e's packed rows start at the padded offset
 * pad_e = sum_{e'<e} roundup(rows_e', 128) in xq [.][K/2], sfx and xs [.][Pp]; size the buffers
 * with fs_grouped_rows(max_rows, E) rows.  Rows of the padding are zero. */
fs_status fs_quantize_splice_grouped(const void* X, int32_t dtype, int32_t E, const int64_t* row_offsets,
                                     int64_t max_rows, int32_t K, int64_t ldx, const uint32_t* masks,
                                     int32_t p, const float* gA, uint32_t opts, uint8_t* xq,
                                     uint8_t* sfx, uint16_t* xs, void* stream);
/* Upper bound of the padded row count for max_rows routed rows over E experts. */
int64_t fs_grouped_rows(int64_t max_rows, int32_t E);

/* ------------------------------------------------------------------------------------------
 * SpliceGEMM — FourSight §4.2 Eq. 5 and §5.1 "Dual-path execution":
 *   Y = alpha * ( sum_k (q sf)_x (q sf)_w  +  X_S W'_S^T )
 * the NVFP4 product over all K lanes (protected lanes hold code 0) and the BF16 product over the
 * protected slice accumulated into the same FP32 accumulator, scaled once by alpha.
 *
 * A plan caches the kernel choice for one weight shape (N, K, p_max) and owns a device error
 * word; creating it is the only call that allocates.  fs_plan_check synchronises `stream` and
 * returns FS_ERR_TIMEOUT if a kernel launched with the plan gave up a bounded wait (the word is
 * then cleared).  A plan may be used from one stream at a time.
 * ---------------------------------------------------------------------------------------- */
typedef struct fs_plan_s* fs_plan;
fs_status fs_plan_create(fs_plan* out, int32_t N, int32_t K, int32_t p_max, uint32_t opts);
fs_status fs_plan_destroy(fs_plan plan);
fs_status fs_plan_check(fs_plan plan, void* stream);

/* Packed operands as written above (activation rows M; weight rows N = the plan's N), p <= the
 * plan's p_max; alpha: device float.  Y [M][ldy] fp32 (bf16 with FS_OUT_BF16 in the plan's
 * opts), ldy >= N, 16-byte aligned rows.  M <= 16 runs the weight-streaming decode kernel (weights
 * as the 128-row operand of tcgen05 block-scaled MMAs with the tokens as N = 16, K split over a
 * thread-block cluster), larger M the tcgen05 prefill kernel (FS_PATH_TENSOR / FS_PATH_DECODE in
 * the plan's opts force one).
 * Plan requirements: N % 16 == 0 and K % 256 == 0 (FS_ERR_UNSUPPORTED otherwise); the packed
 * operands must be 16-byte aligned.  The output is not accumulated into: Y is overwritten.
 * M = 0 (an empty batch) returns FS_OK without reading any operand pointer (the plan must still
 * be valid); the same holds for the segmented, grouped (max_rows = 0) and allocation-free calls. */
fs_status fs_splice_gemm(fs_plan plan, int64_t M, int32_t p, const uint8_t* xq, const uint8_t* sfx,
                         const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                         const float* alpha, void* Y, int64_t ldy, void* stream);

/* Segmented SpliceGEMM: one launch over several projections that read the same activations (q,
 * k and v; gate and up), their packed weights stacked as adjacent row ranges of one operand.
 * FourSight §5.2 applies SpliceGEMM to every linear projection; computing projections that share
 * an input in one launch gives each of them the same result as its own fs_splice_gemm call, up to
 * the order of FP32 partial sums.
 *   plan        N = the total rows (output columns) of all segments; p_max and opts as usual.
 *   nseg        1..8 segments; seg_start: HOST array of nseg + 1 int32, 0 = seg_start[0] < ... <
 *               seg_start[nseg] = N, interior boundaries multiples of 256 (of 128 when N % 256 != 0)
 *               so that every tile of either path lies in one segment.
 *   wq, sfw, ws segment s occupies rows [seg_start[s], seg_start[s+1]) of wq and ws and the scale
 *               bytes from fs_sf_bytes(seg_start[s], K) on, exactly as fs_prepare_weights writes a
 *               projection of seg_start[s+1] - seg_start[s] rows at those offsets; all segments are
 *               prepared with the mask and gain of the shared activations.
 *   alpha       device, nseg floats: segment s's alpha from its fs_prepare_weights.
 *   Y           [M][ldy]: columns [seg_start[s], seg_start[s+1]) are projection s's output.
 * Otherwise (operands, paths, alignment, errors) as fs_splice_gemm; argument errors are returned
 * before anything launches. */
fs_status fs_splice_gemm_segmented(fs_plan plan, int64_t M, int32_t p, const uint8_t* xq, const uint8_t* sfx,
                                   const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                                   int32_t nseg, const int32_t* seg_start, const float* alpha, void* Y,
                                   int64_t ldy, void* stream);

/* Decode-path SpliceGEMM with the activation preparation in the same launch — FourSight §5.1
 * "Low-latency decode path" with its "Data preparation" (Mask S->0, FP4 Quant, Extract X_S).
 * Equivalent, bit for bit, to
 *     fs_quantize_splice(X, FS_DTYPE_BF16, M, K, ldx, mask, p, gA, xopts, xq, sfx, xs)
 *     fs_splice_gemm_segmented(plan, M, p, xq, sfx, xs, wq, sfw, ws, nseg, seg_start, alpha, Y, ldy)
 * on the decode kernel, without the packed activation buffers: every CTA of the weight-streaming
 * kernel encodes its own K range of the (at most 16) token rows into its shared-memory stages, so
 * the activations never make a round trip through global memory and no second kernel runs.
 *   X          device bf16 [M][ldx], ldx >= K (the plan's K), 16-byte aligned rows; 0 <= M <= 16
 *              (FS_ERR_UNSUPPORTED above 16).
 *   mask, p    the protected set as for fs_quantize_splice (mask may be NULL when p == 0);
 *              p <= the plan's p_max.
 *   gA         device float, the frozen activation gain.
 *   xopts      0 or FS_RESIDUAL (the activation encoding; FS_COMPACT_K is not available here).
 *   wq .. ws   the prepared weights of the plan's N rows (fs_prepare_weights, same mask and gA).
 *   nseg, seg_start  as for fs_splice_gemm_segmented; nseg <= 1 with seg_start NULL is one
 *              projection with alpha[0].
 *   alpha, Y, ldy    as for fs_splice_gemm.
 * The plan must not force FS_PATH_TENSOR (FS_ERR_UNSUPPORTED).  Argument errors are returned
 * before anything launches; M = 0 returns FS_OK without reading any operand. */
fs_status fs_decode_splice_gemm(fs_plan plan, int64_t M, int32_t p, const void* X, int64_t ldx,
                                const uint32_t* mask, const float* gA, uint32_t xopts, const uint8_t* wq,
                                const uint8_t* sfw, const uint16_t* ws, int32_t nseg, const int32_t* seg_start,
                                const float* alpha, void* Y, int64_t ldy, void* stream);

/* Grouped SpliceGEMM over E experts (the mixture-of-experts projections).  Activations are the
 * padded-row outputs of fs_quantize_splice_grouped (row_offsets as given there); expert e's
 * weights are rows [e*N, (e+1)*N) of stacked wq [E*N][K/2], sfw (tiled over E*N rows) and
 * ws [E*N][Pp]; alpha [E].  Y [row_offsets[E]][ldy] in the original (unpadded) row order.
 * Needs N % 128 == 0 and E <= 256.  Experts run on the tensor-core kernel (256-row CTA-pair
 * tiles, or 128-row tiles).  With FS_PATH_DECODE in the plan's opts, experts of 1..16 rows run on
 * the weight-streaming decode kernel instead (each 128-row weight tile streamed once against the
 * expert's tokens as 16 columns) and the tensor-core kernel skips them; with max_rows <= 16 only
 * the decode kernel is launched.  Each expert's rows are read from the device offsets inside the
 * kernels, so the split needs no host synchronisation; the results of the two kernels differ
 * only in the fp32 summation order. */
fs_status fs_splice_gemm_grouped(fs_plan plan, int32_t E, const int64_t* row_offsets, int64_t max_rows,
                                 int32_t p, const uint8_t* xq, const uint8_t* sfx, const uint16_t* xs,
                                 const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                                 const float* alpha, void* Y, int64_t ldy, void* stream);

/* SpliceGEMM for callers that cannot allocate device memory.  The paper has no counterpart to
 * this call; it exists for integration.  fs_splice_gemm needs a plan, and fs_plan_create calls
 * cudaMalloc for the tensor-core kernel's error word.  Code that must not allocate at call time
 * (an allocator or memory-pool callback, a runtime that serves every device byte from an arena
 * reserved at start-up, a plugin whose host forbids allocations) calls this instead: same
 * operands, same results, no plan.  Its only scratch is one 32-bit error word in a file-scope
 * __device__ array of the library (1 word, 256-byte aligned); every GPU that loads the library
 * holds it until the process exits.  No problem size needs more scratch than that; shapes beyond
 * the kernels' limits (N % 16, K % 256 or 256 <= K <= 65536, M < 2^31 - 256, p <= min(K, 256)) are
 * rejected with FS_ERR_INVALID_ARGUMENT / FS_ERR_UNSUPPORTED.
 *   N, K, opts  as for fs_plan_create (FS_OUT_BF16, FS_PATH_TENSOR, FS_PATH_DECODE apply);
 *   M .. ldy    as for fs_splice_gemm;
 *   check != 0  synchronise `stream` after the launch and return FS_ERR_TIMEOUT if the kernel gave
 *               up a bounded wait (check == 0: fully asynchronous, no device-to-host read).
 * The call never calls cudaMalloc, cudaFree or any allocating routine.  Its first call on a device
 * looks up the device address of the scratch array (cudaGetSymbolAddress, with that device
 * current); make that first call before any stream capture.  Every call clears the word on
 * `stream` before its kernel; calls that overlap on the GPU (unordered streams) share the word and
 * race on it. */
fs_status fs_splice_gemm_noalloc(int32_t N, int32_t K, uint32_t opts, int64_t M, int32_t p, const uint8_t* xq,
                                 const uint8_t* sfx, const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw,
                                 const uint16_t* ws, const float* alpha, void* Y, int64_t ldy, int32_t check,
                                 void* stream);

/* ------------------------------------------------------------------------------------------
 * TIM-aware sequence filter — FourSight §4.1 "The dual-gate mechanism" and Eq. 3-4; §2.1 for the
 * group advantage; §6.1 for tau = 1e-4, K1 = 0.01 x output_len, K2 = 5.
 *
 * logp [S][ld] fp32 train-engine log-probs; lengths [S] int32 (NULL: every sequence has T tokens;
 * positions >= length are ignored).  A token is a tail token when logp <= log_tau or logp is NaN
 * (log_tau = fl32(ln tau), formed by the caller).  Per sequence:
 *   tail_count [S] int32, max_run [S] int32 (longest run of consecutive tail tokens),
 *   keep [S] uint8 = (tail_count < K1 && max_run < K2).
 * Advantages (optional):
 *   rewards != NULL: adv [S] is written with keep ? (r - mu)/sigma : 0, mu and population sigma
 *     over each group of G consecutive sequences (all of them, dropped ones included), float64
 *     sequential sums rounded to float32, sigma == 0 giving 0; S % G == 0 is required;
 *   rewards == NULL and adv != NULL: adv is masked in place (adv = keep ? adv : 0).
 * The loss denominator stays G: nothing is renormalised by the number of kept sequences.
 * Requirements: S >= 0, T >= 0, ld >= T, K1 >= 1, K2 >= 1, logp 4-byte aligned (rows are read with
 * 16-byte loads when logp is 16-byte aligned and ld % 4 == 0).
 * ---------------------------------------------------------------------------------------- */
fs_status fs_seq_filter(const float* logp, int64_t ld, const int32_t* lengths, int32_t S, int32_t T,
                        float log_tau, int32_t K1, int32_t K2, int32_t G, const float* rewards,
                        float* adv, uint8_t* keep, int32_t* tail_count, int32_t* max_run, void* stream);

/* ------------------------------------------------------------------------------------------
 * Training side — FourSight §5.2 "System Implementation" (backward passes run in BF16 with the
 * straight-through estimator), §4.1 Eq. 4 (GRPO objective with filtered advantages and the original
 * 1/G denominator) and §6.1 (TIM measured by sampled K3 estimates of the KL divergence).
 * ---------------------------------------------------------------------------------------- */

/* Y [M][N] = alpha * A [M][K] . B [N][K]^T with BF16 operands (row-major, K contiguous, leading
 * dimensions lda/ldb in elements, 16-byte aligned rows) and FP32 accumulation on the tcgen05
 * kernel of fs_splice_gemm (every k-tile through its BF16 path).  alpha: device float or NULL
 * (1).  The plan supplies only the error word and FS_OUT_BF16 / FS_FAULT_NO_COPIES (its N and K
 * are not used).  Requirements: N % 16 == 0, K >= 1, M < 2^31 - 256. */
fs_status fs_gemm_bf16(fs_plan plan, int64_t M, int32_t N, int32_t K, const uint16_t* A, int64_t lda,
                       const uint16_t* B, int64_t ldb, const float* alpha, void* Y, int64_t ldy, void* stream);

/* dst [C][ldd] = src [R][lds]^T for bf16 matrices (16-byte vector accesses when both are 16-byte
 * aligned with ld % 8 == 0). */
fs_status fs_transpose_bf16(int64_t R, int64_t C, const uint16_t* src, int64_t lds, uint16_t* dst, int64_t ldd,
                            void* stream);

/* Straight-through backward of Y = SpliceGEMM(X, W): the quantiser's Jacobian is taken as the
 * identity, so the gradients use the BF16 operands:  dX [M][K] = dY [M][N] . W [N][K]  and
 * dW [N][K] = dY^T . X [M][K], FP32 accumulation, FP32 outputs (bf16 with FS_OUT_BF16 in the plan).
 * dY, X, W bf16 row-major with leading dimensions in elements.  work: device scratch of
 * fs_ste_backward_work_bytes(M, N, K) bytes, 256-byte aligned (the transposes dY^T, X^T, W^T).
 * Requirements: N, K multiples of 16, M <= 2^24.  Two fs_gemm_bf16 launches and three transposes. */
int64_t fs_ste_backward_work_bytes(int64_t M, int32_t N, int32_t K);
fs_status fs_ste_backward(fs_plan plan, int64_t M, int32_t N, int32_t K, const uint16_t* dY, int64_t lddy,
                          const uint16_t* X, int64_t ldx, const uint16_t* W, int64_t ldw, void* work,
                          int64_t work_bytes, void* dX, int64_t lddx, void* dW, int64_t lddw, void* stream);

/* GRPO objective of Eq. 4 with the advantages A'_i already filtered (fs_seq_filter's adv: f_i A_i):
 *   rho_it = exp(logp_it - logp_old_it),  l_it = min(rho A', clip(rho, 1 - eps, 1 + eps) A'),
 *   seq_obj [S] = (1/|y_i|) sum_{t < |y_i|} l_it   (|y_i| = lengths[i], or T when lengths == NULL),
 *   J (optional, device float) = (1/S) sum_i seq_obj_i: the mean over groups of (1/G) sum over the
 *     group, so a dropped sequence still counts in the denominator (the original 1/G),
 *   grad [S][ldg] (optional) = dJ/dlogp_it = rho A' / (S |y_i|) where the unclipped term is the
 *     minimum (rho A' <= clip(rho) A'), else 0; positions >= |y_i| get 0.
 * logp, logp_old: fp32 [S][ld].  Sums run in float64 in a fixed order (reproducible).
 * Requirements: 0 <= eps < 1, ld >= T. */
fs_status fs_grpo_objective(const float* logp, const float* logp_old, int64_t ld, const int32_t* lengths,
                            int32_t S, int32_t T, const float* adv, float eps, float* seq_obj, float* J,
                            float* grad, int64_t ldg, void* stream);

/* TIM metric: per token d = logp_train - logp_rollout (fp32 [S][ld], tokens sampled by the rollout
 * engine) and k3 = exp(d) - 1 - d >= 0, the K3 estimate of KL(pi_rollout || pi_train).
 * seq_k3 [S]: mean over each sequence's tokens (0 for an empty one); batch_k3 (optional, device
 * float): mean over all tokens of the batch, which needs work of fs_k3_work_bytes(S) bytes. */
int64_t fs_k3_work_bytes(int32_t S);
fs_status fs_k3_kl(const float* logp_train, const float* logp_roll, int64_t ld, const int32_t* lengths, int32_t S,
                   int32_t T, float* seq_k3, float* batch_k3, void* work, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FOURSIGHT_H */
