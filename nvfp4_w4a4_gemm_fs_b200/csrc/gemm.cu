// SpliceGEMM plans and entry points: argument checks and dispatch between the tensor-core path
// (large M, FourSight §5.1 "High-throughput prefill path") and the weight-streaming decode path
// (M <= 16, the small-M regime of §5.1 "Low-latency decode path").
#include "common.cuh"
#include "gemm.cuh"

struct fs_plan_s {
  int32_t N, K, p_max;
  uint32_t opts;
  uint32_t* err;      // device error word (bounded-wait timeouts)
  int device;
};

using namespace fs;

namespace {

constexpr uint32_t kPathMask = FS_PATH_TENSOR | FS_PATH_DECODE;
constexpr int kDecodeRows = 16;        // token columns of the decode kernel's MMA

fs_status check_operands(const char* who, const fs_plan_s* pl, int32_t p, const uint8_t* xq, const uint8_t* sfx,
                         const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                         const float* alpha, const void* Y, int64_t ldy) {
  if (!pl) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null plan", who);
  if (p < 0 || p > pl->p_max) return fail(FS_ERR_INVALID_ARGUMENT, "%s: p=%d outside [0, p_max=%d]", who, p, pl->p_max);
  if (!xq || !sfx || !wq || !sfw || !alpha || !Y || (p > 0 && (!xs || !ws)))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (!aligned(xq, 16) || !aligned(sfx, 16) || !aligned(wq, 16) || !aligned(sfw, 16) ||
      (p > 0 && (!aligned(xs, 16) || !aligned(ws, 16))))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: packed operands must be 16-byte aligned", who);
  const bool bf16 = pl->opts & FS_OUT_BF16;
  if (ldy < pl->N || !aligned(Y, 16) || (ldy % (bf16 ? 8 : 4)) != 0)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: Y must be 16-byte aligned with ldy >= N and 16-byte rows", who);
  return FS_OK;
}

}  // namespace

extern "C" fs_status fs_plan_create(fs_plan* out, int32_t N, int32_t K, int32_t p_max, uint32_t opts) {
  if (!out) return fail(FS_ERR_INVALID_ARGUMENT, "fs_plan_create: null out");
  *out = nullptr;
  if (N < 16 || N % 16 != 0) return fail(FS_ERR_INVALID_ARGUMENT, "fs_plan_create: need N >= 16 and N %% 16 == 0 (N=%d)", N);
  if (K < 256 || K % 256 != 0 || K > 65536) return fail(FS_ERR_UNSUPPORTED, "fs_plan_create: need K %% 256 == 0, 256 <= K <= 65536 (K=%d)", K);
  if (p_max < 0 || p_max > 256 || p_max > K) return fail(FS_ERR_INVALID_ARGUMENT, "fs_plan_create: need 0 <= p_max <= min(K, 256)");
  if ((opts & kPathMask) == kPathMask) return fail(FS_ERR_INVALID_ARGUMENT, "fs_plan_create: FS_PATH_TENSOR and FS_PATH_DECODE are exclusive");
  auto* pl = new fs_plan_s{N, K, p_max, opts, nullptr, 0};
  cudaGetDevice(&pl->device);
  cudaError_t e = cudaMalloc(&pl->err, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(pl->err, 0, sizeof(uint32_t));
  if (e != cudaSuccess) {
    if (pl->err) cudaFree(pl->err);
    delete pl;
    return cuda_status(e, "fs_plan_create");
  }
  *out = pl;
  return FS_OK;
}

extern "C" fs_status fs_plan_destroy(fs_plan plan) {
  if (!plan) return FS_OK;
  cudaFree(plan->err);
  delete plan;
  return FS_OK;
}

extern "C" fs_status fs_plan_check(fs_plan plan, void* stream) {
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "fs_plan_check: null plan");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t w = 0;
  cudaError_t e = cudaMemcpyAsync(&w, plan->err, sizeof(w), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, "fs_plan_check");
  if (w) {
    cudaMemsetAsync(plan->err, 0, sizeof(uint32_t), s);
    cudaStreamSynchronize(s);
    return fail(FS_ERR_TIMEOUT, "a SpliceGEMM kernel gave up a bounded wait (error word 0x%x)", w);
  }
  return FS_OK;
}

namespace {

fs_status splice_gemm(const char* who, fs_plan plan, int64_t M, int32_t p, const uint8_t* xq, const uint8_t* sfx,
                      const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                      const Segments& seg, const float* alpha, void* Y, int64_t ldy, void* stream) {
  if (M < 0) return fail(FS_ERR_INVALID_ARGUMENT, "%s: M < 0", who);
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null plan", who);
  if (M == 0) return FS_OK;                        // an empty batch reads no operand
  fs_status st = check_operands(who, plan, p, xq, sfx, xs, wq, sfw, ws, alpha, Y, ldy);
  if (st != FS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int pp = side_cols(p);
  const bool decode = (plan->opts & FS_PATH_DECODE) || (!(plan->opts & FS_PATH_TENSOR) && M <= 16);
  if (decode) {
    if (M > 16) return fail(FS_ERR_UNSUPPORTED, "%s: the decode path takes M <= 16 (M=%lld)", who, (long long)M);
    DecodeParams d{};
    d.M = static_cast<int>(M); d.N = plan->N; d.K = plan->K; d.pp = pp;
    d.kb4 = static_cast<int>(round_up(plan->K / 16, 4) / 4);
    d.xq = xq; d.sfx = sfx; d.xs = xs; d.wq = wq; d.sfw = sfw; d.ws = ws; d.alpha = alpha; d.seg = seg;
    d.Y = Y; d.ldy = ldy; d.out_bf16 = (plan->opts & FS_OUT_BF16) ? 1 : 0; d.err = plan->err;
    d.wait_ns = wait_limit_ns(plan->opts); d.no_copies = (plan->opts & FS_FAULT_NO_COPIES) ? 1 : 0;
    return launch_splice_gemm_decode_tc(d, s);
  }
  if (M > (int64_t{1} << 31) - 256) return fail(FS_ERR_UNSUPPORTED, "%s: M too large", who);
  TcParams prm{};
  prm.M = M; prm.N = plan->N; prm.K = plan->K; prm.KT = plan->K / 256; prm.ST = static_cast<int>(ceil_div(pp, 64));
  prm.E = 1; prm.kb4 = plan->K / 64; prm.offsets = nullptr; prm.sfa = sfx; prm.sfb = sfw; prm.alpha = alpha;
  prm.seg = seg; prm.Y = Y; prm.ldy = ldy; prm.out_bf16 = (plan->opts & FS_OUT_BF16) ? 1 : 0; prm.err = plan->err;
  prm.wait_ns = wait_limit_ns(plan->opts); prm.no_copies = (plan->opts & FS_FAULT_NO_COPIES) ? 1 : 0;
  TcLaunch L{};
  L.xq = xq; L.wq = wq; L.xs = xs; L.ws = ws; L.a_rows = M; L.b_rows = plan->N; L.y_rows = M; L.pp = pp;
  L.bn = (plan->N % 256 == 0) ? 256 : 128;
  L.max_tiles = ceil_div(M, 128) * ceil_div(plan->N, L.bn);
  return launch_splice_gemm_tc(L, prm, s);
}

Segments one_segment(int N) {
  Segments sg{};
  sg.n = 1;
  sg.n0[0] = 0;
  sg.n0[1] = N;
  return sg;
}

}  // namespace

extern "C" fs_status fs_splice_gemm(fs_plan plan, int64_t M, int32_t p, const uint8_t* xq, const uint8_t* sfx,
                                    const uint16_t* xs, const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                                    const float* alpha, void* Y, int64_t ldy, void* stream) {
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "fs_splice_gemm: null plan");
  return splice_gemm("fs_splice_gemm", plan, M, p, xq, sfx, xs, wq, sfw, ws, one_segment(plan->N), alpha, Y, ldy,
                     stream);
}

namespace {

// Segments of a launch from the caller's seg_start: every tile of either path must lie in one
// segment.
fs_status build_segments(const char* who, const fs_plan_s* plan, int32_t nseg, const int32_t* seg_start,
                         Segments* sg) {
  if (nseg < 1 || nseg > kMaxSegments || !seg_start)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: need 1 <= nseg <= %d and seg_start", who, kMaxSegments);
  const int gran = (plan->N % 256 == 0) ? 256 : 128;
  if (seg_start[0] != 0 || seg_start[nseg] != plan->N)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: segments must start at 0 and end at N=%d", who, plan->N);
  *sg = Segments{};
  sg->n = nseg;
  for (int i = 0; i <= nseg; ++i) {
    if (i > 0 && seg_start[i] <= seg_start[i - 1])
      return fail(FS_ERR_INVALID_ARGUMENT, "%s: segment starts must increase", who);
    if (i > 0 && i < nseg && seg_start[i] % gran != 0)
      return fail(FS_ERR_INVALID_ARGUMENT, "%s: segment boundaries must be multiples of %d", who, gran);
    sg->n0[i] = seg_start[i];
  }
  return FS_OK;
}

}  // namespace

extern "C" fs_status fs_splice_gemm_segmented(fs_plan plan, int64_t M, int32_t p, const uint8_t* xq,
                                              const uint8_t* sfx, const uint16_t* xs, const uint8_t* wq,
                                              const uint8_t* sfw, const uint16_t* ws, int32_t nseg,
                                              const int32_t* seg_start, const float* alpha, void* Y, int64_t ldy,
                                              void* stream) {
  const char* who = "fs_splice_gemm_segmented";
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null plan", who);
  Segments sg;
  const fs_status st = build_segments(who, plan, nseg, seg_start, &sg);
  if (st != FS_OK) return st;
  return splice_gemm(who, plan, M, p, xq, sfx, xs, wq, sfw, ws, sg, alpha, Y, ldy, stream);
}

extern "C" fs_status fs_decode_splice_gemm(fs_plan plan, int64_t M, int32_t p, const void* X, int64_t ldx,
                                           const uint32_t* mask, const float* gA, uint32_t xopts, const uint8_t* wq,
                                           const uint8_t* sfw, const uint16_t* ws, int32_t nseg,
                                           const int32_t* seg_start, const float* alpha, void* Y, int64_t ldy,
                                           void* stream) {
  const char* who = "fs_decode_splice_gemm";
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null plan", who);
  if (M < 0) return fail(FS_ERR_INVALID_ARGUMENT, "%s: M < 0", who);
  if (M > 16) return fail(FS_ERR_UNSUPPORTED, "%s: the decode path takes M <= 16 (M=%lld)", who, (long long)M);
  if (plan->opts & FS_PATH_TENSOR) return fail(FS_ERR_UNSUPPORTED, "%s: the plan forces the tensor-core path", who);
  if (xopts & ~static_cast<uint32_t>(FS_RESIDUAL))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: xopts may hold FS_RESIDUAL only (0x%x)", who, xopts);
  if (p < 0 || p > plan->p_max) return fail(FS_ERR_INVALID_ARGUMENT, "%s: p=%d outside [0, p_max=%d]", who, p, plan->p_max);
  Segments sg = one_segment(plan->N);
  if (!(nseg <= 1 && !seg_start)) {
    const fs_status st = build_segments(who, plan, nseg, seg_start, &sg);
    if (st != FS_OK) return st;
  }
  if (M == 0) return FS_OK;                        // an empty batch reads no operand
  if (!X || !gA || !wq || !sfw || !alpha || !Y || (p > 0 && (!mask || !ws)))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (ldx < plan->K || (ldx * 2) % 16 != 0 || !aligned(X, 16))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: X must be 16-byte aligned with ldx >= K and 16-byte rows", who);
  if (!aligned(wq, 16) || !aligned(sfw, 16) || (p > 0 && (!aligned(ws, 16) || !aligned(mask, 4))) || !aligned(gA, 4))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: misaligned operand", who);
  const bool bf16 = plan->opts & FS_OUT_BF16;
  if (ldy < plan->N || !aligned(Y, 16) || (ldy % (bf16 ? 8 : 4)) != 0)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: Y must be 16-byte aligned with ldy >= N and 16-byte rows", who);
  DecodeParams d{};
  d.M = static_cast<int>(M); d.N = plan->N; d.K = plan->K; d.pp = side_cols(p);
  d.kb4 = static_cast<int>(round_up(plan->K / 16, 4) / 4);
  d.wq = wq; d.sfw = sfw; d.ws = ws; d.alpha = alpha; d.seg = sg;
  d.Y = Y; d.ldy = ldy; d.out_bf16 = bf16 ? 1 : 0; d.err = plan->err;
  d.wait_ns = wait_limit_ns(plan->opts); d.no_copies = (plan->opts & FS_FAULT_NO_COPIES) ? 1 : 0;
  d.fuse = 1; d.x = static_cast<const uint16_t*>(X); d.ldx = ldx; d.mask = p > 0 ? mask : nullptr; d.p = p;
  d.gA = gA; d.residual = (xopts & FS_RESIDUAL) ? 1 : 0;
  return launch_splice_gemm_decode_tc(d, static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_splice_gemm_grouped(fs_plan plan, int32_t E, const int64_t* row_offsets, int64_t max_rows,
                                            int32_t p, const uint8_t* xq, const uint8_t* sfx, const uint16_t* xs,
                                            const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                                            const float* alpha, void* Y, int64_t ldy, void* stream) {
  if (E <= 0 || !row_offsets || max_rows < 0) return fail(FS_ERR_INVALID_ARGUMENT, "fs_splice_gemm_grouped: need E > 0, row_offsets, max_rows >= 0");
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "fs_splice_gemm_grouped: null plan");
  if (max_rows == 0) return FS_OK;                 // no routed rows: nothing is read or written
  fs_status st = check_operands("fs_splice_gemm_grouped", plan, p, xq, sfx, xs, wq, sfw, ws, alpha, Y, ldy);
  if (st != FS_OK) return st;
  if (plan->N % 128 != 0) return fail(FS_ERR_UNSUPPORTED, "fs_splice_gemm_grouped: need N %% 128 == 0");
  const int64_t a_rows = fs_grouped_rows(max_rows, E);
  if (a_rows > (int64_t{1} << 31) - 256) return fail(FS_ERR_UNSUPPORTED, "fs_splice_gemm_grouped: too many rows");
  const int pp = side_cols(p);
  TcParams prm{};
  prm.M = 0; prm.N = plan->N; prm.K = plan->K; prm.KT = plan->K / 256; prm.ST = static_cast<int>(ceil_div(pp, 64));
  prm.E = E; prm.kb4 = plan->K / 64; prm.offsets = row_offsets; prm.sfa = sfx; prm.sfb = sfw; prm.alpha = alpha;
  prm.seg = one_segment(plan->N);
  prm.Y = Y; prm.ldy = ldy; prm.out_bf16 = (plan->opts & FS_OUT_BF16) ? 1 : 0; prm.err = plan->err;
  prm.wait_ns = wait_limit_ns(plan->opts); prm.no_copies = (plan->opts & FS_FAULT_NO_COPIES) ? 1 : 0;
  // With FS_PATH_DECODE, experts of at most kDecodeRows rows go to the weight-streaming decode
  // kernel (their 128-row weight tiles streamed once against up to 16 token columns) and the
  // tensor-core kernel gives them no tiles; with max_rows <= kDecodeRows only the decode kernel
  // runs.  Not the default: one grouped tensor-core launch already streams a decode batch's
  // weights near the HBM rate (64 experts, 16-64 tokens top-8: within -2% .. +5% of the split).
  const bool split = (plan->opts & FS_PATH_DECODE) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!split || max_rows > kDecodeRows) {
    prm.skip_small = split ? kDecodeRows : 0;
    TcLaunch L{};
    L.xq = xq; L.wq = wq; L.xs = xs; L.ws = ws; L.a_rows = a_rows; L.b_rows = static_cast<int64_t>(E) * plan->N; L.y_rows = max_rows; L.pp = pp;
    L.bn = (plan->N % 256 == 0) ? 256 : 128;
    L.max_tiles = ceil_div(a_rows, 128) * (plan->N / L.bn);
    st = launch_splice_gemm_tc(L, prm, s);
    if (st != FS_OK || !split) return st;
  }
  DecodeParams d{};
  d.M = 0; d.N = plan->N; d.K = plan->K; d.pp = pp; d.kb4 = static_cast<int>(round_up(plan->K / 16, 4) / 4);
  d.xq = xq; d.sfx = sfx; d.xs = xs; d.wq = wq; d.sfw = sfw; d.ws = ws; d.alpha = alpha; d.seg = one_segment(plan->N);
  d.Y = Y; d.ldy = ldy; d.out_bf16 = prm.out_bf16; d.err = plan->err;
  d.wait_ns = prm.wait_ns; d.no_copies = prm.no_copies;
  d.offsets = row_offsets; d.E = E; d.small_max = kDecodeRows; d.a_rows = a_rows;
  return launch_splice_gemm_decode_tc(d, s);
}

// ------------------------------------------------------------------------------------------
// BF16 GEMM on the same tensor-core kernel: no NVFP4 k-tiles, every k-tile through the BF16
// path that carries the protected slice of a SpliceGEMM (kind::f16 MMAs, FP32 accumulation in
// TMEM).  Used by the straight-through backward of FourSight §5.2 ("backward passes run in BF16
// with STE").
// ------------------------------------------------------------------------------------------
namespace fs {

fs_status gemm_bf16(const char* who, fs_plan plan, int64_t M, int32_t N, int32_t K, const uint16_t* A, int64_t lda,
                    const uint16_t* B, int64_t ldb, const float* alpha, void* Y, int64_t ldy, cudaStream_t s) {
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null plan", who);
  if (M < 0 || N < 16 || N % 16 != 0 || K < 1)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: need M >= 0, N %% 16 == 0 (N >= 16), K >= 1", who);
  if (M == 0) return FS_OK;
  if (M > (int64_t{1} << 31) - 256 || K > (1 << 24)) return fail(FS_ERR_UNSUPPORTED, "%s: problem too large", who);
  if (!A || !B || !Y) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (lda < K || ldb < K || lda % 8 != 0 || ldb % 8 != 0 || !aligned(A, 16) || !aligned(B, 16))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: A and B need 16-byte aligned rows with ld >= K", who);
  const bool bf16 = plan->opts & FS_OUT_BF16;
  if (ldy < N || !aligned(Y, 16) || (ldy % (bf16 ? 8 : 4)) != 0)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: Y must be 16-byte aligned with ldy >= N and 16-byte rows", who);
  TcParams prm{};
  prm.M = M; prm.N = N; prm.K = 0; prm.KT = 0; prm.ST = static_cast<int>(ceil_div(K, 64));
  prm.E = 1; prm.kb4 = 0; prm.offsets = nullptr; prm.sfa = nullptr; prm.sfb = nullptr; prm.alpha = alpha;
  prm.seg = one_segment(N); prm.Y = Y; prm.ldy = ldy; prm.out_bf16 = bf16 ? 1 : 0; prm.err = plan->err;
  prm.wait_ns = wait_limit_ns(plan->opts); prm.no_copies = (plan->opts & FS_FAULT_NO_COPIES) ? 1 : 0;
  TcLaunch L{};
  L.xq = A; L.wq = B; L.xs = A; L.ws = B; L.a_rows = M; L.b_rows = N; L.y_rows = M; L.pp = K;
  L.xs_ld = lda; L.ws_ld = ldb;
  L.bn = (N % 256 == 0) ? 256 : 128;
  L.max_tiles = ceil_div(M, 128) * ceil_div(N, L.bn);
  return launch_splice_gemm_tc(L, prm, s);
}

}  // namespace fs

extern "C" fs_status fs_gemm_bf16(fs_plan plan, int64_t M, int32_t N, int32_t K, const uint16_t* A, int64_t lda,
                                  const uint16_t* B, int64_t ldb, const float* alpha, void* Y, int64_t ldy,
                                  void* stream) {
  return gemm_bf16("fs_gemm_bf16", plan, M, N, K, A, lda, B, ldb, alpha, Y, ldy, static_cast<cudaStream_t>(stream));
}

extern "C" int64_t fs_ste_backward_work_bytes(int64_t M, int32_t N, int32_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  const int64_t ldm = round_up(M, 8);
  return 2 * (static_cast<int64_t>(N) * ldm + static_cast<int64_t>(K) * ldm + static_cast<int64_t>(K) * N) + 3 * 256;
}

extern "C" fs_status fs_ste_backward(fs_plan plan, int64_t M, int32_t N, int32_t K, const uint16_t* dY, int64_t lddy,
                                     const uint16_t* X, int64_t ldx, const uint16_t* W, int64_t ldw, void* work,
                                     int64_t work_bytes, void* dX, int64_t lddx, void* dW, int64_t lddw, void* stream) {
  const char* who = "fs_ste_backward";
  if (!plan) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null plan", who);
  if (M < 0 || N < 16 || N % 16 != 0 || K < 16 || K % 16 != 0)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: need M >= 0 and N, K multiples of 16", who);
  if (M == 0) return FS_OK;
  if (M > (int64_t{1} << 24)) return fail(FS_ERR_UNSUPPORTED, "%s: M > 2^24 (the reduction length of dW)", who);
  if (!dY || !X || !W || !work || !dX || !dW) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (work_bytes < fs_ste_backward_work_bytes(M, N, K) || !aligned(work, 256))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: work must be 256-byte aligned with fs_ste_backward_work_bytes bytes", who);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t ldm = round_up(M, 8);
  auto* base = static_cast<uint8_t*>(work);
  auto* dYt = reinterpret_cast<uint16_t*>(base);                                            // [N][ldm]
  auto* Xt = reinterpret_cast<uint16_t*>(base + round_up(2 * N * ldm, 256));                 // [K][ldm]
  auto* Wt = reinterpret_cast<uint16_t*>(base + round_up(2 * N * ldm, 256) + round_up(2 * K * ldm, 256));   // [K][N]
  fs_status st = fs_transpose_bf16(M, N, dY, lddy, dYt, ldm, stream);
  if (st == FS_OK) st = fs_transpose_bf16(M, K, X, ldx, Xt, ldm, stream);
  if (st == FS_OK) st = fs_transpose_bf16(N, K, W, ldw, Wt, N, stream);
  if (st != FS_OK) return st;
  // dX [M][K] = dY [M][N] . W [N][K]: A = dY (reduction over N), B = W^T [K][N]
  st = gemm_bf16(who, plan, M, K, N, dY, lddy, Wt, N, nullptr, dX, lddx, s);
  if (st != FS_OK) return st;
  // dW [N][K] = dY^T [N][M] . X [M][K]: A = dY^T (reduction over M), B = X^T [K][M]
  return gemm_bf16(who, plan, N, K, static_cast<int32_t>(M), dYt, ldm, Xt, ldm, nullptr, dW, lddw, s);
}
