// fs_splice_gemm_noalloc: the SpliceGEMM call for callers that cannot allocate device memory.
//
// fs_splice_gemm needs a plan, and creating a plan calls cudaMalloc for the device word in which
// the tensor-core kernel reports a bounded wait that gave up.  Some callers cannot allocate at
// that point: code running inside a custom allocator or memory-pool callback, inference runtimes
// that hand out every device byte from a pre-reserved arena, or plugins whose host framework
// forbids allocations after start-up.  This entry point does the same work without a plan: its one
// word of scratch lives in the file-scope device array below, which the CUDA module owns; every
// GPU that loads the library holds that array until the process exits.
//
// The array is shared by every call on a device and keeps the last call's contents, so each call
// clears it (cudaMemsetAsync on the caller's stream, no allocation) before its kernel starts.  Two
// calls that overlap on the GPU (different streams, no ordering between them) race on it: a
// timeout reported by one may then come from the other.
#include "common.cuh"
#include "gemm.cuh"

namespace fs {
namespace {

// Scratch of the allocation-free call: the tensor-core kernel's error word.  The kernel needs
// exactly this one 32-bit word, whatever the problem size.
constexpr int kNoAllocScratchWords = 1;
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocScratchWords];

// The device address of the scratch array in the context current on this thread.  In host code
// the array's name is only a host-side stand-in, so kernels must be given this address.  It is
// looked up on every call (cudaGetSymbolAddress allocates nothing): an address cached per device
// number would go stale after cudaDeviceReset or under another context of the same device.  The
// first lookup in a context may load the library's module there, which is why the first call on a
// device should come before any stream capture.
fs_status scratch_for_current_context(uint32_t** out) {
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_status(e, "fs_splice_gemm_noalloc: cudaGetSymbolAddress");
  *out = static_cast<uint32_t*>(ptr);
  return FS_OK;
}

}  // namespace
}  // namespace fs

using namespace fs;

extern "C" fs_status fs_splice_gemm_noalloc(int32_t N, int32_t K, uint32_t opts, int64_t M, int32_t p,
                                            const uint8_t* xq, const uint8_t* sfx, const uint16_t* xs,
                                            const uint8_t* wq, const uint8_t* sfw, const uint16_t* ws,
                                            const float* alpha, void* Y, int64_t ldy, int32_t check,
                                            void* stream) {
  const char* who = "fs_splice_gemm_noalloc";
  if (N < 16 || N % 16 != 0) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need N >= 16 and N %% 16 == 0 (N=%d)", who, N);
  if (K < 256 || K % 256 != 0 || K > 65536) return fail(FS_ERR_UNSUPPORTED, "%s: need K %% 256 == 0, 256 <= K <= 65536 (K=%d)", who, K);
  if (M < 0 || M > (int64_t{1} << 31) - 256) return fail(FS_ERR_UNSUPPORTED, "%s: need 0 <= M < 2^31 - 256", who);
  if (p < 0 || p > 256 || p > K) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need 0 <= p <= min(K, 256)", who);
  if ((opts & (FS_PATH_TENSOR | FS_PATH_DECODE)) == (FS_PATH_TENSOR | FS_PATH_DECODE))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: FS_PATH_TENSOR and FS_PATH_DECODE are exclusive", who);
  if (M == 0) return FS_OK;                        // an empty batch reads no operand
  if (!xq || !sfx || !wq || !sfw || !alpha || !Y || (p > 0 && (!xs || !ws)))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (!aligned(xq, 16) || !aligned(sfx, 16) || !aligned(wq, 16) || !aligned(sfw, 16) ||
      (p > 0 && (!aligned(xs, 16) || !aligned(ws, 16))))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: packed operands must be 16-byte aligned", who);
  const bool bf16 = opts & FS_OUT_BF16;
  if (ldy < N || !aligned(Y, 16) || (ldy % (bf16 ? 8 : 4)) != 0)
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: Y must be 16-byte aligned with ldy >= N and 16-byte rows", who);
  const bool decode = (opts & FS_PATH_DECODE) || (!(opts & FS_PATH_TENSOR) && M <= 16);
  if (decode && M > 16) return fail(FS_ERR_UNSUPPORTED, "%s: the decode path takes M <= 16", who);
  // The kernels need exactly kNoAllocScratchWords words of scratch; no problem size needs more.
  static_assert(kNoAllocScratchWords >= 1, "one error word");

  uint32_t* scratch = nullptr;
  fs_status st = scratch_for_current_context(&scratch);
  if (st != FS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(scratch, 0, kNoAllocScratchWords * sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_status(e, "fs_splice_gemm_noalloc: clearing scratch");

  const int pp = side_cols(p);
  if (decode) {
    DecodeParams d{};
    d.M = static_cast<int>(M); d.N = N; d.K = K; d.pp = pp; d.kb4 = static_cast<int>(round_up(K / 16, 4) / 4);
    d.xq = xq; d.sfx = sfx; d.xs = xs; d.wq = wq; d.sfw = sfw; d.ws = ws; d.alpha = alpha;
    d.Y = Y; d.ldy = ldy; d.out_bf16 = bf16 ? 1 : 0; d.err = scratch;
    d.wait_ns = wait_limit_ns(opts); d.no_copies = (opts & FS_FAULT_NO_COPIES) ? 1 : 0;
    d.seg.n = 1; d.seg.n0[0] = 0; d.seg.n0[1] = N;
    st = launch_splice_gemm_decode_tc(d, s);
  } else {
    TcParams prm{};
    prm.M = M; prm.N = N; prm.K = K; prm.KT = K / 256; prm.ST = static_cast<int>(ceil_div(pp, 64));
    prm.E = 1; prm.kb4 = K / 64; prm.offsets = nullptr; prm.sfa = sfx; prm.sfb = sfw; prm.alpha = alpha;
    prm.Y = Y; prm.ldy = ldy; prm.out_bf16 = bf16 ? 1 : 0; prm.err = scratch;
    prm.wait_ns = wait_limit_ns(opts); prm.no_copies = (opts & FS_FAULT_NO_COPIES) ? 1 : 0;
    prm.seg.n = 1; prm.seg.n0[0] = 0; prm.seg.n0[1] = N;
    TcLaunch L{};
    L.xq = xq; L.wq = wq; L.xs = xs; L.ws = ws; L.a_rows = M; L.b_rows = N; L.y_rows = M; L.pp = pp;
    L.bn = (N % 256 == 0) ? 256 : 128;
    L.max_tiles = ceil_div(M, 128) * ceil_div(N, L.bn);
    st = launch_splice_gemm_tc(L, prm, s);
  }
  if (st != FS_OK || !check) return st;
  uint32_t word = 0;
  e = cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, "fs_splice_gemm_noalloc: reading scratch");
  if (word) return fail(FS_ERR_TIMEOUT, "%s: the kernel gave up a bounded wait (word 0x%x)", who, word);
  return FS_OK;
}
