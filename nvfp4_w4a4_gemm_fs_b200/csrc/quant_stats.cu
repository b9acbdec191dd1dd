// Activation preparation with the channel statistics in the same pass over X.
//
// FourSight §5.2 "System Implementation": a forward hook subsamples token rows BEFORE masking and
// accumulates running channel moments; §5.1 "Data preparation" then masks the protected lanes
// (Mask S->0), quantises the rest to NVFP4 (FP4 Quant) and copies the protected columns to X_S
// (Extract X_S).  Both read the same activations, so this kernel reads each bf16 element of X once
// and does both: the moments of the raw value (exact integers, added to the state the NEXT
// reselection reads) and the masked NVFP4 encoding with the CURRENT protected set.
//
// Layout of the work: CTA (x, y) owns the 256-channel slab x and every (8 * gridDim.y)-th pair of
// rows starting at 2 * (8 y + warp); lane l of a warp holds the 8 channels 8l .. 8l+7 of the slab
// (one 16-byte load per row), so a 16-element block is two adjacent lanes.  A warp takes two rows
// per iteration: the moments take the rows pairwise through the packed fp32x2 arithmetic (each lane
// of a pair is one row), and each row is quantised on its own.  The lane's protected lanes, its
// kill mask and its first side column depend only on the slab, so they are computed once.
//
// Results are bit-identical to fs_channel_stats followed by fs_quantize_splice: the moments are
// exact integers (order-free), and the block rule is the library's (t = fl32(fl32(a_b g)/6),
// sf = UE4M3_RNE(t), v = fl32(fl32(x g)/sf), q = E2M1_RNE(v)).
#include "common.cuh"
#include "moments.cuh"

namespace fs {
namespace {

using namespace moments;

constexpr int kQSWarps = 8;
constexpr int kQSThreads = kQSWarps * 32;
constexpr int kSlab = 256;                       // channels per CTA column (32 lanes x 8)
constexpr int kDepth = 4;                        // row pairs per warp in the shared-memory ring

struct QSArgs {
  const uint16_t* X;
  int64_t ldx;
  int64_t M, Mp;                 // rows, rows padded to 128 (scale rows written as zero past M)
  int K, kb4, p, pp;
  uint32_t opts;
  const uint32_t* mask;          // may be null when p == 0
  const float* gain;
  uint8_t* q;
  uint8_t* sf;
  uint16_t* side;
  int row_stride;
  unsigned long long* n;
  unsigned long long* s1;
  unsigned long long* s2;
  uint32_t* amax;
  uint32_t* flags;
};

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

template <bool kStats>
__global__ void __launch_bounds__(kQSThreads, 2) quantize_stats_kernel(const QSArgs a) {
  __shared__ unsigned long long sh_s1[kSlab];      // per channel of the slab, summed over the warps
  __shared__ unsigned long long sh_s2[kSlab];
  __shared__ uint32_t sh_am[kSlab];                // max |x| as bf16 magnitude bits
  __shared__ float sh_val[128], sh_rcp[128];
  __shared__ int sh_bad;
  __shared__ uint4 ring[kQSWarps][kDepth][2][32];   // per warp: kDepth row pairs x 32 lanes x 16 bytes

  // Programmatic dependent launch: the next kernel (the decode GEMM, which streams its weights
  // into L2 before it waits for this grid) may start now; this grid's own first global access
  // comes after griddepcontrol.wait, i.e. after the previous kernel has finished and flushed.
  // Both instructions are no-ops when the launch carries no programmatic dependency.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * kSlab + lane * 8;
  const bool active = c0 < a.K;                  // K % 64 == 0: whole 8-lane scale groups
  if (threadIdx.x < 128) {
    const int c = threadIdx.x;                   // code 0 and the unused NaN code: d = 1, r = 0
    const bool real = c > 0 && c < 127;
    const float d = real ? ue4m3_value(c) : 1.0f;
    sh_val[c] = d;
    sh_rcp[c] = real ? __frcp_rn(d) : 0.0f;
  }
  if (threadIdx.x == 0) sh_bad = 0;
  for (int c = threadIdx.x; c < kSlab; c += blockDim.x) { sh_s1[c] = 0; sh_s2[c] = 0; sh_am[c] = 0; }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Protected lanes of this lane's 8 channels, the words to clear, and the side column of its
  // first protected channel (protected channels below c0).  The count below the slab is shared by
  // the warp: 32 mask words per step, summed with a warp reduction.
  uint32_t pbits = 0;
  int col0 = 0;
  if (a.p > 0) {
    const int wi = c0 >> 5;
    const int slab_w = (blockIdx.x * kSlab) >> 5;             // first mask word of the slab
    int below = 0;
    for (int w0 = 0; w0 < slab_w; w0 += 32) {
      const int w = w0 + lane;
      int cnt = w < slab_w ? __popc(__ldg(a.mask + w)) : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      below += cnt;
    }
    if (active) {
      for (int w = slab_w; w < wi; ++w) below += __popc(__ldg(a.mask + w));
      const uint32_t mw = __ldg(a.mask + wi);
      below += __popc(mw & ((1u << (c0 & 31)) - 1u));
      pbits = (mw >> (c0 & 31)) & 0xFFu;
    }
    col0 = below;
  }
  uint32_t kill[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t two = (pbits >> (2 * j)) & 3u;
    kill[j] = ((two & 1u) | ((two & 2u) << 15)) * 0xFFFFu;
  }
  const bool residual = a.opts & FS_RESIDUAL;
  const float g = __ldg(a.gain);
  const bool fast = pow2_gain_in_fast_range(g);
  const float inv6 = __frcp_rn(6.0f);
  const int blk = c0 >> 4;                        // this lane's 16-element block
  __syncthreads();

  // moments: raw-bit sums of up to kRawRows rows in wrapping 32-bit registers (see moments.cuh)
  constexpr int kRawRows = 256;
  uint32_t ra1[8], rb1[8], rc2[8], rd2[8];
  uint32_t am[4] = {0u, 0u, 0u, 0u};             // per channel pair: max |x| as bf16 magnitude bits
#pragma unroll
  for (int v = 0; v < 8; ++v) { ra1[v] = 0u; rb1[v] = 0u; rc2[v] = 0u; rd2[v] = 0u; }
  int raw_rows = 0;
  bool bad = false;
  auto flush_raw = [&]() {
    const uint32_t nr = static_cast<uint32_t>(raw_rows);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int A1 = static_cast<int>(ra1[v] - nr * kMagicBits);
      const int B1 = static_cast<int>(rb1[v] - nr * kMagicBits);
      const int C2 = static_cast<int>(rc2[v] - nr * kMagic8Bits);
      const int D2 = static_cast<int>(rd2[v] - nr * kMagicBits);
      // two's complement: adding the 64-bit pattern of a negative sum subtracts it
      atomicAdd(&sh_s1[lane * 8 + v], static_cast<unsigned long long>(static_cast<long long>(A1) * 65536 + B1));
      atomicAdd(&sh_s2[lane * 8 + v], static_cast<unsigned long long>(static_cast<long long>(C2) * 4194304 + D2));
      ra1[v] = 0u; rb1[v] = 0u; rc2[v] = 0u; rd2[v] = 0u;
    }
    raw_rows = 0;
  };

  // Quantise one row's 8 channels (a half block; the partner lane holds the other half).  The row
  // test is uniform across the warp, so every lane reaches the shuffles; lanes past K hold zeros
  // and store nothing.
  auto quantise_row = [&](int64_t r, const uint4& x) {
    uint32_t sfc = 0;
    if (r < a.M) {
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      uint32_t xm[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) xm[j] = w[j] & ~kill[j];
      const uint32_t* src = residual ? w : xm;       // lanes that set the block scale
      uint32_t m = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) m = vmax_u16x2(m, src[j] & 0x7FFF7FFFu);
      uint32_t mb = max(m & 0xFFFFu, m >> 16);
      mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 1));   // the block's other half
      // NaN cannot occur here (finite inputs required); |x| bits order like |x|
      const float amax = __uint_as_float(mb << 16);
      const float t = div_markstein(__fmul_rn(amax, g), 6.0f, inv6);
      sfc = ue4m3_rne(t);
      const float sd = sh_val[sfc], sr = sh_rcp[sfc];
      float v[8];
      if (fast) {
        const float R = __fmul_rn(g, sr);            // exact: g is a power of two in range
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[2 * j] = snap12(__fmul_rn(bf16_lo(xm[j]), R));
          v[2 * j + 1] = snap12(__fmul_rn(bf16_hi(xm[j]), R));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[2 * j] = div_markstein(__fmul_rn(bf16_lo(xm[j]), g), sd, sr);
          v[2 * j + 1] = div_markstein(__fmul_rn(bf16_hi(xm[j]), g), sd, sr);
        }
      }
      if (active)
        *reinterpret_cast<uint32_t*>(a.q + r * (a.K / 2) + (c0 >> 1)) =
            e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
      if (pbits) {                                   // Extract X_S (pbits == 0 for lanes past K)
        uint32_t pb = pbits;
        int col = col0;
        while (pb) {
          const int j = __ffs(pb) - 1;
          pb &= pb - 1;
          a.side[r * a.pp + col++] = static_cast<uint16_t>((w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
        }
      }
    }
    // scale word of blocks 4k..4k+3 (lanes 8k, 8k+2, 8k+4, 8k+6 hold them); zero past M
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sfc, 2);
    const uint32_t s4 = __shfl_down_sync(0xffffffffu, sfc, 4);
    const uint32_t s6 = __shfl_down_sync(0xffffffffu, sfc, 6);
    if (active && (lane & 7) == 0)
      *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, blk, a.kb4)) = sfc | (s2 << 8) | (s4 << 16) | (s6 << 24);
    // padding side columns p .. pp-1 of the row (slab 0 writes them)
    if (blockIdx.x == 0 && r < a.M && lane < a.pp - a.p) a.side[r * a.pp + a.p + lane] = 0;
  };

  // Rows stream through a per-warp ring in shared memory filled by cp.async (each lane copies and
  // later reads only its own 16-byte slots, so no barrier is needed beyond cp.async.wait_group):
  // kDepth - 1 row pairs stay in flight while the warp computes on the current one.
  const int64_t step = static_cast<int64_t>(gridDim.y) * kQSWarps * 2;
  const int64_t first = (static_cast<int64_t>(blockIdx.y) * kQSWarps + warp) * 2;
  auto issue = [&](int64_t r0, int slot) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t r = r0 + h;
      if (active && r < a.M) {
        const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&ring[warp][slot][h][lane]));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(a.X + r * a.ldx + c0) : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll
  for (int d = 0; d < kDepth - 1; ++d) issue(first + d * step, d);
  int slot = 0;
  // r0 % row_stride, kept incrementally (a 64-bit division per row would dominate the loop)
  const int64_t stride = a.row_stride;
  int64_t mod0 = first % stride;
  const int64_t dmod = step % stride;
  for (int64_t r0 = first; r0 < a.Mp; r0 += step) {
    issue(r0 + (kDepth - 1) * step, (slot + kDepth - 1) % kDepth);
    asm volatile("cp.async.wait_group %0;" ::"n"(kDepth - 1) : "memory");
    const int64_t r1 = r0 + 1;
    uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = make_uint4(0u, 0u, 0u, 0u);
    if (active && r0 < a.M) xa = ring[warp][slot][0][lane];
    if (active && r1 < a.M) xb = ring[warp][slot][1][lane];
    slot = slot + 1 == kDepth ? 0 : slot + 1;
    // moments of the raw (unmasked) values of the rows the statistics take
    const int64_t mod1 = mod0 + 1 == stride ? 0 : mod0 + 1;
    const bool ta = r0 < a.M && mod0 == 0;
    const bool tb = r1 < a.M && mod1 == 0;
    mod0 += dmod;
    if (mod0 >= stride) mod0 -= stride;
    if (kStats && active && (ta || tb)) {
      const uint32_t wa[4] = {ta ? xa.x : 0u, ta ? xa.y : 0u, ta ? xa.z : 0u, ta ? xa.w : 0u};
      const uint32_t wb[4] = {tb ? xb.x : 0u, tb ? xb.y : 0u, tb ? xb.z : 0u, tb ? xb.w : 0u};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t m2 = vmax_u16x2(wa[j] & 0x7FFF7FFFu, wb[j] & 0x7FFF7FFFu);   // both channels, both rows
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int v = 2 * j + h;
          const uint32_t mag = h ? (m2 >> 16) : (m2 & 0xFFFFu);
          const float x0 = h ? bf16_hi(wa[j]) : bf16_lo(wa[j]);
          const float x1 = h ? bf16_hi(wb[j]) : bf16_lo(wb[j]);
          if (mag < 0x4700u) {                   // |x| < 2^15 for both rows: select-free path
            add_bf16_pair_in_range(ra1[v], rb1[v], rc2[v], rd2[v], x0, x1);
            am[j] = vmax_u16x2(am[j], m2 & (h ? 0xFFFF0000u : 0x0000FFFFu));
          } else {
            SmallSums s{ra1[v], rb1[v], rc2[v], rd2[v], 0.0f};
            add_bf16(s, x0, bad);
            add_bf16(s, x1, bad);
            ra1[v] = s.a1; rb1[v] = s.b1; rc2[v] = s.c2; rd2[v] = s.d2;
            const uint32_t mb = __float_as_uint(s.amax) >> 16;          // in-range part only
            am[j] = vmax_u16x2(am[j], h ? (mb << 16) : mb);
          }
        }
      }
      raw_rows += 2;                             // a row not taken adds the zero pattern
      if (raw_rows + 2 > kRawRows) flush_raw();
    }
    quantise_row(r0, xa);
    quantise_row(r1, xb);
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");   // nothing left in flight (all past the end)
  if constexpr (!kStats) return;
  flush_raw();
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (am[j] & 0xFFFFu) atomicMax(&sh_am[lane * 8 + 2 * j], am[j] & 0xFFFFu);
    if (am[j] >> 16) atomicMax(&sh_am[lane * 8 + 2 * j + 1], am[j] >> 16);
  }
  if (bad) atomicOr(&sh_bad, 1);
  __syncthreads();
  for (int c = threadIdx.x; c < kSlab; c += blockDim.x) {
    const int ch = blockIdx.x * kSlab + c;
    if (ch >= a.K) continue;
    if (sh_s1[c]) atomicAdd(a.s1 + ch, sh_s1[c]);     // two's complement wraps
    if (sh_s2[c]) atomicAdd(a.s2 + ch, sh_s2[c]);
    if (sh_am[c]) atomicMax(a.amax + ch, sh_am[c] << 16);   // bf16 magnitude bits -> float bits
  }
  if (threadIdx.x == 0) {
    if (sh_bad) atomicOr(a.flags, 1u);
    if (blockIdx.x == 0 && blockIdx.y == 0)
      atomicAdd(a.n, static_cast<unsigned long long>((a.M + a.row_stride - 1) / a.row_stride));
  }
}

}  // namespace

// One wave: as many row groups per slab as fill the resident CTA slots, each with at least 16 row
// pairs per warp when the batch is large enough.
fs_status launch_quantize_rows(const QSArgs& a, bool with_stats, cudaStream_t s, const char* who) {
  // resident CTAs per SM of the instantiation that runs (the moments take twice the registers)
  static PerDevice<int> occ_stats, occ_plain;
  int slots = 1;
  const bool got = with_stats
      ? occ_stats.get(current_device(), &slots, [](int* v) {
          return cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, quantize_stats_kernel<true>, kQSThreads, 0) ==
                     cudaSuccess && *v >= 1;
        })
      : occ_plain.get(current_device(), &slots, [](int* v) {
          return cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, quantize_stats_kernel<false>, kQSThreads, 0) ==
                     cudaSuccess && *v >= 1;
        });
  if (!got) slots = 1;
  const int chunks = static_cast<int>(ceil_div(a.K, kSlab));
  int64_t gy = std::max<int64_t>(1, static_cast<int64_t>(slots) * sm_count() / chunks);
  gy = std::min<int64_t>(gy, std::max<int64_t>(1, ceil_div(a.Mp, 2 * kQSWarps * 16)));
  gy = std::min<int64_t>(gy, 65535);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(chunks, static_cast<unsigned>(gy), 1);
  cfg.blockDim = dim3(kQSThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = with_stats ? cudaLaunchKernelEx(&cfg, quantize_stats_kernel<true>, a)
                                   : cudaLaunchKernelEx(&cfg, quantize_stats_kernel<false>, a);
  if (e != cudaSuccess) return cuda_status(e, who);
  FS_CHECK_LAUNCH(who);
  return FS_OK;
}

// fs_quantize_splice for decode-sized bf16 batches: the same row-streaming kernel without the
// moments (no per-CTA mask tables; each lane derives its protected lanes from the mask directly).
fs_status quantize_rows_bf16(const void* X, int64_t M, int32_t K, int64_t ldx, const uint32_t* mask, int32_t p,
                             const float* gA, uint32_t opts, uint8_t* xq, uint8_t* sfx, uint16_t* xs, cudaStream_t s) {
  QSArgs a{};
  a.X = static_cast<const uint16_t*>(X); a.ldx = ldx; a.M = M; a.Mp = round_up(M, 128); a.K = K;
  a.kb4 = static_cast<int>(round_up(K / 16, 4) / 4); a.p = p; a.pp = side_cols(p); a.opts = opts;
  a.mask = p > 0 ? mask : nullptr; a.gain = gA; a.q = xq; a.sf = sfx; a.side = xs; a.row_stride = 1;
  return launch_quantize_rows(a, false, s, "fs_quantize_splice");
}

}  // namespace fs

using namespace fs;

extern "C" fs_status fs_quantize_splice_stats(const void* X, int32_t dtype, int64_t M, int32_t K, int64_t ldx,
                                              const uint32_t* mask, int32_t p, const float* gA, uint32_t opts,
                                              uint8_t* xq, uint8_t* sfx, uint16_t* xs, int32_t row_stride,
                                              int64_t* n, int64_t* s1, int64_t* s2, uint32_t* amax,
                                              uint32_t* flags, void* stream) {
  const char* who = "fs_quantize_splice_stats";
  if (M < 0) return fail(FS_ERR_INVALID_ARGUMENT, "%s: M < 0", who);
  if (dtype != FS_DTYPE_BF16 && dtype != FS_DTYPE_F32) return fail(FS_ERR_INVALID_ARGUMENT, "%s: bad dtype %d", who, dtype);
  if (dtype != FS_DTYPE_BF16) return fail(FS_ERR_UNSUPPORTED, "%s: bf16 activations only", who);
  if (K <= 0 || K % 64 != 0 || K > 16384) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need K %% 64 == 0 and 0 < K <= 16384 (K=%d)", who, K);
  if (p < 0 || p > K || p > 256) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need 0 <= p <= min(K,256) (p=%d)", who, p);
  if (row_stride < 1) return fail(FS_ERR_INVALID_ARGUMENT, "%s: row_stride must be >= 1", who);
  if (ldx < K || (ldx * 2) % 16 != 0) return fail(FS_ERR_INVALID_ARGUMENT, "%s: leading dimension must be >= K with 16-byte rows", who);
  if (!gA || !xq || !sfx || (p > 0 && (!mask || !xs)) || !n || !s1 || !s2 || !amax || !flags || (M > 0 && !X))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (!aligned(X, 16) || !aligned(xq, 16) || !aligned(sfx, 16) || (xs && !aligned(xs, 16)) || (mask && !aligned(mask, 4)) ||
      !aligned(s1, 8) || !aligned(s2, 8) || !aligned(n, 8) || !aligned(amax, 4) || !aligned(flags, 4))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: misaligned pointer", who);
  if (M == 0) return FS_OK;
  QSArgs a{};
  a.X = static_cast<const uint16_t*>(X); a.ldx = ldx; a.M = M; a.Mp = round_up(M, 128); a.K = K;
  a.kb4 = static_cast<int>(round_up(K / 16, 4) / 4); a.p = p; a.pp = side_cols(p); a.opts = opts;
  a.mask = p > 0 ? mask : nullptr; a.gain = gA; a.q = xq; a.sf = sfx; a.side = xs; a.row_stride = row_stride;
  a.n = reinterpret_cast<unsigned long long*>(n); a.s1 = reinterpret_cast<unsigned long long*>(s1);
  a.s2 = reinterpret_cast<unsigned long long*>(s2); a.amax = amax; a.flags = flags;
  return launch_quantize_rows(a, true, static_cast<cudaStream_t>(stream), who);
}
