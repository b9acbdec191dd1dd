// Running channel moments and top-s protected-channel reselection.
//
// FourSight §5.2 "System Implementation": a forward hook subsamples token rows before masking
// and accumulates running channel moments in a GPU buffer; after each optimizer step the
// protected set is reselected as the top-s channels by the variance of the previous step
// (§9.3 Prop. 2 / Cor. 1 justify variance and second moment as the key; §6.1: s = 64).
//
// Moments are exact integers (s1 = sum rint(x 2^16), s2 = sum rint(x^2 2^14)), so every
// reduction order gives the same state and the selection is reproducible bit for bit.
#include <type_traits>

#include "common.cuh"
#include "moments.cuh"

namespace fs {
namespace {

using namespace moments;

constexpr int kStatsWarps = 8;
#ifndef FS_STATS_MIN_CTAS
#define FS_STATS_MIN_CTAS 3
#endif
#ifndef FS_STATS_VEC
#define FS_STATS_VEC 8
#endif
// bf16 channels per lane: 8 (16-byte loads).  4 channels with 4 CTAs per SM was faster on an
// L2-resident input but 10% slower on a 16384 x 4096 input read from HBM.
constexpr int kStatsVecBf16 = FS_STATS_VEC;
// fp32 inputs (small problems): convert directly.
__device__ __forceinline__ void add_f32(long long& s1, long long& s2, float& amax, float x, bool& bad) {
  const float ax = fabsf(x);
  if (!(ax < kRangeLimit)) {
    bad = true;
    return;
  }
  amax = fmaxf(amax, ax);
  s1 += __float2ll_rn(x * 65536.0f);
  const double xd = static_cast<double>(x);
  s2 += __double2ll_rn(__dmul_rn(__dmul_rn(xd, xd), kS2Scale));
}

// Grid: x = channel chunks (32*VEC channels), y = row groups.  Block: kStatsWarps warps; warp w
// takes rows (blockIdx.y*W + w) + i*gridDim.y*W of the subsampled rows, kUnroll rows per pass
// with all loads issued first.  Lane l holds VEC consecutive channels.  Each thread keeps its
// 64-bit totals in its own shared-memory slots ([warp][v][lane], conflict-free); the CTA reduces
// them over warps and adds to the global state with integer atomics.
template <typename T, int VEC>
__global__ void __launch_bounds__(kStatsWarps * 32, FS_STATS_MIN_CTAS)
channel_stats_kernel(const T* __restrict__ X, int64_t M, int K, int64_t ldx, int row_stride,
                     unsigned long long* n, unsigned long long* s1, unsigned long long* s2,
                     uint32_t* amax, uint32_t* flags) {
  constexpr bool kF32 = sizeof(T) == 4;
  constexpr int kUnroll = 4;
  __shared__ long long sh_s1[kStatsWarps][VEC][32];
  __shared__ long long sh_s2[kStatsWarps][VEC][32];
  __shared__ float sh_am[kStatsWarps][VEC][32];
  __shared__ int sh_bad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * 32 * VEC + lane * VEC;
  const bool active = c0 < K;
  if (threadIdx.x == 0) sh_bad = 0;
#pragma unroll
  for (int v = 0; v < VEC; ++v) { sh_s1[warp][v][lane] = 0; sh_s2[warp][v][lane] = 0; }
  bool bad = false;
  float am[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) am[v] = 0.0f;
  // bf16: raw-bit sums of up to kRawRows rows in wrapping 32-bit registers.  The largest term,
  // yh/2^8 < 2^22, keeps the exact sum of 256 rows inside int32.
  constexpr int kRawRows = 256;
  uint32_t ra1[VEC], rb1[VEC], rc2[VEC], rd2[VEC];
  int raw_rows = 0;
#pragma unroll
  for (int v = 0; v < VEC; ++v) { ra1[v] = 0u; rb1[v] = 0u; rc2[v] = 0u; rd2[v] = 0u; }
  auto flush_raw = [&]() {
    const uint32_t n_rows = static_cast<uint32_t>(raw_rows);
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      const int A1 = static_cast<int>(ra1[v] - n_rows * kMagicBits);
      const int B1 = static_cast<int>(rb1[v] - n_rows * kMagicBits);
      const int C2 = static_cast<int>(rc2[v] - n_rows * kMagic8Bits);
      const int D2 = static_cast<int>(rd2[v] - n_rows * kMagicBits);
      sh_s1[warp][v][lane] += static_cast<long long>(A1) * 65536 + B1;
      sh_s2[warp][v][lane] += static_cast<long long>(C2) * 4194304 + D2;   // yh*2^14 = (yh/2^8)*2^22
      ra1[v] = 0u; rb1[v] = 0u; rc2[v] = 0u; rd2[v] = 0u;
    }
    raw_rows = 0;
  };

  const int64_t taken = (M + row_stride - 1) / row_stride;     // rows 0, s, 2s, ...
  const int64_t step = static_cast<int64_t>(gridDim.y) * kStatsWarps;
  if (active) {
    for (int64_t i = static_cast<int64_t>(blockIdx.y) * kStatsWarps + warp; i < taken; i += kUnroll * step) {
      using Load = typename std::conditional<sizeof(T) * VEC == 16, uint4, uint2>::type;   // VEC elements
      Load q[kUnroll];
      int rows = 0;
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t idx = i + u * step;
        if (idx < taken) {
          q[u] = __ldg(reinterpret_cast<const Load*>(X + idx * row_stride * ldx + c0));
          ++rows;
        } else {
          q[u] = Load{};
        }
      }
      if constexpr (kF32) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          if (u >= rows) break;
          const float xs[4] = {__uint_as_float(q[u].x), __uint_as_float(q[u].y), __uint_as_float(q[u].z), __uint_as_float(q[u].w)};
#pragma unroll
          for (int v = 0; v < 4; ++v) add_f32(sh_s1[warp][v][lane], sh_s2[warp][v][lane], am[v], xs[v], bad);
        }
      } else {
        // Zero rows past the end contribute rint(0) = 0: their raw bits are the magic patterns,
        // removed with the row count.  The batch maximum of |x| per channel comes from the bf16
        // bits: the low 15 bits order like |x| (infinity and NaN above every finite value), and
        // |x| < 2^15 exactly when they are below 0x4700.  A batch of kUnroll rows of a channel
        // whose maximum is in range takes the select-free path; otherwise (rare) each element is
        // checked, out-of-range ones add the zero pattern and raise the flag.
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          uint32_t m2 = 0;                         // both channels of the word, packed
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            const uint32_t w = (&q[u].x)[v >> 1] & 0x7FFF7FFFu;
            asm("max.u16x2 %0, %1, %2;" : "=r"(m2) : "r"(m2), "r"(w));
          }
          float xs[kUnroll];
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            const uint32_t w = (&q[u].x)[v >> 1];
            xs[u] = (v & 1) ? bf16_hi(w) : bf16_lo(w);
          }
          const uint32_t mag = (v & 1) ? (m2 >> 16) : (m2 & 0xFFFFu);
          if (mag < 0x4700u) {
            static_assert(kUnroll % 2 == 0, "rows are taken in pairs");
#pragma unroll
            for (int u = 0; u < kUnroll; u += 2) add_bf16_pair_in_range(ra1[v], rb1[v], rc2[v], rd2[v], xs[u], xs[u + 1]);
            am[v] = fmaxf(am[v], __uint_as_float(mag << 16));
          } else {
            SmallSums a{ra1[v], rb1[v], rc2[v], rd2[v], am[v]};
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) add_bf16(a, xs[u], bad);
            ra1[v] = a.a1; rb1[v] = a.b1; rc2[v] = a.c2; rd2[v] = a.d2; am[v] = a.amax;
          }
        }
        raw_rows += kUnroll;
        if (raw_rows + kUnroll > kRawRows) flush_raw();
      }
    }
  }
  if constexpr (!kF32) flush_raw();
#pragma unroll
  for (int v = 0; v < VEC; ++v) sh_am[warp][v][lane] = am[v];
  if (bad) atomicOr(&sh_bad, 1);
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * VEC; c += blockDim.x) {
    const int ch = blockIdx.x * 32 * VEC + c;
    if (ch >= K) continue;
    const int v = c % VEC, l = c / VEC;
    long long a = 0, b = 0;
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kStatsWarps; ++w) {
      a += sh_s1[w][v][l];
      b += sh_s2[w][v][l];
      m = fmaxf(m, sh_am[w][v][l]);
    }
    if (a) atomicAdd(s1 + ch, static_cast<unsigned long long>(a));    // two's complement wraps
    if (b) atomicAdd(s2 + ch, static_cast<unsigned long long>(b));
    if (m > 0.0f) atomicMax(amax + ch, __float_as_uint(m));             // non-negative floats order as uints
  }
  if (threadIdx.x == 0) {
    if (sh_bad) atomicOr(flags, 1u);
    if (blockIdx.x == 0 && blockIdx.y == 0) atomicAdd(n, static_cast<unsigned long long>(taken));
  }
}

// ------------------------------------------------------------------------------------------
// Reselection: one CTA per problem.
// ------------------------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kMaxK = 16384;

// Map a double key to an unsigned integer with the same order (-0 folded onto +0 first).
__device__ __forceinline__ unsigned long long order_bits(double k) {
  if (k == 0.0) k = 0.0;
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(k));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ double channel_key(long long n, long long s1, long long s2, bool m2_only) {
  if (n == 0) return 0.0;
  const double dn = __ll2double_rn(n);
  const double m2 = __ddiv_rn(__ll2double_rn(s2) / kS2Scale, dn);   // /2^14 exact
  if (m2_only) return m2;
  const double m1 = __ddiv_rn(__ll2double_rn(s1) / kS1Scale, dn);   // /2^16 exact
  return __dsub_rn(m2, __dmul_rn(m1, m1));
}

__global__ void __launch_bounds__(kSelThreads)
select_topk_kernel(int K, long long* n_all, long long* s1_all, long long* s2_all, uint32_t* amax_all,
                   uint32_t* flags_all, int p, uint32_t opts, int32_t* P_all, uint32_t* mask_all,
                   float* gA_all, int reset) {
  extern __shared__ unsigned long long sh_keys[];         // [K]
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long sh_prefix;
  __shared__ int sh_need, sh_binc, sh_ties;
  __shared__ int sh_scan[kSelThreads / 32];
  __shared__ uint32_t sh_amax[kSelThreads / 32];

  const int prob = blockIdx.x;
  const long long n = n_all[prob];
  const long long* s1 = s1_all + static_cast<int64_t>(prob) * K;
  const long long* s2 = s2_all + static_cast<int64_t>(prob) * K;
  const uint32_t* amax = amax_all + static_cast<int64_t>(prob) * K;
  int32_t* P = P_all + static_cast<int64_t>(prob) * p;
  const int words = (K + 31) / 32;
  uint32_t* mask = mask_all + static_cast<int64_t>(prob) * words;
  const bool m2_only = opts & FS_KEY_M2;
  const int tid = threadIdx.x;

  for (int j = tid; j < K; j += blockDim.x) sh_keys[j] = order_bits(channel_key(n, s1[j], s2[j], m2_only));
  if (tid == 0) { sh_prefix = 0; sh_need = p; }
  __syncthreads();

  // Radix select of the p-th largest ordered key, 8 bits at a time from the top.  Histogram
  // updates are aggregated per warp (lanes with the same digit add once), and warp 0 finds the
  // threshold digit with a suffix scan over 8 bins per lane.  Once the bin holding the p-th key
  // is taken whole (its count equals the keys still needed), every key at or above the bin's
  // prefix is selected: the passes stop with T = that prefix and `need` = the keys equal to it.
  unsigned long long prefix = 0;
  int need = p;
  const int lane = tid & 31, warp_id = tid >> 5;
  if (p > 0) {
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      const unsigned long long hi_mask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
      for (int j0 = 0; j0 < K; j0 += blockDim.x) {
        const int j = j0 + tid;
        int bin = -1;
        if (j < K) {
          const unsigned long long k = sh_keys[j];
          if ((k & hi_mask) == prefix) bin = static_cast<int>((k >> shift) & 0xFF);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<unsigned>(__popc(peers)));
      }
      __syncthreads();
      if (warp_id == 0) {
        int c[8], local = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { c[i] = static_cast<int>(hist[8 * lane + i]); local += c[i]; }
        int incl = local;                                  // sum over lanes >= this lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += y;
        }
        const int above = incl - local;
        if (above < need && need <= incl) {
          int r = need - above, d = 8 * lane, bc = 0;
#pragma unroll
          for (int i = 7; i >= 0; --i) {
            if (c[i] >= r) { d = 8 * lane + i; bc = c[i]; break; }
            r -= c[i];
          }
          sh_prefix = prefix | (static_cast<unsigned long long>(d) << shift);
          sh_need = r;
          sh_binc = bc;
        }
      }
      if (tid == 0) sh_ties = 0;
      __syncthreads();
      prefix = sh_prefix;
      need = sh_need;
      if (shift > 0 && sh_binc == need) {          // uniform: the whole bin is selected
        int eq = 0;
        for (int j = tid; j < K; j += blockDim.x) eq += sh_keys[j] == prefix;
        if (eq) atomicAdd(&sh_ties, eq);
        __syncthreads();
        need = sh_ties;
        break;
      }
      __syncthreads();
    }
  }
  // Selected: key > T, plus the `need` lowest-index channels with key == T (T = prefix).
  // Channels are visited in index order, chunk per thread, with block-wide exclusive scans.
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int j0 = tid * per, j1 = min(K, j0 + per);
  int n_gt = 0, n_eq = 0;
  if (p > 0) {
    for (int j = j0; j < j1; ++j) {
      n_gt += sh_keys[j] > prefix;
      n_eq += sh_keys[j] == prefix;
    }
  }
  // exclusive scan of n_eq over threads (to rank ties by index)
  auto block_exclusive_scan = [&](int v) -> int {
    const int lane = tid & 31, warp = tid >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh_scan[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int s = (lane < (int)(blockDim.x >> 5)) ? sh_scan[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      if (lane < (int)(blockDim.x >> 5)) sh_scan[lane] = s;
    }
    __syncthreads();
    const int excl = x - v + (warp > 0 ? sh_scan[warp - 1] : 0);
    __syncthreads();
    return excl;
  };
  const int eq_before = block_exclusive_scan(n_eq);
  // count selected in this chunk
  int n_sel = 0;
  if (p > 0) {
    int eq_seen = eq_before;
    for (int j = j0; j < j1; ++j) {
      const unsigned long long k = sh_keys[j];
      if (k > prefix || (k == prefix && eq_seen++ < need)) ++n_sel;
    }
  }
  const int sel_before = block_exclusive_scan(n_sel);
  // write P (ascending) and the mask; unselected amax feed the gain
  float am_unprot = 0.0f;
  {
    int eq_seen = eq_before, out = sel_before;
    for (int j = j0; j < j1; ++j) {
      const unsigned long long k = sh_keys[j];
      const bool sel = p > 0 && (k > prefix || (k == prefix && eq_seen++ < need));
      if (sel) P[out++] = j;
      const float a = __uint_as_float(amax[j]);
      if (!sel || (opts & FS_RESIDUAL)) am_unprot = fmaxf(am_unprot, a);
      sh_keys[j] = sel ? 1ull : 0ull;       // reuse as the selection flag
    }
  }
  __syncthreads();
  for (int w = tid; w < words; w += blockDim.x) {
    uint32_t bits = 0;
    for (int b = 0; b < 32; ++b) {
      const int j = w * 32 + b;
      if (j < K && sh_keys[j]) bits |= 1u << b;
    }
    mask[w] = bits;
  }
  // block max of the unprotected amax
  uint32_t am = __float_as_uint(am_unprot);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
  if ((tid & 31) == 0) sh_amax[tid >> 5] = am;
  __syncthreads();
  if (tid == 0) {
    uint32_t m = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = max(m, sh_amax[w]);
    const float a = __uint_as_float(m);
    gA_all[prob] = (opts & FS_GAIN_EXACT) ? gain_exact(a) : gain_pow2(a);
  }
  if (reset) {
    __syncthreads();
    for (int j = tid; j < K; j += blockDim.x) {
      s1_all[static_cast<int64_t>(prob) * K + j] = 0;
      s2_all[static_cast<int64_t>(prob) * K + j] = 0;
      amax_all[static_cast<int64_t>(prob) * K + j] = 0;
    }
    if (tid == 0) { n_all[prob] = 0; flags_all[prob] = 0; }
  }
}

}  // namespace
}  // namespace fs

using namespace fs;

extern "C" fs_status fs_channel_stats(const void* X, int32_t dtype, int64_t M, int32_t K, int64_t ldx,
                                      int32_t row_stride, int64_t* n, int64_t* s1, int64_t* s2,
                                      uint32_t* amax, uint32_t* flags, void* stream) {
  if (M < 0 || K <= 0 || K % 8 != 0) return fail(FS_ERR_INVALID_ARGUMENT, "fs_channel_stats: need M >= 0, K > 0, K %% 8 == 0 (M=%lld K=%d)", (long long)M, K);
  if (row_stride < 1) return fail(FS_ERR_INVALID_ARGUMENT, "fs_channel_stats: row_stride must be >= 1");
  if (dtype != FS_DTYPE_BF16 && dtype != FS_DTYPE_F32) return fail(FS_ERR_INVALID_ARGUMENT, "fs_channel_stats: bad dtype %d", dtype);
  if (!n || !s1 || !s2 || !amax || !flags || (M > 0 && !X)) return fail(FS_ERR_INVALID_ARGUMENT, "fs_channel_stats: null pointer");
  const int esz = dtype == FS_DTYPE_BF16 ? 2 : 4;
  if (ldx < K || (ldx * esz) % 16 != 0 || !aligned(X, 16)) return fail(FS_ERR_INVALID_ARGUMENT, "fs_channel_stats: X rows must be 16-byte aligned and ldx >= K");
  if (!aligned(s1, 8) || !aligned(s2, 8) || !aligned(n, 8) || !aligned(amax, 4) || !aligned(flags, 4)) return fail(FS_ERR_INVALID_ARGUMENT, "fs_channel_stats: misaligned state");
  if (M == 0) return FS_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == FS_DTYPE_BF16;
  const int vec = bf16 ? kStatsVecBf16 : 4;
  const int chunks = static_cast<int>(ceil_div(K, 32 * vec));
  const int64_t taken = ceil_div(M, row_stride);
  // One wave: as many row groups per channel chunk as fill the resident CTA slots (a second,
  // partial wave would run at a fraction of the occupancy), each reading at least 128 rows.
  const void* kernel = bf16 ? reinterpret_cast<const void*>(channel_stats_kernel<uint16_t, kStatsVecBf16>)
                            : reinterpret_cast<const void*>(channel_stats_kernel<float, 4>);
  static PerDevice<int> per_sm[2];
  int slots = 1;
  if (!per_sm[bf16 ? 0 : 1].get(current_device(), &slots, [kernel](int* v) {
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, kernel, kStatsWarps * 32, 0) == cudaSuccess && *v >= 1;
      }))
    slots = 1;
  int64_t gy = std::max<int64_t>(1, static_cast<int64_t>(slots) * sm_count() / chunks);
  gy = std::min<int64_t>(gy, std::max<int64_t>(1, ceil_div(taken, 128)));
  gy = std::min<int64_t>(gy, 65535);
  dim3 grid(chunks, static_cast<unsigned>(gy));
  auto* un = reinterpret_cast<unsigned long long*>(n);
  auto* u1 = reinterpret_cast<unsigned long long*>(s1);
  auto* u2 = reinterpret_cast<unsigned long long*>(s2);
  if (bf16)
    channel_stats_kernel<uint16_t, kStatsVecBf16><<<grid, kStatsWarps * 32, 0, s>>>(static_cast<const uint16_t*>(X), M, K, ldx, row_stride, un, u1, u2, amax, flags);
  else
    channel_stats_kernel<float, 4><<<grid, kStatsWarps * 32, 0, s>>>(static_cast<const float*>(X), M, K, ldx, row_stride, un, u1, u2, amax, flags);
  FS_CHECK_LAUNCH("fs_channel_stats");
  return FS_OK;
}

extern "C" fs_status fs_stats_check(const uint32_t* flags, int32_t nprob, void* stream) {
  if (nprob < 0 || (nprob > 0 && !flags)) return fail(FS_ERR_INVALID_ARGUMENT, "fs_stats_check: bad arguments");
  if (nprob == 0) return FS_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host[64];
  for (int32_t i0 = 0; i0 < nprob; i0 += 64) {
    const int cnt = std::min(64, nprob - i0);
    cudaError_t e = cudaMemcpyAsync(host, flags + i0, cnt * sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e, "fs_stats_check");
    for (int i = 0; i < cnt; ++i)
      if (host[i]) return fail(FS_ERR_RANGE, "statistics input out of range (|x| >= 2^15 or not finite) in problem %d", i0 + i);
  }
  return FS_OK;
}

extern "C" fs_status fs_select_topk(int32_t nprob, int32_t K, int64_t* n, int64_t* s1, int64_t* s2,
                                    uint32_t* amax, uint32_t* flags, int32_t p, uint32_t opts,
                                    int32_t* P, uint32_t* mask, float* gA, int32_t reset, void* stream) {
  if (nprob < 0 || K <= 0 || K > kMaxK) return fail(FS_ERR_INVALID_ARGUMENT, "fs_select_topk: need 0 < K <= %d", kMaxK);
  if (p < 0 || p > K || p > 256) return fail(FS_ERR_INVALID_ARGUMENT, "fs_select_topk: need 0 <= p <= min(K, 256)");
  if (nprob == 0) return FS_OK;
  if (!n || !s1 || !s2 || !amax || !flags || !mask || !gA || (p > 0 && !P)) return fail(FS_ERR_INVALID_ARGUMENT, "fs_select_topk: null pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t smem = static_cast<size_t>(K) * sizeof(unsigned long long);
  static PerDevice<int> attr;
  fs_status ast = set_max_dynamic_smem(attr, reinterpret_cast<const void*>(select_topk_kernel), kMaxK * 8,
                                       "fs_select_topk: smem attribute");
  if (ast != FS_OK) return ast;
  select_topk_kernel<<<nprob, kSelThreads, smem, s>>>(K, reinterpret_cast<long long*>(n), reinterpret_cast<long long*>(s1),
                                                     reinterpret_cast<long long*>(s2), amax, flags, p, opts,
                                                     P, mask, gA, reset);
  FS_CHECK_LAUNCH("fs_select_topk");
  return FS_OK;
}
