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
#include "ptx.cuh"

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
// Reselection: one cluster of kSelCluster CTAs per problem.
// ------------------------------------------------------------------------------------------
constexpr int kSelCluster = 8;
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelMaxR = 4;                   // rounds of 32 channels per warp
constexpr int kMaxK = kSelCluster * kSelThreads * kSelMaxR;   // 16384

// Map a double key to an unsigned integer with the same order (-0 folded onto +0 first).
__device__ __forceinline__ unsigned long long order_bits(double k) {
  if (k == 0.0) k = 0.0;
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(k));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Correctly rounded y / d in fp64 from r = RN(1/d), by Markstein's correction (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev.
// 34(1), 1990), the fp64 counterpart of the library's fp32 division: q0 = RN(y*r) is within two
// ulps; the first remainder step makes it faithful (pre-rounding error below 4u^2 |y/d|, u = 2^-53),
// after which the remainder y - d*q1 is exact in one fused multiply-add and the second step
// rounds correctly.  Used with d = n >= 1 and y a scaled integer moment, so nothing underflows.
__device__ __forceinline__ double div_rn_by(double y, double d, double r) {
  const double q0 = __dmul_rn(y, r);
  const double e0 = __fma_rn(-q0, d, y);
  const double q1 = __fma_rn(e0, r, q0);
  const double e1 = __fma_rn(-q1, d, y);
  return __fma_rn(e1, r, q1);
}

// Key of one channel: fl64(m2 - fl64(m1 * m1)) with m1 = fl64(fl64(s1 / 2^16) / n),
// m2 = fl64(fl64(s2 / 2^14) / n); dn = n and rn = RN(1/n) are the problem's (n > 0).
__device__ __forceinline__ double channel_key(double dn, double rn, long long s1, long long s2, bool m2_only) {
  const double m2 = div_rn_by(__ll2double_rn(s2) / kS2Scale, dn, rn);   // /2^14 exact
  if (m2_only) return m2;
  const double m1 = div_rn_by(__ll2double_rn(s1) / kS1Scale, dn, rn);   // /2^16 exact
  return __dsub_rn(m2, __dmul_rn(m1, m1));
}

// The cluster's CTAs split the channels: CTA c takes [c*chunk, (c+1)*chunk), chunk = 512*R, and
// its warp w the 32*R channels from c*chunk + 32*R*w, one round of 32 consecutive channels (one
// mask word) per step, so every thread holds at most kSelMaxR keys in registers.
//
// The p-th largest key is found by a radix select over the cluster, 8 bits at a time from the top:
// each CTA histograms its keys that match the prefix so far (warp-aggregated shared atomics), and
// after a cluster barrier every CTA sums the 8 histograms through distributed shared memory and
// takes the same decision.  Histograms are double-buffered, so one barrier per pass suffices: a
// CTA rewrites a buffer only after the next pass's barrier, which every other CTA reaches after
// reading it.  Once the bin holding the p-th key is taken whole (its count equals the keys still
// needed) every key from the bin's prefix up is selected and the passes stop.
//
// Selected: key > T, plus the `need` lowest-index channels with key == T.  The CTAs exchange
// their counts of keys > T and == T (one barrier), which fixes each warp's first tie rank and
// first output slot; the warps then walk their rounds with ballots, writing P in ascending order
// and one mask word per round.  The maximum of the unprotected channels' amax goes to CTA 0 by
// remote atomics; after the last barrier CTA 0 writes the gain.
__global__ void __cluster_dims__(kSelCluster, 1, 1) __launch_bounds__(kSelThreads)
select_topk_kernel(int K, int R, long long* n_all, long long* s1_all, long long* s2_all, uint32_t* amax_all,
                   uint32_t* flags_all, int p, uint32_t opts, int32_t* P_all, uint32_t* mask_all,
                   float* gA_all, int reset) {
  __shared__ unsigned int hist[2][256];          // this CTA's histogram of the pass (double-buffered)
  __shared__ unsigned int tot[256];              // the cluster's histogram of the pass
  __shared__ unsigned long long sh_prefix;
  __shared__ int sh_need, sh_binc;
  __shared__ int sh_wgt[kSelWarps], sh_weq[kSelWarps];
  __shared__ int sh_cnt[2];                      // this CTA's keys > T and == T (read by the cluster)
  __shared__ uint32_t sh_wam[kSelWarps];
  __shared__ uint32_t sh_am_cluster;             // CTA 0: maximum over the cluster

  const int prob = blockIdx.x / kSelCluster;
  const uint32_t rank = ptx::cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const long long n = n_all[prob];
  long long* s1 = s1_all + static_cast<int64_t>(prob) * K;
  long long* s2 = s2_all + static_cast<int64_t>(prob) * K;
  uint32_t* amax = amax_all + static_cast<int64_t>(prob) * K;
  int32_t* P = P_all + static_cast<int64_t>(prob) * p;
  const int words = (K + 31) / 32;
  uint32_t* mask = mask_all + static_cast<int64_t>(prob) * words;
  const bool m2_only = opts & FS_KEY_M2;
  const int j_warp = static_cast<int>(rank) * kSelThreads * R + warp * 32 * R;   // first channel of the warp

  if (tid == 0) sh_am_cluster = 0;               // ordered before any remote access by a cluster barrier

  // Keys and maxima into registers, every load in flight at once; the moments are cleared (reset)
  // by the thread that read them.
  const double dn = __ll2double_rn(n);
  const double rn = n > 0 ? __drcp_rn(dn) : 0.0;
  unsigned long long key[kSelMaxR];
  uint32_t am[kSelMaxR];
  bool valid[kSelMaxR];
  {
    long long a1[kSelMaxR], a2[kSelMaxR];
#pragma unroll
    for (int r = 0; r < kSelMaxR; ++r) {
      const int j = j_warp + r * 32 + lane;
      valid[r] = r < R && j < K;
      a1[r] = 0; a2[r] = 0; am[r] = 0;
      if (valid[r]) { a1[r] = __ldcg(s1 + j); a2[r] = __ldcg(s2 + j); am[r] = __ldcg(amax + j); }
    }
#pragma unroll
    for (int r = 0; r < kSelMaxR; ++r) {
      key[r] = order_bits(n == 0 ? 0.0 : channel_key(dn, rn, a1[r], a2[r], m2_only));
      if (valid[r] && reset) {
        const int j = j_warp + r * 32 + lane;
        s1[j] = 0; s2[j] = 0; amax[j] = 0;
      }
    }
  }

  // Threshold T and the number of keys equal to T to take (p = 0: nothing is selected).
  unsigned long long T = ~0ull;
  int need = 0;
  if (p > 0) {
    unsigned long long prefix = 0;
    need = p;
    int buf = 0;
    for (int shift = 56; shift >= 0; shift -= 8, buf ^= 1) {
      for (int i = tid; i < 256; i += kSelThreads) hist[buf][i] = 0;
      __syncthreads();
      const unsigned long long hi_mask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
#pragma unroll
      for (int r = 0; r < kSelMaxR; ++r) {
        if (r < R) {                                  // uniform
          const int bin = (valid[r] && (key[r] & hi_mask) == prefix) ? static_cast<int>((key[r] >> shift) & 0xFF) : -1;
          const unsigned peers = __match_any_sync(0xffffffffu, bin);
          if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[buf][bin], static_cast<unsigned>(__popc(peers)));
        }
      }
      ptx::cluster_sync();                            // every CTA's histogram of this pass is complete
      if (tid < 256) {
        const uint32_t addr = ptx::smem_u32(&hist[buf][tid]);
        unsigned int part[kSelCluster];
#pragma unroll
        for (int c = 0; c < kSelCluster; ++c) part[c] = ptx::ld_shared_cluster_u32(ptx::mapa_shared(addr, c));
        unsigned int sum = 0;
#pragma unroll
        for (int c = 0; c < kSelCluster; ++c) sum += part[c];
        tot[tid] = sum;
      }
      __syncthreads();
      if (warp == 0) {
        // suffix scan over 8 bins per lane: the digit holding the need-th largest remaining key
        int c[8], local = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { c[i] = static_cast<int>(tot[8 * lane + i]); local += c[i]; }
        int incl = local;                                  // keys in the bins of lanes >= this lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += y;
        }
        const int above = incl - local;
        if (above < need && need <= incl) {
          int rem = need - above, d = 8 * lane, bc = 0;
#pragma unroll
          for (int i = 7; i >= 0; --i) {
            if (c[i] >= rem) { d = 8 * lane + i; bc = c[i]; break; }
            rem -= c[i];
          }
          sh_prefix = prefix | (static_cast<unsigned long long>(d) << shift);
          sh_need = rem;
          sh_binc = bc;
        }
      }
      __syncthreads();
      prefix = sh_prefix;
      need = sh_need;
      const bool whole_bin = shift > 0 && sh_binc == need;   // uniform over the cluster
      if (whole_bin || shift == 0) {
        T = prefix;
        if (whole_bin) need = p;                     // every key == T lies in the bin: take them all
        break;
      }
    }
  }

  // Per warp: keys > T and == T; per CTA: their sums, exchanged over the cluster.
  int gt = 0, eq = 0;
#pragma unroll
  for (int r = 0; r < kSelMaxR; ++r) {
    gt += __popc(__ballot_sync(0xffffffffu, valid[r] && key[r] > T));
    eq += __popc(__ballot_sync(0xffffffffu, valid[r] && key[r] == T));
  }
  if (lane == 0) { sh_wgt[warp] = gt; sh_weq[warp] = eq; }
  __syncthreads();
  if (tid == 0) {
    int cg = 0, ce = 0;
    for (int w = 0; w < kSelWarps; ++w) { cg += sh_wgt[w]; ce += sh_weq[w]; }
    sh_cnt[0] = cg;
    sh_cnt[1] = ce;
  }
  ptx::cluster_sync();                               // every CTA's counts are visible
  // Ties of lower-ranked CTAs and warps come first; a group with `e_before` ties before it and
  // g, e of its own takes g + clamp(need - e_before, 0, e) channels.
  int cta_g = 0, cta_e = 0;
  if (lane < kSelCluster) {
    const uint32_t base = ptx::smem_u32(&sh_cnt[0]);
    cta_g = static_cast<int>(ptx::ld_shared_cluster_u32(ptx::mapa_shared(base, lane)));
    cta_e = static_cast<int>(ptx::ld_shared_cluster_u32(ptx::mapa_shared(base + 4, lane)));
  }
  auto taken = [&](int g, int e, int e_before) { return g + min(max(need - e_before, 0), e); };
  int e_before = 0, out = 0;
  for (int c = 0; c < static_cast<int>(rank); ++c) {
    const int g = __shfl_sync(0xffffffffu, cta_g, c), e = __shfl_sync(0xffffffffu, cta_e, c);
    out += taken(g, e, e_before);
    e_before += e;
  }
  for (int w = 0; w < warp; ++w) {
    out += taken(sh_wgt[w], sh_weq[w], e_before);
    e_before += sh_weq[w];
  }
  // The warp's rounds in channel order: P entries, mask words, the unprotected maximum.
  uint32_t am_unprot = 0;
#pragma unroll
  for (int r = 0; r < kSelMaxR; ++r) {
    if (r < R) {                                      // uniform
      const uint32_t eqb = __ballot_sync(0xffffffffu, valid[r] && key[r] == T);
      const bool sel = valid[r] && (key[r] > T || (key[r] == T && e_before + __popc(eqb & lt) < need));
      const uint32_t selb = __ballot_sync(0xffffffffu, sel);
      const int j = j_warp + r * 32 + lane;
      const int slot = out + __popc(selb & lt);
      if (sel && slot < p) P[slot] = j;
      const int word = (j_warp + r * 32) >> 5;
      if (lane == 0 && word < words) mask[word] = selb;
      if (valid[r] && (!sel || (opts & FS_RESIDUAL))) am_unprot = max(am_unprot, am[r]);   // floats >= 0 order as uints
      out += __popc(selb);
      e_before += __popc(eqb);
    }
  }
  am_unprot = __reduce_max_sync(0xffffffffu, am_unprot);
  if (lane == 0) sh_wam[warp] = am_unprot;
  __syncthreads();
  if (tid == 0) {
    uint32_t m = 0;
    for (int w = 0; w < kSelWarps; ++w) m = max(m, sh_wam[w]);
    ptx::red_max_shared_cluster_u32(ptx::mapa_shared(ptx::smem_u32(&sh_am_cluster), 0), m);
  }
  ptx::cluster_sync();                               // the maxima have arrived; no CTA reads another's memory after this
  if (rank == 0 && tid == 0) {
    const float a = __uint_as_float(sh_am_cluster);
    gA_all[prob] = (opts & FS_GAIN_EXACT) ? gain_exact(a) : gain_pow2(a);
    if (reset) { n_all[prob] = 0; flags_all[prob] = 0; }   // every CTA read n before the first barrier
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
  const int R = static_cast<int>(ceil_div(K, kSelCluster * kSelThreads));   // 1..kSelMaxR
  select_topk_kernel<<<static_cast<unsigned>(nprob) * kSelCluster, kSelThreads, 0, s>>>(
      K, R, reinterpret_cast<long long*>(n), reinterpret_cast<long long*>(s1), reinterpret_cast<long long*>(s2), amax,
      flags, p, opts, P, mask, gA, reset);
  FS_CHECK_LAUNCH("fs_select_topk");
  return FS_OK;
}
