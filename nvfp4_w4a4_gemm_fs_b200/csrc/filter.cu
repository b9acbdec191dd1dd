// TIM-aware dual-gate sequence filter with advantage masking.
//
// FourSight §4.1 "The dual-gate mechanism": a token is a tail token when its training
// probability is at most tau; G1 drops a trajectory with at least K1 tail tokens, G2 one with
// at least K2 consecutive tail tokens (Eq. 3: keep iff count < K1 and run < K2).  Eq. 4 masks
// the advantage (A' = f A) and keeps the original 1/G loss denominator.  §2.1 gives the group
// advantage A = (r - mu) / sigma.
//
// One CTA per sequence, plus one warp that computes the group advantage meanwhile.  Each of the
// kFThreads scanning threads summarises a contiguous chunk of tokens as
// (length, count, leading run, trailing run, longest run); the summaries combine associatively
// in token order, first within a warp with shuffles, then across warps in shared memory.
#include "common.cuh"

namespace fs {
namespace {

constexpr int kFThreads = 256;

struct RunSum {
  int len, cnt, pre, suf, best;
};

__device__ __forceinline__ RunSum combine(const RunSum& a, const RunSum& b) {
  RunSum r;
  r.len = a.len + b.len;
  r.cnt = a.cnt + b.cnt;
  r.pre = (a.pre == a.len) ? a.len + b.pre : a.pre;
  r.suf = (b.suf == b.len) ? b.len + a.suf : b.suf;
  r.best = max(max(a.best, b.best), a.suf + b.pre);
  return r;
}

__device__ __forceinline__ void push(RunSum& s, bool tail) {
  // append one token to the right of s
  if (tail) {
    s.cnt += 1;
    if (s.pre == s.len) s.pre += 1;
    s.suf += 1;
    s.best = max(s.best, s.suf);
  } else {
    s.suf = 0;
  }
  s.len += 1;
}

__device__ __forceinline__ RunSum shfl_down(const RunSum& s, int o) {
  RunSum r;
  r.len = __shfl_down_sync(0xffffffffu, s.len, o);
  r.cnt = __shfl_down_sync(0xffffffffu, s.cnt, o);
  r.pre = __shfl_down_sync(0xffffffffu, s.pre, o);
  r.suf = __shfl_down_sync(0xffffffffu, s.suf, o);
  r.best = __shfl_down_sync(0xffffffffu, s.best, o);
  return r;
}

__global__ void __launch_bounds__(kFThreads + 32)
seq_filter_kernel(const float* __restrict__ logp, int64_t ld, const int32_t* __restrict__ lengths, int T,
                  float log_tau, int K1, int K2, int G, const float* __restrict__ rewards, float* adv,
                  uint8_t* keep, int32_t* tail_count, int32_t* max_run, bool vec_rows) {
  __shared__ RunSum sh[kFThreads / 32];
  __shared__ float sh_adv;
  const int s = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // The group advantage (§2.1) does not depend on the tokens: an extra warp computes it while the
  // kFThreads others scan (one thread, sequential float64 order, as the oracle sums).
  // Barrier 1 joins the scanning warps and, when it works, the extra warp (whole warps only).
  const uint32_t nbar = kFThreads + (rewards ? 32 : 0);
  auto bar_sync = [&]() { asm volatile("bar.sync 1, %0;" ::"r"(nbar) : "memory"); };
  if (warp == kFThreads / 32) {
    if (!rewards) return;                          // the whole warp: not counted in nbar
    if (lane == 0) {
      const int g0 = (s / G) * G;
      double sum = 0.0;
      for (int i = 0; i < G; ++i) sum = __dadd_rn(sum, static_cast<double>(__ldg(rewards + g0 + i)));
      const double mu = __ddiv_rn(sum, static_cast<double>(G));
      double q = 0.0;
      for (int i = 0; i < G; ++i) {
        const double d = __dsub_rn(static_cast<double>(__ldg(rewards + g0 + i)), mu);
        q = __dadd_rn(q, __dmul_rn(d, d));
      }
      const double sigma = __dsqrt_rn(__ddiv_rn(q, static_cast<double>(G)));
      float A = 0.0f;
      if (sigma > 0.0) A = __double2float_rn(__ddiv_rn(__dsub_rn(static_cast<double>(__ldg(rewards + s)), mu), sigma));
      sh_adv = A;
    }
    bar_sync();
    return;
  }
  int L = lengths ? __ldg(lengths + s) : T;
  L = L < 0 ? 0 : (L > T ? T : L);
  const float* row = logp + static_cast<int64_t>(s) * ld;
  // chunk of 4*per4 tokens per thread, contiguous, in thread order
  const int per4 = (L + 4 * kFThreads - 1) / (4 * kFThreads);
  const int t0 = tid * per4 * 4;
  RunSum acc{0, 0, 0, 0, 0};
  for (int c = 0; c < per4; ++c) {
    const int t = t0 + 4 * c;
    if (t >= L) break;
    float v[4];
    if (vec_rows && t + 4 <= L) {
      const float4 q = __ldg(reinterpret_cast<const float4*>(row + t));
      v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
      for (int j = 0; j < 4; ++j) v[j] = (t + j < L) ? __ldg(row + t + j) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (t + j < L) push(acc, !(v[j] > log_tau));     // logp <= log_tau, or NaN
  }
  // ordered reduction: lane i's segment precedes lane i+o's
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const RunSum other = shfl_down(acc, o);
    if (lane + o < 32 && (lane & (2 * o - 1)) == 0) acc = combine(acc, other);
  }
  if (lane == 0) sh[warp] = acc;
  bar_sync();
  if (tid == 0) {
    RunSum tot = sh[0];
    for (int w = 1; w < kFThreads / 32; ++w) tot = combine(tot, sh[w]);
    const int k = (tot.cnt < K1 && tot.best < K2) ? 1 : 0;
    keep[s] = static_cast<uint8_t>(k);
    tail_count[s] = tot.cnt;
    max_run[s] = tot.best;
    if (rewards) {
      adv[s] = k ? sh_adv : 0.0f;                  // written before the barrier above
    } else if (adv) {
      adv[s] = k ? adv[s] : 0.0f;
    }
  }
}

}  // namespace
}  // namespace fs

using namespace fs;

extern "C" fs_status fs_seq_filter(const float* logp, int64_t ld, const int32_t* lengths, int32_t S, int32_t T,
                                   float log_tau, int32_t K1, int32_t K2, int32_t G, const float* rewards,
                                   float* adv, uint8_t* keep, int32_t* tail_count, int32_t* max_run, void* stream) {
  if (S < 0 || T < 0 || K1 < 1 || K2 < 1) return fail(FS_ERR_INVALID_ARGUMENT, "fs_seq_filter: need S, T >= 0 and K1, K2 >= 1");
  if (S == 0) return FS_OK;
  if (ld < T) return fail(FS_ERR_INVALID_ARGUMENT, "fs_seq_filter: need ld >= T");
  if ((T > 0 && !logp) || !keep || !tail_count || !max_run) return fail(FS_ERR_INVALID_ARGUMENT, "fs_seq_filter: null pointer");
  if (logp && !aligned(logp, 4)) return fail(FS_ERR_INVALID_ARGUMENT, "fs_seq_filter: logp must be 4-byte aligned");
  const bool vec_rows = aligned(logp, 16) && ld % 4 == 0;   // float4 loads when every row is 16-byte aligned
  if (rewards) {
    if (!adv) return fail(FS_ERR_INVALID_ARGUMENT, "fs_seq_filter: rewards given without adv output");
    if (G < 1 || S % G != 0) return fail(FS_ERR_INVALID_ARGUMENT, "fs_seq_filter: need G >= 1 and S %% G == 0 with rewards");
  }
  seq_filter_kernel<<<S, kFThreads + 32, 0, static_cast<cudaStream_t>(stream)>>>(logp, ld, lengths, T, log_tau, K1, K2, G,
                                                                           rewards, adv, keep, tail_count, max_run, vec_rows);
  FS_CHECK_LAUNCH("fs_seq_filter");
  return FS_OK;
}
