// Training-side kernels around SpliceGEMM (FourSight §5.2 "System Implementation", §4.1 Eq. 4, §6.1).
//
// - fs_transpose_bf16: the operand transposes of the straight-through backward (dX = dY W and
//   dW = dY^T X run as K-major BF16 GEMMs on the tensor-core kernel).
// - fs_grpo_objective: Eq. 4's clipped surrogate with the filtered advantages A' = f A of the
//   dual-gate filter, the 1/|y_i| token weight and the ORIGINAL 1/G group denominator, fused with
//   its gradient with respect to the current policy's log-probs.
// - fs_k3_kl: the TIM metric of §6.1, sampled K3 estimates of KL(pi_rollout || pi_train) from the
//   rollout tokens: k3 = exp(d) - 1 - d with d = logp_train - logp_rollout.
// The per-sequence kernels use one CTA per sequence; sums run in a fixed order (thread chunk,
// warp tree, CTA tree), so results are reproducible run to run.
#include "common.cuh"

namespace fs {
namespace {

// ------------------------------------------------------------------------------------------ transpose
constexpr int kTile = 64;

// dst[c][r] = src[r][c] for a 64 x 64 tile per CTA: 16-byte loads along src rows into shared
// memory, 16-byte stores along dst rows.  Rows of the tile are padded to 66 elements (33 words):
// the load phase's writes are then free of bank conflicts (4-way unpadded) and the store phase's
// column reads (8 threads 8 rows apart) at most 2-way (8-way unpadded; rows 4 x 8 apart share a bank).
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t* __restrict__ src, int64_t lds, uint16_t* dst,
                                                             int64_t ldd, int64_t R, int64_t C, bool vec) {
  __shared__ uint16_t tile[kTile][kTile + 2];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTile, c0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int t = threadIdx.x;
  // load: 64 rows x 8 chunks of 8 elements; thread t takes chunk t % 8 of rows t / 8 and t / 8 + 32
  for (int rr = t >> 3; rr < kTile; rr += 32) {
    const int cc = (t & 7) * 8;
    const int64_t r = r0 + rr, c = c0 + cc;
    uint16_t v[8];
    if (vec && r < R && c + 8 <= C) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(src + r * lds + c));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) { v[2 * j] = w[j] & 0xFFFFu; v[2 * j + 1] = w[j] >> 16; }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (r < R && c + j < C) ? __ldg(src + r * lds + c + j) : 0;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) tile[rr][cc + j] = v[j];
  }
  __syncthreads();
  for (int cc = t >> 3; cc < kTile; cc += 32) {
    const int rr = (t & 7) * 8;
    const int64_t c = c0 + cc, r = r0 + rr;
    if (c >= C) continue;
    uint16_t v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = tile[rr + j][cc];
    if (vec && r + 8 <= R) {
      uint4 q;
      q.x = v[0] | (static_cast<uint32_t>(v[1]) << 16); q.y = v[2] | (static_cast<uint32_t>(v[3]) << 16);
      q.z = v[4] | (static_cast<uint32_t>(v[5]) << 16); q.w = v[6] | (static_cast<uint32_t>(v[7]) << 16);
      *reinterpret_cast<uint4*>(dst + c * ldd + r) = q;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (r + j < R) dst[c * ldd + r + j] = v[j];
    }
  }
}

// ------------------------------------------------------------------------------------------ per sequence
constexpr int kSThreads = 256;

// Block-wide sum in a fixed order: each thread's partial, then a warp tree, then warp 0 over the
// warps' partials.  Returns the total in thread 0.
__device__ __forceinline__ double block_sum(double v, double* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < kSThreads / 32; ++w) t += sh[w];
  __syncthreads();
  return t;
}

// Eq. 4 per token: rho = exp(logp - logp_old); l = min(rho A, clip(rho, 1-eps, 1+eps) A); the
// gradient of l with respect to logp is rho A when the unclipped term is the minimum, else 0.
__global__ void __launch_bounds__(kSThreads)
grpo_objective_kernel(const float* __restrict__ logp, const float* __restrict__ logp_old, int64_t ld,
                      const int32_t* __restrict__ lengths, int T, int S, const float* __restrict__ adv, float eps,
                      float* seq_obj, float* grad, int64_t ldg) {
  __shared__ double sh[kSThreads / 32];
  const int s = blockIdx.x;
  int L = lengths ? __ldg(lengths + s) : T;
  L = L < 0 ? 0 : (L > T ? T : L);
  const float A = __ldg(adv + s);
  const float* lp = logp + static_cast<int64_t>(s) * ld;
  const float* lo = logp_old + static_cast<int64_t>(s) * ld;
  float* gr = grad ? grad + static_cast<int64_t>(s) * ldg : nullptr;
  // the token weight of Eq. 4 with the group denominator folded over all S sequences: J is the
  // mean over sequences of (1/|y_i|) sum_t l_it, so dJ/dlogp_it = rho A / (S |y_i|) on the active branch
  const float wtok = L > 0 ? __fdiv_rn(1.0f, static_cast<float>(L)) : 0.0f;
  const float wgrad = L > 0 ? __fdiv_rn(wtok, static_cast<float>(S)) : 0.0f;
  const float lo_c = 1.0f - eps, hi_c = 1.0f + eps;
  double part = 0.0;
  for (int t = threadIdx.x; t < T; t += kSThreads) {
    float g = 0.0f;
    if (t < L) {
      const float rho = expf(__fsub_rn(__ldg(lp + t), __ldg(lo + t)));
      const float unc = __fmul_rn(rho, A);
      const float clp = __fmul_rn(fminf(fmaxf(rho, lo_c), hi_c), A);
      const bool unclipped = unc <= clp;
      part += static_cast<double>(unclipped ? unc : clp);
      g = unclipped ? __fmul_rn(unc, wgrad) : 0.0f;
    }
    if (gr) gr[t] = g;
  }
  const double tot = block_sum(part, sh);
  if (threadIdx.x == 0) seq_obj[s] = __double2float_rn(tot * static_cast<double>(wtok));
}

// k3(d) = exp(d) - 1 - d >= 0.  For |d| < 1/16 the cancellation is avoided with the Taylor series
// of exp about 0 (terms to d^7; the first omitted term is below 2^-30 of the result); otherwise
// expm1f(d) - d.
__device__ __forceinline__ float k3_of(float d) {
  if (fabsf(d) < 0.0625f) {
    // d^2/2 (1 + d/3 (1 + d/4 (1 + d/5 (1 + d/6 (1 + d/7)))))
    float p = __fmaf_rn(d, 1.0f / 7.0f, 1.0f);
    p = __fmaf_rn(d * (1.0f / 6.0f), p, 1.0f);
    p = __fmaf_rn(d * (1.0f / 5.0f), p, 1.0f);
    p = __fmaf_rn(d * (1.0f / 4.0f), p, 1.0f);
    p = __fmaf_rn(d * (1.0f / 3.0f), p, 1.0f);
    return 0.5f * d * d * p;
  }
  return expm1f(d) - d;
}

__global__ void __launch_bounds__(kSThreads)
k3_kl_kernel(const float* __restrict__ logp_train, const float* __restrict__ logp_roll, int64_t ld,
             const int32_t* __restrict__ lengths, int T, float* seq_k3, double* seq_sum, bool vec) {
  __shared__ double sh[kSThreads / 32];
  const int s = blockIdx.x;
  int L = lengths ? __ldg(lengths + s) : T;
  L = L < 0 ? 0 : (L > T ? T : L);
  const float* a = logp_train + static_cast<int64_t>(s) * ld;
  const float* b = logp_roll + static_cast<int64_t>(s) * ld;
  // per-thread partials in float over 4 tokens at a time (16-byte loads of both rows when the rows
  // are 16-byte aligned), accumulated into a double per group of four
  double part = 0.0;
  int t0 = 0;
  if (vec) {
    const int L4 = L & ~3;
    for (int t = 4 * threadIdx.x; t < L4; t += 4 * kSThreads) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(a + t));
      const float4 y = __ldg(reinterpret_cast<const float4*>(b + t));
      const float q = (k3_of(__fsub_rn(x.x, y.x)) + k3_of(__fsub_rn(x.y, y.y))) +
                      (k3_of(__fsub_rn(x.z, y.z)) + k3_of(__fsub_rn(x.w, y.w)));
      part += static_cast<double>(q);
    }
    t0 = L4;
  }
  for (int t = t0 + threadIdx.x; t < L; t += kSThreads) part += static_cast<double>(k3_of(__fsub_rn(__ldg(a + t), __ldg(b + t))));
  const double tot = block_sum(part, sh);
  if (threadIdx.x == 0) {
    seq_k3[s] = L > 0 ? __double2float_rn(tot / static_cast<double>(L)) : 0.0f;
    if (seq_sum) seq_sum[s] = tot;
  }
}

// Fixed-order batch reductions over the S per-sequence values (one CTA).
__global__ void __launch_bounds__(kSThreads) mean_of_seq_kernel(const float* seq_obj, int S, float* out) {
  __shared__ double sh[kSThreads / 32];
  double part = 0.0;
  for (int i = threadIdx.x; i < S; i += kSThreads) part += static_cast<double>(seq_obj[i]);
  const double tot = block_sum(part, sh);
  if (threadIdx.x == 0) *out = __double2float_rn(tot / static_cast<double>(S));
}

__global__ void __launch_bounds__(kSThreads)
k3_batch_kernel(const double* seq_sum, const int32_t* lengths, int S, int T, float* out) {
  __shared__ double sh[kSThreads / 32];
  double part = 0.0, cnt = 0.0;
  for (int i = threadIdx.x; i < S; i += kSThreads) {
    int L = lengths ? lengths[i] : T;
    L = L < 0 ? 0 : (L > T ? T : L);
    part += seq_sum[i];
    cnt += static_cast<double>(L);
  }
  const double tot = block_sum(part, sh);
  const double n = block_sum(cnt, sh);
  if (threadIdx.x == 0) *out = n > 0.0 ? __double2float_rn(tot / n) : 0.0f;
}

}  // namespace
}  // namespace fs

using namespace fs;

extern "C" fs_status fs_transpose_bf16(int64_t R, int64_t C, const uint16_t* src, int64_t lds, uint16_t* dst, int64_t ldd,
                                       void* stream) {
  if (R < 0 || C < 0 || lds < C || ldd < R) return fail(FS_ERR_INVALID_ARGUMENT, "fs_transpose_bf16: need R, C >= 0, lds >= C, ldd >= R");
  if (R == 0 || C == 0) return FS_OK;
  if (!src || !dst || !aligned(src, 2) || !aligned(dst, 2)) return fail(FS_ERR_INVALID_ARGUMENT, "fs_transpose_bf16: null or misaligned pointer");
  if (ceil_div(R, kTile) > 65535) return fail(FS_ERR_UNSUPPORTED, "fs_transpose_bf16: R too large");
  const bool vec = aligned(src, 16) && aligned(dst, 16) && lds % 8 == 0 && ldd % 8 == 0;
  dim3 grid(static_cast<unsigned>(ceil_div(C, kTile)), static_cast<unsigned>(ceil_div(R, kTile)));
  transpose_bf16_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(src, lds, dst, ldd, R, C, vec);
  FS_CHECK_LAUNCH("fs_transpose_bf16");
  return FS_OK;
}

extern "C" fs_status fs_grpo_objective(const float* logp, const float* logp_old, int64_t ld, const int32_t* lengths,
                                       int32_t S, int32_t T, const float* adv, float eps, float* seq_obj, float* J,
                                       float* grad, int64_t ldg, void* stream) {
  const char* who = "fs_grpo_objective";
  if (S < 0 || T < 0 || ld < T || !(eps >= 0.0f) || !(eps < 1.0f))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: need S, T >= 0, ld >= T and 0 <= eps < 1", who);
  if (S == 0) return FS_OK;
  if ((T > 0 && (!logp || !logp_old)) || !adv || !seq_obj) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (grad && ldg < T) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need ldg >= T", who);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  grpo_objective_kernel<<<S, kSThreads, 0, s>>>(logp, logp_old, ld, lengths, T, S, adv, eps, seq_obj, grad, ldg);
  FS_CHECK_LAUNCH(who);
  if (J) {
    mean_of_seq_kernel<<<1, kSThreads, 0, s>>>(seq_obj, S, J);
    FS_CHECK_LAUNCH(who);
  }
  return FS_OK;
}

extern "C" int64_t fs_k3_work_bytes(int32_t S) { return S < 0 ? 0 : static_cast<int64_t>(S) * 8; }

extern "C" fs_status fs_k3_kl(const float* logp_train, const float* logp_roll, int64_t ld, const int32_t* lengths,
                              int32_t S, int32_t T, float* seq_k3, float* batch_k3, void* work, void* stream) {
  const char* who = "fs_k3_kl";
  if (S < 0 || T < 0 || ld < T) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need S, T >= 0 and ld >= T", who);
  if (S == 0) return FS_OK;
  if ((T > 0 && (!logp_train || !logp_roll)) || !seq_k3 || (batch_k3 && !work))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (work && !aligned(work, 8)) return fail(FS_ERR_INVALID_ARGUMENT, "%s: work must be 8-byte aligned", who);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* sums = static_cast<double*>(work);      // per-sequence sums for the batch mean (may be null)
  const bool vec = aligned(logp_train, 16) && aligned(logp_roll, 16) && ld % 4 == 0;
  k3_kl_kernel<<<S, kSThreads, 0, s>>>(logp_train, logp_roll, ld, lengths, T, seq_k3, sums, vec);
  FS_CHECK_LAUNCH(who);
  if (batch_k3) {
    k3_batch_kernel<<<1, kSThreads, 0, s>>>(sums, lengths, S, T, batch_k3);
    FS_CHECK_LAUNCH(who);
  }
  return FS_OK;
}
