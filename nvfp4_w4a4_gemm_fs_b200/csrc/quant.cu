// Activation preparation and weight pre-split.
//
// FourSight §5.1 "Data preparation": one pass over X in which each thread owns one 16-element
// NVFP4 block, zeroes the protected lanes with a precomputed register bitmask (Mask S->0),
// quantises the remaining lanes (FP4 Quant) and copies the protected lanes to the compact BF16
// side buffer X_S (Extract X_S).  The weights are pre-split the same way after each policy
// update into the NVFP4 pack of W_{~S} and W'_S = BF16(W_S / alpha) (Eq. 5).
//
// Block rule (FourSight §9.3.1 Eq. 9, with the fp32 operation order this library fixes):
//   a_b = max |x| over the block's unprotected lanes (all lanes in the residual form)
//   t   = fl32(fl32(a_b*g)/6);  sf = UE4M3_RNE_satfinite(t)
//   v   = fl32(fl32(x*g)/sf);   q  = E2M1_RNE_satfinite(v)   (sf == 0: q = +-0)
#include "common.cuh"

namespace fs {
namespace {

constexpr int kQThreads = 256;

enum class Side { Activation, Weight };

struct QuantArgs {
  const void* X;
  int64_t ldx;
  int K;
  int nb;             // K / 16
  int kb4;            // roundup(K/16, 4) / 4
  int p, pp;          // protected count, padded side columns
  uint32_t opts;
  const uint32_t* masks;     // [E][K/32] (E = 1 for the plain call); may be null when p == 0
  const float* gains;        // [E]
  const float* alpha;        // weight side only: alpha [1]
  uint8_t* q;                // [rows][K/2]
  uint8_t* sf;               // tiled
  uint16_t* side;            // [rows][pp]
  // row mapping
  int E;
  const int64_t* offsets;    // [E+1] device (grouped); null for the plain call
  int64_t rows;              // plain call: M
  int rows_per_cta;          // divides 128
};

template <typename T>
__device__ __forceinline__ void load_block(const T* src, float (&x)[16]) {
  if constexpr (sizeof(T) == 2) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) { x[2 * j] = bf16_lo(w[j]); x[2 * j + 1] = bf16_hi(w[j]); }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src) + j);
      x[4 * j] = v.x; x[4 * j + 1] = v.y; x[4 * j + 2] = v.z; x[4 * j + 3] = v.w;
    }
  }
}

// One CTA covers `rows_per_cta` consecutive packed rows, all inside one expert's padded region.
template <typename T, Side kSide, bool kGrouped>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(QuantArgs a) {
  __shared__ int sh_prefix[16384 / 32 + 1];       // protected channels before each mask word
  __shared__ int sh_expert;
  __shared__ int64_t sh_src_row0, sh_valid;        // source row of the CTA's first row, valid rows

  const int tid = threadIdx.x;
  const int64_t prow0 = static_cast<int64_t>(blockIdx.x) * a.rows_per_cta;   // first packed row

  // ---- locate the expert and the source rows -------------------------------------------
  if constexpr (kGrouped) {
    if (tid == 0) {
      int64_t pad = 0;
      int e = -1;
      int64_t src0 = 0, valid = 0;
      for (int i = 0; i < a.E; ++i) {
        const int64_t r0 = a.offsets[i], r1 = a.offsets[i + 1];
        const int64_t span = ((r1 - r0) + 127) / 128 * 128;
        if (prow0 < pad + span) {
          e = i;
          const int64_t local = prow0 - pad;
          src0 = r0 + local;
          valid = (r1 - r0) - local;
          break;
        }
        pad += span;
      }
      sh_expert = e;
      sh_src_row0 = src0;
      sh_valid = valid;
    }
    __syncthreads();
    if (sh_expert < 0) return;                 // beyond the last expert's padded region
  } else {
    if (tid == 0) {
      sh_expert = 0;
      sh_src_row0 = prow0;
      sh_valid = a.rows - prow0;
    }
    __syncthreads();
  }
  const int e = sh_expert;
  const int64_t src_row0 = sh_src_row0;
  const int64_t valid = sh_valid;               // rows of this CTA with data (may be <= 0)
  const int words = a.K / 32;
  const uint32_t* mask = (a.p > 0) ? a.masks + static_cast<int64_t>(e) * words : nullptr;

  // ---- protected-channel prefix counts per mask word (for the X_S column of a lane) -----
  if (a.p > 0) {
    if (tid < 32) {
      int carry = 0;
      for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + tid;
        const int c = (w < words) ? __popc(__ldg(mask + w)) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += y;
        }
        if (w < words) sh_prefix[w] = carry + incl - c;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    __syncthreads();
  }

  const float g = __ldg(a.gains + e);
  float alpha_v = 0.0f;
  if constexpr (kSide == Side::Weight) alpha_v = __ldg(a.alpha);
  const bool residual = a.opts & FS_RESIDUAL;
  const T* X = static_cast<const T*>(a.X);
  const int total = a.rows_per_cta * a.nb;

  for (int i0 = 0; i0 < total; i0 += kQThreads) {
    const int i = i0 + tid;
    const bool in_range = i < total;
    const int r = in_range ? i / a.nb : 0;
    const int b = in_range ? i % a.nb : 0;
    const int64_t prow = prow0 + r;
    const bool has_data = in_range && r < valid;
    uint32_t sfc = 0;
    if (has_data) {
      const int64_t srow = src_row0 + r;
      float x[16];
      load_block<T>(X + srow * a.ldx + static_cast<int64_t>(b) * 16, x);
      const uint32_t mbits = mask ? ((__ldg(mask + (b >> 1)) >> ((b & 1) * 16)) & 0xFFFFu) : 0u;
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const bool prot = (mbits >> j) & 1u;
        if (residual || !prot) amax = fmaxf(amax, fabsf(x[j]));
      }
      const float t = div_small_divisor(__fmul_rn(amax, g), kInvSix);
      sfc = ue4m3_rne(t);
      const double inv = sfc ? __drcp_rn(static_cast<double>(ue4m3_value(sfc))) : 0.0;
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float x0 = ((mbits >> j) & 1u) ? 0.0f : x[j];
        const float x1 = ((mbits >> (j + 1)) & 1u) ? 0.0f : x[j + 1];
        const float v0 = div_small_divisor(__fmul_rn(x0, g), inv);
        const float v1 = div_small_divisor(__fmul_rn(x1, g), inv);
        const uint32_t byte = e2m1x2(v0, v1);
        if (j < 8) lo |= byte << (j * 4); else hi |= byte << ((j - 8) * 4);
      }
      *reinterpret_cast<uint2*>(a.q + prow * (a.K / 2) + static_cast<int64_t>(b) * 8) = make_uint2(lo, hi);
      // Extract the protected lanes into the side buffer.
      if (mbits) {
        int col = sh_prefix[b >> 1] + ((b & 1) ? __popc(__ldg(mask + (b >> 1)) & 0xFFFFu) : 0);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if ((mbits >> j) & 1u) {
            uint16_t h;
            if constexpr (kSide == Side::Activation) {
              h = f32_to_bf16_bits(x[j]);
            } else {
              const float wb = __uint_as_float(static_cast<uint32_t>(f32_to_bf16_bits(x[j])) << 16);
              h = f32_to_bf16_bits(__fdiv_rn(wb, alpha_v));
            }
            a.side[prow * a.pp + col] = h;
            ++col;
          }
        }
      }
      if (b == 0)
        for (int c = a.p; c < a.pp; ++c) a.side[prow * a.pp + c] = 0;
    } else if (in_range && kGrouped) {
      // padding rows of a grouped buffer: zero codes and side columns
      *reinterpret_cast<uint2*>(a.q + prow * (a.K / 2) + static_cast<int64_t>(b) * 8) = make_uint2(0, 0);
      if (b == 0)
        for (int c = 0; c < a.pp; ++c) a.side[prow * a.pp + c] = 0;
    }
    // Gather the 4 scales of blocks b..b+3 (same row since K/16 % 4 == 0) into one word.
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sfc, 1);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sfc, 2);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sfc, 3);
    if (in_range && (b & 3) == 0)
      *reinterpret_cast<uint32_t*>(a.sf + sf_offset(prow, b, a.kb4)) = sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
}

// Max |W| over the unprotected columns (all columns in the residual form) as float bits.
template <typename T>
__global__ void __launch_bounds__(256) weight_amax_kernel(const T* __restrict__ W, int64_t N, int K, int64_t ldw,
                                                          const uint32_t* __restrict__ mask, uint32_t opts,
                                                          uint32_t* out_bits) {
  const bool residual = opts & FS_RESIDUAL;
  const int64_t total = N * (K / 16);
  float m = 0.0f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / (K / 16);
    const int b = static_cast<int>(i % (K / 16));
    float x[16];
    load_block<T>(W + r * ldw + static_cast<int64_t>(b) * 16, x);
    const uint32_t mbits = (mask && !residual) ? ((__ldg(mask + (b >> 1)) >> ((b & 1) * 16)) & 0xFFFFu) : 0u;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (!((mbits >> j) & 1u)) m = fmaxf(m, fabsf(x[j]));
  }
  uint32_t bits = __float_as_uint(m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bits = max(bits, __shfl_xor_sync(0xffffffffu, bits, o));
  if ((threadIdx.x & 31) == 0 && bits) atomicMax(out_bits, bits);
}

// gW from the reduced amax bits (stored in the gW slot), then alpha = fl32(1/fl32(gA*gW)).
__global__ void weight_gain_kernel(float* gW, float* alpha, const float* gA, uint32_t opts) {
  const float amax = __uint_as_float(*reinterpret_cast<uint32_t*>(gW));
  const float g = (opts & FS_GAIN_EXACT) ? gain_exact(amax) : gain_pow2(amax);
  *gW = g;
  *alpha = __fdiv_rn(1.0f, __fmul_rn(*gA, g));
}

template <Side kSide, bool kGrouped>
fs_status launch_quantize(int dtype, QuantArgs& a, int64_t padded_rows, cudaStream_t s) {
  // rows per CTA: a power of two dividing 128, so a CTA never straddles a 128-row tile
  int rpc = 1;
  while (rpc < 128 && rpc * a.nb < kQThreads) rpc *= 2;
  a.rows_per_cta = rpc;
  const int64_t ctas = ceil_div(padded_rows, rpc);
  if (ctas == 0) return FS_OK;
  if (ctas > 0x7FFFFFFF) return fail(FS_ERR_UNSUPPORTED, "too many rows");
  if (dtype == FS_DTYPE_BF16)
    quantize_kernel<uint16_t, kSide, kGrouped><<<static_cast<unsigned>(ctas), kQThreads, 0, s>>>(a);
  else
    quantize_kernel<float, kSide, kGrouped><<<static_cast<unsigned>(ctas), kQThreads, 0, s>>>(a);
  FS_CHECK_LAUNCH("quantize kernel");
  return FS_OK;
}

fs_status check_common(const char* who, int32_t dtype, int32_t K, int64_t ld, const void* X, int32_t p,
                       const uint32_t* mask, const void* gain, const uint8_t* q, const uint8_t* sf,
                       const uint16_t* side) {
  if (dtype != FS_DTYPE_BF16 && dtype != FS_DTYPE_F32) return fail(FS_ERR_INVALID_ARGUMENT, "%s: bad dtype %d", who, dtype);
  if (K <= 0 || K % 64 != 0 || K > 16384) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need K %% 64 == 0 and 0 < K <= 16384 (K=%d)", who, K);
  if (p < 0 || p > K || p > 256) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need 0 <= p <= min(K,256) (p=%d)", who, p);
  const int esz = dtype == FS_DTYPE_BF16 ? 2 : 4;
  if (ld < K || (ld * esz) % 16 != 0) return fail(FS_ERR_INVALID_ARGUMENT, "%s: leading dimension must be >= K with 16-byte rows", who);
  if (!X || !gain || !q || !sf || (p > 0 && (!mask || !side))) return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (!aligned(X, 16) || !aligned(q, 16) || !aligned(sf, 16) || (side && !aligned(side, 16)) || (mask && !aligned(mask, 4)))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: misaligned pointer", who);
  return FS_OK;
}

}  // namespace
}  // namespace fs

using namespace fs;

extern "C" fs_status fs_quantize_splice(const void* X, int32_t dtype, int64_t M, int32_t K, int64_t ldx,
                                        const uint32_t* mask, int32_t p, const float* gA, uint32_t opts,
                                        uint8_t* xq, uint8_t* sfx, uint16_t* xs, void* stream) {
  if (M < 0) return fail(FS_ERR_INVALID_ARGUMENT, "fs_quantize_splice: M < 0");
  if (M == 0) return FS_OK;
  fs_status st = check_common("fs_quantize_splice", dtype, K, ldx, X, p, mask, gA, xq, sfx, xs);
  if (st != FS_OK) return st;
  QuantArgs a{};
  a.X = X; a.ldx = ldx; a.K = K; a.nb = K / 16; a.kb4 = static_cast<int>(round_up(K / 16, 4) / 4);
  a.p = p; a.pp = side_cols(p); a.opts = opts; a.masks = mask; a.gains = gA; a.alpha = nullptr;
  a.q = xq; a.sf = sfx; a.side = xs; a.E = 1; a.offsets = nullptr; a.rows = M;
  return launch_quantize<Side::Activation, false>(dtype, a, round_up(M, 128), static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_quantize_splice_grouped(const void* X, int32_t dtype, int32_t E, const int64_t* row_offsets,
                                                int64_t max_rows, int32_t K, int64_t ldx, const uint32_t* masks,
                                                int32_t p, const float* gA, uint32_t opts, uint8_t* xq,
                                                uint8_t* sfx, uint16_t* xs, void* stream) {
  if (E <= 0 || E > 1024 || max_rows < 0 || !row_offsets) return fail(FS_ERR_INVALID_ARGUMENT, "fs_quantize_splice_grouped: need 0 < E <= 1024, max_rows >= 0, row_offsets");
  if (max_rows == 0) return FS_OK;
  fs_status st = check_common("fs_quantize_splice_grouped", dtype, K, ldx, X, p, masks, gA, xq, sfx, xs);
  if (st != FS_OK) return st;
  QuantArgs a{};
  a.X = X; a.ldx = ldx; a.K = K; a.nb = K / 16; a.kb4 = static_cast<int>(round_up(K / 16, 4) / 4);
  a.p = p; a.pp = side_cols(p); a.opts = opts; a.masks = masks; a.gains = gA; a.alpha = nullptr;
  a.q = xq; a.sf = sfx; a.side = xs; a.E = E; a.offsets = row_offsets; a.rows = 0;
  return launch_quantize<Side::Activation, true>(dtype, a, fs_grouped_rows(max_rows, E), static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_prepare_weights(const void* W, int32_t dtype, int32_t N, int32_t K, int64_t ldw,
                                        const uint32_t* mask, int32_t p, uint32_t opts, const float* gA,
                                        uint8_t* wq, uint8_t* sfw, uint16_t* ws, float* gW, float* alpha,
                                        void* stream) {
  if (N <= 0) return fail(FS_ERR_INVALID_ARGUMENT, "fs_prepare_weights: N must be >= 1");
  fs_status st = check_common("fs_prepare_weights", dtype, K, ldw, W, p, mask, gA, wq, sfw, ws);
  if (st != FS_OK) return st;
  if (!gW || !alpha) return fail(FS_ERR_INVALID_ARGUMENT, "fs_prepare_weights: null gW/alpha");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(gW, 0, sizeof(float), s);
  if (e != cudaSuccess) return cuda_status(e, "fs_prepare_weights: memset");
  const int64_t blocks = static_cast<int64_t>(N) * (K / 16);
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ceil_div(blocks, 256), 148 * 8));
  const uint32_t* m = p > 0 ? mask : nullptr;
  if (dtype == FS_DTYPE_BF16)
    weight_amax_kernel<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(W), N, K, ldw, m, opts, reinterpret_cast<uint32_t*>(gW));
  else
    weight_amax_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(W), N, K, ldw, m, opts, reinterpret_cast<uint32_t*>(gW));
  FS_CHECK_LAUNCH("fs_prepare_weights: amax");
  weight_gain_kernel<<<1, 1, 0, s>>>(gW, alpha, gA, opts);
  FS_CHECK_LAUNCH("fs_prepare_weights: gain");
  QuantArgs a{};
  a.X = W; a.ldx = ldw; a.K = K; a.nb = K / 16; a.kb4 = static_cast<int>(round_up(K / 16, 4) / 4);
  a.p = p; a.pp = side_cols(p); a.opts = opts; a.masks = mask; a.gains = gW; a.alpha = alpha;
  a.q = wq; a.sf = sfw; a.side = ws; a.E = 1; a.offsets = nullptr; a.rows = N;
  return launch_quantize<Side::Weight, false>(dtype, a, round_up(N, 128), s);
}
