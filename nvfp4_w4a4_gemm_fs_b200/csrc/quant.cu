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
#include "moments.cuh"

namespace fs {

// Row-streaming quantiser (quant_stats.cu) used for bf16 batches of at most kSmallBatchRows rows.
constexpr int64_t kSmallBatchRows = 64;
fs_status quantize_rows_bf16(const void* X, int64_t M, int32_t K, int64_t ldx, const uint32_t* mask, int32_t p,
                             const float* gA, uint32_t opts, uint8_t* xq, uint8_t* sfx, uint16_t* xs, cudaStream_t s);

namespace {

constexpr int kQThreads = 256;
#ifndef FS_Q_PASS_ROWS
#define FS_Q_PASS_ROWS 4
#endif

enum class Side { Activation, Weight };

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

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

// Raw 16-element block as loaded: bf16 pairs packed in 8 words (widened on use) or 16 floats.
template <typename T>
struct RawBlock {
  static constexpr int kWords = sizeof(T) == 2 ? 8 : 16;
  uint32_t w[kWords];
  __device__ __forceinline__ float get(int j) const {
    if constexpr (sizeof(T) == 2) return (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
    else return __uint_as_float(w[j]);
  }
  // The block with the lanes whose bit is set in `mbits` replaced by +0.
  __device__ __forceinline__ RawBlock masked(uint32_t mbits) const {
    RawBlock m;
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t two = (mbits >> (2 * j)) & 3u;                        // lanes 2j, 2j+1
        const uint32_t kill = ((two & 1u) | ((two & 2u) << 15)) * 0xFFFFu;   // 16-bit fields to clear
        m.w[j] = w[j] & ~kill;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) m.w[j] = ((mbits >> j) & 1u) ? 0u : w[j];
    }
    return m;
  }
};

template <typename T>
__device__ __forceinline__ void load_raw(const T* src, RawBlock<T>& x) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int v = 0; v < RawBlock<T>::kWords / 4; ++v) {
    const uint4 q = __ldg(p + v);
    x.w[4 * v] = q.x; x.w[4 * v + 1] = q.y; x.w[4 * v + 2] = q.z; x.w[4 * v + 3] = q.w;
  }
}

constexpr int kMaxGroupedExperts = 256;

// Where a chunk of `rows_per_cta` packed rows lives: its expert, first source row and how many
// of its rows carry data (the rest are padding of the expert's 128-row-aligned region).
struct ChunkLoc {
  int e;              // -1: past the last expert (or past the padded rows)
  int64_t prow0;      // first packed row
  int64_t src_row0;   // first source row of X
  int64_t valid;      // rows of the chunk with data (may be <= 0)
};

// Persistent CTAs loop over chunks of `rows_per_cta` packed rows; a chunk never straddles an
// expert's padded region (rows_per_cta divides 128).  Each thread owns one 16-element block per
// pass; the load of the next pass (or of the next chunk) is issued before the current block is
// computed, so every thread keeps a load in flight.  Divisions by the UE4M3 scale use per-code
// tables of the scale value and its reciprocal in shared memory; for bf16 input under a
// power-of-two gain the division is replaced by one multiply and a 12-bit snap (snap12), which
// yields the same codes.
template <typename T, Side kSide, bool kGrouped, bool kRowPasses>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(QuantArgs a, int64_t nchunks) {
  __shared__ uint16_t sh_mbits[16384 / 16];             // protected lanes of each 16-element block
  __shared__ uint4 sh_kill[sizeof(T) == 2 ? 2 * 16384 / 16 : 1];   // bf16: per block, 8 words of lanes to clear
  __shared__ uint16_t sh_col[16384 / 16];               // side-buffer column of each block's first protected lane
  __shared__ uint16_t sh_pidx[256];                     // channel of each side-buffer column (p <= 256)
  __shared__ float sh_val[128], sh_rcp[128];            // UE4M3 value and RN(1/value) per code
  __shared__ int sh_wsum[kQThreads / 32];               // per-warp totals of the mask scan
  __shared__ int64_t sh_pad[kGrouped ? kMaxGroupedExperts + 1 : 1];   // padded start of each expert
  __shared__ int64_t sh_off[kGrouped ? kMaxGroupedExperts + 1 : 1];   // row offsets of the experts

  const int tid = threadIdx.x;
  if (tid < 128) {
    // code 0 (zero scale) and the unused NaN code: d = 1, r = 0 gives +-0 with the sign of x
    const bool real = tid > 0 && tid < 127;
    const float d = real ? ue4m3_value(tid) : 1.0f;
    sh_val[tid] = d;
    sh_rcp[tid] = real ? __frcp_rn(d) : 0.0f;
  }
  if constexpr (kGrouped) {
    if (tid == 0) {
      sh_pad[0] = 0;
      for (int i = 0; i < a.E; ++i) {
        sh_off[i] = a.offsets[i];
        sh_pad[i + 1] = sh_pad[i] + (a.offsets[i + 1] - a.offsets[i] + 127) / 128 * 128;
      }
      sh_off[a.E] = a.offsets[a.E];
    }
  }
  __syncthreads();
  auto locate = [&](int64_t chunk) {
    ChunkLoc L;
    L.prow0 = chunk * a.rows_per_cta;
    if (chunk >= nchunks) { L.e = -1; L.src_row0 = 0; L.valid = 0; return L; }
    if constexpr (kGrouped) {
      if (L.prow0 >= sh_pad[a.E]) { L.e = -1; L.src_row0 = 0; L.valid = 0; return L; }
      int lo = 0, hi = a.E - 1;                   // expert with pad[e] <= prow0 < pad[e+1]
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sh_pad[mid] <= L.prow0) lo = mid; else hi = mid - 1;
      }
      L.e = lo;
      const int64_t local = L.prow0 - sh_pad[lo];
      L.src_row0 = sh_off[lo] + local;
      L.valid = (sh_off[lo + 1] - sh_off[lo]) - local;
    } else {
      L.e = 0;
      L.src_row0 = L.prow0;
      L.valid = a.rows - L.prow0;
    }
    return L;
  };

  const int words = a.K / 32;
  const bool residual = a.opts & FS_RESIDUAL;
  const T* X = static_cast<const T*>(a.X);
  const int total = a.rows_per_cta * a.nb;            // blocks per chunk
  float alpha_v = 0.0f;
  if constexpr (kSide == Side::Weight) alpha_v = __ldg(a.alpha);
  const float inv6 = __frcp_rn(6.0f);

  // General chunks: block i of the chunk is (row i / nb, block i % nb), the quotient taken as
  // trunc((i + 1/2) / nb) in fp32: i < 2^19 and nb <= 1024, so (i + 1/2) / nb lies at least 1/(2 nb)
  // from every integer while the fp32 product errs by under 2^-23 of it, and the result is exact.
  // kRowPasses (nb a multiple of the CTA size): every pass covers kQThreads blocks of one row, its
  // row and first block kept incrementally, so a pass costs no division and its row addresses
  // are uniform.
  const float inv_nb = 1.0f / static_cast<float>(a.nb);
  auto row_of = [&](int i) { return static_cast<int>((static_cast<float>(i) + 0.5f) * inv_nb); };
  auto load_one = [&](const ChunkLoc& L, int i0, RawBlock<T>& x) {
    const int i = i0 + tid;
    const int r = row_of(i);
    if (L.e >= 0 && i < total && r < L.valid) {
      const int b = i - r * a.nb;
      load_raw<T>(X + (L.src_row0 + r) * a.ldx + static_cast<int64_t>(b) * 16, x);
    }
  };
  auto load_pass = [&](const ChunkLoc& L, int r, int b0, RawBlock<T>& x) {
    if (L.e >= 0 && r < L.valid) load_raw<T>(X + (L.src_row0 + r) * a.ldx + static_cast<int64_t>(b0 + tid) * 16, x);
  };

  // Chunks per CTA: grouped problems take a contiguous range (consecutive chunks mostly share an
  // expert, so the expert's mask tables are built once per range instead of once per chunk); the
  // plain call deals them round-robin (every wave of CTAs sweeps the matrix in order).
  int64_t c_first = blockIdx.x, c_end = nchunks, c_step = gridDim.x;
  if constexpr (kGrouped) {
    const int64_t per = (nchunks + gridDim.x - 1) / gridDim.x;
    c_first = static_cast<int64_t>(blockIdx.x) * per;
    c_end = c_first + per < nchunks ? c_first + per : nchunks;
    c_step = 1;
  }
  ChunkLoc L = locate(c_first < c_end ? c_first : nchunks);
  RawBlock<T> xc;
  if constexpr (kRowPasses) load_pass(L, 0, 0, xc);
  else load_one(L, 0, xc);
  int cur_e = -1;
  const uint32_t* mask = nullptr;
  float g = 1.0f;
  bool fast = false;                               // snap12 path (bf16 input, power-of-two gain)

  for (int64_t chunk = c_first; chunk < c_end && L.e >= 0; chunk += c_step) {
    if (L.e != cur_e) {                            // uniform across the CTA
      cur_e = L.e;
      mask = (a.p > 0) ? a.masks + static_cast<int64_t>(cur_e) * words : nullptr;
      g = __ldg(a.gains + cur_e);
      fast = sizeof(T) == 2 && pow2_gain_in_fast_range(g);
      if (a.p > 0) {
        __syncthreads();                           // previous expert's tables no longer read
        // per block: its 16 mask bits and the side column of its first protected lane
        // (protected channels before it).  Thread t takes the contiguous blocks
        // [t*per, t*per + per) (per <= 4 for K <= 16384): all mask words are loaded in one round
        // trip, then an exclusive scan of the per-thread counts over the CTA.
        const int nb = a.nb;
        const int per = (nb + kQThreads - 1) / kQThreads;
        const int bt0 = tid * per;
        uint32_t mbv[4];
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int b = bt0 + j;
          mbv[j] = (j < per && b < nb) ? ((__ldg(mask + (b >> 1)) >> ((b & 1) * 16)) & 0xFFFFu) : 0u;
          cnt += __popc(mbv[j]);
        }
        const int lane = tid & 31, wid = tid >> 5;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) sh_wsum[wid] = incl;
        __syncthreads();
        int col = incl - cnt;
        for (int w = 0; w < wid; ++w) col += sh_wsum[w];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int b = bt0 + j;
          if (j < per && b < nb) {
            sh_mbits[b] = static_cast<uint16_t>(mbv[j]);
            sh_col[b] = static_cast<uint16_t>(col);
            col += __popc(mbv[j]);
          }
        }
        __syncthreads();
        // channel of every side column: the protected channels in ascending order
        for (int b = tid; b < nb; b += kQThreads) {
          uint32_t mb = sh_mbits[b];
          int col = sh_col[b];
          while (mb) {
            const int j = __ffs(mb) - 1;
            mb &= mb - 1;
            sh_pidx[col++] = static_cast<uint16_t>(b * 16 + j);
          }
        }
        if constexpr (sizeof(T) == 2) {
          for (int b = tid; b < nb; b += kQThreads) {
            const uint32_t mb = sh_mbits[b];
            uint32_t k[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t two = (mb >> (2 * j)) & 3u;
              k[j] = ((two & 1u) | ((two & 2u) << 15)) * 0xFFFFu;
            }
            sh_kill[2 * b] = make_uint4(k[0], k[1], k[2], k[3]);
            sh_kill[2 * b + 1] = make_uint4(k[4], k[5], k[6], k[7]);
          }
        }
        __syncthreads();
      }
    }
    const ChunkLoc Ln = locate(chunk + c_step < c_end ? chunk + c_step : nchunks);
    int r_cur = 0, b_cur = 0;                      // kRowPasses: row and first block of this pass
    for (int i0 = 0; i0 < total; i0 += kQThreads) {
      RawBlock<T> xn;
      int r_nxt = r_cur, b_nxt = b_cur + kQThreads;
      if constexpr (kRowPasses) {
        if (b_nxt == a.nb) { b_nxt = 0; ++r_nxt; }
        if (i0 + kQThreads < total) load_pass(L, r_nxt, b_nxt, xn);   // prefetch the next pass
        else load_pass(Ln, 0, 0, xn);                                  // or the next chunk's first
      } else {
        if (i0 + kQThreads < total) load_one(L, i0 + kQThreads, xn);
        else load_one(Ln, 0, xn);
      }
      const RawBlock<T>& x = xc;
      int r, b;
      bool in_range;
      if constexpr (kRowPasses) {
        r = r_cur; b = b_cur + tid; in_range = true;
      } else {
        const int i = i0 + tid;
        in_range = i < total;
        r = in_range ? row_of(i) : 0;
        b = in_range ? i - r * a.nb : 0;
      }
      const int64_t prow = L.prow0 + r;
      const bool has_data = in_range && r < L.valid;
      uint32_t sfc = 0;
      if (has_data) {
        const uint32_t mbits = mask ? sh_mbits[b] : 0u;
        RawBlock<T> xm;
        if constexpr (sizeof(T) == 2) {
          if (mask) {                                // uniform: clear protected lanes, no branch per block
            const uint4 k0 = sh_kill[2 * b], k1 = sh_kill[2 * b + 1];
            xm.w[0] = x.w[0] & ~k0.x; xm.w[1] = x.w[1] & ~k0.y; xm.w[2] = x.w[2] & ~k0.z; xm.w[3] = x.w[3] & ~k0.w;
            xm.w[4] = x.w[4] & ~k1.x; xm.w[5] = x.w[5] & ~k1.y; xm.w[6] = x.w[6] & ~k1.z; xm.w[7] = x.w[7] & ~k1.w;
          } else {
            xm = x;
          }
        } else {
          xm = mbits ? x.masked(mbits) : x;
        }
        const RawBlock<T>& xs = residual ? x : xm;    // lanes that set the block scale
        float amax = 0.0f;
        if constexpr (sizeof(T) == 2) {
          // bf16: |x| orders like its low 15 bits, so the block maximum is a packed 16-bit max of
          // the magnitudes (finite inputs), shifted back into a float
          uint32_t m = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) m = vmax_u16x2(m, xs.w[j] & 0x7FFF7FFFu);
          amax = __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(xs.get(j)));
        }
        const float t = div_markstein(__fmul_rn(amax, g), 6.0f, inv6);
        sfc = ue4m3_rne(t);
        const float sd = sh_val[sfc], sr = sh_rcp[sfc];
        float v[16];
        if (fast) {
          const float R = __fmul_rn(g, sr);        // exact: g is a power of two in range
          if constexpr (sizeof(T) == 2) {
            // two elements per packed multiply (each lane the IEEE RN product of the scalar form)
            const uint64_t R2 = moments::pack_f32x2(R, R);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint64_t pr = moments::mul_f32x2(moments::pack_f32x2(bf16_lo(xm.w[j]), bf16_hi(xm.w[j])), R2);
              v[2 * j] = snap12(__uint_as_float(static_cast<uint32_t>(pr)));
              v[2 * j + 1] = snap12(__uint_as_float(static_cast<uint32_t>(pr >> 32)));
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = snap12(__fmul_rn(xm.get(j), R));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = div_markstein(__fmul_rn(xm.get(j), g), sd, sr);
        }
        const uint32_t lo = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
        const uint32_t hi = e2m1x8(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
        *reinterpret_cast<uint2*>(a.q + prow * (a.K / 2) + static_cast<int64_t>(b) * 8) = make_uint2(lo, hi);
      } else if (in_range && kGrouped) {
        // padding rows of a grouped buffer: zero codes (their side columns are zeroed below)
        *reinterpret_cast<uint2*>(a.q + prow * (a.K / 2) + static_cast<int64_t>(b) * 8) = make_uint2(0, 0);
      }
      // Gather the 4 scales of blocks b..b+3 (same row since K/16 % 4 == 0) into one word.
      const uint32_t s1 = __shfl_down_sync(0xffffffffu, sfc, 1);
      const uint32_t s2 = __shfl_down_sync(0xffffffffu, sfc, 2);
      const uint32_t s3 = __shfl_down_sync(0xffffffffu, sfc, 3);
      if (in_range && (b & 3) == 0)
        *reinterpret_cast<uint32_t*>(a.sf + sf_offset(prow, b, a.kb4)) = sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
      xc = xn;
      r_cur = r_nxt;
      b_cur = b_nxt;
    }
    // Extract X_S: side column c of each row is channel sh_pidx[c] (the block data is still in
    // L1/L2), zero in the padding columns p..pp-1 and in the padding rows of a grouped buffer.
    if (a.pp > 0) {
      for (int idx = tid; idx < a.rows_per_cta * a.pp; idx += kQThreads) {
        const int r = idx / a.pp;
        const int c = idx - r * a.pp;
        const bool data = r < L.valid;
        if (!data && !kGrouped) continue;
        uint16_t hv = 0;
        if (data && c < a.p) {
          const T* src = X + (L.src_row0 + r) * a.ldx + sh_pidx[c];
          float xv;
          if constexpr (sizeof(T) == 2) xv = __uint_as_float(static_cast<uint32_t>(__ldg(src)) << 16);
          else xv = __ldg(src);
          if constexpr (kSide == Side::Activation) {
            hv = f32_to_bf16_bits(xv);
          } else {
            const float wb = __uint_as_float(static_cast<uint32_t>(f32_to_bf16_bits(xv)) << 16);
            hv = f32_to_bf16_bits(__fdiv_rn(wb, alpha_v));
          }
        }
        a.side[(L.prow0 + r) * a.pp + c] = hv;
      }
    }
    L = Ln;
  }
}

// Compacted-K form (FS_COMPACT_K): the NVFP4 operand holds the unprotected channels in ascending
// order, so the 16-element blocks are re-formed over them, zero padded to Kc = roundup(K - p, 256)
// columns; the side buffer is the same as in the split form.  One thread per (row, compacted
// block): its 16 elements are gathered through a table of source channels built once per CTA by
// a block-wide scan of the mask.  Same block arithmetic as quantize_kernel.
template <typename T, Side kSide>
__global__ void __launch_bounds__(kQThreads) quantize_compact_kernel(QuantArgs a, int Kc, int64_t rows_padded) {
  __shared__ uint16_t sh_src[16384];                  // source channel of compacted column j
  __shared__ uint16_t sh_pidx[256];                   // protected channels, ascending
  __shared__ int sh_scan[kQThreads / 32][2];
  __shared__ float sh_val[128], sh_rcp[128];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 128) {
    const bool real = tid > 0 && tid < 127;
    const float d = real ? ue4m3_value(tid) : 1.0f;
    sh_val[tid] = d;
    sh_rcp[tid] = real ? __frcp_rn(d) : 0.0f;
  }
  // channel lists: thread t scans channels [t*per, (t+1)*per); exclusive scans of both counts
  const int per = (a.K + kQThreads - 1) / kQThreads;
  const int c0 = tid * per, c1 = min(a.K, c0 + per);
  auto is_prot = [&](int ch) { return a.masks && ((__ldg(a.masks + (ch >> 5)) >> (ch & 31)) & 1u); };
  int nu = 0, np = 0;
  for (int ch = c0; ch < c1; ++ch) { if (is_prot(ch)) ++np; else ++nu; }
  int xu = nu, xp = np;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yu = __shfl_up_sync(0xffffffffu, xu, o), yp = __shfl_up_sync(0xffffffffu, xp, o);
    if (lane >= o) { xu += yu; xp += yp; }
  }
  if (lane == 31) { sh_scan[warp][0] = xu; sh_scan[warp][1] = xp; }
  __syncthreads();
  int bu = xu - nu, bp = xp - np;
  for (int w = 0; w < warp; ++w) { bu += sh_scan[w][0]; bp += sh_scan[w][1]; }
  for (int ch = c0; ch < c1; ++ch) {
    if (is_prot(ch)) { if (bp < 256) sh_pidx[bp] = static_cast<uint16_t>(ch); ++bp; }
    else sh_src[bu++] = static_cast<uint16_t>(ch);
  }
  __syncthreads();
  const int nkeep = a.K - a.p;
  const int nbc = Kc / 16;
  const T* X = static_cast<const T*>(a.X);
  const float g = __ldg(a.gains);
  const bool fast = sizeof(T) == 2 && pow2_gain_in_fast_range(g);
  const float inv6 = __frcp_rn(6.0f);
  const int64_t items = rows_padded * nbc;          // nbc % 4 == 0: a warp's aligned groups of 4 share a row
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * kQThreads; i0 < items; i0 += static_cast<int64_t>(gridDim.x) * kQThreads) {
    const int64_t i = i0 + tid;
    const bool in_range = i < items;
    const int64_t r = in_range ? i / nbc : 0;
    const int jb = in_range ? static_cast<int>(i - r * nbc) : 0;
    uint32_t sfc = 0;
    if (in_range && r < a.rows) {
      float x[16];
      const T* row = X + r * a.ldx;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int jc = jb * 16 + e;
        float v = 0.0f;
        if (jc < nkeep) {
          if constexpr (sizeof(T) == 2) v = __uint_as_float(static_cast<uint32_t>(__ldg(row + sh_src[jc])) << 16);
          else v = __ldg(row + sh_src[jc]);
        }
        x[e] = v;
      }
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[e]));
      const float t = div_markstein(__fmul_rn(amax, g), 6.0f, inv6);
      sfc = ue4m3_rne(t);
      const float sd = sh_val[sfc], sr = sh_rcp[sfc];
      float v[16];
      if (fast) {
        const float R = __fmul_rn(g, sr);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = snap12(__fmul_rn(x[e], R));
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = div_markstein(__fmul_rn(x[e], g), sd, sr);
      }
      const uint32_t lo = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
      const uint32_t hi = e2m1x8(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
      *reinterpret_cast<uint2*>(a.q + r * (Kc / 2) + static_cast<int64_t>(jb) * 8) = make_uint2(lo, hi);
    }
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sfc, 1);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sfc, 2);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sfc, 3);
    if (in_range && (jb & 3) == 0)
      *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, jb, a.kb4)) = sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
  // side columns (as in the split form): the protected channels in ascending order, zero padded
  if (a.pp > 0) {
    const float alpha_v = kSide == Side::Weight ? __ldg(a.alpha) : 1.0f;
    const int64_t sitems = a.rows * a.pp;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kQThreads + tid; i < sitems;
         i += static_cast<int64_t>(gridDim.x) * kQThreads) {
      const int64_t r = i / a.pp;
      const int c = static_cast<int>(i - r * a.pp);
      uint16_t hv = 0;
      if (c < a.p) {
        const T* src = X + r * a.ldx + sh_pidx[c];
        float xv;
        if constexpr (sizeof(T) == 2) xv = __uint_as_float(static_cast<uint32_t>(__ldg(src)) << 16);
        else xv = __ldg(src);
        if constexpr (kSide == Side::Activation) {
          hv = f32_to_bf16_bits(xv);
        } else {
          const float wb = __uint_as_float(static_cast<uint32_t>(f32_to_bf16_bits(xv)) << 16);
          hv = f32_to_bf16_bits(__fdiv_rn(wb, alpha_v));
        }
      }
      a.side[r * a.pp + c] = hv;
    }
  }
}

template <Side kSide>
fs_status launch_quantize_compact(int dtype, QuantArgs& a, cudaStream_t s) {
  const int Kc = static_cast<int>(round_up(a.K - a.p, 256));
  a.kb4 = Kc / 64;
  const int64_t rows_padded = round_up(a.rows, 128);
  const int64_t items = rows_padded * (Kc / 16);
  if (items == 0) return FS_OK;
  auto kernel = dtype == FS_DTYPE_BF16 ? quantize_compact_kernel<uint16_t, kSide> : quantize_compact_kernel<float, kSide>;
  const int64_t grid = std::min<int64_t>(ceil_div(items, kQThreads), static_cast<int64_t>(sm_count()) * 4);
  kernel<<<static_cast<unsigned>(grid), kQThreads, 0, s>>>(a, Kc, rows_padded);
  FS_CHECK_LAUNCH("quantize (compacted K)");
  return FS_OK;
}

// Max |W| over the unprotected columns (all columns in the residual form) as float bits.
// fp32 weights (small problems): one 16-element block per thread.
__global__ void __launch_bounds__(256) weight_amax_f32_kernel(const float* __restrict__ W, int64_t N, int K, int64_t ldw,
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
    load_block<float>(W + r * ldw + static_cast<int64_t>(b) * 16, x);
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

// bf16 weights: a streaming reduction over the whole matrix (the gain needs one maximum, so rows
// play no role): the work is the N x K/256 stripes of 256 columns, dealt round-robin to the
// warps, kAmaxDepth stripes (16-byte loads, lane l the 8 columns 8l..8l+7) in flight per warp.
// |w| of a bf16 value orders like its low 15 bits, so the maximum is taken on packed 16-bit
// halves (max.u16x2) after clearing sign bits and protected lanes; the result, shifted to the
// high half, is the float.  One atomic per CTA.
#ifndef FS_AMAX_DEPTH
#define FS_AMAX_DEPTH 8
#endif
constexpr int kAmaxDepth = FS_AMAX_DEPTH;
constexpr int kAmaxThreads = 256;

__global__ void __launch_bounds__(kAmaxThreads) weight_amax_bf16_kernel(const uint16_t* __restrict__ W, int64_t N,
                                                                        int K, int64_t ldw,
                                                                        const uint32_t* __restrict__ mask,
                                                                        uint32_t opts, uint32_t* out_bits) {
  __shared__ uint32_t sh_max[kAmaxThreads / 32];
  const bool use_mask = mask && !(opts & FS_RESIDUAL);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int stripes = K / 256;                 // K % 64 == 0; a ragged last stripe is handled below
  const int tail_cols = K - stripes * 256;
  uint32_t m = 0;
  // Clears the lanes of column c0..c0+7 that are protected, and every sign bit.
  auto keep = [&](int c0) -> uint4 {
    uint32_t k8 = 0;
    if (use_mask) k8 = (__ldg(mask + (c0 >> 5)) >> (c0 & 31)) & 0xFFu;
    uint4 r;
    uint32_t* rw = &r.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t two = (k8 >> (2 * j)) & 3u;
      rw[j] = 0x7FFF7FFFu & ~(((two & 1u) | ((two & 2u) << 15)) * 0xFFFFu);
    }
    return r;
  };
  auto fold = [&](const uint4& v, const uint4& k) {
    m = vmax_u16x2(m, v.x & k.x);
    m = vmax_u16x2(m, v.y & k.y);
    m = vmax_u16x2(m, v.z & k.z);
    m = vmax_u16x2(m, v.w & k.w);
  };
  if (stripes > 0) {
    // stripe u = r * stripes + s; this warp takes u = warp, warp + nwarps, ...
    int64_t r = warp / stripes;
    int s = static_cast<int>(warp - r * stripes);
    const int64_t dr = nwarps / stripes;
    const int ds = static_cast<int>(nwarps - dr * stripes);
    while (r < N) {
      uint4 v[kAmaxDepth];
      int c[kAmaxDepth];
#pragma unroll
      for (int d = 0; d < kAmaxDepth; ++d) {
        c[d] = 0;
        v[d] = make_uint4(0u, 0u, 0u, 0u);
        if (r < N) {
          c[d] = s * 256 + lane * 8;
          v[d] = __ldg(reinterpret_cast<const uint4*>(W + r * ldw + c[d]));
          r += dr;
          s += ds;
          if (s >= stripes) { s -= stripes; ++r; }
        }
      }
#pragma unroll
      for (int d = 0; d < kAmaxDepth; ++d) fold(v[d], keep(c[d]));
    }
  }
  if (tail_cols && lane * 8 < tail_cols) {
    const int c0 = stripes * 256 + lane * 8;
    for (int64_t r = warp; r < N; r += nwarps) fold(__ldg(reinterpret_cast<const uint4*>(W + r * ldw + c0)), keep(c0));
  }
  uint32_t bits = max(m & 0xFFFFu, m >> 16) << 16;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bits = max(bits, __shfl_xor_sync(0xffffffffu, bits, o));
  if (lane == 0) sh_max[threadIdx.x >> 5] = bits;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
#pragma unroll
    for (int w = 0; w < kAmaxThreads / 32; ++w) b = max(b, sh_max[w]);
    if (b) atomicMax(out_bits, b);
  }
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
  // rows per chunk: a power of two dividing 128, so a chunk never straddles a 128-row tile.  With
  // nb a multiple of the CTA size, 4 rows (4 or more passes) per chunk amortise the per-chunk work.
  const bool passes = a.nb % kQThreads == 0;
  int rpc = 1;
  if (passes) rpc = FS_Q_PASS_ROWS;
  else
    while (rpc < 128 && rpc * a.nb < kQThreads) rpc *= 2;
  a.rows_per_cta = rpc;
  const int64_t chunks = ceil_div(padded_rows, rpc);
  if (chunks == 0) return FS_OK;
  auto kernel = dtype == FS_DTYPE_BF16
                    ? (passes ? quantize_kernel<uint16_t, kSide, kGrouped, true> : quantize_kernel<uint16_t, kSide, kGrouped, false>)
                    : (passes ? quantize_kernel<float, kSide, kGrouped, true> : quantize_kernel<float, kSide, kGrouped, false>);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQThreads, 0) != cudaSuccess || per_sm < 1) per_sm = 2;
  const int64_t grid = std::min<int64_t>(chunks, static_cast<int64_t>(sm_count()) * per_sm);
  kernel<<<static_cast<unsigned>(grid), kQThreads, 0, s>>>(a, chunks);
  FS_CHECK_LAUNCH("quantize kernel");
  return FS_OK;
}

fs_status check_common(const char* who, int32_t dtype, int32_t K, int64_t ld, const void* X, int32_t p,
                       const uint32_t* mask, const void* gain, const uint8_t* q, const uint8_t* sf,
                       const uint16_t* side, uint32_t opts = 0) {
  if (dtype != FS_DTYPE_BF16 && dtype != FS_DTYPE_F32) return fail(FS_ERR_INVALID_ARGUMENT, "%s: bad dtype %d", who, dtype);
  if (K <= 0 || K % 64 != 0 || K > 16384) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need K %% 64 == 0 and 0 < K <= 16384 (K=%d)", who, K);
  if (p < 0 || p > K || p > 256) return fail(FS_ERR_INVALID_ARGUMENT, "%s: need 0 <= p <= min(K,256) (p=%d)", who, p);
  const int esz = dtype == FS_DTYPE_BF16 ? 2 : 4;
  if (ld < K || (ld * esz) % 16 != 0) return fail(FS_ERR_INVALID_ARGUMENT, "%s: leading dimension must be >= K with 16-byte rows", who);
  // a compacted operand of no columns (FS_COMPACT_K with p == K) has no codes or scales
  const bool need_q = !((opts & FS_COMPACT_K) && p == K);
  if (!X || !gain || (need_q && (!q || !sf)) || (p > 0 && (!mask || !side)))
    return fail(FS_ERR_INVALID_ARGUMENT, "%s: null pointer", who);
  if (!aligned(X, 16) || (q && !aligned(q, 16)) || (sf && !aligned(sf, 16)) || (side && !aligned(side, 16)) ||
      (mask && !aligned(mask, 4)))
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
  fs_status st = check_common("fs_quantize_splice", dtype, K, ldx, X, p, mask, gA, xq, sfx, xs, opts);
  if (st != FS_OK) return st;
  QuantArgs a{};
  a.X = X; a.ldx = ldx; a.K = K; a.nb = K / 16; a.kb4 = static_cast<int>(round_up(K / 16, 4) / 4);
  a.p = p; a.pp = side_cols(p); a.opts = opts; a.masks = mask; a.gains = gA; a.alpha = nullptr;
  a.q = xq; a.sf = sfx; a.side = xs; a.E = 1; a.offsets = nullptr; a.rows = M;
  if (opts & FS_COMPACT_K) {
    if (opts & FS_RESIDUAL) return fail(FS_ERR_INVALID_ARGUMENT, "fs_quantize_splice: FS_COMPACT_K excludes FS_RESIDUAL");
    return launch_quantize_compact<Side::Activation>(dtype, a, static_cast<cudaStream_t>(stream));
  }
  if (dtype == FS_DTYPE_BF16 && M <= kSmallBatchRows)       // decode-sized batches
    return quantize_rows_bf16(X, M, K, ldx, mask, p, gA, opts, xq, sfx, xs, static_cast<cudaStream_t>(stream));
  return launch_quantize<Side::Activation, false>(dtype, a, round_up(M, 128), static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_quantize_splice_grouped(const void* X, int32_t dtype, int32_t E, const int64_t* row_offsets,
                                                int64_t max_rows, int32_t K, int64_t ldx, const uint32_t* masks,
                                                int32_t p, const float* gA, uint32_t opts, uint8_t* xq,
                                                uint8_t* sfx, uint16_t* xs, void* stream) {
  if (E <= 0 || E > kMaxGroupedExperts || max_rows < 0 || !row_offsets)
    return fail(FS_ERR_INVALID_ARGUMENT, "fs_quantize_splice_grouped: need 0 < E <= %d, max_rows >= 0, row_offsets", kMaxGroupedExperts);
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
  fs_status st = check_common("fs_prepare_weights", dtype, K, ldw, W, p, mask, gA, wq, sfw, ws, opts);
  if (st != FS_OK) return st;
  if (!gW || !alpha) return fail(FS_ERR_INVALID_ARGUMENT, "fs_prepare_weights: null gW/alpha");
  if ((opts & FS_COMPACT_K) && (opts & FS_RESIDUAL))
    return fail(FS_ERR_INVALID_ARGUMENT, "fs_prepare_weights: FS_COMPACT_K excludes FS_RESIDUAL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(gW, 0, sizeof(float), s);
  if (e != cudaSuccess) return cuda_status(e, "fs_prepare_weights: memset");
  const uint32_t* m = p > 0 ? mask : nullptr;
  if (dtype == FS_DTYPE_BF16) {
    // one wave of resident CTAs, each warp with at least kAmaxDepth stripes
    static PerDevice<int> occ;
    int per_sm = 1;
    if (!occ.get(current_device(), &per_sm, [](int* v) {
          return cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, weight_amax_bf16_kernel, kAmaxThreads, 0) ==
                     cudaSuccess && *v >= 1;
        }))
      per_sm = 1;
    const int64_t work = static_cast<int64_t>(N) * std::max(1, K / 256);
    const unsigned grid = static_cast<unsigned>(std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(work, (kAmaxThreads / 32) * kAmaxDepth), static_cast<int64_t>(sm_count()) * per_sm)));
    weight_amax_bf16_kernel<<<grid, kAmaxThreads, 0, s>>>(static_cast<const uint16_t*>(W), N, K, ldw, m, opts, reinterpret_cast<uint32_t*>(gW));
  } else {
    const int64_t blocks = static_cast<int64_t>(N) * (K / 16);
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ceil_div(blocks, 256), 148 * 8));
    weight_amax_f32_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(W), N, K, ldw, m, opts, reinterpret_cast<uint32_t*>(gW));
  }
  FS_CHECK_LAUNCH("fs_prepare_weights: amax");
  weight_gain_kernel<<<1, 1, 0, s>>>(gW, alpha, gA, opts);
  FS_CHECK_LAUNCH("fs_prepare_weights: gain");
  QuantArgs a{};
  a.X = W; a.ldx = ldw; a.K = K; a.nb = K / 16; a.kb4 = static_cast<int>(round_up(K / 16, 4) / 4);
  a.p = p; a.pp = side_cols(p); a.opts = opts; a.masks = mask; a.gains = gW; a.alpha = alpha;
  a.q = wq; a.sf = sfw; a.side = ws; a.E = 1; a.offsets = nullptr; a.rows = N;
  if (opts & FS_COMPACT_K) return launch_quantize_compact<Side::Weight>(dtype, a, s);
  return launch_quantize<Side::Weight, false>(dtype, a, round_up(N, 128), s);
}
