// SpliceGEMM decode path (M <= 16 tokens) on the 5th-generation tensor cores.
//
// FourSight §5.1 "Dual-path execution": for small M the product is bound by streaming the packed
// weights once.  Here the weights are the MMA's 128-row A operand and the (at most 16) tokens its
// N = 16 B operand, so the block-scaled tcgen05 MMA (kind::mxf4nvf4) applies the UE4M3 scales in
// hardware and the SMs only move bytes.  To put every SM on the weight stream, the K range of
// each 128-row tile is split over the CTAs of a thread-block cluster (up to 8 along grid y); each
// CTA accumulates its part in TMEM, and the partials are summed in a fixed order through
// distributed shared memory, scaled by alpha once and stored.  The protected slice X_S W'_S^T
// (§4.2 Eq. 5) runs as BF16 MMAs (kind::f16) into the TMEM accumulator of the cluster's last CTA.
//   warp 0      TMA producer: per k-tile a 128 x 128-byte box of W and a 16 x 128-byte box of the
//               packed activations (rows past M read as zero), plus both tiles' scale atoms (bulk
//               copies); the BF16 side tiles use the same boxes, 64 bf16 wide
//   warp 1      TMEM allocation; one thread copies the scale atoms to TMEM (tcgen05.cp, ordered
//               before its MMAs) and issues the MMAs
//   warps 2..5  epilogue: TMEM -> shared-memory partial; after a cluster barrier each CTA sums a
//               contiguous share of the tile's outputs over all CTAs of the cluster, x alpha, store
// The kFuse form (fs_decode_splice_gemm) takes bf16 activations instead of packed ones: the
// producer loads only the weight side, and warps 2..5, before their epilogue, encode this CTA's K
// range of the tokens into each stage (Mask S->0, FP4 Quant, Extract X_S of §5.1 "Data
// preparation") and hand it to the MMA thread through a second per-stage barrier.
// The grouped form (mixture-of-experts projections, FS_PATH_DECODE on fs_splice_gemm_grouped)
// runs one 128-row weight tile of one expert per cluster: the expert's rows come from the device
// offsets after the programmatic-launch wait, its tokens from the first rows of its 128-row padded
// range of the grouped activations, its weights from rows e*N .. of the stacked operand; a cluster
// whose expert has no rows or more than 16 leaves before any copy.
// Every mbarrier wait is bounded; on expiry the kernel records a timeout in the error word and
// still reaches both cluster barriers and releases TMEM.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemm.cuh"
#include "moments.cuh"
#include "ptx.cuh"

namespace fs {
namespace {

constexpr int kDThreads = 192;
constexpr int kDRows = 128;          // weight rows per tile (MMA M)
constexpr int kDTok = 16;            // token columns (MMA N)
#ifndef FS_DEC_STAGES
#define FS_DEC_STAGES 3
#endif
#ifndef FS_DEC_CTAS_PER_SM
#define FS_DEC_CTAS_PER_SM 3
#endif
// Three stages of 22 KB (the partial sums reuse stage 0) let three CTAs share an SM, so the K
// split can be wider without a second wave; against four stages at two CTAs per SM this measured
// 14.9 -> 8.6 us for the 12288 x 4096 projection at M = 1.
constexpr int kDStages = FS_DEC_STAGES;
constexpr int kDCtasPerSm = FS_DEC_CTAS_PER_SM;   // residency the shared-memory budget allows
#ifndef FS_DEC_MAX_SPLIT
#define FS_DEC_MAX_SPLIT 8
#endif
constexpr int kDMaxSplit = FS_DEC_MAX_SPLIT;   // at most a portable cluster (8)
constexpr uint64_t kDDrainNs = 50000000ull;

struct DCfg {
  static constexpr int W_BYTES = kDRows * 128;      // 256 fp4 or 64 bf16 per row
  static constexpr int X_BYTES = kDTok * 128;
  static constexpr int SFW_BYTES = 2048;            // four 512-byte atoms, one per MMA
  static constexpr int SFX_BYTES = 2048;
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES + SFW_BYTES + SFX_BYTES;   // multiple of 1024
  static constexpr int RED_BYTES = kDRows * kDTok * 4;   // partial [token][row], in stage 0 after the MMAs
  static_assert(RED_BYTES <= STAGE_BYTES, "the partial fits in a stage");
  // full, empty, xfull per stage; acc_full; drain; the TMEM slot and abort flag; the protected
  // channel list of the fused activation preparation (at most 256 uint16); the UE4M3 value and
  // reciprocal tables of the preparation (128 floats each)
  static constexpr int BAR_BYTES = 8 * (3 * kDStages + 2);
  static constexpr int SMEM_BYTES = 1024 + kDStages * STAGE_BYTES + BAR_BYTES + 16 + 2 * 256 + 2 * 128 * 4;
  static constexpr int TMEM_COLS = 128;
  static constexpr int SF_COL = 32;                 // scale buffer b: SFA at SF_COL+32b, SFB at SF_COL+32b+16
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the 128-byte swizzle");
  static_assert(SF_COL + 64 <= TMEM_COLS, "TMEM budget");
};
// (+ 1 KB the hardware reserves per CTA)
static_assert(kDCtasPerSm * (DCfg::SMEM_BYTES + 1024) <= 233472, "CTAs per SM must fit the SM's shared memory");

struct DecTcParams {
  int M, N, KT, ST, kb4, kt_per, S;
  const uint8_t* sfw;
  const uint8_t* sfx;
  const float* alpha;
  Segments seg;
  void* Y;
  int64_t ldy;
  int out_bf16;
  uint32_t* err;
  uint64_t wait_ns;
  int no_copies;
  // fused activation preparation (the kFuse kernel): bf16 X [M][ldx], the protected set as a
  // bitmask of p channels, the frozen gain, the residual form
  const uint16_t* x;
  int64_t ldx;
  const uint32_t* mask;
  int p;
  const float* gA;
  int residual;
  // grouped (offsets != null): blockIdx.x = expert * n_tiles + tile; experts with 1..small_max rows
  const int64_t* offsets;
  int n_tiles, small_max;
};

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* err,
                                         uint64_t limit_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1;; ++i) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 0) {
      if (*abort_flag) return false;
      if (now_ns() - t0 > limit_ns) {
        if (err) atomicOr(err, ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = now_ns();
  while (!ptx::mbar_try_wait(bar, parity))
    if (now_ns() - t0 > limit_ns) return;
}

// Fused activation preparation (kFuse): §5.1 "Data preparation" for this CTA's K range of the (at
// most 16) token rows, written straight into the stage in the layout the TMA path would have
// loaded: the E2M1 codes of row r as the 128-byte row r of the X box (128-byte swizzle: 16-byte
// chunk c at position c ^ (r % 8)), the UE4M3 scales as bytes r*16 + (b % 4) of the b/4-th
// 512-byte atom, and for the side k-tiles the bf16 values of the protected channels.  The block
// rule is the library's (t = fl32(fl32(a_b g)/6), sf = UE4M3_RNE(t), v = fl32(fl32(x g)/sf),
// q = E2M1_RNE(v)), so the stage bytes equal those fs_quantize_splice writes and the product is
// bit-identical to the unfused call.
struct PrepBlock {
  uint32_t codes0, codes1;   // elements 0..7, 8..15
  uint32_t sfc;
};

__device__ __forceinline__ uint32_t dec_vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// One 16-element block: w = its 8 bf16 pairs (element 2j in the low half of w[j]), kb = its 16
// protected-lane bits.
// sf_val / sf_rcp: per UE4M3 code its value and RN(1 / value) (code 0 and the unused NaN code:
// 1 and 0, the zero-scale rule).
__device__ __forceinline__ PrepBlock prep_block(const uint32_t (&w)[8], uint32_t kb, bool residual, float g,
                                                bool fast, float inv6, const float* sf_val, const float* sf_rcp) {
  uint32_t xm[8];
  uint32_t m = 0;
  if (kb == 0) {                                   // no protected lane in the block (the common case)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      xm[j] = w[j];
      m = dec_vmax_u16x2(m, w[j] & 0x7FFF7FFFu);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t two = (kb >> (2 * j)) & 3u;
      const uint32_t kill = ((two & 1u) | ((two & 2u) << 15)) * 0xFFFFu;
      xm[j] = w[j] & ~kill;
      m = dec_vmax_u16x2(m, (residual ? w[j] : xm[j]) & 0x7FFF7FFFu);
    }
  }
  const uint32_t mb = max(m & 0xFFFFu, m >> 16);
  const float amax = __uint_as_float(mb << 16);
  PrepBlock out;
  out.sfc = ue4m3_rne(div_markstein(__fmul_rn(amax, g), 6.0f, inv6));
  const float sd = sf_val[out.sfc], sr = sf_rcp[out.sfc];
  float v[16];
  if (fast) {
    const float R = __fmul_rn(g, sr);              // exact: g is a power of two in range
    // two elements per packed multiply (each lane the IEEE RN product of the scalar form)
    const uint64_t R2 = moments::pack_f32x2(R, R);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint64_t pr = moments::mul_f32x2(moments::pack_f32x2(bf16_lo(xm[j]), bf16_hi(xm[j])), R2);
      v[2 * j] = snap12(__uint_as_float(static_cast<uint32_t>(pr)));
      v[2 * j + 1] = snap12(__uint_as_float(static_cast<uint32_t>(pr >> 32)));
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[2 * j] = div_markstein(__fmul_rn(bf16_lo(xm[j]), g), sd, sr);
      v[2 * j + 1] = div_markstein(__fmul_rn(bf16_hi(xm[j]), g), sd, sr);
    }
  }
  out.codes0 = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
  out.codes1 = e2m1x8(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
  return out;
}

template <bool kFuse>
__global__ void __launch_bounds__(kDThreads, kDCtasPerSm)
splice_gemm_decode_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                             const __grid_constant__ CUtensorMap tmWS, const __grid_constant__ CUtensorMap tmXS,
                             const DecTcParams p) {
  using C = DCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // The partial sums reuse stage 0: it is written only after every MMA (hence every stage's use)
  // has completed (acc_full), and every load this CTA issues is consumed by one of those MMAs.
  float* red = reinterpret_cast<float*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDStages * C::STAGE_BYTES);
  uint64_t* empty = full + kDStages;
  uint64_t* xfull = empty + kDStages;              // kFuse: the prepared X / SFX bytes are in the stage
  uint64_t* acc_full = xfull + kDStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint16_t* pidx = reinterpret_cast<uint16_t*>(tmem_slot + 4);   // kFuse: protected channels, ascending
  float* sf_val = reinterpret_cast<float*>(pidx + 256);          // kFuse: UE4M3 code -> value
  float* sf_rcp = sf_val + 128;                                   //        and RN(1 / value)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(ptx::cluster_ctarank());     // K split inside the tile's cluster
  // Output columns n0.. of the tile; its weight rows start at wrow0 (grouped: expert e's weights
  // are rows e*N .. e*N + N - 1 of the stacked operand).
  const int expert = p.offsets ? static_cast<int>(blockIdx.x) / p.n_tiles : 0;
  const int n0 = (static_cast<int>(blockIdx.x) - expert * (p.offsets ? p.n_tiles : 0)) * kDRows;
  const int wrow0 = expert * p.N + n0;
  const int kt0 = rank * p.kt_per;
  const int kt1 = kt0 + p.kt_per < p.KT ? kt0 + p.kt_per : p.KT;
  const int nf = kt1 - kt0;                                       // FP4 k-tiles of this CTA (>= 1)
  const int nk = nf + (rank == p.S - 1 ? p.ST : 0);              // + the BF16 side k-tiles
  auto W_at = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto X_at = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES; };
  auto SFW_at = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES + C::X_BYTES; };
  auto SFX_at = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES + C::X_BYTES + C::SFW_BYTES; };

  // Programmatic dependent launch: the next kernel may start its prologue now.  Pulling this
  // CTA's weight boxes into L2 is safe before the wait (an L2 prefetch only); every real load and
  // store comes after griddepcontrol.wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kDStages; ++s) {
      ptx::mbar_init(full + s, 1);
      ptx::mbar_init(empty + s, 1);
      ptx::mbar_init(xfull + s, 8 * p.M);          // the 8 M threads of the group preparing it
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tmW);
    if constexpr (!kFuse) ptx::prefetch_tensormap(&tmX);
    if (p.ST > 0) {
      ptx::prefetch_tensormap(&tmWS);
      if constexpr (!kFuse) ptx::prefetch_tensormap(&tmXS);
    }
    // (not in the fused form, whose preparing warps read X meanwhile: measured faster without it
    // at 16 tokens and equal at 1)
    // (nor in the grouped form, which learns only after the wait whether its expert is its own)
    if (!kFuse && !p.no_copies && !p.offsets)
      for (int kt = kt0; kt < kt1; ++kt) ptx::tma_prefetch_2d(&tmW, kt * 128, wrow0);
  }
  if (warp == 1) {
    ptx::tmem_alloc<1>(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish<1>();
  }
  if constexpr (kFuse) {
    if (threadIdx.x < 128) {
      const int c = threadIdx.x;
      const bool real = c > 0 && c < 127;
      const float d = real ? ue4m3_value(c) : 1.0f;
      sf_val[c] = d;
      sf_rcp[c] = real ? __frcp_rn(d) : 0.0f;
    }
    // The X rows M..15 and the scale bytes that no token row < M owns stay zero, as in a packed
    // buffer (and as the TMA path's out-of-range fill); the preparing warps rewrite the bytes of
    // rows 0..M-1 every k-tile.  X and SFX are adjacent in a stage: X_BYTES + SFW_BYTES lie
    // between them, so the two are cleared separately.
    constexpr int kX16 = C::X_BYTES / 16, kS16 = C::SFX_BYTES / 16;
    for (int i = threadIdx.x; i < kDStages * (kX16 + kS16); i += kDThreads) {
      const int s = i / (kX16 + kS16), o = i % (kX16 + kS16);
      uint8_t* dst = o < kX16 ? X_at(s) + 16 * o : SFX_at(s) + 16 * (o - kX16);
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    ptx::fence_proxy_async_smem();                 // visible to tcgen05.cp
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  // Token rows: the problem's M, or expert e's rows r0 .. r1 - 1 of the output, packed from row
  // xrow0 of the grouped activations (every expert's rows start at a 128-row boundary).  A cluster
  // whose expert has no rows, or more than small_max (the tensor-core kernel's), leaves at once:
  // all its CTAs decide alike and none has touched another's memory.
  int M = p.M;
  int64_t yrow0 = 0, xrow0 = 0;
  if (p.offsets) {
    const int64_t r0 = __ldg(p.offsets + expert), r1 = __ldg(p.offsets + expert + 1);
    if (r1 - r0 <= 0 || r1 - r0 > p.small_max) {
      ptx::tc_fence_before();
      __syncthreads();
      if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc<1>(tmem, C::TMEM_COLS);
      }
      return;
    }
    M = static_cast<int>(r1 - r0);
    yrow0 = r0;
    if (warp == 0) {
      int64_t pad = 0;
      for (int i = lane; i < expert; i += 32) {
        const int64_t n = __ldg(p.offsets + i + 1) - __ldg(p.offsets + i);
        pad += (n + 127) / 128 * 128;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) pad += __shfl_xor_sync(0xffffffffu, pad, o);
      xrow0 = pad;
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // (p.no_copies, the failure-detection test hook: nothing is issued; the MMA and epilogue
    // waits run out and every CTA still reaches both cluster barriers)
    if (lane == 0 && !p.no_copies) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      for (int i = 0; i < nk; ++i) {
        if (!wait_bar(empty + stage, phase ^ 1, abort_flag, p.err, p.wait_ns)) break;
        // (kFuse: the weight side only; the preparing warps fill X and SFX)
        if (i < nf) {
          const int kt = kt0 + i;
          ptx::mbar_arrive_expect_tx(full + stage, kFuse ? C::W_BYTES + C::SFW_BYTES : C::STAGE_BYTES);
          ptx::tma_load_2d(W_at(stage), &tmW, kt * 128, wrow0, full + stage);
          if constexpr (!kFuse) ptx::tma_load_2d(X_at(stage), &tmX, kt * 128, static_cast<int32_t>(xrow0), full + stage);
          ptx::bulk_load(SFW_at(stage), p.sfw + (static_cast<int64_t>(wrow0 / kDRows) * p.kb4 + kt * 4) * 512,
                         C::SFW_BYTES, full + stage);
          if constexpr (!kFuse)
            ptx::bulk_load(SFX_at(stage), p.sfx + ((xrow0 / kDRows) * p.kb4 + static_cast<int64_t>(kt) * 4) * 512,
                           C::SFX_BYTES, full + stage);
        } else {
          const int sk = i - nf;
          ptx::mbar_arrive_expect_tx(full + stage, kFuse ? C::W_BYTES : C::W_BYTES + C::X_BYTES);
          ptx::tma_load_2d(W_at(stage), &tmWS, sk * 64, wrow0, full + stage);
          if constexpr (!kFuse) ptx::tma_load_2d(X_at(stage), &tmXS, sk * 64, static_cast<int32_t>(xrow0), full + stage);
        }
        ++issued;
        if (++stage == kDStages) { stage = 0; phase ^= 1; }
      }
      {
        // Copies issued but possibly not landed: the last min(issued, stages) stages, drained
        // whether or not a wait has given up yet (another role may give up later, and the CTA
        // must not exit with a copy landing in its shared memory).  The waits replay the
        // (stage, parity) pairs the MMA waits on; on the normal path they are met before the
        // epilogue starts.
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < kDStages && i < issued; ++i) {
          if (--s < 0) { s = kDStages - 1; ph ^= 1; }
          drain_bar(full + s, ph, kDDrainNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ scale copies + MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_f4 = ptx::idesc_nvf4(kDRows, kDTok);
      constexpr uint32_t idesc_bf = ptx::idesc_bf16(kDRows, kDTok);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        if (!wait_bar(full + stage, phase, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
        if constexpr (kFuse)
          if (!wait_bar(xfull + stage, phase, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint64_t adesc = ptx::desc_kmajor_sw128(ptx::smem_u32(W_at(stage)));
        const uint64_t bdesc = ptx::desc_kmajor_sw128(ptx::smem_u32(X_at(stage)));
        if (i < nf) {
          const uint32_t sfa = tmem + C::SF_COL + 32 * (i & 1);
          const uint32_t sfb = sfa + 16;
          const uint32_t sw = ptx::smem_u32(SFW_at(stage)), sx = ptx::smem_u32(SFX_at(stage));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ptx::tc_cp_32x128b_warpx4(sfa + 4 * j, ptx::desc_sf_block(sw + 512 * j));
            ptx::tc_cp_32x128b_warpx4(sfb + 4 * j, ptx::desc_sf_block(sx + 512 * j));
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            ptx::tc_mma_nvf4<1>(tmem, adesc + 2 * j, bdesc + 2 * j, idesc_f4, sfa + 4 * j, sfb + 4 * j, (i | j) != 0);
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) ptx::tc_mma_bf16<1>(tmem, adesc + 2 * j, bdesc + 2 * j, idesc_bf, (i | j) != 0);
        }
        ptx::tc_commit<1>(empty + stage);
        if (++stage == kDStages) { stage = 0; phase ^= 1; }
      }
      if (ok) ptx::tc_commit<1>(acc_full);
      ptx::tc_commit<1>(drain);                    // every MMA issued above has completed
      drain_bar(drain, 0, p.wait_ns);
    }
  } else {
    if constexpr (kFuse) {
      // ---------------------------------------------------------------- activation preparation
      // The 128 threads form R = min(128 / (8 M), stages) groups of 8 M threads; group j prepares
      // the k-tiles j, j + R, j + 2R, ... of this CTA (FP4 first, then the side k-tiles), so a
      // small batch issues the loads of several k-tiles at once.  R <= stages keeps every parity
      // wait within one phase: a group reaches k-tile i (stage i % S) only after its k-tile
      // i - R passed its own wait, i.e. after the MMAs of k-tile i - R - S >= i - 2S were done,
      // and its first k-tile is j < S.  In a group, thread (r, c) takes token row r
      // and the 32 channels c*32 .. c*32+31 of each FP4 k-tile (two scale blocks, one mask word,
      // four 16-byte loads of X; the next k-tile's are issued right after the current one is handed
      // over) or the side columns c*8 .. c*8+7.
      __shared__ int warp_tot[4];
      const int t = threadIdx.x - 64;
      const int G = 8 * p.M, R = min(128 / G, kDStages);
      const int grp = t / G, r = (t - grp * G) >> 3, c = t & 7;
      const uint16_t* xrow = p.x + static_cast<int64_t>(grp < R ? r : 0) * p.ldx;
      const float g = __ldg(p.gA);
      const bool fast = pow2_gain_in_fast_range(g);
      const float inv6 = __frcp_rn(6.0f);
      const bool residual = p.residual != 0;
      // X loads of each group's first k-tile and the mask words of the channel list go out
      // together, so the list's scan waits for the same round trip as the first encode.
      uint4 cur[4];
      uint32_t mc = 0;
      auto load = [&](int kt, uint4 (&v)[4], uint32_t& mw) {
        const int ch = kt * 256 + c * 32;
        const uint4* src = reinterpret_cast<const uint4*>(xrow + ch);
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = __ldg(src + j);
        mw = p.p > 0 ? __ldg(p.mask + (ch >> 5)) : 0u;
      };
      if (grp < R && grp < nf) load(kt0 + grp, cur, mc);
      if (nk > nf) {
        // Protected channel list for the side k-tiles: the set bits of the mask in ascending
        // order, from contiguous word ranges per thread (up to 4 words kept in registers) and an
        // exclusive scan of their counts.
        pidx[t] = 0;
        pidx[t + 128] = 0;
        const int nw = p.KT * 8;
        const int per = (nw + 127) / 128;
        const int w0 = min(t * per, nw), w1 = min(w0 + per, nw);
        uint32_t mw4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) mw4[j] = w0 + j < w1 ? __ldg(p.mask + w0 + j) : 0u;
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) cnt += __popc(mw4[j]);
        for (int w = w0 + 4; w < w1; ++w) cnt += __popc(__ldg(p.mask + w));
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (lane == 31) warp_tot[warp - 2] = incl;
        ptx::named_bar_sync(1, 128);
        int pos = incl - cnt;
        for (int q = 0; q < warp - 2; ++q) pos += warp_tot[q];
        auto scatter = [&](uint32_t mw, int w) {
          while (mw) {
            const int b = __ffs(mw) - 1;
            mw &= mw - 1;
            if (pos < 256) pidx[pos] = static_cast<uint16_t>(w * 32 + b);
            ++pos;
          }
        };
#pragma unroll
        for (int j = 0; j < 4; ++j) scatter(mw4[j], w0 + j);   // words past w1 are zero
        for (int w = w0 + 4; w < w1; ++w) scatter(__ldg(p.mask + w), w);
        ptx::named_bar_sync(1, 128);
      }
      if (grp < R) {
        const int xoff = r * 128 + ((c ^ (r & 7)) << 4);   // 128-byte swizzle of the X box
        const int sfoff = 512 * (c >> 1) + r * 16 + ((2 * c) & 3);
        bool ok = true;
        for (int i = grp; i < nf; i += R) {
          const int stage = i % kDStages;
          const uint32_t phase = (i / kDStages) & 1;
          if (!wait_bar(empty + stage, phase ^ 1, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
          const uint32_t wa[8] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y, cur[1].z, cur[1].w};
          const uint32_t wb[8] = {cur[2].x, cur[2].y, cur[2].z, cur[2].w, cur[3].x, cur[3].y, cur[3].z, cur[3].w};
          const PrepBlock b0 = prep_block(wa, mc & 0xFFFFu, residual, g, fast, inv6, sf_val, sf_rcp);
          const PrepBlock b1 = prep_block(wb, mc >> 16, residual, g, fast, inv6, sf_val, sf_rcp);
          *reinterpret_cast<uint4*>(X_at(stage) + xoff) = make_uint4(b0.codes0, b0.codes1, b1.codes0, b1.codes1);
          *reinterpret_cast<uint16_t*>(SFX_at(stage) + sfoff) = static_cast<uint16_t>(b0.sfc | (b1.sfc << 8));
          ptx::fence_proxy_async_smem();           // generic writes -> the MMA's async reads
          ptx::mbar_arrive(xfull + stage);
          if (i + R < nf) load(kt0 + i + R, cur, mc);   // after the handover (it is a release)
        }
        // side k-tiles: the indices nf .. nk-1 that fall to this group
        for (int i = nf + ((grp - nf % R) % R + R) % R; ok && i < nk; i += R) {
          const int sk = i - nf;
          const int stage = i % kDStages;
          const uint32_t phase = (i / kDStages) & 1;
          if (!wait_bar(empty + stage, phase ^ 1, abort_flag, p.err, p.wait_ns)) break;
          uint32_t hv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int col = sk * 64 + c * 8 + e;
            hv[e] = col < p.p ? static_cast<uint32_t>(__ldg(xrow + pidx[col])) : 0u;
          }
          *reinterpret_cast<uint4*>(X_at(stage) + xoff) =
              make_uint4(hv[0] | (hv[1] << 16), hv[2] | (hv[3] << 16), hv[4] | (hv[5] << 16), hv[6] | (hv[7] << 16));
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(xfull + stage);
        }
      }
    }
    // ------------------------------------------------------------------ epilogue: TMEM -> partial
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    if (wait_bar(acc_full, 0, abort_flag, p.err, p.wait_ns)) {
      ptx::tc_fence_after();
      uint32_t r[16];
      ptx::tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quad * 32) << 16), r);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < kDTok; ++t) red[t * kDRows + row] = __uint_as_float(r[t]);
    } else {
#pragma unroll
      for (int t = 0; t < kDTok; ++t) red[t * kDRows + row] = 0.0f;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();                             // every CTA's partial is in its shared memory
  if (warp >= 2) {
    // This CTA's share of the tile's outputs (token-major: consecutive rows of one token), four
    // consecutive outputs per thread, summed over the cluster in rank order.  The S remote loads
    // of a group are all issued before the first add, so their latencies overlap.
    const int e = threadIdx.x - 64;
    constexpr int kOut = kDRows * kDTok;
    const int share = ((kOut + p.S - 1) / p.S + 3) & ~3;
    const int v0 = rank * share;
    const int v1 = v0 + share < kOut ? v0 + share : kOut;
    const float alpha = __ldg(p.alpha + (p.offsets ? expert : segment_of(n0, p.seg)));
    const uint32_t red_addr = ptx::smem_u32(red);
    for (int v = v0 + 4 * e; v < v1; v += 4 * 128) {
      const int t = v / kDRows, rr = v - t * kDRows;   // 4 rows rr..rr+3 of token t
      if (t >= M || n0 + rr >= p.N) continue;
      float4 part[kDMaxSplit];
#pragma unroll
      for (int s2 = 0; s2 < kDMaxSplit; ++s2)
        if (s2 < p.S) part[s2] = ptx::ld_shared_cluster_v4(ptx::mapa_shared(red_addr + 4u * v, s2));
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s2 = 0; s2 < kDMaxSplit; ++s2)
        if (s2 < p.S) { sum.x += part[s2].x; sum.y += part[s2].y; sum.z += part[s2].z; sum.w += part[s2].w; }
      const float y[4] = {sum.x * alpha, sum.y * alpha, sum.z * alpha, sum.w * alpha};
      const int64_t off = (yrow0 + t) * p.ldy + n0 + rr;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (n0 + rr + q >= p.N) break;
        if (p.out_bf16) static_cast<uint16_t*>(p.Y)[off + q] = f32_to_bf16_bits(y[q]);
        else static_cast<float*>(p.Y)[off + q] = y[q];
      }
    }
  }
  ptx::cluster_sync();                             // no CTA leaves while another reads its partial
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc<1>(tmem, C::TMEM_COLS);
  }
}

}  // namespace

fs_status launch_splice_gemm_decode_tc(const DecodeParams& d, cudaStream_t s) {
  using C = DCfg;
  using Kernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, DecTcParams);
  const Kernel kernel = d.fuse ? splice_gemm_decode_tc_kernel<true> : splice_gemm_decode_tc_kernel<false>;
  const char* who = d.fuse ? "fs_decode_splice_gemm" : "fs_splice_gemm (decode path)";
  static PerDevice<int> attr, attr_fused;
  fs_status ast = set_max_dynamic_smem(d.fuse ? attr_fused : attr, reinterpret_cast<const void*>(kernel),
                                       C::SMEM_BYTES, "fs_splice_gemm (decode): smem attribute");
  if (ast != FS_OK) return ast;
  DecTcParams p{};
  p.M = d.M; p.N = d.N; p.KT = d.K / 256; p.ST = static_cast<int>(ceil_div(d.pp, 64)); p.kb4 = d.kb4;
  p.sfw = d.sfw; p.sfx = d.sfx; p.alpha = d.alpha; p.seg = d.seg; p.Y = d.Y; p.ldy = d.ldy; p.out_bf16 = d.out_bf16;
  p.err = d.err; p.wait_ns = d.wait_ns; p.no_copies = d.no_copies;
  p.x = d.x; p.ldx = d.ldx; p.mask = d.mask; p.p = d.p; p.gA = d.gA; p.residual = d.residual;
  if (d.offsets && d.fuse) return fail(FS_ERR_UNSUPPORTED, "%s: the grouped form takes packed activations", who);
  const int n_tiles = static_cast<int>(ceil_div(d.N, kDRows));
  p.offsets = d.offsets; p.n_tiles = n_tiles; p.small_max = d.small_max;
  const int64_t w_rows = d.offsets ? static_cast<int64_t>(d.E) * d.N : d.N;   // weight operand rows
  const int64_t x_rows = d.offsets ? d.a_rows : d.M;                          // activation operand rows
  // K split: as many CTAs per 128-row tile as fill the SMs at the resident CTAs per SM, at most 8
  // (a portable cluster);
  // every split keeps at least one FP4 k-tile.
  const int tiles = n_tiles * (d.offsets ? d.E : 1);
  int S = static_cast<int>(std::max<int64_t>(1, (kDCtasPerSm * static_cast<int64_t>(sm_count())) / tiles));
  S = std::min(S, std::min(kDMaxSplit, p.KT));
  p.kt_per = static_cast<int>(ceil_div(p.KT, S));
  p.S = static_cast<int>(ceil_div(p.KT, p.kt_per));

  // (the fused kernel reads X itself; its activation maps are placeholders it never uses)
  CUtensorMap tmW, tmX, tmWS, tmXS;
  const uint64_t kbytes = static_cast<uint64_t>(d.K) / 2;
  fs_status st = make_map(&tmW, d.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, w_rows, kbytes, 128, kDRows);
  if (st == FS_OK && !d.fuse) st = make_map(&tmX, d.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, x_rows, kbytes, 128, kDTok);
  if (st != FS_OK) return st;
  if (d.fuse) tmX = tmW;
  if (p.ST > 0) {
    const uint64_t pp = static_cast<uint64_t>(d.pp);
    st = make_map(&tmWS, d.ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, w_rows, pp * 2, 64, kDRows);
    if (st == FS_OK && !d.fuse) st = make_map(&tmXS, d.xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, x_rows, pp * 2, 64, kDTok);
    if (st != FS_OK) return st;
    if (d.fuse) tmXS = tmWS;
  } else {
    tmWS = tmW;
    tmXS = tmX;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(p.S), 1);
  cfg.blockDim = dim3(kDThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = 1;
  attrs[0].val.clusterDim.y = static_cast<unsigned>(p.S);
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tmW, tmX, tmWS, tmXS, p);
  if (e != cudaSuccess) return cuda_status(e, who);
  FS_CHECK_LAUNCH(who);
  return FS_OK;
}

}  // namespace fs
