// SpliceGEMM decode path (M <= 16 tokens), persistent stream-K form.
//
// FourSight §5.1 "Dual-path execution": for small M the product is bound by streaming the packed
// weights once.  The weights are the 128-row A operand of tcgen05 block-scaled MMAs
// (kind::mxf4nvf4, M = 128, N = 16) and the tokens the B operand, so the tensor core applies the
// UE4M3 scales and the SMs only move bytes; the protected slice X_S W'_S^T (§4.2 Eq. 5) runs as
// BF16 MMAs (kind::f16) into the same TMEM accumulator.
//
// Work decomposition: a 128-row output tile needs U = K/256 NVFP4 units plus ceil(Pp/64) BF16
// units (one k-tile each, about 22 KB of operands).  The T = tiles * U units are cut into G
// contiguous, balanced ranges, one per persistent CTA (one per SM), so every SM streams the same
// number of bytes whatever N and K are, and a CTA pays its prologue once per launch.  A range can
// start or end inside a tile: the CTA then writes its partial sums of that tile to the plan's
// workspace, and the last of the tile's contributors (per 32-row quadrant, found with a counter)
// adds the partials in CTA order, scales by alpha once and stores Y; a tile held whole by one
// CTA is stored directly.  Results do not depend on arrival order.
//   warp 0      TMA producer: weight boxes (and scale atoms) of its first stages are issued
//               BEFORE griddepcontrol.wait (they do not depend on the previous kernel), the
//               activation boxes after it; then both per unit through a ring of stages
//   warp 1      TMEM allocation; one thread copies the scale atoms to TMEM (tcgen05.cp) and
//               issues the MMAs, one accumulator buffer per tile segment (two buffers)
//   warps 2..5  epilogue: TMEM -> registers, direct store or partial + fix-up
// The launch allows programmatic dependent launch, and a CTA uses under half of an SM's shared
// memory, so the next decode launch's CTAs become resident early and stream their weights while
// this one finishes.  Every mbarrier wait is bounded; on expiry the kernel records a timeout,
// drains its copies (bounded), releases TMEM and returns; fs_plan_check then also clears the
// workspace counters, which an aborted launch may have left behind.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace fs {
namespace {

constexpr int kKThreads = 192;
constexpr int kKRows = 128;          // weight rows per tile (MMA M)
constexpr int kKTok = 16;            // token columns (MMA N)
#ifndef FS_DSK_STAGES
#define FS_DSK_STAGES 4
#endif
constexpr int kKStages = FS_DSK_STAGES;
constexpr uint64_t kKDrainNs = 50000000ull;

struct KCfg {
  static constexpr int W_BYTES = kKRows * 128;      // 256 fp4 or 64 bf16 per row
  static constexpr int X_BYTES = kKTok * 128;
  static constexpr int SFW_BYTES = 2048;            // four 512-byte atoms, one per MMA
  static constexpr int SFX_BYTES = 2048;
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES + SFW_BYTES + SFX_BYTES;   // multiple of 1024
  static constexpr int SMEM_BYTES = 1024 + kKStages * STAGE_BYTES + 8 * (2 * kKStages + 5) + 16;
  static constexpr int TMEM_COLS = 128;
  static constexpr int ACC_COLS = 16;               // accumulator buffer b at column 16 b
  static constexpr int SF_COL = 32;                 // scale buffer i: SFW at 32+32i, SFX at 32+32i+16
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the 128-byte swizzle");
  static_assert(SF_COL + 64 <= TMEM_COLS, "TMEM budget");
  static_assert(2 * SMEM_BYTES <= 232448, "two CTAs (this launch and the next) fit one SM");
};

struct SkParams {
  int M, N, KT, ST, U, kb4;
  int64_t T, q, r;           // units; CTA c owns q units (q + 1 for c < r)
  const uint8_t* sfw;
  const uint8_t* sfx;
  const float* alpha;
  Segments seg;
  void* Y;
  int64_t ldy;
  int out_bf16;
  float* part;               // [2 G][16 tokens][128 rows] partial sums
  int* counter;              // [tiles][4] arrivals per 32-row quadrant (0 between launches)
  uint32_t* err;
  uint64_t wait_ns;
  int no_copies;
};

__device__ __forceinline__ int64_t unit0(int64_t c, const SkParams& p) { return c * p.q + (c < p.r ? c : p.r); }
__device__ __forceinline__ int64_t cta_of(int64_t u, const SkParams& p) {
  const int64_t b = p.r * (p.q + 1);
  return u < b ? u / (p.q + 1) : p.r + (u - b) / p.q;
}

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
        atomicOr(err, ERR_TIMEOUT);
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

__device__ __forceinline__ int atomic_add_acq_rel(int* addr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}

__global__ void __launch_bounds__(kKThreads, 1)
splice_gemm_decode_sk_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                             const __grid_constant__ CUtensorMap tmWS, const __grid_constant__ CUtensorMap tmXS,
                             const SkParams p) {
  using C = KCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kKStages * C::STAGE_BYTES);
  uint64_t* empty = full + kKStages;
  uint64_t* acc_full = empty + kKStages;            // [2]
  uint64_t* acc_empty = acc_full + 2;               // [2], 4 epilogue warps arrive
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  const int64_t u_begin = unit0(c, p), u_end = unit0(c + 1, p);
  auto W_at = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto X_at = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES; };
  auto SFW_at = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES + C::X_BYTES; };
  auto SFX_at = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES + C::X_BYTES + C::SFW_BYTES; };

  // The next launch may become resident now: it only streams its own weights before its wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kKStages; ++s) { ptx::mbar_init(full + s, 1); ptx::mbar_init(empty + s, 1); }
    for (int b = 0; b < 2; ++b) { ptx::mbar_init(acc_full + b, 1); ptx::mbar_init(acc_empty + b, 4); }
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tmW); ptx::prefetch_tensormap(&tmX);
    if (p.ST > 0) { ptx::prefetch_tensormap(&tmWS); ptx::prefetch_tensormap(&tmXS); }
  }
  if (warp == 1) {
    ptx::tmem_alloc<1>(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish<1>();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && !p.no_copies) {
      auto weight_part = [&](int64_t u, int s) {
        const int tile = static_cast<int>(u / p.U), k = static_cast<int>(u % p.U);
        if (k < p.KT) {
          ptx::mbar_arrive_expect_tx(full + s, C::STAGE_BYTES);
          ptx::tma_load_2d(W_at(s), &tmW, k * 128, tile * kKRows, full + s);
          ptx::bulk_load(SFW_at(s), p.sfw + (static_cast<int64_t>(tile) * p.kb4 + k * 4) * 512, C::SFW_BYTES, full + s);
        } else {
          ptx::mbar_arrive_expect_tx(full + s, C::W_BYTES + C::X_BYTES);
          ptx::tma_load_2d(W_at(s), &tmWS, (k - p.KT) * 64, tile * kKRows, full + s);
        }
      };
      auto activation_part = [&](int64_t u, int s) {
        const int k = static_cast<int>(u % p.U);
        if (k < p.KT) {
          ptx::tma_load_2d(X_at(s), &tmX, k * 128, 0, full + s);
          ptx::bulk_load(SFX_at(s), p.sfx + static_cast<int64_t>(k) * 4 * 512, C::SFX_BYTES, full + s);
        } else {
          ptx::tma_load_2d(X_at(s), &tmXS, (k - p.KT) * 64, 0, full + s);
        }
      };
      const int pre = static_cast<int>(u_end - u_begin < kKStages ? u_end - u_begin : kKStages);
      for (int i = 0; i < pre; ++i) weight_part(u_begin + i, i);      // stages start free
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int i = 0; i < pre; ++i) activation_part(u_begin + i, i);
      int stage = pre % kKStages;
      uint32_t phase = pre == kKStages ? 1u : 0u;
      int issued = pre;
      for (int64_t u = u_begin + pre; u < u_end; ++u) {
        if (!wait_bar(empty + stage, phase ^ 1, abort_flag, p.err, p.wait_ns)) break;
        weight_part(u, stage);
        activation_part(u, stage);
        ++issued;
        if (++stage == kKStages) { stage = 0; phase ^= 1; }
      }
      if (*abort_flag) {
        // copies issued but possibly not landed: the last min(issued, stages) stages
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < kKStages && i < issued; ++i) {
          if (--s < 0) { s = kKStages - 1; ph ^= 1; }
          drain_bar(full + s, ph, kKDrainNs);
        }
      }
    } else if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ scale copies + MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_f4 = ptx::idesc_nvf4(kKRows, kKTok);
      constexpr uint32_t idesc_bf = ptx::idesc_bf16(kKRows, kKTok);
      int stage = 0, si = 0;
      uint32_t phase = 0;
      int64_t uc = 0;                               // units issued (scale buffer parity)
      bool ok = true;
      for (int64_t u = u_begin; u < u_end && ok; ++si) {
        const int64_t tile = u / p.U;
        const int64_t seg_end = (tile + 1) * p.U < u_end ? (tile + 1) * p.U : u_end;
        const int buf = si & 1;
        if (!wait_bar(acc_empty + buf, ((si >> 1) & 1) ^ 1, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t d = tmem + C::ACC_COLS * buf;
        for (int64_t v = u; v < seg_end; ++v, ++uc) {
          if (!wait_bar(full + stage, phase, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
          ptx::tc_fence_after();
          const int k = static_cast<int>(v % p.U);
          const uint64_t adesc = ptx::desc_kmajor_sw128(ptx::smem_u32(W_at(stage)));
          const uint64_t bdesc = ptx::desc_kmajor_sw128(ptx::smem_u32(X_at(stage)));
          const bool first = v == u;
          if (k < p.KT) {
            const uint32_t sfa = tmem + C::SF_COL + 32 * static_cast<uint32_t>(uc & 1);
            const uint32_t sfb = sfa + 16;
            const uint32_t sw = ptx::smem_u32(SFW_at(stage)), sx = ptx::smem_u32(SFX_at(stage));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              ptx::tc_cp_32x128b_warpx4(sfa + 4 * j, ptx::desc_sf_block(sw + 512 * j));
              ptx::tc_cp_32x128b_warpx4(sfb + 4 * j, ptx::desc_sf_block(sx + 512 * j));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              ptx::tc_mma_nvf4<1>(d, adesc + 2 * j, bdesc + 2 * j, idesc_f4, sfa + 4 * j, sfb + 4 * j, !(first && j == 0));
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) ptx::tc_mma_bf16<1>(d, adesc + 2 * j, bdesc + 2 * j, idesc_bf, !(first && j == 0));
          }
          ptx::tc_commit<1>(empty + stage);
          if (++stage == kKStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        ptx::tc_commit<1>(acc_full + buf);
        u = seg_end;
      }
      ptx::tc_commit<1>(drain);                    // every MMA issued above has completed
      drain_bar(drain, 0, p.wait_ns);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");      // global writes only after the previous launch
    const int quad = warp & 3;
    const int rowl = quad * 32 + lane;              // row of the tile held by this thread
    const int64_t first_tile = u_begin / p.U;
    int si = 0;
    for (int64_t u = u_begin; u < u_end; ++si) {
      const int64_t tile = u / p.U;
      const int64_t seg_end = (tile + 1) * p.U < u_end ? (tile + 1) * p.U : u_end;
      const int buf = si & 1;
      if (!wait_bar(acc_full + buf, (si >> 1) & 1, abort_flag, p.err, p.wait_ns)) break;
      ptx::tc_fence_after();
      uint32_t r[16];
      ptx::tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quad * 32) << 16) + C::ACC_COLS * buf, r);
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty + buf);
      const int n0 = static_cast<int>(tile) * kKRows;
      const int row = n0 + rowl;
      const float alpha = p.alpha ? __ldg(p.alpha + segment_of(n0, p.seg)) : 1.0f;
      auto store = [&](const float (&y)[kKTok]) {
        if (row >= p.N) return;
#pragma unroll
        for (int t = 0; t < kKTok; ++t) {
          if (t >= p.M) break;
          const int64_t off = static_cast<int64_t>(t) * p.ldy + row;
          if (p.out_bf16) static_cast<uint16_t*>(p.Y)[off] = f32_to_bf16_bits(y[t] * alpha);
          else static_cast<float*>(p.Y)[off] = y[t] * alpha;
        }
      };
      if (u == tile * p.U && seg_end == (tile + 1) * p.U) {
        float y[kKTok];
#pragma unroll
        for (int t = 0; t < kKTok; ++t) y[t] = __uint_as_float(r[t]);
        store(y);                                   // the whole tile is this CTA's
      } else {
        const int64_t slot = 2 * c + (tile == first_tile ? 0 : 1);
        float* mine = p.part + slot * (kKTok * kKRows);
#pragma unroll
        for (int t = 0; t < kKTok; ++t)
          if (t < p.M) mine[t * kKRows + rowl] = __uint_as_float(r[t]);
        __threadfence();
        __syncwarp();
        const int64_t c_first = cta_of(tile * p.U, p), c_last = cta_of((tile + 1) * p.U - 1, p);
        const int contributors = static_cast<int>(c_last - c_first + 1);
        int* cnt = p.counter + tile * 4 + quad;
        int old = 0;
        if (lane == 0) old = atomic_add_acq_rel(cnt, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == contributors - 1) {
          // last of this quadrant's contributors: sum the partials in CTA order
          __threadfence();
          float y[kKTok];
#pragma unroll
          for (int t = 0; t < kKTok; ++t) y[t] = 0.0f;
          for (int64_t cc = c_first; cc <= c_last; ++cc) {
            const int64_t sl = 2 * cc + (tile == unit0(cc, p) / p.U ? 0 : 1);
            const float* src = p.part + sl * (kKTok * kKRows);
#pragma unroll
            for (int t = 0; t < kKTok; ++t)
              if (t < p.M) y[t] += __ldcg(src + t * kKRows + rowl);
          }
          store(y);
          if (lane == 0) *cnt = 0;                  // ready for the next launch
        }
      }
      u = seg_end;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc<1>(tmem, C::TMEM_COLS);
  }
}

}  // namespace

int64_t decode_sk_ctas() { return sm_count(); }

int64_t decode_sk_workspace_bytes(int N) {
  const int64_t tiles = ceil_div(N, kKRows);
  return round_up(2 * decode_sk_ctas() * kKTok * kKRows * 4, 256) + tiles * 4 * 4;
}

fs_status launch_splice_gemm_decode_sk(const DecodeParams& d, void* workspace, int64_t ws_bytes, cudaStream_t s) {
  using C = KCfg;
  static PerDevice<int> attr;
  fs_status ast = set_max_dynamic_smem(attr, reinterpret_cast<const void*>(splice_gemm_decode_sk_kernel),
                                       C::SMEM_BYTES, "fs_splice_gemm (decode): smem attribute");
  if (ast != FS_OK) return ast;
  if (ws_bytes < decode_sk_workspace_bytes(d.N)) return fail(FS_ERR_INVALID_ARGUMENT, "decode workspace too small");
  SkParams p{};
  p.M = d.M; p.N = d.N; p.KT = d.K / 256; p.ST = static_cast<int>(ceil_div(d.pp, 64)); p.U = p.KT + p.ST;
  p.kb4 = d.kb4;
  const int64_t tiles = ceil_div(d.N, kKRows);
  p.T = tiles * p.U;
  const int64_t G = std::min<int64_t>(p.T, decode_sk_ctas());
  p.q = p.T / G; p.r = p.T % G;
  p.sfw = d.sfw; p.sfx = d.sfx; p.alpha = d.alpha; p.seg = d.seg; p.Y = d.Y; p.ldy = d.ldy; p.out_bf16 = d.out_bf16;
  auto* base = static_cast<uint8_t*>(workspace);
  p.part = reinterpret_cast<float*>(base);
  p.counter = reinterpret_cast<int*>(base + round_up(2 * decode_sk_ctas() * kKTok * kKRows * 4, 256));
  p.err = d.err; p.wait_ns = d.wait_ns; p.no_copies = d.no_copies;

  CUtensorMap tmW, tmX, tmWS, tmXS;
  const uint64_t kbytes = static_cast<uint64_t>(d.K) / 2;
  fs_status st = make_map(&tmW, d.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, d.N, kbytes, 128, kKRows);
  if (st == FS_OK) st = make_map(&tmX, d.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, d.M, kbytes, 128, kKTok);
  if (st != FS_OK) return st;
  if (p.ST > 0) {
    const uint64_t pp = static_cast<uint64_t>(d.pp);
    st = make_map(&tmWS, d.ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, d.N, pp * 2, 64, kKRows);
    if (st == FS_OK) st = make_map(&tmXS, d.xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, d.M, pp * 2, 64, kKTok);
    if (st != FS_OK) return st;
  } else {
    tmWS = tmW;
    tmXS = tmX;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(G), 1, 1);
  cfg.blockDim = dim3(kKThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, splice_gemm_decode_sk_kernel, tmW, tmX, tmWS, tmXS, p);
  if (e != cudaSuccess) return cuda_status(e, "fs_splice_gemm (decode path)");
  FS_CHECK_LAUNCH("fs_splice_gemm (decode path)");
  return FS_OK;
}

}  // namespace fs
