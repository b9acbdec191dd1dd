// SpliceGEMM on the 5th-generation tensor cores (tcgen05), the large-M path.
//
// FourSight §4.2 Eq. 5 and §5.1 "Dual-path execution" (Fig. 6): the NVFP4 product runs as
// block-scaled MMAs, then the BF16 tiles of the protected slice (X_S, W'_S) are loaded into the
// SAME shared-memory stage buffers and their BF16 MMAs accumulate into the SAME FP32 TMEM
// accumulator; the epilogue moves TMEM to registers, multiplies by alpha once and stores Y.
//
// Per CTA (persistent, one per SM): a 128 x BN output tile at a time.
//   warp 0      TMA producer: per k-tile one 128x128-byte box of A and a BNx128-byte box of B
//               (128-byte swizzle) plus the tile's UE4M3 scale atoms (plain bulk copies); the
//               BF16 side tiles use the same boxes, 64 bf16 wide.
//   warp 1      allocates TMEM; one thread issues tcgen05.cp (scales SMEM->TMEM) and
//               tcgen05.mma: kind::mxf4nvf4 (K = 64 per instruction) over all of K, then
//               kind::f16 (K = 16) over the protected slice, then commits to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns at a time, x alpha, store.
// Every mbarrier wait is bounded; on expiry the kernel records a timeout in the plan's error
// word, all roles stop issuing work, and TMEM is still released.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace fs {
namespace {

constexpr int kBM = 128;
constexpr int kThreads = 320;                  // producer, MMA, 4 epilogue and 4 scale warps
constexpr int kMaxExperts = 256;
constexpr uint64_t kWaitNs = 4000000000ull;     // 4 s bound on any single wait

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = kBM * 128;            // 128 rows x 128 bytes (256 fp4 or 64 bf16)
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = kBM * 16;           // 16 scales per row per k-tile
  static constexpr int SFB_BYTES = BN * 16;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = BN == 256 ? 3 : 4;
  static constexpr int NUM_ACC = BN == 256 ? 1 : 2;    // TMEM accumulator buffers
  static constexpr int ACC_COLS = BN * NUM_ACC;
  // Scale factors in TMEM, double-buffered by k-tile parity so that the copy for k-tile kt+1
  // does not overwrite columns the MMAs of k-tile kt may still read.
  static constexpr int SF_COLS = 16 + 4 * (BN / 32);   // SFA: 4 MMAs x 4 columns; SFB: 4 MMAs x BN/32
  static constexpr int SFA_COL = ACC_COLS;
  static constexpr int SFB_COL = ACC_COLS + 16;
  static constexpr int TMEM_COLS = 512;
  static_assert(ACC_COLS + 2 * SF_COLS <= TMEM_COLS, "TMEM budget");
  static constexpr int STAGING_BUFS = 3;                // per epilogue warp
  static constexpr int STAGING_BYTES = 4 * STAGING_BUFS * 4096;  // 4 warps x buffers x (32 rows x 128 B)
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGING_BYTES + 1024 + 4 * (kMaxExperts + 1);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget of one CTA");
};

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait with a deadline and an abort flag shared by the CTA's roles.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* err) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1;; ++i) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 0) {
      if (*abort_flag) return false;
      if (now_ns() - t0 > kWaitNs) {
        atomicOr(err, ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

struct TileMap {
  int e;           // expert
  int64_t arow;    // first row in the packed activation buffers (padded for experts)
  int64_t yrow;    // first output row
  int rows;        // valid rows in this tile
  int64_t brow;    // first row in the (stacked) weight buffers
  int n0;          // first output column
};

__device__ __forceinline__ TileMap map_tile(int t, const TcParams& p, const int* cum_m) {
  TileMap m;
  const int total_m = cum_m[p.E];
  const int mt = t % total_m;
  const int nt = t / total_m;
  int lo = 0, hi = p.E - 1;                   // expert with cum_m[e] <= mt < cum_m[e+1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cum_m[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  m.e = lo;
  const int local = mt - cum_m[lo];
  m.arow = static_cast<int64_t>(mt) * kBM;    // experts start at 128-row boundaries
  if (p.offsets) {
    const int64_t r0 = p.offsets[lo], r1 = p.offsets[lo + 1];
    m.yrow = r0 + static_cast<int64_t>(local) * kBM;
    const int64_t left = r1 - m.yrow;
    m.rows = static_cast<int>(left < kBM ? left : kBM);
  } else {
    m.yrow = m.arow;
    const int64_t left = p.M - m.arow;
    m.rows = static_cast<int>(left < kBM ? left : kBM);
  }
  m.n0 = nt * p.BN;
  m.brow = static_cast<int64_t>(lo) * p.N + m.n0;
  return m;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
splice_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                      const __grid_constant__ CUtensorMap tmY, const TcParams p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;           // 1024-byte aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::STAGING_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + C::NUM_ACC;
  uint64_t* sf_full = acc_empty + C::NUM_ACC;      // [2]: scales of a k-tile are in TMEM
  uint64_t* sf_empty = sf_full + 2;                // [2]: the MMAs reading a scale buffer are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* cum_m = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto A_at = [&](int s) { return stages + s * C::STAGE_BYTES; };
  auto B_at = [&](int s) { return stages + s * C::STAGE_BYTES + C::A_BYTES; };
  auto SFA_at = [&](int s) { return stages + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES; };
  auto SFB_at = [&](int s) { return stages + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES + C::SFA_BYTES; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    cum_m[0] = 0;
    if (p.offsets) {
      for (int e = 0; e < p.E; ++e) {
        const int64_t rows = p.offsets[e + 1] - p.offsets[e];
        cum_m[e + 1] = cum_m[e] + static_cast<int>((rows + kBM - 1) / kBM);
      }
    } else {
      cum_m[1] = static_cast<int>((p.M + kBM - 1) / kBM);
    }
    for (int s = 0; s < C::STAGES; ++s) { ptx::mbar_init(full + s, 1); ptx::mbar_init(empty + s, 1); }
    for (int a = 0; a < C::NUM_ACC; ++a) { ptx::mbar_init(acc_full + a, 1); ptx::mbar_init(acc_empty + a, 128); }
    for (int b = 0; b < 2; ++b) { ptx::mbar_init(sf_full + b, 4); ptx::mbar_init(sf_empty + b, 1); }
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tmA); ptx::prefetch_tensormap(&tmB); ptx::prefetch_tensormap(&tmY);
    if (p.ST > 0) { ptx::prefetch_tensormap(&tmSA); ptx::prefetch_tensormap(&tmSB); }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total_tiles = cum_m[p.E] * p.n_tiles;
  const int ktiles = p.KT + p.ST;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const TileMap m = map_tile(t, p, cum_m);
        for (int kt = 0; kt < ktiles; ++kt) {
          if (!wait_bar(empty + stage, phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          if (kt < p.KT) {
            ptx::mbar_arrive_expect_tx(full + stage, C::STAGE_BYTES);
            ptx::tma_load_2d(A_at(stage), &tmA, kt * 128, static_cast<int32_t>(m.arow), full + stage);
            ptx::tma_load_2d(B_at(stage), &tmB, kt * 128, static_cast<int32_t>(m.brow), full + stage);
            ptx::bulk_load(SFA_at(stage), p.sfa + ((m.arow / kBM) * p.kb4 + kt * 4) * 512, C::SFA_BYTES, full + stage);
#pragma unroll
            for (int rg = 0; rg < BN / 128; ++rg)
              ptx::bulk_load(SFB_at(stage) + rg * 2048, p.sfb + ((m.brow / kBM + rg) * p.kb4 + kt * 4) * 512, 2048,
                             full + stage);
          } else {
            ptx::mbar_arrive_expect_tx(full + stage, C::A_BYTES + C::B_BYTES);
            ptx::tma_load_2d(A_at(stage), &tmSA, (kt - p.KT) * 64, static_cast<int32_t>(m.arow), full + stage);
            ptx::tma_load_2d(B_at(stage), &tmSB, (kt - p.KT) * 64, static_cast<int32_t>(m.brow), full + stage);
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_f4 = ptx::idesc_nvf4(kBM, BN);
      constexpr uint32_t idesc_bf = ptx::idesc_bf16(kBM, BN);
      int stage = 0, acc = 0, sf_count = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        if (!wait_bar(acc_empty + acc, acc_phase ^ 1, abort_flag, p.err)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kt = 0; kt < ktiles; ++kt) {
          if (!wait_bar(full + stage, phase, abort_flag, p.err)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t adesc = ptx::desc_kmajor_sw128(ptx::smem_u32(A_at(stage)));
          const uint64_t bdesc = ptx::desc_kmajor_sw128(ptx::smem_u32(B_at(stage)));
          if (kt < p.KT) {
            const int buf = sf_count & 1;
            if (!wait_bar(sf_full + buf, (sf_count >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t sf_off = buf * C::SF_COLS;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              ptx::tc_mma_nvf4(d, adesc + 2 * j, bdesc + 2 * j, idesc_f4, tmem + C::SFA_COL + sf_off + 4 * j,
                               tmem + C::SFB_COL + sf_off + (BN / 32) * j, (kt | j) != 0);
            ptx::tc_commit(sf_empty + buf);
            ++sf_count;
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) ptx::tc_mma_bf16(d, adesc + 2 * j, bdesc + 2 * j, idesc_bf, 1u);
          }
          ptx::tc_commit(empty + stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        ptx::tc_commit(acc_full + acc);
        if (++acc == C::NUM_ACC) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------------ scale warps
    // Each warp owns one TMEM lane quadrant and writes, for every FP4 k-tile, the block scales
    // of its 32 lanes exactly as tcgen05.cp.32x128b.warpx4 would lay them out: lane l, columns
    // 4c..4c+3 of an atom's slot hold the atom's 16-byte row l (SFA: one atom per MMA; SFB: the
    // BN/128 row-group atoms side by side).  Scales are double-buffered in TMEM by k-tile parity.
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int stage = 0, sf_count = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      for (int kt = 0; kt < ktiles; ++kt) {
        if (kt < p.KT) {
          const int buf = sf_count & 1;
          if (!wait_bar(sf_empty + buf, ((sf_count >> 1) & 1) ^ 1, abort_flag, p.err)) { ok = false; break; }
          if (!wait_bar(full + stage, phase, abort_flag, p.err)) { ok = false; break; }
          const uint8_t* sfa = SFA_at(stage);
          const uint8_t* sfb = SFB_at(stage);
          const uint32_t col = tmem + lane_base + buf * C::SF_COLS;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 a = *reinterpret_cast<const uint4*>(sfa + 512 * j + lane * 16);
            ptx::tmem_st_32x32b_x4(col + C::SFA_COL + 4 * j, a.x, a.y, a.z, a.w);
            if constexpr (BN == 256) {
              const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + 512 * j + lane * 16);
              const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + 2048 + 512 * j + lane * 16);
              ptx::tmem_st_32x32b_x8(col + C::SFB_COL + 8 * j, b0, b1);
            } else {
              const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + 512 * j + lane * 16);
              ptx::tmem_st_32x32b_x4(col + C::SFB_COL + 4 * j, b0.x, b0.y, b0.z, b0.w);
            }
          }
          ptx::tmem_st_wait();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(sf_full + buf);
          ++sf_count;
        }
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // TMEM -> registers (x alpha) -> swizzled staging in shared memory -> TMA store of a
    // 32-row x 32-column box per warp; the accumulator is released right after the last TMEM
    // load, so the next tile's MMAs overlap the stores.  Partial tiles of an expert (rows that
    // end inside the output) use direct stores instead, since a box would cross into the next
    // expert's rows.
    const int quad = warp & 3;                  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;           // row of the tile held by this thread
    uint8_t* stage_buf = staging + quad * C::STAGING_BUFS * 4096;
    int acc = 0, nbuf = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const TileMap m = map_tile(t, p, cum_m);
      if (!wait_bar(acc_full + acc, acc_phase, abort_flag, p.err)) break;
      ptx::tc_fence_after();
      const float alpha = __ldg(p.alpha + m.e);
      const bool use_tma = !(p.offsets && m.rows < kBM);
      const bool row_ok = row < m.rows;
      const int64_t yrow = m.yrow + row;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN + c * 32, r);
        ptx::tmem_ld_wait();
        if (c == BN / 32 - 1) {
          ptx::tc_fence_before();
          ptx::mbar_arrive(acc_empty + acc);
        }
        const int col0 = m.n0 + c * 32;
        if (col0 >= p.N) continue;
        if (use_tma) {
          if (quad * 32 >= m.rows) continue;            // this warp's rows are all past the end
          uint8_t* buf = stage_buf + (nbuf % C::STAGING_BUFS) * 4096;
          if (lane == 0) ptx::bulk_wait_read<C::STAGING_BUFS - 1>();   // the store that last used `buf` has read it
          __syncwarp();
          if (p.out_bf16) {
            // 32 rows x 64 bytes, 64-byte swizzle: 16-byte chunk j of row r sits at j ^ ((r >> 1) & 3)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t w[4];
#pragma unroll
              for (int h = 0; h < 4; ++h)
                w[h] = static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[8 * j + 2 * h]) * alpha)) |
                       (static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[8 * j + 2 * h + 1]) * alpha)) << 16);
              *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
            // 32 rows x 128 bytes, 128-byte swizzle: 16-byte chunk j of row r sits at j ^ (r & 7)
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<float4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                  make_float4(__uint_as_float(r[4 * j]) * alpha, __uint_as_float(r[4 * j + 1]) * alpha,
                              __uint_as_float(r[4 * j + 2]) * alpha, __uint_as_float(r[4 * j + 3]) * alpha);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(&tmY, col0, static_cast<int32_t>(m.yrow + quad * 32), buf);
            ptx::bulk_commit();
          }
          ++nbuf;
        } else if (row_ok) {
          if (p.out_bf16) {
            uint16_t* y = static_cast<uint16_t*>(p.Y) + yrow * p.ldy + col0;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + i < p.N) y[i] = f32_to_bf16_bits(__uint_as_float(r[i]) * alpha);
          } else {
            float* y = static_cast<float*>(p.Y) + yrow * p.ldy + col0;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + i < p.N) y[i] = __uint_as_float(r[i]) * alpha;
          }
        }
      }
      if (++acc == C::NUM_ACC) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------
// Host: tensor maps and launch
// ------------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2D K-major map with a 128-byte-wide, `box_rows`-high box and 128-byte swizzle.
fs_status make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t inner_elems,
                   uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(FS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {inner_elems, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FS_OK;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int BN>
fs_status launch_bn(const TcLaunch& L, TcParams prm, cudaStream_t s) {
  using C = Cfg<BN>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(splice_gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_status(e, "fs_splice_gemm: smem attribute");
    attr = true;
  }
  prm.BN = BN;
  prm.n_tiles = static_cast<int>(ceil_div(prm.N, BN));
  CUtensorMap tmA, tmB, tmSA, tmSB;
  const uint64_t kbytes = static_cast<uint64_t>(prm.K) / 2;
  fs_status st = make_map(&tmA, L.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, L.a_rows, kbytes, 128, kBM);
  if (st == FS_OK) st = make_map(&tmB, L.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, L.b_rows, kbytes, 128, BN);
  if (st != FS_OK) return st;
  if (prm.ST > 0) {
    const uint64_t pp = static_cast<uint64_t>(L.pp);
    st = make_map(&tmSA, L.xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, L.a_rows, pp * 2, 64, kBM);
    if (st == FS_OK) st = make_map(&tmSB, L.ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, L.b_rows, pp * 2, 64, BN);
    if (st != FS_OK) return st;
  } else {
    tmSA = tmA;
    tmSB = tmB;
  }
  CUtensorMap tmY;
  {
    auto fn = encode_fn();
    const int esz = prm.out_bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(prm.N), static_cast<cuuint64_t>(L.y_rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(prm.ldy) * esz};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&tmY, prm.out_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, prm.Y,
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    prm.out_bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FS_ERR_CUDA, "cuTensorMapEncodeTiled (Y) failed (%d)", static_cast<int>(r));
  }
  const int grid = static_cast<int>(std::min<int64_t>(std::max<int64_t>(L.max_tiles, 1), sm_count()));
  splice_gemm_tc_kernel<BN><<<grid, kThreads, C::SMEM_BYTES, s>>>(tmA, tmB, tmSA, tmSB, tmY, prm);
  FS_CHECK_LAUNCH("fs_splice_gemm (tensor-core path)");
  return FS_OK;
}

}  // namespace

fs_status launch_splice_gemm_tc(const TcLaunch& L, const TcParams& prm, cudaStream_t s) {
  if (prm.E > kMaxExperts) return fail(FS_ERR_UNSUPPORTED, "fs_splice_gemm: at most %d experts", kMaxExperts);
  if (L.bn == 256) return launch_bn<256>(L, prm, s);
  return launch_bn<128>(L, prm, s);
}

}  // namespace fs
