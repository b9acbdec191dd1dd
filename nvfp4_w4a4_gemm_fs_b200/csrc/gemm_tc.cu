// SpliceGEMM on the 5th-generation tensor cores (tcgen05), the large-M path.
//
// FourSight §4.2 Eq. 5 and §5.1 "Dual-path execution" (Fig. 6): the NVFP4 product runs as
// block-scaled MMAs, then the BF16 tiles of the protected slice (X_S, W'_S) are loaded into the
// SAME shared-memory stage buffers and their BF16 MMAs accumulate into the SAME FP32 TMEM
// accumulator; the epilogue moves TMEM to registers, multiplies by alpha once and stores Y.
//
// Persistent kernel, one CTA per SM.  Output tiles are 128 x BN per CTA.  With CG = 2 two CTAs of
// a cluster form a pair that computes a 256 x 256 tile with cta_group::2 MMAs: each CTA loads
// its own 128 rows of A and half (128 rows) of the B tile, the leader CTA issues the MMAs for
// both, and each CTA's TMEM receives its 128 output rows.  Halving B per CTA cuts the operand
// bytes per k-tile from 48 KB to 32 KB, which buys pipeline depth and L2->SM bandwidth.
//   warp 0      TMA producer: per k-tile one 128x128-byte box of A and a (BN/CG)x128-byte box of
//               B (128-byte swizzle), plus the tile's UE4M3 scale atoms (plain bulk copies of
//               this CTA's A rows and all BN columns of B); the BF16 side tiles use the same
//               boxes, 64 bf16 wide.
//   warp 1      allocates TMEM; one thread of the leader issues tcgen05.mma: kind::mxf4nvf4
//               (K = 64 per instruction) over all of K, then kind::f16 (K = 16) over the
//               protected slice, and commits the stage / scale / accumulator barriers.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns, x alpha, staged in shared memory
//               and written with TMA stores.
//   warps 6..9  scale warps: tcgen05.st of each k-tile's block scales into TMEM.
// Accumulators (BN = 256) overlap in TMEM: tile i uses columns [128*(i&1), 128*(i&1) + 256), so
// consecutive tiles share columns [128, 256).  The epilogue loads that shared half into
// registers first and releases it at once; the next tile's MMAs then run while the epilogue
// drains the other half and the stores, so output traffic overlaps the main loop.
// Every mbarrier wait is bounded; on expiry the kernel records a timeout in the error word,
// stops issuing work, waits (bounded) for its own copies in flight and still releases TMEM.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace fs {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

namespace {

constexpr int kBM = 128;
constexpr int kThreads = 320;                  // producer, MMA, 4 epilogue and 4 scale warps
constexpr int kMaxExperts = 256;
constexpr uint64_t kDrainNs = 50000000ull;      // 50 ms bound on each wait of the abort path

#ifndef FS_TC_PAIR_STAGES
#define FS_TC_PAIR_STAGES 5
#endif
#ifndef FS_TC_PAIR_STAGING
#define FS_TC_PAIR_STAGING 2
#endif
#ifndef FS_TC_SF_BUFS
#define FS_TC_SF_BUFS 2
#endif
#ifndef FS_TC_SF_SPLIT
#define FS_TC_SF_SPLIT 1
#endif
#ifndef FS_TC_OVERLAP_ACC
#define FS_TC_OVERLAP_ACC 1
#endif

template <int BN, int CG>
struct Cfg {
  static_assert(CG == 1 || (CG == 2 && BN == 256), "CTA pairs use 256 x 256 tiles");
  static constexpr int B_ROWS = BN / CG;               // rows of the B tile this CTA loads
  static constexpr int A_BYTES = kBM * 128;            // 128 rows x 128 bytes (256 fp4 or 64 bf16)
  static constexpr int B_BYTES = B_ROWS * 128;
  static constexpr int SFA_BYTES = kBM * 16;           // 16 scales per row per k-tile
  static constexpr int SFB_BYTES = BN * 16;            // every CTA holds the scales of all BN columns
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int TX_BYTES = CG * (A_BYTES + B_BYTES);   // A/B bytes landing per stage in the pair
  static constexpr int STAGES = CG == 2 ? FS_TC_PAIR_STAGES : (BN == 256 ? 3 : 4);
  static constexpr int STAGING_BUFS = CG == 2 ? FS_TC_PAIR_STAGING : 3;   // per epilogue warp
  // Accumulators: BN = 256 overlaps two 256-column buffers in 384 columns (OVERLAP; otherwise
  // one 256-column buffer); BN = 128 keeps two disjoint 128-column buffers.  With two buffers
  // tile i starts at column 128 * (i & 1).
  static constexpr bool OVERLAP = BN == 128 || FS_TC_OVERLAP_ACC;
  static constexpr int ACC_SLOTS = BN == 256 ? 1 : 2;  // accumulator barrier pairs
  static constexpr int ACC_SPAN = BN == 256 ? (OVERLAP ? 384 : 256) : 256;
  // Scale factors in TMEM: SF_BUFS k-tiles' worth, handed over in units of MPU MMAs (SF_SPLIT
  // units per k-tile) that rotate over a ring of SF_UNITS slots.  The scales of unit u may be
  // written once the MMAs of unit u - SF_UNITS are done.  Finer units give the scale warps more
  // slack but add handoffs; on B200 one unit per k-tile measured fastest (two: +13%, four: +40%
  // on an 8192 x 4096 x 4096 GEMM).
  static constexpr int SF_BUFS = FS_TC_SF_BUFS;
  static constexpr int SF_SPLIT = FS_TC_SF_SPLIT;
  static constexpr int MPU = 4 / SF_SPLIT;                 // MMAs per scale unit
  static constexpr int SF_COLS = 16 + 4 * (BN / 32);       // per k-tile: SFA 4 MMAs x 4 columns; SFB 4 MMAs x BN/32
  static constexpr int UNIT_COLS = SF_COLS / SF_SPLIT;     // SFA MPU x 4, then SFB MPU x BN/32
  static constexpr int SF_UNITS = SF_BUFS * SF_SPLIT;
  static constexpr int SF_COL = ACC_SPAN;
  static constexpr int TMEM_COLS = 512;
  static_assert(SF_SPLIT == 1 || SF_SPLIT == 2 || SF_SPLIT == 4, "scale units divide the k-tile's 4 MMAs");
  static_assert(ACC_SPAN + SF_UNITS * UNIT_COLS <= TMEM_COLS, "TMEM budget");
  static constexpr int STAGING_BYTES = 4 * STAGING_BUFS * 4096;  // 4 warps x buffers x (32 rows x 128 B)
  // full, sf_loaded, empty per stage; acc_full, acc_empty per slot; sf_full, sf_empty per scale
  // unit slot; drain
  static constexpr int NUM_BARS = 3 * STAGES + 2 * ACC_SLOTS + 2 * SF_UNITS + 1;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGING_BYTES + 8 * NUM_BARS + 16 +
                                    2 * 4 * (kMaxExperts + 1);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget of one CTA");
};

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait with a deadline (`limit_ns`) and an abort flag shared by the CTA's roles.
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

// Abort path: wait up to `limit_ns` for one phase of a barrier, ignoring the abort flag.
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = now_ns();
  while (!ptx::mbar_try_wait(bar, parity))
    if (now_ns() - t0 > limit_ns) return;
}

struct TileMap {
  int e;           // expert
  int64_t arow;    // first row of this CTA's A rows in the packed activation buffers
  int64_t yrow;    // first output row of this CTA
  int rows;        // valid rows of this CTA (may be <= 0 for the second CTA of a pair)
  int64_t brow;    // first row of the tile in the (stacked) weight buffers
  int n0;          // first output column
};

// Tile t -> rows / columns.  cum_m[e] counts the (kBM * CG)-row M-tiles before expert e, cum_g[e]
// the 128-row groups before it (expert e's packed rows start at row 128 cum_g[e]).  The
// operand whose tiles vary fastest is read whole by every wave of CTAs, so the order keeps the
// smaller operand there (it stays in L2) and streams the larger one once: M-tiles fastest when A
// is the smaller, N-tiles fastest otherwise and for experts.
template <int CG>
__device__ __forceinline__ TileMap map_tile(int t, const TcParams& p, const int* cum_m, const int* cum_g, int rank) {
  TileMap m;
  const int total_m = cum_m[p.E];
  const int mt = p.n_fast ? t / p.n_tiles : t % total_m;
  const int nt = p.n_fast ? t % p.n_tiles : t / total_m;
  int lo = 0, hi = p.E - 1;                   // expert with cum_m[e] <= mt < cum_m[e+1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cum_m[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  m.e = lo;
  const int local = mt - cum_m[lo];
  if (p.offsets) {
    // A pair's second CTA may start past the expert's last row: it then has no valid rows, reads
    // zero fill (or a following expert's rows) and stores nothing.
    const int64_t r0 = p.offsets[lo], r1 = p.offsets[lo + 1];
    const int64_t off = static_cast<int64_t>(local) * (kBM * CG) + rank * kBM;
    m.arow = static_cast<int64_t>(cum_g[lo]) * kBM + off;
    m.yrow = r0 + off;
    const int64_t left = r1 - m.yrow;
    m.rows = static_cast<int>(left < kBM ? left : kBM);
  } else {
    m.arow = static_cast<int64_t>(mt) * (kBM * CG) + rank * kBM;
    m.yrow = m.arow;
    const int64_t left = p.M - m.arow;
    m.rows = static_cast<int>(left < kBM ? (left < 0 ? 0 : left) : kBM);
  }
  m.n0 = nt * p.BN;
  m.brow = static_cast<int64_t>(lo) * p.N + m.n0;
  return m;
}

template <int BN, int CG>
__global__ void __launch_bounds__(kThreads, 1)
splice_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                      const __grid_constant__ CUtensorMap tmY, const TcParams p) {
  using C = Cfg<BN, CG>;
  extern __shared__ uint8_t smem_raw[];
  // The same offset in both CTAs of a pair: the dynamic shared memory base is identical.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;           // 1024-byte aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::STAGING_BYTES);   // A/B landed (leader's counts both CTAs)
  uint64_t* sfl = full + C::STAGES;                // this CTA's scale atoms landed
  uint64_t* empty = sfl + C::STAGES;               // the MMAs reading a stage are done
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + C::ACC_SLOTS;   // leader: released by the epilogues of both CTAs
  uint64_t* sf_full = acc_empty + C::ACC_SLOTS;    // leader: scales of a unit are in TMEM (both CTAs)
  uint64_t* sf_empty = sf_full + C::SF_UNITS;      // the MMAs reading a scale slot are done
  uint64_t* drain = sf_empty + C::SF_UNITS;        // leader: all MMAs issued so far are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* cum_m = reinterpret_cast<int*>(tmem_slot + 4);
  int* cum_g = cum_m + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = CG == 2 ? static_cast<int>(ptx::cluster_ctarank()) : 0;
  const int unit = CG == 2 ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);   // CTA or pair
  const int nunits = CG == 2 ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  auto A_at = [&](int s) { return stages + s * C::STAGE_BYTES; };
  auto B_at = [&](int s) { return stages + s * C::STAGE_BYTES + C::A_BYTES; };
  auto SFA_at = [&](int s) { return stages + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES; };
  auto SFB_at = [&](int s) { return stages + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES + C::SFA_BYTES; };
  // Leader-CTA barriers as shared::cluster addresses (the CTA's own address when CG = 1).
  auto leader = [&](uint64_t* bar) { return CG == 2 ? ptx::mapa_shared(ptx::smem_u32(bar), 0) : ptx::smem_u32(bar); };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    cum_m[0] = 0;
    cum_g[0] = 0;
    if (p.offsets) {
      for (int e = 0; e < p.E; ++e) {
        const int64_t rows = p.offsets[e + 1] - p.offsets[e];
        cum_m[e + 1] = cum_m[e] + (rows <= p.skip_small ? 0 : static_cast<int>((rows + kBM * CG - 1) / (kBM * CG)));
        cum_g[e + 1] = cum_g[e] + static_cast<int>((rows + kBM - 1) / kBM);
      }
    } else {
      cum_m[1] = static_cast<int>((p.M + kBM * CG - 1) / (kBM * CG));
    }
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(full + s, 1);
      ptx::mbar_init(sfl + s, 1);
      ptx::mbar_init(empty + s, 1);
    }
    for (int a = 0; a < C::ACC_SLOTS; ++a) { ptx::mbar_init(acc_full + a, 1); ptx::mbar_init(acc_empty + a, 4 * CG); }
    for (int b = 0; b < C::SF_UNITS; ++b) { ptx::mbar_init(sf_full + b, 4 * CG); ptx::mbar_init(sf_empty + b, 1); }
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tmA); ptx::prefetch_tensormap(&tmB); ptx::prefetch_tensormap(&tmY);
    if (p.ST > 0) { ptx::prefetch_tensormap(&tmSA); ptx::prefetch_tensormap(&tmSB); }
  }
  if (warp == 1) {
    ptx::tmem_alloc<CG>(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish<CG>();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) ptx::cluster_sync();     // the peer's barriers exist before anyone signals them
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total_tiles = cum_m[p.E] * p.n_tiles;
  const int ktiles = p.KT + p.ST;
  // 128-row scale groups of the activation buffer (for experts: the padded rows it holds)
  const int64_t m_groups = p.offsets ? p.a_groups : (p.M + kBM - 1) / kBM;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // (p.no_copies, the failure-detection test hook: nothing is issued, so every other role's
    // first wait runs out and the kernel takes its abort path with no copy in flight)
    if (lane == 0 && !p.no_copies) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      uint32_t sfl_bits = 0, last_fp4 = 0;   // per stage: parity of its next FP4 use; last use was FP4
      bool ok = true;
      for (int t = unit; t < total_tiles && ok; t += nunits) {
        const TileMap m = map_tile<CG>(t, p, cum_m, cum_g, rank);
        // Scale atoms of rows past the end of the activation buffer (a dense problem's last pair,
        // an expert's last pair at the end of the buffer) are not there: skip them (those output
        // rows are discarded).
        const bool sfa_ok = (m.arow / kBM) < m_groups;
        const int64_t brow = m.brow + rank * C::B_ROWS;
        for (int kt = 0; kt < ktiles; ++kt) {
          if (!wait_bar(empty + stage, phase ^ 1, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
          const bool fp4 = kt < p.KT;
          last_fp4 = (last_fp4 & ~(1u << stage)) | (static_cast<uint32_t>(fp4) << stage);
          if (fp4) {
            sfl_bits ^= 1u << stage;
            ptx::mbar_arrive_expect_tx(sfl + stage, (sfa_ok ? C::SFA_BYTES : 0) + C::SFB_BYTES);
            if (sfa_ok)
              ptx::bulk_load(SFA_at(stage), p.sfa + ((m.arow / kBM) * p.kb4 + kt * 4) * 512, C::SFA_BYTES, sfl + stage);
#pragma unroll
            for (int rg = 0; rg < BN / 128; ++rg)
              ptx::bulk_load(SFB_at(stage) + rg * 2048, p.sfb + ((m.brow / kBM + rg) * p.kb4 + kt * 4) * 512, 2048,
                             sfl + stage);
          }
          if (rank == 0) ptx::mbar_arrive_expect_tx(full + stage, C::TX_BYTES);
          const CUtensorMap* ma = fp4 ? &tmA : &tmSA;
          const CUtensorMap* mb = fp4 ? &tmB : &tmSB;
          const int32_t kx = fp4 ? kt * 128 : (kt - p.KT) * 64;
          if constexpr (CG == 1) {
            ptx::tma_load_2d(A_at(stage), ma, kx, static_cast<int32_t>(m.arow), full + stage);
            ptx::tma_load_2d(B_at(stage), mb, kx, static_cast<int32_t>(brow), full + stage);
          } else {
            const uint32_t bar = leader(full + stage);
            ptx::tma_load_2d_pair(A_at(stage), ma, kx, static_cast<int32_t>(m.arow), bar);
            ptx::tma_load_2d_pair(B_at(stage), mb, kx, static_cast<int32_t>(brow), bar);
          }
          ++issued;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      {
        // Copies issued but possibly not landed: the last min(issued, STAGES) stages.  Drained
        // whether this loop finished or gave up, since another role may still give up after it
        // finished, and the CTA must not exit with a copy landing in its shared memory.  The
        // waits replay the (stage, parity) pairs the consumers wait on, and no later phase can
        // complete once nothing more is issued; on the normal path they are met before the last
        // tile's epilogue starts.  The leader can observe both CTAs' A/B bytes; every CTA
        // observes its own scale atoms.
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < C::STAGES && i < issued; ++i) {
          if (--s < 0) { s = C::STAGES - 1; ph ^= 1; }
          if (rank == 0) drain_bar(full + s, ph, kDrainNs);
          if ((last_fp4 >> s) & 1) drain_bar(sfl + s, ((sfl_bits >> s) & 1) ^ 1, kDrainNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_f4 = ptx::idesc_nvf4(kBM * CG, BN);
      constexpr uint32_t idesc_bf = ptx::idesc_bf16(kBM * CG, BN);
      int stage = 0, acc = 0, sf_unit = 0, i = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = unit; t < total_tiles && ok; t += nunits, ++i) {
        if (!wait_bar(acc_empty + acc, acc_phase ^ 1, abort_flag, p.err, p.wait_ns)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(C::OVERLAP ? (i & 1) * 128 : 0);
        for (int kt = 0; kt < ktiles; ++kt) {
          if (!wait_bar(full + stage, phase, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t adesc = ptx::desc_kmajor_sw128(ptx::smem_u32(A_at(stage)));
          const uint64_t bdesc = ptx::desc_kmajor_sw128(ptx::smem_u32(B_at(stage)));
          if (kt < p.KT) {
#pragma unroll
            for (int h = 0; h < C::SF_SPLIT; ++h) {
              const int slot = sf_unit % C::SF_UNITS;
              if (!wait_bar(sf_full + slot, (sf_unit / C::SF_UNITS) & 1, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
              ptx::tc_fence_after();
              const uint32_t sf = tmem + C::SF_COL + slot * C::UNIT_COLS;
#pragma unroll
              for (int jj = 0; jj < C::MPU; ++jj) {
                const int j = h * C::MPU + jj;
                ptx::tc_mma_nvf4<CG>(d, adesc + 2 * j, bdesc + 2 * j, idesc_f4, sf + 4 * jj,
                                     sf + 4 * C::MPU + (BN / 32) * jj, (kt | j) != 0);
              }
              ptx::tc_commit<CG>(sf_empty + slot);
              ++sf_unit;
            }
            if (!ok) break;
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) ptx::tc_mma_bf16<CG>(d, adesc + 2 * j, bdesc + 2 * j, idesc_bf, (kt | j) != 0);
          }
          ptx::tc_commit<CG>(empty + stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        ptx::tc_commit<CG>(acc_full + acc);
        if (++acc == C::ACC_SLOTS) { acc = 0; acc_phase ^= 1; }
      }
      // Every MMA issued above has completed before TMEM can be released.
      ptx::tc_commit<CG>(drain);
      drain_bar(drain, 0, p.wait_ns);
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------------ scale warps
    // Each warp owns one TMEM lane quadrant and writes, for every FP4 k-tile, the block scales
    // of its 32 lanes exactly as tcgen05.cp.32x128b.warpx4 would lay them out: lane l, columns
    // 4c..4c+3 of an atom's slot hold the atom's 16-byte row l (SFA: one atom per MMA; SFB: the
    // BN/128 row-group atoms side by side).  A k-tile's atoms are read from shared memory first,
    // then written unit by unit as each ring slot frees up.
    // The scale-atom barrier of a stage completes one phase per FP4 use of that stage only, so
    // its parity is tracked per stage (the producer keeps the same bits).
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int stage = 0, sf_unit = 0;
    uint32_t sfl_bits = 0;
    bool ok = true;
    for (int t = unit; t < total_tiles && ok; t += nunits) {
      for (int kt = 0; kt < ktiles; ++kt) {
        if (kt < p.KT) {
          if (!wait_bar(sfl + stage, (sfl_bits >> stage) & 1, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
          sfl_bits ^= 1u << stage;
          const uint8_t* sfa = SFA_at(stage);
          const uint8_t* sfb = SFB_at(stage);
          uint4 a[4], b0[4], b1[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a[j] = *reinterpret_cast<const uint4*>(sfa + 512 * j + lane * 16);
            b0[j] = *reinterpret_cast<const uint4*>(sfb + 512 * j + lane * 16);
            if constexpr (BN == 256) b1[j] = *reinterpret_cast<const uint4*>(sfb + 2048 + 512 * j + lane * 16);
          }
#pragma unroll
          for (int h = 0; h < C::SF_SPLIT; ++h) {
            const int slot = sf_unit % C::SF_UNITS;
            if (!wait_bar(sf_empty + slot, ((sf_unit / C::SF_UNITS) & 1) ^ 1, abort_flag, p.err, p.wait_ns)) { ok = false; break; }
            const uint32_t col = tmem + lane_base + C::SF_COL + slot * C::UNIT_COLS;
#pragma unroll
            for (int jj = 0; jj < C::MPU; ++jj) {
              const int j = h * C::MPU + jj;
              ptx::tmem_st_32x32b_x4(col + 4 * jj, a[j].x, a[j].y, a[j].z, a[j].w);
              if constexpr (BN == 256) ptx::tmem_st_32x32b_x8(col + 4 * C::MPU + 8 * jj, b0[j], b1[j]);
              else ptx::tmem_st_32x32b_x4(col + 4 * C::MPU + 4 * jj, b0[j].x, b0[j].y, b0[j].z, b0[j].w);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if constexpr (CG == 1) ptx::mbar_arrive(sf_full + slot);
              else ptx::mbar_arrive_remote(leader(sf_full + slot));
            }
            ++sf_unit;
          }
          if (!ok) break;
        }
        if (++stage == C::STAGES) stage = 0;
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // Part 1: the 128 accumulator columns the next tile will overwrite are loaded into registers
    // and released at once (BN = 128: the whole tile).  Part 2 (BN = 256): the other 128 columns,
    // 32 at a time, while the next tile's MMAs run.  Each 32 x 32 chunk is scaled by alpha,
    // staged in shared memory with the TMA swizzle and written by a TMA store.  In a partial tile
    // of an expert (rows that end inside the output) the warp whose 32 rows hold the expert's last
    // row stores directly, since its box would cross into the next expert's rows; warps whose rows
    // all belong to the expert still use TMA.
    const int quad = warp & 3;                  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;           // row of the tile held by this thread
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    uint8_t* stage_buf = staging + quad * C::STAGING_BUFS * 4096;
    int acc = 0, nbuf = 0, i = 0;
    uint32_t acc_phase = 0;
    for (int t = unit; t < total_tiles; t += nunits, ++i) {
      const TileMap m = map_tile<CG>(t, p, cum_m, cum_g, rank);
      if (!wait_bar(acc_full + acc, acc_phase, abort_flag, p.err, p.wait_ns)) break;
      ptx::tc_fence_after();
      const float alpha = p.alpha ? __ldg(p.alpha + (p.offsets ? m.e : segment_of(m.n0, p.seg))) : 1.0f;
      const bool use_tma = !p.offsets || (quad + 1) * 32 <= m.rows;
      const bool row_ok = row < m.rows;
      const int64_t yrow = m.yrow + row;
      const int base = C::OVERLAP ? (i & 1) * 128 : 0;
      // TMEM column and output column of each part.
      const int p1_tcol = BN == 256 ? 128 : base;
      const int p1_ocol = BN == 256 ? 128 - base : 0;
      const int p2_tcol = base == 0 ? 0 : 256;
      const int p2_ocol = base == 0 ? 0 : 128;

      auto emit = [&](const uint32_t (&r)[32], int col0) {
        if (col0 >= p.N) return;
        if (use_tma) {
          if (quad * 32 >= m.rows) return;              // this warp's rows are all past the end
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
          // Y's base and row pitch are 16-byte aligned (the Y tensor map requires it) and col0 is
          // a multiple of 32, so whole 32-column chunks go out as 16-byte stores.
          const bool whole = col0 + 32 <= p.N;
          if (p.out_bf16) {
            uint16_t* y = static_cast<uint16_t*>(p.Y) + yrow * p.ldy + col0;
            if (whole) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 4; ++h)
                  w[h] = static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[8 * j + 2 * h]) * alpha)) |
                         (static_cast<uint32_t>(f32_to_bf16_bits(__uint_as_float(r[8 * j + 2 * h + 1]) * alpha)) << 16);
                *reinterpret_cast<uint4*>(y + 8 * j) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (col0 + c < p.N) y[c] = f32_to_bf16_bits(__uint_as_float(r[c]) * alpha);
            }
          } else {
            float* y = static_cast<float*>(p.Y) + yrow * p.ldy + col0;
            if (whole) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(y + 4 * j) =
                    make_float4(__uint_as_float(r[4 * j]) * alpha, __uint_as_float(r[4 * j + 1]) * alpha,
                                __uint_as_float(r[4 * j + 2]) * alpha, __uint_as_float(r[4 * j + 3]) * alpha);
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (col0 + c < p.N) y[c] = __uint_as_float(r[c]) * alpha;
            }
          }
        }
      };

      // The accumulator columns the next tile writes have been read: hand them back.
      auto release = [&]() {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CG == 1) ptx::mbar_arrive(acc_empty + acc);
          else ptx::mbar_arrive_remote(leader(acc_empty + acc));
        }
      };
      {
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld_32x32b_x32(lane_addr + p1_tcol + c * 32, r[c]);
        ptx::tmem_ld_wait();
        if constexpr (C::OVERLAP) release();
#pragma unroll
        for (int c = 0; c < 4; ++c) emit(r[c], m.n0 + p1_ocol + c * 32);
      }
      if constexpr (BN == 256) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          ptx::tmem_ld_32x32b_x32(lane_addr + p2_tcol + c * 32, r);
          ptx::tmem_ld_wait();
          if (!C::OVERLAP && c == 3) release();
          emit(r, m.n0 + p2_ocol + c * 32);
        }
      }
      if (++acc == C::ACC_SLOTS) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) {
    // Neither CTA leaves (or frees TMEM) while the other may still signal its barriers or, for
    // the leader's MMAs, write its TMEM.
    ptx::cluster_sync();
  }
  if (*abort_flag) {
    // Copies of the peer that this CTA could not observe: give them time to land.
    const uint64_t t0 = now_ns();
    while (now_ns() - t0 < 100000ull) {}
  }
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc<CG>(tmem, C::TMEM_COLS);
  }
}

template <int BN, int CG>
fs_status set_smem_attr() {
  static PerDevice<int> cache;
  return set_max_dynamic_smem(cache, reinterpret_cast<const void*>(splice_gemm_tc_kernel<BN, CG>),
                              Cfg<BN, CG>::SMEM_BYTES, "fs_splice_gemm: smem attribute");
}

// Number of CTA pairs that can be resident at once on the current device (clusters must fit
// inside a GPC, so this can be below half the SM count); 0 when the query fails.
int pair_slots() {
  static PerDevice<int> cache;
  int n = 0;
  if (cache.get(current_device(), &n, [](int* out) {
    *out = 0;
    if (set_smem_attr<256, 2>() != FS_OK) return false;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(sm_count() & ~1));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Cfg<256, 2>::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, splice_gemm_tc_kernel<256, 2>, &cfg) == cudaSuccess && c > 0) *out = c;
    else cudaGetLastError();
    return true;
  }))
    return n;
  return 0;
}

template <int BN, int CG>
fs_status launch_cfg(const TcLaunch& L, TcParams prm, int units, cudaStream_t s) {
  using C = Cfg<BN, CG>;
  fs_status st = set_smem_attr<BN, CG>();
  if (st != FS_OK) return st;
  prm.BN = BN;
  prm.n_tiles = static_cast<int>(ceil_div(prm.N, BN));
  // N-tiles fastest when the weights (B) are the smaller operand of a dense problem, and for experts:
  // then the tiles in flight belong to a few consecutive experts, whose weights stay in L2 while
  // each of their 128-row activation tiles meets every N-tile.
  prm.n_fast = (prm.offsets || (prm.E == 1 && static_cast<int64_t>(prm.N) <= L.a_rows)) ? 1 : 0;
  prm.a_groups = ceil_div(L.a_rows, kBM);
  CUtensorMap tmA, tmB, tmSA, tmSB;
  const uint64_t kbytes = static_cast<uint64_t>(prm.K) / 2;
  if (prm.KT > 0) {
    st = make_map(&tmA, L.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, L.a_rows, kbytes, 128, kBM);
    if (st == FS_OK) st = make_map(&tmB, L.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, L.b_rows, kbytes, 128, C::B_ROWS);
    if (st != FS_OK) return st;
  }
  if (prm.ST > 0) {
    const uint64_t pp = static_cast<uint64_t>(L.pp);
    const uint64_t lds = static_cast<uint64_t>(L.xs_ld ? L.xs_ld : L.pp), ldw = static_cast<uint64_t>(L.ws_ld ? L.ws_ld : L.pp);
    st = make_map(&tmSA, L.xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, L.a_rows, lds * 2, 64, kBM);
    if (st == FS_OK) st = make_map(&tmSB, L.ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pp, L.b_rows, ldw * 2, 64, C::B_ROWS);
    if (st != FS_OK) return st;
  }
  if (prm.KT == 0) {            // BF16 only: the FP4 maps are never used for loads
    tmA = tmSA;
    tmB = tmSB;
  } else if (prm.ST == 0) {
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
  if constexpr (CG == 1) {
    splice_gemm_tc_kernel<BN, 1><<<units, kThreads, C::SMEM_BYTES, s>>>(tmA, tmB, tmSA, tmSB, tmY, prm);
  } else {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * units));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, splice_gemm_tc_kernel<256, 2>, tmA, tmB, tmSA, tmSB, tmY, prm);
    if (e != cudaSuccess) return cuda_status(e, "fs_splice_gemm (tensor-core path, CTA pairs)");
  }
  FS_CHECK_LAUNCH("fs_splice_gemm (tensor-core path)");
  return FS_OK;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// Host: tensor maps and launch
// ------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

fs_status launch_splice_gemm_tc(const TcLaunch& L, const TcParams& prm, cudaStream_t s) {
  if (prm.E > kMaxExperts) return fail(FS_ERR_UNSUPPORTED, "fs_splice_gemm: at most %d experts", kMaxExperts);
  const int64_t m_tiles = ceil_div(L.a_rows, kBM);
  // Problems with N % 256 == 0 and at least two 128-row tiles run on CTA pairs (experts: each
  // expert's rows in 256-row pair tiles, at most one more pair tile per expert than dense).
  if (L.bn == 256 && m_tiles >= 2) {
    const int slots = pair_slots();
    if (slots > 0) {
      const int64_t tiles = (ceil_div(L.a_rows, 2 * kBM) + (prm.offsets ? prm.E : 0)) * (prm.N / 256);
      const int units = static_cast<int>(std::min<int64_t>(tiles, slots));
      return launch_cfg<256, 2>(L, prm, units, s);
    }
  }
  const int units = static_cast<int>(std::min<int64_t>(std::max<int64_t>(L.max_tiles, 1), sm_count()));
  if (L.bn == 256) return launch_cfg<256, 1>(L, prm, units, s);
  return launch_cfg<128, 1>(L, prm, units, s);
}

}  // namespace fs
