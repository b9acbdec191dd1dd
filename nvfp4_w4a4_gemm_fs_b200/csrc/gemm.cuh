// Internal launch interface shared by the SpliceGEMM kernels and the ABI layer.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace fs {

// Output segments of one launch: weight rows (= output columns) [seg_n0[s], seg_n0[s+1]) use
// alpha[s] (projections that share an input, packed as adjacent row ranges).
constexpr int kMaxSegments = 8;
struct Segments {
  int n;                           // 1 .. kMaxSegments
  int n0[kMaxSegments + 1];        // first row of each segment, n0[n] = N
};

// Segment holding row `row` (segments are whole tiles, so any row of a tile will do).
__device__ __forceinline__ int segment_of(int row, const Segments& sg) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < kMaxSegments; ++i)
    if (i < sg.n && row >= sg.n0[i]) s = i;
  return s;
}

// Kernel parameters of the tensor-core path (plain: E = 1, offsets = null).
struct TcParams {
  int64_t M;
  int N, K, KT, ST, BN, n_tiles, E, kb4;
  int n_fast;         // tile order: 1 = N-tiles vary fastest (B stays in L2), 0 = M-tiles fastest
  int64_t a_groups;   // 128-row groups of the activation buffers (scale atoms past them are not read)
  const int64_t* offsets;
  int skip_small;     // experts: those with at most this many rows get no tiles (the decode kernel's)
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* alpha;     // [E] for experts, else [segments]
  Segments seg;
  void* Y;
  int64_t ldy;
  int out_bf16;
  uint32_t* err;
  uint64_t wait_ns;   // limit of every bounded wait
  int no_copies;      // failure-detection test hook: the producer issues no copies
};

// Host-side description of the operand buffers for tensor-map encoding.
struct TcLaunch {
  const void* xq;
  const void* wq;
  const void* xs;
  const void* ws;
  int64_t a_rows;     // rows of the activation buffers (padded rows for experts)
  int64_t b_rows;     // rows of the weight buffers (E * N for experts)
  int64_t y_rows;     // rows of Y
  int pp;               // columns of the side (BF16) operands
  int64_t xs_ld, ws_ld; // their leading dimensions in elements (0: pp)
  int bn;
  int64_t max_tiles;
};

fs_status launch_splice_gemm_tc(const TcLaunch& L, const TcParams& prm, cudaStream_t s);

// 2D K-major tensor map, 128-byte swizzle, box `box_inner` elements x `box_rows` rows.
fs_status make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t inner_elems, uint64_t rows,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows);

struct DecodeParams {
  int M, N, K, pp, kb4;
  const uint8_t* xq;
  const uint8_t* sfx;
  const uint16_t* xs;
  const uint8_t* wq;
  const uint8_t* sfw;
  const uint16_t* ws;
  const float* alpha;  // [segments]
  Segments seg;
  void* Y;
  int64_t ldy;
  int out_bf16;
  uint32_t* err;      // device error word (bounded-wait timeouts of the tensor-core decode kernel)
  uint64_t wait_ns;   // limit of every bounded wait
  int no_copies;      // failure-detection test hook: the producer issues no copies
  // fuse != 0: the kernel prepares the activations itself from bf16 X (xq, sfx, xs unused)
  int fuse;
  const uint16_t* x;
  int64_t ldx;
  const uint32_t* mask;
  int p;
  const float* gA;
  int residual;
  // grouped (offsets != null): experts with 1..small_max rows, E stacked weight operands of N rows,
  // packed activations in the grouped layout (each expert's rows from a 128-row boundary) with
  // a_rows rows in all; xq, sfx, xs, wq, sfw, ws, alpha as for fs_splice_gemm_grouped
  const int64_t* offsets;
  int E;
  int small_max;
  int64_t a_rows;
};

// Wait limits: the normal bound, and the short one of the failure-detection test option
// (FS_FAULT_NO_COPIES), under which every launch gives up its waits and reports a timeout.
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint64_t kFaultWaitLimitNs = 20000000ull;
inline uint64_t wait_limit_ns(uint32_t opts) { return (opts & FS_FAULT_NO_COPIES) ? kFaultWaitLimitNs : kWaitLimitNs; }

fs_status launch_splice_gemm_decode_tc(const DecodeParams& p, cudaStream_t s);

}  // namespace fs
