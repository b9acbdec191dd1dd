// SpliceGEMM decode path (M <= 16 tokens): a weight-streaming kernel.
//
// FourSight §5.1 "Dual-path execution" describes a low-latency decode path for small M; here the
// whole product streams the packed NVFP4 weights once with 128-bit loads, dequantises them in
// registers and multiplies on the warp-level tensor cores:
//   * a quad of threads covers 128 contiguous bytes (256 elements) of one weight row; each
//     thread's 32 bytes feed its MMA fragment slots directly, the K order inside a chunk being
//     permuted identically for weights and activations (thread c of the quad owns elements
//     64c .. 64c+63 of the chunk; in k-step j it supplies elements 64c+4j .. 64c+4j+3);
//   * E2M1 codes and UE4M3 scales convert exactly to f16 (a product of the two has at most 6
//     significant bits and lies in [2^-10, 2688]), so the f16 MMA with FP32 accumulation sums the
//     same dequantised values as the tensor-core path;
//   * the protected slice X_S W'_S^T runs as BF16 MMAs into the same FP32 accumulators;
//   * the warps of a CTA split K, each with its next chunk's loads in flight; the partial sums
//     are reduced in shared memory, scaled once by alpha and stored.
#include "common.cuh"
#include "gemm.cuh"

namespace fs {
namespace {


__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(r) : "r"(byte));
  return r;
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t r;
  asm("{\n\t.reg .b16 h;\n\tcvt.u16.u32 h, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}" : "=r"(r) : "r"(two_bytes));
  return r;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 32 packed bytes (64 elements) of one row plus its 4 scale bytes, dequantised lazily.
struct Span {
  uint4 lo, hi;     // bytes 0..15, 16..31
  uint32_t sf;      // 4 UE4M3 scales (blocks 0..3 of the span)
};

__device__ __forceinline__ uint32_t span_word(const Span& s, int w) {
  switch (w) {
    case 0: return s.lo.x; case 1: return s.lo.y; case 2: return s.lo.z; case 3: return s.lo.w;
    case 4: return s.hi.x; case 5: return s.hi.y; case 6: return s.hi.z; default: return s.hi.w;
  }
}

// f16x2 of elements 4j+2h, 4j+2h+1 of the span (h = 0 or 1), scaled by their block scale.
__device__ __forceinline__ uint32_t span_pair(const Span& s, int j, int h, uint32_t scale2) {
  const uint32_t word = span_word(s, j >> 1);
  const uint32_t byte = (word >> (((j & 1) * 2 + h) * 8)) & 0xFFu;
  return hmul2(e2m1x2_to_f16x2(byte), scale2);
}

__device__ __forceinline__ Span load_span(const uint8_t* q_row, const uint8_t* sf, int64_t row, int k0, int kb4) {
  Span s;
  const uint4* p = reinterpret_cast<const uint4*>(q_row + k0 / 2);
  s.lo = __ldg(p);
  s.hi = __ldg(p + 1);
  s.sf = __ldg(reinterpret_cast<const uint32_t*>(sf + sf_offset(row, k0 / 16, kb4)));
  return s;
}

// scales of blocks b and b broadcast into both halves of an f16x2
__device__ __forceinline__ uint32_t scale_pair(uint32_t sf4, int b) {
  const uint32_t byte = (sf4 >> (8 * b)) & 0xFFu;
  return e4m3x2_to_f16x2(byte | (byte << 8));
}

constexpr int kRowsPerWarp = 16;

struct ChunkData {
  Span wa, wb, x0, x1;
};

template <int NT>
__device__ __forceinline__ ChunkData load_chunk(const DecodeParams& p, const uint8_t* wA, const uint8_t* wB,
                                                int64_t rowA, int64_t rowB, int tok0, int tok1, bool t0ok,
                                                bool t1ok, int k0) {
  ChunkData d;
  const int64_t kbytes = p.K / 2;
  d.wa = load_span(wA, p.sfw, rowA, k0, p.kb4);
  d.wb = load_span(wB, p.sfw, rowB, k0, p.kb4);
  d.x0.lo = d.x0.hi = make_uint4(0, 0, 0, 0);
  d.x0.sf = 0;
  d.x1 = d.x0;
  if (t0ok) d.x0 = load_span(p.xq + tok0 * kbytes, p.sfx, tok0, k0, p.kb4);
  if (NT == 2 && t1ok) d.x1 = load_span(p.xq + tok1 * kbytes, p.sfx, tok1, k0, p.kb4);
  return d;
}

template <int NT>
__device__ __forceinline__ void mma_chunk(const ChunkData& d, float (&acc)[NT][4]) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {                 // the span's 4 blocks, 4 k-steps each
    const uint32_t ssa = scale_pair(d.wa.sf, b), ssb = scale_pair(d.wb.sf, b);
    const uint32_t sx0 = scale_pair(d.x0.sf, b);
    const uint32_t sx1 = NT == 2 ? scale_pair(d.x1.sf, b) : 0u;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = 4 * b + jj;
      const uint32_t a0 = span_pair(d.wa, j, 0, ssa), a2 = span_pair(d.wa, j, 1, ssa);
      const uint32_t a1 = span_pair(d.wb, j, 0, ssb), a3 = span_pair(d.wb, j, 1, ssb);
      mma_f16(acc[0], a0, a1, a2, a3, span_pair(d.x0, j, 0, sx0), span_pair(d.x0, j, 1, sx0));
      if (NT == 2) mma_f16(acc[NT - 1], a0, a1, a2, a3, span_pair(d.x1, j, 0, sx1), span_pair(d.x1, j, 1, sx1));
    }
  }
}

// Grid: one CTA per 16 output features.  The WARPS warps of a CTA split K in 256-element chunks
// (warp w takes chunks w, w+WARPS, ...), each keeping its next chunk's loads in flight; the
// partial sums are reduced in shared memory, the protected BF16 slice is added by the warps
// (one 16-wide k-step each), and warp 0 scales by alpha and stores Y.
template <int NT, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
splice_gemm_decode_kernel(const DecodeParams p) {
  __shared__ float red[WARPS][32][4 * NT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kRowsPerWarp;
  const int64_t rowA = n0 + g, rowB = n0 + g + 8;
  const int64_t kbytes = p.K / 2;
  // Programmatic dependent launch: let the next kernel in the stream start its own prologue now,
  // and pull this CTA's weight rows (and their BF16 protected columns) into L2 while the previous
  // kernel may still be running.  An L2 prefetch is safe whatever that kernel writes (L2 is
  // coherent); every real load and store below comes after griddepcontrol.wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp == 0 && lane < kRowsPerWarp && n0 + lane < p.N) {
    const uint8_t* row = p.wq + (n0 + lane) * kbytes;
    for (int64_t off = 0; off < kbytes; off += 16384) {
      const uint32_t bytes = static_cast<uint32_t>(kbytes - off < 16384 ? kbytes - off : 16384);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(row + off), "r"(bytes) : "memory");
    }
    if (p.pp > 0)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.ws + (n0 + lane) * p.pp),
                   "r"(static_cast<uint32_t>(p.pp * 2)) : "memory");
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint8_t* wA = p.wq + rowA * kbytes;
  const uint8_t* wB = p.wq + rowB * kbytes;
  const int tok0 = g, tok1 = g + 8;
  const bool t0ok = tok0 < p.M, t1ok = tok1 < p.M;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;

  const int chunks = p.K / 256;
  if (warp < chunks) {
    ChunkData cur = load_chunk<NT>(p, wA, wB, rowA, rowB, tok0, tok1, t0ok, t1ok, warp * 256 + c * 64);
    for (int ch = warp; ch < chunks; ch += WARPS) {
      ChunkData nxt;
      const bool more = ch + WARPS < chunks;
      if (more) nxt = load_chunk<NT>(p, wA, wB, rowA, rowB, tok0, tok1, t0ok, t1ok, (ch + WARPS) * 256 + c * 64);
      mma_chunk<NT>(cur, acc);
      if (more) cur = nxt;
    }
  }
  // protected slice in BF16 (natural K order), one 16-wide k-step per warp
  if (p.pp > 0) {
    const uint32_t* wsA = reinterpret_cast<const uint32_t*>(p.ws + rowA * p.pp);
    const uint32_t* wsB = reinterpret_cast<const uint32_t*>(p.ws + rowB * p.pp);
    for (int ks = warp; ks < p.pp / 16; ks += WARPS) {
      const int e0 = ks * 8 + c;                   // 32-bit word index of elements 16ks + 2c
      const uint32_t a0 = __ldg(wsA + e0), a2 = __ldg(wsA + e0 + 4);
      const uint32_t a1 = __ldg(wsB + e0), a3 = __ldg(wsB + e0 + 4);
      uint32_t b0 = 0, b1 = 0;
      if (t0ok) {
        const uint32_t* xs0 = reinterpret_cast<const uint32_t*>(p.xs + static_cast<int64_t>(tok0) * p.pp);
        b0 = __ldg(xs0 + e0); b1 = __ldg(xs0 + e0 + 4);
      }
      mma_bf16(acc[0], a0, a1, a2, a3, b0, b1);
      if (NT == 2) {
        uint32_t d0 = 0, d1 = 0;
        if (t1ok) {
          const uint32_t* xs1 = reinterpret_cast<const uint32_t*>(p.xs + static_cast<int64_t>(tok1) * p.pp);
          d0 = __ldg(xs1 + e0); d1 = __ldg(xs1 + e0 + 4);
        }
        mma_bf16(acc[NT - 1], a0, a1, a2, a3, d0, d1);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane][4 * t + i] = acc[t][i];
  __syncthreads();
  if (warp == 0) {
    const float alpha = __ldg(p.alpha);
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) v += red[w][lane][4 * t + i];
        // D fragment: c0,c1 -> (feature g, tokens 2c, 2c+1); c2,c3 -> (feature g+8, same tokens)
        const int tok = 8 * t + 2 * c + (i & 1);
        const int64_t feat = n0 + g + (i >> 1) * 8;
        if (tok < p.M && feat < p.N) {
          v *= alpha;
          if (p.out_bf16) static_cast<uint16_t*>(p.Y)[tok * p.ldy + feat] = f32_to_bf16_bits(v);
          else static_cast<float*>(p.Y)[tok * p.ldy + feat] = v;
        }
      }
  }
}

}  // namespace

fs_status launch_splice_gemm_decode(const DecodeParams& p, cudaStream_t s) {
  constexpr int kWarps = 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(p.N, kRowsPerWarp)), 1, 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = (p.M <= 8) ? cudaLaunchKernelEx(&cfg, splice_gemm_decode_kernel<1, kWarps>, p)
                             : cudaLaunchKernelEx(&cfg, splice_gemm_decode_kernel<2, kWarps>, p);
  if (e != cudaSuccess) return cuda_status(e, "fs_splice_gemm (decode path)");
  FS_CHECK_LAUNCH("fs_splice_gemm (decode path)");
  return FS_OK;
}

}  // namespace fs
