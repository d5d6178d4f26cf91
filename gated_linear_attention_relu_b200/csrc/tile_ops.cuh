// tile_ops.cuh -- shared pieces of the single-stage tensor-core kernels (token-causal, backward):
// operand descriptors and row addressing of a 128 x 128 bf16 tile in the canonical 128B-swizzled
// layout (two 64-channel halves of 128 rows x 128 B, as TMA writes it), and the RoPE of a span of a
// row and its transpose.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace la {
namespace tile {

constexpr uint32_t HALF = 128 * 128;  // one 64-channel half: 128 rows x 128 B

// K-major operand (rows of 128 channels, 128B swizzle, two 64-channel halves): K step kk.
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int kk) {
  return smem_desc_sw128(base + static_cast<uint32_t>(kk >> 2) * HALF + static_cast<uint32_t>(kk & 3) * 32u, 16,
                         1024);
}
// MN-major operand (the same row layout read along rows): K step kk = rows 16kk .. 16kk+15.
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int kk) {
  return smem_desc_sw128(base + static_cast<uint32_t>(kk) * 2048u, HALF, 1024);
}
// Shared-memory address of 16-byte chunk ck (0..15) of row r in that layout.
__device__ __forceinline__ uint32_t row_chunk(uint32_t base, int r, int ck) {
  return base + static_cast<uint32_t>(ck >> 3) * HALF + static_cast<uint32_t>(r) * 128u +
         ((static_cast<uint32_t>(ck & 7) ^ static_cast<uint32_t>(r & 7)) << 4);
}

__device__ __forceinline__ float sigmoid_tanh(float g) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(0.5f * g));
  return 0.5f + 0.5f * y;
}

// In place over the NP bf16 pairs of a row starting at pair P0 (channels [2 P0, 2 P0 + 2 NP),
// already ReLU'd): a <- RoPE(a) at grid position (pt, ph, pw).  P0 and NP are even, so the span
// covers whole 16-byte table entries.
template <int DT, int DH, int P0, int NP>
__device__ __forceinline__ void rotate_span(uint32_t (&a)[NP], const float2* __restrict__ tab,
                                            const float4* __restrict__ tab2, const Rope& rope, const Plan& p,
                                            int pt, int ph, int pw) {
  static_assert(P0 % 2 == 0 && NP % 2 == 0, "spans of whole table entries");
  if constexpr (DT >= 0 && DH >= 0) {
    constexpr int DW = 128 - DT - DH;
    static_assert(DT % 4 == 0 && DH % 4 == 0 && DW % 4 == 0, "bands of whole 16-byte entries");
    const float4* bt = tab2 + pt * (DT / 4);
    const float4* bh = tab2 + rope.tab_off_h / 2 + ph * (DH / 4);
    const float4* bw = tab2 + rope.tab_off_w / 2 + pw;
    const int W = static_cast<int>(p.W);
#pragma unroll
    for (int j = 0; j < NP / 2; ++j) {
      const int pi = P0 + 2 * j;
      const int bnd = band_of<DT, DH>(pi, rope);
      const int e = pair_in_band<DT, DH>(pi, rope) / 2;
      const float4 cs = __ldg(bnd == 0 ? bt + e : (bnd == 1 ? bh + e : bw + e * W));
      const float x0 = bf16lo(a[2 * j]), x1 = bf16hi(a[2 * j]);
      const float y0 = bf16lo(a[2 * j + 1]), y1 = bf16hi(a[2 * j + 1]);
      a[2 * j] = pack_bf16(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
      a[2 * j + 1] = pack_bf16(y0 * cs.z - y1 * cs.w, y0 * cs.w + y1 * cs.z);
    }
  } else {
    const int ext[3] = {static_cast<int>(p.T), static_cast<int>(p.Hh), static_cast<int>(p.W)};
    const int off[3] = {0, static_cast<int>(rope.tab_off_h), static_cast<int>(rope.tab_off_w)};
    const int pos[3] = {pt, ph, pw};
#pragma unroll 4
    for (int j = 0; j < NP; ++j) {
      const int pi = P0 + j;
      const int bnd = band_of<DT, DH>(pi, rope);
      const int loc = pair_in_band<DT, DH>(pi, rope);
      const float2 cs = __ldg(tab + off[bnd] + loc * ext[bnd] + pos[bnd]);
      const float x0 = bf16lo(a[j]), x1 = bf16hi(a[j]);
      a[j] = pack_bf16(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
    }
  }
}

// In place over the fp32 values of NP pairs starting at pair P0 (channels [2 P0, 2 P0 + 2 NP)):
// x <- RoPE^T(x).  P0 and NP are even.
template <int DT, int DH, int P0, int NP>
__device__ __forceinline__ void rotate_span_t(float (&x)[2 * NP], const float2* __restrict__ tab,
                                              const float4* __restrict__ tab2, const Rope& rope, const Plan& p,
                                              int pt, int ph, int pw) {
  static_assert(P0 % 2 == 0 && NP % 2 == 0, "spans of whole table entries");
  if constexpr (DT >= 0 && DH >= 0) {
    const float4* bt = tab2 + pt * (DT / 4);
    const float4* bh = tab2 + rope.tab_off_h / 2 + ph * (DH / 4);
    const float4* bw = tab2 + rope.tab_off_w / 2 + pw;
    const int W = static_cast<int>(p.W);
#pragma unroll
    for (int j = 0; j < NP / 2; ++j) {
      const int pi = P0 + 2 * j;
      const int bnd = band_of<DT, DH>(pi, rope);
      const int e = pair_in_band<DT, DH>(pi, rope) / 2;
      const float4 cs = __ldg(bnd == 0 ? bt + e : (bnd == 1 ? bh + e : bw + e * W));
      const float x0 = x[4 * j], x1 = x[4 * j + 1], y0 = x[4 * j + 2], y1 = x[4 * j + 3];
      x[4 * j] = x0 * cs.x + x1 * cs.y;
      x[4 * j + 1] = x1 * cs.x - x0 * cs.y;
      x[4 * j + 2] = y0 * cs.z + y1 * cs.w;
      x[4 * j + 3] = y1 * cs.z - y0 * cs.w;
    }
  } else {
    const int ext[3] = {static_cast<int>(p.T), static_cast<int>(p.Hh), static_cast<int>(p.W)};
    const int off[3] = {0, static_cast<int>(rope.tab_off_h), static_cast<int>(rope.tab_off_w)};
    const int pos[3] = {pt, ph, pw};
#pragma unroll 4
    for (int j = 0; j < NP; ++j) {
      const int pi = P0 + j;
      const int bnd = band_of<DT, DH>(pi, rope);
      const int loc = pair_in_band<DT, DH>(pi, rope);
      const float2 cs = __ldg(tab + off[bnd] + loc * ext[bnd] + pos[bnd]);
      const float x0 = x[2 * j], x1 = x[2 * j + 1];
      x[2 * j] = x0 * cs.x + x1 * cs.y;
      x[2 * j + 1] = x1 * cs.x - x0 * cs.y;
    }
  }
}

}  // namespace tile
}  // namespace la
