// Byte dot products of Q4_K rows against 16-bit fixed-point activations,
// shared by the single-token decode kernels.  Device code only.
//
// For a 32-bit quant word w (four quants of sub-block 2c in its low nibbles
// and four of sub-block 2c+1 in its high nibbles) the thread forms
//   lo = w & 0x0F0F0F0F,  hi = w & 0xF0F0F0F0  (16 x the high quants)
// and accumulates dp4a(lo, x_hi) and dp4a(lo, x_lo) (and the same for hi),
// where the activations are x = (256*x_hi + x_lo) * 2^-s per 32-element run
// (x_hi signed, x_lo unsigned bytes), so the integer sums are exact.  Per
// (row, sub-block) the fp32 epilogue adds d*sc * 2^-s * (256*C_hi + C_lo) -
// dmin*m * X (X the run's sum of the represented activations; the 1/16 of
// the high nibbles folded into the scale, exactly).
#pragma once

#include "moe_internal.h"
#include "q4k_decode.cuh"

namespace moe {

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {  // u8 x s8
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {  // u8 x u8
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Chunk c of R rows' super-blocks (blk[r]: the rows' 144-byte blocks) against
// one token's activations of that super-block: xh/xl the 256 high/low
// activation bytes, sc the eight runs' (2^-s, X).  The chunk's activations are
// loaded once for the R rows.  Adds row r's partial dot product to acc[r].
template <int R>
__device__ __forceinline__ void gv_chunk_rows(const uint8_t* const (&blk)[R], int c, const uint8_t* xh,
                                              const uint8_t* xl, const float2* sc, float (&acc)[R]) {
  // activations: sub-block 2c at bytes 64c..64c+31, sub-block 2c+1 at 64c+32..
  const uint4* ph = reinterpret_cast<const uint4*>(xh + 64 * c);
  const uint4* pl = reinterpret_cast<const uint4*>(xl + 64 * c);
  const uint4 h0 = ph[0], h1 = ph[1], h2 = ph[2], h3 = ph[3];
  const uint4 l0 = pl[0], l1 = pl[1], l2 = pl[2], l3 = pl[3];
  const uint32_t xhl[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  const uint32_t xhh[8] = {h2.x, h2.y, h2.z, h2.w, h3.x, h3.y, h3.z, h3.w};
  const uint32_t xll[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
  const uint32_t xlh[8] = {l2.x, l2.y, l2.z, l2.w, l3.x, l3.y, l3.z, l3.w};
  const float2 sl = sc[2 * c], sh = sc[2 * c + 1];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const uint4 hdr = *reinterpret_cast<const uint4*>(blk[r]);
    const uint4 qa = *reinterpret_cast<const uint4*>(blk[r] + 16 + 32 * c);
    const uint4 qb = *reinterpret_cast<const uint4*>(blk[r] + 32 + 32 * c);
    const uint32_t q[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    int chl = 0, cll = 0, chh = 0, clh = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      // high nibbles left in place: 16x the quant, so the sums are 16x too
      const uint32_t lo = q[k] & 0x0F0F0F0Fu, hi = q[k] & 0xF0F0F0F0u;
      chl = dp4a_us(lo, xhl[k], chl);
      cll = dp4a_uu(lo, xll[k], cll);
      chh = dp4a_us(hi, xhh[k], chh);
      clh = dp4a_uu(hi, xlh[k], clh);
    }
    const RowScales rs = decode_scales(hdr, c);
    acc[r] += rs.s_lo * sl.x * (float)(chl * 256 + cll) + (rs.s_hi * 0.0625f) * sh.x * (float)(chh * 256 + clh) -
              (rs.m_lo * sl.y + rs.m_hi * sh.y);
  }
}

}  // namespace moe
