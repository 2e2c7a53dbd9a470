// Dot products of one 64-weight chunk of weight rows, for every GGUF block
// type the single-token kernel reads, against one token's activations in
// 16-bit fixed point per 32-element run (x = (256*x_hi + x_lo) * 2^-s, x_hi
// signed and x_lo unsigned bytes; run scale (2^-s, X) with X the run's sum of
// the represented values).  Device code only.
//
// Weights are stored per 256-weight group ("super-block") in the device
// layout of their type (moe_internal.h, dev_sb_bytes): the GGUF block bytes,
// with Q6_K blocks padded to 224 bytes and MXFP4 blocks grouped eight at a
// time into 144 bytes.  Chunk c holds weights 64c..64c+63 of the group, i.e.
// runs 2c and 2c+1.  Integer sums are exact (dp4a); each (row, scale group)
// adds its float scale times the sum, plus the min term where the type has
// one, in fp32.  The Q4_K case is gv_chunk_rows in gemv_dot.cuh.
#pragma once

#include "gemv_dot.cuh"
#include "moe_internal.h"

namespace moe {

__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {  // s8 x s8
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {  // s8 x u8
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ float half_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu))); }
__device__ __forceinline__ float half_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }

// The chunk's activations: run 2c in xa*, run 2c+1 in xb*, eight words each.
struct ChunkX {
  uint32_t ah[8], al[8], bh[8], bl[8];
  float2 sa, sb;
};
__device__ __forceinline__ ChunkX load_chunk_x(const uint8_t* xh, const uint8_t* xl, const float2* sc, int c) {
  ChunkX x;
  const uint4* ph = reinterpret_cast<const uint4*>(xh + 64 * c);
  const uint4* pl = reinterpret_cast<const uint4*>(xl + 64 * c);
  const uint4 h0 = ph[0], h1 = ph[1], h2 = ph[2], h3 = ph[3];
  const uint4 l0 = pl[0], l1 = pl[1], l2 = pl[2], l3 = pl[3];
  const uint32_t ah[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  const uint32_t bh[8] = {h2.x, h2.y, h2.z, h2.w, h3.x, h3.y, h3.z, h3.w};
  const uint32_t al[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
  const uint32_t bl[8] = {l2.x, l2.y, l2.z, l2.w, l3.x, l3.y, l3.z, l3.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x.ah[k] = ah[k];
    x.al[k] = al[k];
    x.bh[k] = bh[k];
    x.bl[k] = bl[k];
  }
  x.sa = sc[2 * c];
  x.sb = sc[2 * c + 1];
  return x;
}

// ---- Q5_K: d, dmin, the 12 Q4_K scale bytes, qh[32] (fifth bits), qs[128]
__device__ __forceinline__ float q5k_chunk(const uint8_t* blk, int c, const ChunkX& x) {
  const uint4 hdr = *reinterpret_cast<const uint4*>(blk);
  const uint4 h0 = *reinterpret_cast<const uint4*>(blk + 16), h1 = *reinterpret_cast<const uint4*>(blk + 32);
  const uint4 qa = *reinterpret_cast<const uint4*>(blk + 48 + 32 * c);
  const uint4 qb = *reinterpret_cast<const uint4*>(blk + 64 + 32 * c);
  const uint32_t qh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  const uint32_t q[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
  int ahs = 0, als = 0, bhs = 0, bls = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    // quants of run 2c: low nibbles + bit 2c of qh; run 2c+1: high nibbles + bit 2c+1
    const uint32_t ua = (q[k] & 0x0F0F0F0Fu) | (((qh[k] >> (2 * c)) & 0x01010101u) << 4);
    const uint32_t ub = ((q[k] >> 4) & 0x0F0F0F0Fu) | (((qh[k] >> (2 * c + 1)) & 0x01010101u) << 4);
    ahs = dp4a_us(ua, x.ah[k], ahs);
    als = dp4a_uu(ua, x.al[k], als);
    bhs = dp4a_us(ub, x.bh[k], bhs);
    bls = dp4a_uu(ub, x.bl[k], bls);
  }
  const RowScales rs = decode_scales(hdr, c);
  return rs.s_lo * x.sa.x * (float)(ahs * 256 + als) + rs.s_hi * x.sb.x * (float)(bhs * 256 + bls) -
         (rs.m_lo * x.sa.y + rs.m_hi * x.sb.y);
}

// ---- Q6_K (device block 224 bytes): ql[128], qh[64], scales[16] (s8), d, pad
// 6-bit value u in 0..63 -> the signed byte u - 32: flipping bit 5 gives the
// 6-bit two's complement, then bits 6-7 copy bit 5.
__device__ __forceinline__ uint32_t q6_signed(uint32_t u) {
  const uint32_t v = u ^ 0x20202020u;
  return v | ((v & 0x20202020u) * 6u);
}
__device__ __forceinline__ float q6k_chunk(const uint8_t* blk, int c, const ChunkX& x) {
  const int h = c >> 1, odd = c & 1;
  const uint4 la0 = *reinterpret_cast<const uint4*>(blk + 64 * h), la1 = *reinterpret_cast<const uint4*>(blk + 64 * h + 16);
  const uint4 lb0 = *reinterpret_cast<const uint4*>(blk + 64 * h + 32),
              lb1 = *reinterpret_cast<const uint4*>(blk + 64 * h + 48);
  const uint4 h0 = *reinterpret_cast<const uint4*>(blk + 128 + 32 * h),
              h1 = *reinterpret_cast<const uint4*>(blk + 144 + 32 * h);
  const uint4 sc4 = *reinterpret_cast<const uint4*>(blk + 192);
  const uint32_t la[8] = {la0.x, la0.y, la0.z, la0.w, la1.x, la1.y, la1.z, la1.w};
  const uint32_t lb[8] = {lb0.x, lb0.y, lb0.z, lb0.w, lb1.x, lb1.y, lb1.z, lb1.w};
  const uint32_t qh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  const int ns = 4 * odd, pa = 2 * odd, pb = 2 * odd + 1;   // nibble shift, parts of runs 2c, 2c+1
  int s[8] = {0, 0, 0, 0, 0, 0, 0, 0};                       // (run a, b) x (group 0, 1) x (hi, lo)
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t ua = ((la[k] >> ns) & 0x0F0F0F0Fu) | (((qh[k] >> (2 * pa)) & 0x03030303u) << 4);
    const uint32_t ub = ((lb[k] >> ns) & 0x0F0F0F0Fu) | (((qh[k] >> (2 * pb)) & 0x03030303u) << 4);
    const uint32_t qa = q6_signed(ua), qb = q6_signed(ub);
    const int g = (k >> 2) * 2;
    s[g] = dp4a_ss(qa, x.ah[k], s[g]);
    s[g + 1] = dp4a_su(qa, x.al[k], s[g + 1]);
    s[4 + g] = dp4a_ss(qb, x.bh[k], s[4 + g]);
    s[4 + g + 1] = dp4a_su(qb, x.bl[k], s[4 + g + 1]);
  }
  const float d = half_lo(*reinterpret_cast<const uint32_t*>(blk + 208));
  const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
  // scale index of part p, group g: 8h + 2p + g
  auto scale = [&](int p, int g) {
    const int i = 8 * h + 2 * p + g;
    return (float)(int8_t)((scw[i >> 2] >> (8 * (i & 3))) & 0xFFu);
  };
  const float fa = d * x.sa.x, fb = d * x.sb.x;
  return fa * (scale(pa, 0) * (float)(s[0] * 256 + s[1]) + scale(pa, 1) * (float)(s[2] * 256 + s[3])) +
         fb * (scale(pb, 0) * (float)(s[4] * 256 + s[5]) + scale(pb, 1) * (float)(s[6] * 256 + s[7]));
}

// ---- Q8_0 (eight 34-byte blocks, 272 bytes): fp16 d then 32 s8 quants
__device__ __forceinline__ float q8_0_chunk(const uint8_t* blk, int c, const ChunkX& x) {
  // blocks 2c and 2c+1 fill bytes 68c .. 68c+67: seventeen aligned words
  const uint32_t* w = reinterpret_cast<const uint32_t*>(blk + 68 * c);
  uint32_t v[17];
#pragma unroll
  for (int i = 0; i < 17; ++i) v[i] = w[i];
  int ah = 0, al = 0, bh = 0, bl = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t qa = __funnelshift_r(v[k], v[k + 1], 16);   // block 2c: bytes 2..33
    const uint32_t qb = v[9 + k];                                // block 2c+1: bytes 36..67
    ah = dp4a_ss(qa, x.ah[k], ah);
    al = dp4a_su(qa, x.al[k], al);
    bh = dp4a_ss(qb, x.bh[k], bh);
    bl = dp4a_su(qb, x.bl[k], bl);
  }
  const float da = half_lo(v[0]), db = half_hi(v[8]);
  return da * x.sa.x * (float)(ah * 256 + al) + db * x.sb.x * (float)(bh * 256 + bl);
}

// ---- MXFP4 (eight 17-byte blocks in 144 bytes): E8M0 scale, 16 bytes of
// FP4 E2M1 codes (element i: low nibble of byte i, element 16+i: high nibble)
// Four codes -> four signed bytes of twice their E2M1 value (0, 1, 2, 3, 4,
// 6, 8, 12 and negatives).
__device__ __forceinline__ uint32_t e2m1x2_bytes(uint32_t codes) {
  constexpr uint32_t kPos0 = 0x03020100u, kPos1 = 0x0C080604u;   // 0 1 2 3 | 4 6 8 12
  constexpr uint32_t kNeg0 = 0xFDFEFF00u, kNeg1 = 0xF4F8FAFCu;   // -0 -1 -2 -3 | -4 -6 -8 -12
  // byte i's 3-bit magnitude code becomes the selector nibble i
  const uint32_t sel = codes & 0x07070707u;
  const uint32_t idx = (sel & 0x7u) | ((sel >> 4) & 0x70u) | ((sel >> 8) & 0x700u) | ((sel >> 12) & 0x7000u);
  const uint32_t pos = __byte_perm(kPos0, kPos1, idx), neg = __byte_perm(kNeg0, kNeg1, idx);
  const uint32_t m = ((codes >> 3) & 0x01010101u) * 0xFFu;      // sign bit -> byte mask
  return (pos & ~m) | (neg & m);
}
// four bytes starting at byte `off` (any alignment) of the word array w
__device__ __forceinline__ uint32_t bytes_at(const uint32_t* w, int off) {
  return __byte_perm(w[off >> 2], w[(off >> 2) + 1], (uint32_t)(off & 3) * 0x1111u + 0x3210u);
}
__device__ __forceinline__ float mxfp4_chunk(const uint8_t* blk, int c, const ChunkX& x) {
  // blocks 2c, 2c+1: bytes 34c .. 34c+33, read as eleven aligned words
  const int base = 34 * c, wb = base & ~3, o = base - wb;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(blk + wb);
  uint32_t v[11];
#pragma unroll
  for (int i = 0; i < 11; ++i) v[i] = w[i];
  int ah = 0, al = 0, bh = 0, bl = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t ca = bytes_at(v, o + 1 + 4 * k), cb = bytes_at(v, o + 18 + 4 * k);
    const uint32_t la = e2m1x2_bytes(ca), ha = e2m1x2_bytes(ca >> 4);   // elements 4k.., 16+4k..
    const uint32_t lb = e2m1x2_bytes(cb), hb = e2m1x2_bytes(cb >> 4);
    ah = dp4a_ss(la, x.ah[k], ah);
    al = dp4a_su(la, x.al[k], al);
    ah = dp4a_ss(ha, x.ah[4 + k], ah);
    al = dp4a_su(ha, x.al[4 + k], al);
    bh = dp4a_ss(lb, x.bh[k], bh);
    bl = dp4a_su(lb, x.bl[k], bl);
    bh = dp4a_ss(hb, x.bh[4 + k], bh);
    bl = dp4a_su(hb, x.bl[4 + k], bl);
  }
  const uint32_t ea = (bytes_at(v, o) & 0xFFu), eb = (bytes_at(v, o + 17) & 0xFFu);
  // 2^(e-128): the codes above are twice the E2M1 values
  const float fa = ea ? __uint_as_float((ea - 1u) << 23) : 0x1p-128f;
  const float fb = eb ? __uint_as_float((eb - 1u) << 23) : 0x1p-128f;
  return fa * x.sa.x * (float)(ah * 256 + al) + fb * x.sb.x * (float)(bh * 256 + bl);
}

// One chunk of R rows of type Q (blk[r]: the rows' super-blocks) against the
// chunk's activations; adds each row's partial dot product to acc[r].
template <int Q, int R>
__device__ __forceinline__ void q_chunk_rows(const uint8_t* const (&blk)[R], int c, const uint8_t* xh,
                                             const uint8_t* xl, const float2* sc, float (&acc)[R]) {
  if (Q == kQ4_K) {
    gv_chunk_rows<R>(blk, c, xh, xl, sc, acc);
  } else {
    const ChunkX x = load_chunk_x(xh, xl, sc, c);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (Q == kQ5_K) acc[r] += q5k_chunk(blk[r], c, x);
      if (Q == kQ6_K) acc[r] += q6k_chunk(blk[r], c, x);
      if (Q == kQ8_0) acc[r] += q8_0_chunk(blk[r], c, x);
      if (Q == kMXFP4) acc[r] += mxfp4_chunk(blk[r], c, x);
    }
  }
}

}  // namespace moe
