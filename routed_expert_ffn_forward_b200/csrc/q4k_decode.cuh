// Q4_K scale decoding shared by the decode-path kernels.  Device code only.
#pragma once

#include "moe_internal.h"

namespace moe {

// Decoded scales of one row for the thread's sub-blocks 2c (lo) and 2c+1 (hi):
// weight = s * q - m.
struct RowScales {
  float s_lo, s_hi, m_lo, m_hi;
};

// hdr: the 16-byte block header (fp16 d, fp16 dmin, 12 packed scale bytes).
__device__ __forceinline__ RowScales decode_scales(uint4 hdr, int c) {
  const float d = __half2float(__ushort_as_half((unsigned short)(hdr.x & 0xFFFFu)));
  const float dmin = __half2float(__ushort_as_half((unsigned short)(hdr.x >> 16)));
  const uint32_t sh = 16u * (uint32_t)(c & 1);
  const uint32_t s0 = hdr.y >> sh, s1 = hdr.z >> sh, s2 = hdr.w >> sh;
  uint32_t vsc, vm;
  if (c < 2) {  // sub-blocks 0..3: low 6 bits of bytes j and j+4
    vsc = s0 & 0x3F3Fu;
    vm = s1 & 0x3F3Fu;
  } else {      // sub-blocks 4..7: nibbles of byte j+4, top 2 bits of bytes j-4 / j
    vsc = (s2 & 0x0F0Fu) | ((s0 >> 2) & 0x3030u);
    vm = ((s2 >> 4) & 0x0F0Fu) | ((s1 >> 2) & 0x3030u);
  }
  // byte b -> float exactly: the bits 0x4B0000bb are the float 2^23 + b
  constexpr uint32_t kMagic = 0x4B000000u;
  constexpr float kMagicF = 8388608.f;
  RowScales r;
  r.s_lo = d * (__uint_as_float(__byte_perm(vsc, kMagic, 0x7650)) - kMagicF);
  r.s_hi = d * (__uint_as_float(__byte_perm(vsc, kMagic, 0x7651)) - kMagicF);
  r.m_lo = dmin * (__uint_as_float(__byte_perm(vm, kMagic, 0x7650)) - kMagicF);
  r.m_hi = dmin * (__uint_as_float(__byte_perm(vm, kMagic, 0x7651)) - kMagicF);
  return r;
}

}  // namespace moe
