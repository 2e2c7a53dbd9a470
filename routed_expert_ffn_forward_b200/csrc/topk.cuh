// Warp-level top-k selection and gating of one token's router logits.
#pragma once

#include <cfloat>

#include "moe_internal.h"

namespace moe {

// Order-preserving map of a logit to an unsigned key (larger logit, larger
// key; -0 is taken as +0 so that equal logits get equal keys).  Key 0 is
// reserved for "no candidate" (it would be the key of a negative NaN).
__device__ __forceinline__ uint32_t topk_key(float v) {
  const uint32_t b = __float_as_uint(v + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float topk_unkey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Called by a full warp.  lt: the token's E logits.  Lane l holds logits
// l, l+32, ... (PL per lane, E <= 32*PL).  k rounds pick the experts in
// decreasing order -- larger logit first, equal logits to the lower expert
// index -- each round one warp max-reduction of the keys and one
// min-reduction of the indices that hold the max; lane r keeps round r's pick.
// With `forced` (k ids) the picks are given.  Gating over the k picks: softmax
// (gating 0) or sigmoid renormalised to sum 1 (gating 1).  Writes ids[0..k)
// and w[0..k).  kL2 reads the logits through L2 only (they were written by
// other CTAs of the same kernel).
template <int PL, bool kL2 = false>
__device__ __forceinline__ void warp_topk_gate(const float* __restrict__ lt, int E, int k, int gating,
                                               const int* __restrict__ forced, int* __restrict__ ids,
                                               float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  int my_e = 0;
  float my_l = 0.f;
  if (forced) {
    if (lane < k) {
      my_e = forced[lane];
      my_l = kL2 ? __ldcg(lt + my_e) : lt[my_e];
    }
  } else {
    uint32_t key[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      key[i] = e < E ? topk_key(kL2 ? __ldcg(lt + e) : lt[e]) : 0u;
    }
    for (int r = 0; r < k; ++r) {
      uint32_t bk = 0u, bi = 0xFFFFFFFFu;
#pragma unroll
      for (int i = 0; i < PL; ++i)
        if (key[i] > bk) {
          bk = key[i];
          bi = (uint32_t)(lane + 32 * i);
        }
      const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t win = __reduce_min_sync(0xffffffffu, bk == m ? bi : 0xFFFFFFFFu);
      if (lane == r) {
        my_e = (int)win;
        my_l = topk_unkey(m);
      }
      if ((int)(win & 31u) == lane) {
#pragma unroll
        for (int i = 0; i < PL; ++i)
          if (i == (int)(win >> 5)) key[i] = 0u;
      }
    }
  }
  float m = lane < k ? my_l : -FLT_MAX;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.f;
  if (lane < k) z = gating == 0 ? expf(my_l - m) : 1.0f / (1.0f + expf(-my_l));
  float sum = z;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    ids[lane] = my_e;
    w[lane] = z / sum;
  }
}

}  // namespace moe
