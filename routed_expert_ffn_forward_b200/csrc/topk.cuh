// Warp-level top-k selection and gating of one token's router logits.
#pragma once

#include <cfloat>

#include "moe_internal.h"

namespace moe {

// (value, index) order of the top-k: larger logit first, equal logits to the
// lower expert index.  `ok` false means "no candidate".
struct TopkCand {
  float v;
  int e;
  bool ok;
};
__device__ __forceinline__ bool topk_better(const TopkCand& a, const TopkCand& b) {
  if (a.ok != b.ok) return a.ok;
  if (!a.ok) return false;
  return a.v > b.v || (a.v == b.v && a.e < b.e);
}

// Called by a full warp.  lt: the token's E logits.  Lane l holds logits
// l, l+32, ... (PL per lane, E <= 32*PL); k rounds of a warp arg-max pick the
// experts in decreasing order and lane r keeps round r's pick.  With `forced`
// (k ids) the picks are given.  Gating over the k picks: softmax (gating 0) or
// sigmoid renormalised to sum 1 (gating 1).  Writes ids[0..k) and w[0..k).
// kL2 reads the logits through L2 only (they were written by other CTAs of the
// same kernel).
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
    float v[PL];
    bool taken[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      taken[i] = e >= E;
      v[i] = taken[i] ? 0.f : (kL2 ? __ldcg(lt + e) : lt[e]);
    }
    for (int r = 0; r < k; ++r) {
      TopkCand c{0.f, 0, false};
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        const TopkCand d{v[i], lane + 32 * i, !taken[i]};
        if (topk_better(d, c)) c = d;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        TopkCand d;
        d.v = __shfl_xor_sync(0xffffffffu, c.v, o);
        d.e = __shfl_xor_sync(0xffffffffu, c.e, o);
        d.ok = __shfl_xor_sync(0xffffffffu, (int)c.ok, o);
        if (topk_better(d, c)) c = d;
      }
      if (lane == r) {
        my_e = c.e;
        my_l = c.v;
      }
      if ((c.e & 31) == lane) {
#pragma unroll
        for (int i = 0; i < PL; ++i)
          if (i == (c.e >> 5)) taken[i] = true;
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
