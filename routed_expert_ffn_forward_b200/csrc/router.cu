// Router: fp32 logits l[t,e] = x[t,:] . Wr[e,:] + b[e], then top-k selection and
// gating per token.  (LayerStoRm README, "TL;DR": the router tells each token
// which few experts it activates.)
#include <cfloat>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRouterTokTile = 8;   // tokens per block
constexpr int kRouterWarps = 8;     // experts per block (one per warp)

// One warp per expert row, kRouterTokTile tokens per block.  Each lane walks
// the row in float4 steps; partial sums are reduced with a fixed xor tree, so
// the result is the same on every run.
__global__ void __launch_bounds__(kRouterWarps * 32)
router_logits_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ W,
                     const float* __restrict__ b, float* __restrict__ logits, int T, int H, int E) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kRouterWarps + warp;
  const int t0 = blockIdx.y * kRouterTokTile;
  if (e >= E) return;
  const int nt = min(kRouterTokTile, T - t0);
  const float* wrow = W + (size_t)e * H;
  const __nv_bfloat16* xb = x + (size_t)t0 * H;
  float acc[kRouterTokTile];
#pragma unroll
  for (int i = 0; i < kRouterTokTile; ++i) acc[i] = 0.f;
  for (int h = lane * 4; h < H; h += 128) {
    const float4 w4 = __ldg(reinterpret_cast<const float4*>(wrow + h));
#pragma unroll
    for (int i = 0; i < kRouterTokTile; ++i) {
      if (i < nt) {
        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(xb + (size_t)i * H + h));
        acc[i] = fmaf(w4.x, bf16lo(xv.x), acc[i]);
        acc[i] = fmaf(w4.y, bf16hi(xv.x), acc[i]);
        acc[i] = fmaf(w4.z, bf16lo(xv.y), acc[i]);
        acc[i] = fmaf(w4.w, bf16hi(xv.y), acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kRouterTokTile; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
  const float bias = b ? b[e] : 0.f;
#pragma unroll
  for (int i = 0; i < kRouterTokTile; ++i)
    if (lane == i && i < nt) logits[(size_t)(t0 + i) * E + e] = acc[i] + bias;
}

// (value, index) ordering of the top-k: larger logit first, equal logits to the
// lower expert index.  `ok` false means "no candidate".
struct Cand {
  float v;
  int e;
  bool ok;
};
__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  if (a.ok != b.ok) return a.ok;
  if (!a.ok) return false;
  return a.v > b.v || (a.v == b.v && a.e < b.e);
}

// One warp per token.  Lane l holds logits l, l+32, ...; k rounds of a warp
// arg-max pick the experts in decreasing order.  Lane r keeps round r's pick.
template <int PL>
__global__ void topk_kernel(const float* __restrict__ logits, int T, int E, int k, int gating,
                            const int* __restrict__ forced, int* __restrict__ ids,
                            float* __restrict__ w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  const float* lt = logits + (size_t)t * E;
  int my_e = 0;
  float my_l = 0.f;
  if (forced) {
    if (lane < k) {
      my_e = forced[(size_t)t * k + lane];
      my_l = lt[my_e];
    }
  } else {
    float v[PL];
    bool taken[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      taken[i] = e >= E;
      v[i] = taken[i] ? 0.f : lt[e];
    }
    for (int r = 0; r < k; ++r) {
      Cand c{0.f, 0, false};
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        const Cand d{v[i], lane + 32 * i, !taken[i]};
        if (better(d, c)) c = d;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        Cand d;
        d.v = __shfl_xor_sync(0xffffffffu, c.v, o);
        d.e = __shfl_xor_sync(0xffffffffu, c.e, o);
        d.ok = __shfl_xor_sync(0xffffffffu, (int)c.ok, o);
        if (better(d, c)) c = d;
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
  // gating over the k picks (lanes >= k contribute zero)
  float m = lane < k ? my_l : -FLT_MAX;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.f;
  if (lane < k) z = gating == 0 ? expf(my_l - m) : 1.0f / (1.0f + expf(-my_l));
  float sum = z;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    ids[(size_t)t * k + lane] = my_e;
    w[(size_t)t * k + lane] = z / sum;
  }
}

}  // namespace

cudaError_t launch_router_logits(const __nv_bfloat16* x, const float* W, const float* b,
                                 float* logits, int T, int H, int E, cudaStream_t st) {
  dim3 grid((E + kRouterWarps - 1) / kRouterWarps, (T + kRouterTokTile - 1) / kRouterTokTile);
  router_logits_kernel<<<grid, kRouterWarps * 32, 0, st>>>(x, W, b, logits, T, H, E);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int T, int E, int k, int gating, const int* forced,
                        int* ids, float* w, cudaStream_t st) {
  const int warps = 8;
  const int grid = (T + warps - 1) / warps;
  const int pl = (E + 31) / 32;
  if (pl <= 8)
    topk_kernel<8><<<grid, warps * 32, 0, st>>>(logits, T, E, k, gating, forced, ids, w);
  else
    topk_kernel<32><<<grid, warps * 32, 0, st>>>(logits, T, E, k, gating, forced, ids, w);
  return cudaGetLastError();
}

}  // namespace moe
