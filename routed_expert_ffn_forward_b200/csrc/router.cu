// Router: fp32 logits l[t,e] = x[t,:] . Wr[e,:] + b[e], then top-k selection and
// gating per token.  (LayerStoRm README, "TL;DR": the router tells each token
// which few experts it activates.)
#include <cfloat>

#include "moe_internal.h"
#include "topk.cuh"

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

// One warp per token.
template <int PL>
__global__ void topk_kernel(const float* __restrict__ logits, int T, int E, int k, int gating,
                            const int* __restrict__ forced, int* __restrict__ ids,
                            float* __restrict__ w) {
  const int warp = threadIdx.x >> 5;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  warp_topk_gate<PL>(logits + (size_t)t * E, E, k, gating, forced ? forced + (size_t)t * k : nullptr,
                     ids + (size_t)t * k, w + (size_t)t * k);
}

// One block per token: G groups of 128 threads each sum a G-th of the K
// splits (in split order) for every expert, the parts are added in order and
// the bias after them (writing the logits to `logits` and shared memory),
// then warp 0 selects and gates.  With many splits (112 at T = 64) four
// groups put four times as many partial-logit loads in flight; with few
// (4 at T = 4096) one group keeps the blocks small.
constexpr int kSumGroup = 128;
template <int PL, int G>
__global__ void __launch_bounds__(kSumGroup * G)
    topk_sum_kernel(float* __restrict__ logits, int E, int k, int gating, const int* __restrict__ forced,
                    int* __restrict__ ids, float* __restrict__ w, const float* __restrict__ part, int nsplit,
                    size_t split_stride, const float* __restrict__ bias) {
  constexpr int kSumGroups = G, kSumThreads = kSumGroup * G;
  __shared__ float s_l[32 * PL];
  __shared__ float s_q[kSumGroups][32 * PL];
  const int t = blockIdx.x;
  const int q = threadIdx.x / kSumGroup, lt = threadIdx.x - q * kSumGroup;
  const int s0 = q * nsplit / kSumGroups, s1 = (q + 1) * nsplit / kSumGroups;
  for (int e = lt; e < E; e += kSumGroup) {
    const float* p = part + (size_t)t * E + e;
    float v = 0.f;
#pragma unroll 8
    for (int s = s0; s < s1; ++s) v += p[(size_t)s * split_stride];
    s_q[q][e] = v;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kSumThreads) {
    float v = s_q[0][e];
#pragma unroll
    for (int g = 1; g < kSumGroups; ++g) v += s_q[g][e];
    v += bias ? bias[e] : 0.f;
    logits[(size_t)t * E + e] = v;
    s_l[e] = v;
  }
  __syncthreads();
  if (threadIdx.x < 32)
    warp_topk_gate<PL>(s_l, E, k, gating, forced ? forced + (size_t)t * k : nullptr, ids + (size_t)t * k,
                       w + (size_t)t * k);
}

}  // namespace

cudaError_t launch_router_logits(const __nv_bfloat16* x, const float* W, const float* b,
                                 float* logits, int T, int H, int E, cudaStream_t st) {
  dim3 grid((E + kRouterWarps - 1) / kRouterWarps, (T + kRouterTokTile - 1) / kRouterTokTile);
  router_logits_kernel<<<grid, kRouterWarps * 32, 0, st>>>(x, W, b, logits, T, H, E);
  return cudaGetLastError();
}

cudaError_t launch_topk(float* logits, int T, int E, int k, int gating, const int* forced,
                        int* ids, float* w, cudaStream_t st, const float* part, int nsplit, size_t split_stride,
                        const float* bias) {
  const int pl = (E + 31) / 32;
  if (part) {
    const bool wide = nsplit >= 16;
    auto kern = pl <= 8 ? (wide ? topk_sum_kernel<8, 4> : topk_sum_kernel<8, 1>)
                        : (wide ? topk_sum_kernel<32, 4> : topk_sum_kernel<32, 1>);
    kern<<<T, kSumGroup * (wide ? 4 : 1), 0, st>>>(logits, E, k, gating, forced, ids, w, part, nsplit, split_stride,
                                                   bias);
    return cudaGetLastError();
  }
  const int warps = 8;
  const int grid = (T + warps - 1) / warps;
  if (pl <= 8)
    topk_kernel<8><<<grid, warps * 32, 0, st>>>(logits, T, E, k, gating, forced, ids, w);
  else
    topk_kernel<32><<<grid, warps * 32, 0, st>>>(logits, T, E, k, gating, forced, ids, w);
  return cudaGetLastError();
}

}  // namespace moe
