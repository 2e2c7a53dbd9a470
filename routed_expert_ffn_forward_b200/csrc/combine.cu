// Gate-weighted combine: out[t] = bf16_rne( sum_j w[t,j] * y[inv(t,j)] + sum_s y[inv(t,k+s)] ).
// Each output element is summed by one thread in the fixed order j = 0..k-1,
// then the shared experts, with no atomics: the result does not depend on
// scheduling (LayerStoRm README, "Notes": a deterministic expert combine).
//
// Expert parallelism (the same "Notes": EP across GPUs with a deterministic
// combine): a rank sums only the pairs whose expert it owns, in the same
// order, and writes the unrounded fp32 sum; the ranks' partial sums are then
// added in rank order and rounded once (combine_partials_kernel).
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void combine_kernel(const float* __restrict__ y, const float* __restrict__ w,
                               const int* __restrict__ inv, const int* __restrict__ ids, int H, int E, int k, int S,
                               __nv_bfloat16* __restrict__ out, float* __restrict__ partial, int ep_rank,
                               int ep_world, int n_rows, unsigned* err) {
  constexpr int kMaxKS = 40;  // top_k + n_shared at most
  __shared__ int s_row[kMaxKS];
  __shared__ float s_w[kMaxKS];
  const int t = blockIdx.y, kS = k + S;
  // the token's y rows and weights, once per block, so the y loads below are
  // independent of each other.  They come from the routing kernels, at least
  // two launches back: every kernel of a forward waits for its predecessor
  // before it lets its dependents launch, so those are complete when this
  // kernel starts, and the loads go ahead of the wait for the down kernel.
  // A pair whose expert another rank owns gets row -1 (skipped).
  if (threadIdx.x < kS) {
    const int j = threadIdx.x;
    const int ex = j < k ? __ldcg(ids + (size_t)t * k + j) : E + (j - k);
    const bool own = ep_owned(ex, ep_rank, ep_world);
    s_row[j] = own ? in_range(__ldcg(inv + t * kS + j), n_rows, err) : -1;
    s_w[j] = j < k ? __ldcg(w + (size_t)t * k + j) : 1.f;
  }
  // launched as a programmatic dependent of the down kernel: wait for it (a
  // no-op when launched normally)
  ptx::pdl_wait();
  __syncthreads();
  const int o = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (o >= H) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < kS; j0 += 8) {
    float4 v[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj)
      if (j0 + jj < kS && s_row[j0 + jj] >= 0)
        v[jj] = *reinterpret_cast<const float4*>(y + (size_t)s_row[j0 + jj] * H + o);
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = j0 + jj;
      if (j >= kS || s_row[j] < 0) continue;
      if (j < k) {  // routed experts: weighted, in order
        acc.x = fmaf(s_w[j], v[jj].x, acc.x);
        acc.y = fmaf(s_w[j], v[jj].y, acc.y);
        acc.z = fmaf(s_w[j], v[jj].z, acc.z);
        acc.w = fmaf(s_w[j], v[jj].w, acc.w);
      } else {  // then the shared experts
        acc.x += v[jj].x;
        acc.y += v[jj].y;
        acc.z += v[jj].z;
        acc.w += v[jj].w;
      }
    }
  }
  if (partial) {
    *reinterpret_cast<float4*>(partial + (size_t)t * H + o) = acc;
    return;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + (size_t)t * H + o) = pk;
}

__global__ void combine_partials_kernel(const float4* __restrict__ p, uint2* __restrict__ out, size_t n4,
                                        int world) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    float4 acc = __ldg(p + i);
    for (int r = 1; r < world; ++r) {
      const float4 v = __ldg(p + (size_t)r * n4 + i);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    out[i] = pk;
  }
}

}  // namespace

cudaError_t launch_combine(const Work& wk, int T, const Shape& s, __nv_bfloat16* out, cudaStream_t st, bool pdl,
                           float* partial, int ep_rank, int ep_world) {
  const int threads = 64;  // more, smaller blocks: the combine is latency-bound at small T
  dim3 grid((s.H / 4 + threads - 1) / threads, T);
  const int n_rows = T * (s.k + s.S);
  if (!pdl) {
    combine_kernel<<<grid, threads, 0, st>>>(wk.y, wk.w, wk.inv, wk.ids, s.H, s.E, s.k, s.S, out, partial, ep_rank,
                                             ep_world, n_rows, wk.err);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, (const float*)wk.y, (const float*)wk.w, (const int*)wk.inv,
                            (const int*)wk.ids, s.H, s.E, s.k, s.S, out, partial, ep_rank, ep_world, n_rows, wk.err);
}

cudaError_t launch_combine_partials(const float* partials, __nv_bfloat16* out, int T, int H, int world,
                                    cudaStream_t st) {
  const size_t n4 = (size_t)T * H / 4;
  if (n4 == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)std::min<size_t>((n4 + 255) / 256, 4096);
  combine_partials_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4*>(partials),
                                                  reinterpret_cast<uint2*>(out), n4, world);
  return cudaGetLastError();
}

}  // namespace moe
