// Gate-weighted combine: out[t] = bf16_rne( sum_j w[t,j] * y[inv(t,j)] + sum_s y[inv(t,k+s)] ).
// Each output element is summed by one thread in the fixed order j = 0..k-1,
// then the shared experts, with no atomics: the result does not depend on
// scheduling (LayerStoRm README, "Notes": a deterministic expert combine).
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void combine_kernel(const float* __restrict__ y, const float* __restrict__ w,
                               const int* __restrict__ inv, int H, int k, int S,
                               __nv_bfloat16* __restrict__ out, int n_rows, unsigned* err) {
  constexpr int kMaxKS = 40;  // top_k + n_shared at most
  __shared__ int s_row[kMaxKS];
  __shared__ float s_w[kMaxKS];
  const int t = blockIdx.y, kS = k + S;
  // the token's y rows and weights, once per block, so the y loads below are
  // independent of each other.  They come from the routing kernels, at least
  // two launches back: every kernel of a forward waits for its predecessor
  // before it lets its dependents launch, so those are complete when this
  // kernel starts, and the loads go ahead of the wait for the down kernel.
  if (threadIdx.x < kS) {
    s_row[threadIdx.x] = in_range(__ldcg(inv + t * kS + threadIdx.x), n_rows, err);
    s_w[threadIdx.x] = threadIdx.x < k ? __ldcg(w + (size_t)t * k + threadIdx.x) : 1.f;
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
      if (j0 + jj < kS) v[jj] = *reinterpret_cast<const float4*>(y + (size_t)s_row[j0 + jj] * H + o);
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = j0 + jj;
      if (j < k) {  // routed experts: weighted, in order
        acc.x = fmaf(s_w[j], v[jj].x, acc.x);
        acc.y = fmaf(s_w[j], v[jj].y, acc.y);
        acc.z = fmaf(s_w[j], v[jj].z, acc.z);
        acc.w = fmaf(s_w[j], v[jj].w, acc.w);
      } else if (j < kS) {  // then the shared experts
        acc.x += v[jj].x;
        acc.y += v[jj].y;
        acc.z += v[jj].z;
        acc.w += v[jj].w;
      }
    }
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + (size_t)t * H + o) = pk;
}

}  // namespace

cudaError_t launch_combine(const Work& wk, int T, const Shape& s, __nv_bfloat16* out, cudaStream_t st, bool pdl) {
  const int threads = 64;  // more, smaller blocks: the combine is latency-bound at small T
  dim3 grid((s.H / 4 + threads - 1) / threads, T);
  if (!pdl) {
    combine_kernel<<<grid, threads, 0, st>>>(wk.y, wk.w, wk.inv, s.H, s.k, s.S, out, T * (s.k + s.S), wk.err);
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
  return cudaLaunchKernelEx(&cfg, combine_kernel, (const float*)wk.y, (const float*)wk.w, (const int*)wk.inv, s.H,
                            s.k, s.S, out, T * (s.k + s.S), wk.err);
}

}  // namespace moe
