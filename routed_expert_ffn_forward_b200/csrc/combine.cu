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
                               __nv_bfloat16* __restrict__ out) {
  // launched as a programmatic dependent of the down kernel on the decode path:
  // wait for it (a no-op when launched normally)
  ptx::pdl_wait();
  const int t = blockIdx.y;
  const int o = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (o >= H) return;
  const int kS = k + S;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int r = inv[t * kS + j];
    const float wj = w[(size_t)t * k + j];
    const float4 v = *reinterpret_cast<const float4*>(y + (size_t)r * H + o);
    acc.x = fmaf(wj, v.x, acc.x);
    acc.y = fmaf(wj, v.y, acc.y);
    acc.z = fmaf(wj, v.z, acc.z);
    acc.w = fmaf(wj, v.w, acc.w);
  }
  for (int s = 0; s < S; ++s) {
    const int r = inv[t * kS + k + s];
    const float4 v = *reinterpret_cast<const float4*>(y + (size_t)r * H + o);
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
  *reinterpret_cast<uint2*>(out + (size_t)t * H + o) = pk;
}

}  // namespace

cudaError_t launch_combine(const Work& wk, int T, const Shape& s, __nv_bfloat16* out, cudaStream_t st, bool pdl) {
  const int threads = 128;
  dim3 grid((s.H / 4 + threads - 1) / threads, T);
  if (!pdl) {
    combine_kernel<<<grid, threads, 0, st>>>(wk.y, wk.w, wk.inv, s.H, s.k, s.S, out);
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
                            s.k, s.S, out);
}

}  // namespace moe
