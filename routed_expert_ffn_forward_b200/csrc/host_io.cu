// Host-buffer forward on the decode path: the token activations are read
// straight from mapped pinned host memory into the device buffer the forward
// reads, by a kernel that the route kernel runs behind as a programmatic
// dependent (its constant router weights are in flight while x crosses the
// host link).
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void stage_in_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  // the route kernel may launch now: it waits for this kernel before it reads x
  ptx::pdl_launch_dependents();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __ldcv(src + i);  // host memory: fetched, not cached
}

}  // namespace

cudaError_t launch_stage_in(const void* src, void* dst, size_t bytes, cudaStream_t st) {
  if ((bytes & 15u) || (reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(dst) & 15u))
    return cudaErrorInvalidValue;
  const size_t n16 = bytes / 16;
  if (n16 == 0) return cudaSuccess;
  constexpr int kThreads = 128;
  const unsigned blocks = (unsigned)std::min<size_t>((n16 + kThreads - 1) / kThreads, 1024);
  stage_in_kernel<<<blocks, kThreads, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16);
  return cudaGetLastError();
}

}  // namespace moe
