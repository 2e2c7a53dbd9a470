// Counting-sort permutation of (token, slot) pairs by expert.
//
// Pairs are numbered p = t*(k+S) + j: j < k are the routed picks of token t,
// j >= k its shared experts E + (j-k).  Rows of the expert-sorted order are
// grouped by expert (routed experts ascending, then the shared ones) and, inside
// an expert, ordered by (t, j): a stable counting sort.
//
// One block per expert.  Block e finds its offset by counting the picks with a
// smaller id and its rows by a stable block-wide compaction of the picks equal
// to e; no block depends on another, and the last block to finish lists the
// experts that have rows.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kPermThreads = 256;

// Block-wide exclusive scan of one int per thread; returns the prefix and
// writes the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int wv = lane < nw ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += n;
    }
    if (lane < nw) s_warp[lane] = wv;  // inclusive prefix over warps
  }
  __syncthreads();
  const int before = warp ? s_warp[warp - 1] : 0;
  *total = s_warp[nw - 1];
  __syncthreads();
  return before + incl - v;
}

__device__ __forceinline__ int block_sum(int v, int* s_warp) {
  int total;
  block_exclusive_scan(v, &total, s_warp);
  return total;
}

__global__ void __launch_bounds__(kPermThreads)
permute_kernel(const int* __restrict__ ids, int T, int E, int k, int S, int* __restrict__ counts,
               int* __restrict__ offsets, int* __restrict__ perm, int* __restrict__ inv,
               int* __restrict__ act, int* __restrict__ n_act, unsigned* __restrict__ ticket) {
  __shared__ int s_warp[32];
  __shared__ bool s_last;
  const int e = blockIdx.x;
  const int kS = k + S;
  const int N = T * k;
  int offset, count;
  if (e < E) {
    int lt = 0, eq = 0;
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      const int v = ids[i];
      lt += v < e;
      eq += v == e;
    }
    offset = block_sum(lt, s_warp);
    count = block_sum(eq, s_warp);
    int base = 0;
    for (int c0 = 0; c0 < N && base < count; c0 += blockDim.x) {
      const int i = c0 + threadIdx.x;
      const int m = (i < N && ids[i] == e) ? 1 : 0;
      int tot;
      const int rank = block_exclusive_scan(m, &tot, s_warp);
      if (m) {
        const int t = i / k, j = i - t * k;
        const int r = offset + base + rank;
        perm[r] = t * kS + j;
        inv[t * kS + j] = r;
      }
      base += tot;
    }
  } else {
    const int s = e - E;
    offset = N + s * T;
    count = T;
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const int r = offset + t;
      perm[r] = t * kS + k + s;
      inv[t * kS + k + s] = r;
    }
  }
  if (threadIdx.x == 0) {
    counts[e] = count;
    offsets[e] = offset;
    if (e == E + S - 1) offsets[E + S] = T * kS;
  }
  // the last block to finish lists the experts with rows, in ascending order
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int base = 0;
  for (int c0 = 0; c0 < E + S; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const int m = (i < E + S && __ldcg(counts + i) > 0) ? 1 : 0;
    int tot;
    const int pos = block_exclusive_scan(m, &tot, s_warp);
    if (m) act[base + pos] = i;
    base += tot;
  }
  if (threadIdx.x == 0) {
    *n_act = base;
    *ticket = 0u;
  }
}

__global__ void set_slots_kernel(int* slot_of, SlotUpdate u) {
  const int i = threadIdx.x;
  if (i < u.n) slot_of[u.expert[i]] = u.slot[i];
}

}  // namespace

cudaError_t launch_permute(const int* ids, int T, const Shape& s, const Work& wk, cudaStream_t st) {
  permute_kernel<<<s.E + s.S, kPermThreads, 0, st>>>(ids, T, s.E, s.k, s.S, wk.counts, wk.offsets,
                                                     wk.perm, wk.inv, wk.act, wk.n_act, wk.ticket);
  return cudaGetLastError();
}

cudaError_t launch_set_slots(int* slot_of, const SlotUpdate& u, cudaStream_t st) {
  set_slots_kernel<<<1, SlotUpdate::kMax, 0, st>>>(slot_of, u);
  return cudaGetLastError();
}

}  // namespace moe
