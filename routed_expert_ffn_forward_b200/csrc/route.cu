// Decode-path routing in one launch (T <= 64): router logits, top-k + gating,
// the counting-sort permutation, the lists of active experts, and the fp16
// fixed-point copy of x that the expert kernels read.
//
// One CTA per expert computes that expert's logits for every token (all 1024
// threads share the row, four tokens at a time).  Independently
// of routing, every CTA also converts a slice of x: each 32-element run of x
// becomes 16-bit fixed point with its own power-of-two scale, stored as a
// high-byte and a low-byte plane, with the run's scale and sum.
// The last CTA to finish (a ticket counter) does the top-k for all tokens and
// the stable permutation in shared memory.
#include "moe_internal.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {
namespace {

constexpr int kRouteThreads = 256;


template <int PL>
__global__ void __launch_bounds__(kRouteThreads) route_decode_kernel(RouteArgs a) {
  extern __shared__ float4 smem_f4[];
  __shared__ float s_red[kRouteThreads / 32][4];
  const int e = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, T = a.T, E = a.E;
  // the first kernel of a forward: let the expert kernel start launching now
  ptx::pdl_launch_dependents();

  // (1) x prep: 16-bit fixed point per 32-element run, with the run scales
  const int runs_per_tok = H / 32;
  for (int run = e + gridDim.x * warp; run < T * runs_per_tok; run += gridDim.x * (kRouteThreads / 32)) {
    const int t = run / runs_per_tok, r = run - t * runs_per_tok;
    const int h = r * 32 + lane;
    float2 rsc;
    int8_t xh;
    uint8_t xl;
    quant_run16(__bfloat162float(a.x[(size_t)t * H + h]), xh, xl, rsc);
    a.xq[(size_t)t * H + h] = xh;
    reinterpret_cast<uint8_t*>(a.xq + a.xq_plane)[(size_t)t * H + h] = xl;
    if (lane == 0) a.xsc[(size_t)t * runs_per_tok + r] = rsc;
  }

  // (2) logits of expert e: every thread takes 4-element pieces of the row
  // (h = 4*tid + 4096*i) for up to 4 tokens at a time; partial sums are
  // reduced in a fixed order (warp xor tree, then warps in index order).
  const float4* wrow = reinterpret_cast<const float4*>(a.W + (size_t)e * H);
  const float bias = a.b ? a.b[e] : 0.f;
  for (int t0 = 0; t0 < T; t0 += 4) {
    const int nt = min(4, T - t0);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int q = tid; q < H / 4; q += kRouteThreads) {
      const float4 w4 = __ldg(wrow + q);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i < nt) {
          const uint2 xv = __ldg(reinterpret_cast<const uint2*>(a.x + (size_t)(t0 + i) * H) + q);
          acc[i] = fmaf(w4.x, bf16lo(xv.x), acc[i]);
          acc[i] = fmaf(w4.y, bf16hi(xv.x), acc[i]);
          acc[i] = fmaf(w4.z, bf16lo(xv.y), acc[i]);
          acc[i] = fmaf(w4.w, bf16hi(xv.y), acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
      if (lane == 0) s_red[warp][i] = acc[i];
    }
    __syncthreads();
    if (warp == 0 && lane < nt) {
      float v = 0.f;
      for (int w = 0; w < kRouteThreads / 32; ++w) v += s_red[w][lane];
      a.logits[(size_t)(t0 + lane) * E + e] = v + bias;
    }
    __syncthreads();
  }

  // (4) the last CTA finishes the routing
  __shared__ bool s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int k = a.k, S = a.S, kS = k + S, N = T * k, ES = E + S;
  int* s_ids = reinterpret_cast<int*>(smem_f4);   // [N]
  float* s_wt = reinterpret_cast<float*>(s_ids + N);
  int* s_cnt = reinterpret_cast<int*>(s_wt + N);  // [ES]
  int* s_off = s_cnt + ES;                        // [ES + 1]
  __shared__ int s_scan[32];
  __syncthreads();

  // top-k + gating, one warp per token (logits read from L2: other CTAs wrote them)
  for (int t = warp; t < T; t += kRouteThreads / 32)
    warp_topk_gate<PL, true>(a.logits + (size_t)t * E, E, k, a.gating, a.forced ? a.forced + (size_t)t * k : nullptr,
                             s_ids + (size_t)t * k, s_wt + (size_t)t * k);
  for (int i = tid; i < ES; i += kRouteThreads) s_cnt[i] = i < E ? 0 : T;
  __syncthreads();
  for (int i = tid; i < N; i += kRouteThreads) {
    atomicAdd(&s_cnt[s_ids[i]], 1);
    a.ids[i] = s_ids[i];
    a.w[i] = s_wt[i];
  }
  __syncthreads();
  // exclusive scan of the counts (routed experts, then shared) and the active lists
  int base = 0, base1 = 0, base2 = 0;
  for (int c0 = 0; c0 < ES; c0 += kRouteThreads) {
    const int i = c0 + tid;
    const int cnt = i < ES ? s_cnt[i] : 0;
    const int small = (cnt > 0 && cnt <= kD1MaxTok) ? 1 : 0, big = cnt > kD1MaxTok ? 1 : 0;
    // three scans share s_scan: do them one after another
    int tot;
    const int pre = block_exclusive_scan_1024(cnt, &tot, s_scan);
    if (i < ES) {
      s_off[i] = base + pre;
      a.counts[i] = cnt;
      a.offsets[i] = base + pre;
    }
    base += tot;
    const int p1 = block_exclusive_scan_1024(small, &tot, s_scan);
    if (small) a.act1[base1 + p1] = i;
    base1 += tot;
    const int p2 = block_exclusive_scan_1024(big, &tot, s_scan);
    if (big) a.act2[base2 + p2] = i;
    base2 += tot;
  }
  if (tid == 0) {
    a.offsets[ES] = base;
    *a.n_act1 = base1;
    *a.n_act2 = base2;
    *a.n_act = base1 + base2;
  }
  __syncthreads();
  // stable scatter: rank of pick i among the earlier picks of the same expert
  for (int i = tid; i < N; i += kRouteThreads) {
    const int ex = s_ids[i];
    int rank = 0;
    for (int j = 0; j < i; ++j) rank += s_ids[j] == ex;
    const int t = i / k, j = i - t * k;
    const int r = s_off[ex] + rank;
    a.perm[r] = t * kS + j;
    a.inv[t * kS + j] = r;
  }
  for (int i = tid; i < T * S; i += kRouteThreads) {
    const int s = i / T, t = i - s * T;
    const int r = N + s * T + t;
    a.perm[r] = t * kS + k + s;
    a.inv[t * kS + k + s] = r;
  }
  if (tid == 0) *a.ticket = 0u;
}

}  // namespace

size_t route_decode_smem(int H, int T, int E, int k, int S) {
  (void)H;
  return (size_t)T * k * 8 + (size_t)(E + S) * 4 + (size_t)(E + S + 1) * 4;
}

cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st) {
  const size_t smem = route_decode_smem(a.H, a.T, a.E, a.k, a.S);
  const int pl = (a.E + 31) / 32;
  cudaError_t err;
  if (pl <= 8) {
    err = cudaFuncSetAttribute(route_decode_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    route_decode_kernel<8><<<a.E, kRouteThreads, smem, st>>>(a);
  } else {
    err = cudaFuncSetAttribute(route_decode_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    route_decode_kernel<32><<<a.E, kRouteThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace moe
