// Decode-path routing (T <= 4): one kernel.
//
// Each of E CTAs computes one expert's logits for every token (256 threads
// share the weight row; partial sums reduced in a fixed order).  Independently of routing, every CTA also converts a slice of
// x: each 32-element run becomes 16-bit fixed point with its own power-of-two
// scale (a high-byte and a low-byte plane), with the run's scale and sum --
// the form the expert kernels read.
//
// The last CTA to write its logits (a device-wide ticket) then does the top-k + gating
// of every token (a warp per token) and the stable counting-sort permutation
// of the T*k picks.  With few picks each pick's sorted position is found by
// counting the picks before it in (expert, token, slot) order, so no pass over
// all E expert counters is needed; only experts with rows get counts and
// offsets.
#include "moe_internal.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {
namespace {

constexpr int kLogitThreads = 256;

template <int PL>
__device__ void route_finish(const RouteArgs& a, int* s_ids);

// kT: 1 (decode of one token) or kD1MaxTok (up to that many tokens)
template <int PL, int kT>
__global__ void __launch_bounds__(kLogitThreads, 2) route_kernel(RouteArgs a) {
  extern __shared__ int s_dyn[];  // the finishing CTA's pick lists
  __shared__ float s_red[kLogitThreads / 32][kD1MaxTok];
  __shared__ bool s_last;
  const int e = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, T = a.T, E = a.E;
  // the first kernel of a forward: let the expert kernel start launching now
  // (it waits for this kernel's completion before it reads anything)
  ptx::pdl_launch_dependents();

  // (1) logits of expert e for the T <= 4 tokens (first: the weight row is the
  // long-latency load); thread takes 4-element pieces h = 4*tid + 1024*i
  // The thread's weight and activation pieces of a pass are all loaded before
  // any arithmetic, so the CTA waits for one memory round trip per pass.
  // Launched as a programmatic dependent (of the kernel that stages x from
  // host memory, or of whatever precedes the forward), the kernel issues the
  // constant router weights before it waits for its predecessor; x and every
  // write come after the wait.
  constexpr int kPieces = 8;                     // per pass: H <= 8192 takes one pass
  const float4* wrow = reinterpret_cast<const float4*>(a.W + (size_t)e * H);
  const float bias = a.b ? a.b[e] : 0.f;
  const int nq = H / 4;
  float acc[kT];
#pragma unroll
  for (int t = 0; t < kT; ++t) acc[t] = 0.f;
  for (int base = 0; base < nq; base += kPieces * kLogitThreads) {
    float4 w4[kPieces];
    uint2 xv[kT][kPieces];
#pragma unroll
    for (int i = 0; i < kPieces; ++i) {
      const int q = base + tid + kLogitThreads * i;
      if (q < nq) w4[i] = __ldg(wrow + q);
    }
    ptx::pdl_wait();  // returns at once after the first pass
#pragma unroll
    for (int i = 0; i < kPieces; ++i) {
      const int q = base + tid + kLogitThreads * i;
      if (q < nq) {
#pragma unroll
        for (int t = 0; t < kT; ++t)
          if (t < T) xv[t][i] = __ldcg(reinterpret_cast<const uint2*>(a.x + (size_t)t * H) + q);
      }
    }
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      if (t < T) {
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          if (base + tid + kLogitThreads * i < nq) {
            acc[t] = fmaf(w4[i].x, bf16lo(xv[t][i].x), acc[t]);
            acc[t] = fmaf(w4[i].y, bf16hi(xv[t][i].x), acc[t]);
            acc[t] = fmaf(w4[i].z, bf16lo(xv[t][i].y), acc[t]);
            acc[t] = fmaf(w4[i].w, bf16hi(xv[t][i].y), acc[t]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kT; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    if (lane == 0) s_red[warp][t] = acc[t];
  }
  __syncthreads();
  if (warp == 0 && lane < T) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kLogitThreads / 32; ++w) v += s_red[w][lane];
    a.logits[(size_t)lane * E + e] = v + bias;
  }
  // (2) the ticket, as soon as the logits are written: the last CTA to take
  // it does the routing of every token.  One release-acquire atomic per CTA,
  // cumulative over the writes the barrier orders before it.
  __syncthreads();
  if (tid == 0) s_last = ptx::atom_add_acq_rel_gpu(a.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  // (3) x prep: 16-bit fixed point per 32-element run, with the run scales;
  // the highest warps take the runs (the finishing CTA's top-k runs on warp 0)
  const int runs_per_tok = H / 32;
  const int xw = kLogitThreads / 32 - 1 - warp;
  for (int run = e + gridDim.x * xw; run < T * runs_per_tok; run += gridDim.x * (kLogitThreads / 32)) {
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

  if (!s_last) return;
  route_finish<PL>(a, s_dyn);
  if (tid == 0) *a.ticket = 0u;
}

template <int PL>
__device__ void route_finish(const RouteArgs& a, int* s_ids) {
  __shared__ int s_cnt_small, s_cnt_big;  // distinct routed experts with <= / > kD1MaxTok rows
  const int tid = threadIdx.x, warp = tid >> 5;
  const int T = a.T, E = a.E, k = a.k, S = a.S, kS = k + S, N = T * k;
  int* s_first = s_ids + N;               // [N] 1 if pick i is its expert's first pick
  int* s_count = s_first + N;             // [N] rows of pick i's expert
  // top-k + gating, one warp per token (no barrier before it: the CTA's last
  // x-prep run, on the highest warp, overlaps it)
  for (int t = warp; t < T; t += kLogitThreads / 32)
    warp_topk_gate<PL, true>(a.logits + (size_t)t * E, E, k, a.gating, a.forced ? a.forced + (size_t)t * k : nullptr,
                             s_ids + t * k, a.w + (size_t)t * k);
  if (tid == 0) {
    s_cnt_small = 0;
    s_cnt_big = 0;
  }
  __syncthreads();
  // per pick: rows of its expert, whether it is the expert's first pick
  for (int i = tid; i < N; i += kLogitThreads) {
    const int ex = s_ids[i];
    int cnt = 0, before = 0;
    for (int j = 0; j < N; ++j) {
      const int kj = s_ids[j];
      cnt += kj == ex;
      before += (kj == ex) & (j < i);
    }
    s_first[i] = before == 0;
    s_count[i] = cnt;
    a.ids[i] = ex;
  }
  __syncthreads();
  // sorted positions: picks of smaller experts first, then earlier picks of
  // the same expert; first picks also place their expert in the active lists
  for (int i = tid; i < N; i += kLogitThreads) {
    const int ex = s_ids[i];
    int lt = 0, eq_before = 0, d_small = 0, d_big = 0;
    for (int j = 0; j < N; ++j) {
      const int kj = s_ids[j];
      lt += kj < ex;
      eq_before += (kj == ex) & (j < i);
      const bool distinct_lt = (kj < ex) & (s_first[j] != 0) & ep_owned(kj, a.ep_rank, a.ep_world);
      d_small += distinct_lt & (s_count[j] <= kD1MaxTok);
      d_big += distinct_lt & (s_count[j] > kD1MaxTok);
    }
    const int t = i / k, j = i - t * k;
    const int r = lt + eq_before;
    a.perm[r] = t * kS + j;
    a.inv[t * kS + j] = r;
    if (s_first[i]) {
      a.counts[ex] = s_count[i];
      a.offsets[ex] = lt;
      if (!ep_owned(ex, a.ep_rank, a.ep_world)) {
        // another rank's expert: no work here
      } else if (s_count[i] <= kD1MaxTok) {
        a.act1[d_small] = ex;
        atomicAdd(&s_cnt_small, 1);
      } else {
        a.act2[d_big] = ex;
        atomicAdd(&s_cnt_big, 1);
      }
    }
  }
  // shared experts: all T tokens, after the routed rows
  for (int i = tid; i < T * S; i += kLogitThreads) {
    const int s = i / T, t = i - s * T;
    const int r = N + s * T + t;
    a.perm[r] = t * kS + k + s;
    a.inv[t * kS + k + s] = r;
  }
  __syncthreads();
  int own_shared = 0;  // owned shared experts (uniform across the block)
  for (int q = 0; q < S; ++q) own_shared += ep_owned(E + q, a.ep_rank, a.ep_world);
  if (tid < S) {
    const int ex = E + tid;
    a.counts[ex] = T;
    a.offsets[ex] = N + tid * T;
    if (ep_owned(ex, a.ep_rank, a.ep_world)) {
      int pos = 0;
      for (int q = 0; q < tid; ++q) pos += ep_owned(E + q, a.ep_rank, a.ep_world);
      if (T <= kD1MaxTok)
        a.act1[s_cnt_small + pos] = ex;
      else
        a.act2[s_cnt_big + pos] = ex;
    }
  }
  if (tid == 0) {
    const int n1 = s_cnt_small + (T <= kD1MaxTok ? own_shared : 0),
              n2 = s_cnt_big + (T <= kD1MaxTok ? 0 : own_shared);
    *a.n_act1 = n1;
    *a.n_act2 = n2;
    *a.n_act = n1 + n2;
    a.offsets[E + S] = T * kS;
  }
}

}  // namespace

size_t route_decode_smem(int H, int T, int E, int k, int S) {
  (void)H;
  (void)E;
  (void)S;
  return (size_t)T * k * 3 * sizeof(int);
}

cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st) {
  const size_t smem = route_decode_smem(a.H, a.T, a.E, a.k, a.S);
  if (a.T > kD1MaxTok) return cudaErrorInvalidValue;
  const bool small_e = (a.E + 31) / 32 <= 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.E);
  cfg.blockDim = dim3(kLogitThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.T == 1)
    return small_e ? cudaLaunchKernelEx(&cfg, route_kernel<8, 1>, a) : cudaLaunchKernelEx(&cfg, route_kernel<32, 1>, a);
  return small_e ? cudaLaunchKernelEx(&cfg, route_kernel<8, kD1MaxTok>, a)
                 : cudaLaunchKernelEx(&cfg, route_kernel<32, kD1MaxTok>, a);
}

}  // namespace moe
