// Expert SwiGLU FFN on Q4_K weights, plain SIMT version (exact fp32 dequant).
//
// For every expert with rows (act list) and each of its rows r (one (token,
// slot) pair): h[r] = silu(W_g x_t) * (W_u x_t) and y[r] = W_d h[r].
// One warp per weight row; lane l takes 16-byte quant segments l, l+32, ... of
// the row, so a warp's loads of a super-block are contiguous.  Each segment
// holds 32 weights: the low nibbles of 16 bytes (sub-block 2c) and their high
// nibbles (sub-block 2c+1), dequantised exactly in fp32 as d*sc*q - dmin*m.
// Work units are (active expert, 8-row tile), walked by a grid-stride loop
// because the number of active experts is only known on the device.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRowsPerBlock = 8;   // one row per warp
constexpr int kTokChunk = 4;       // tokens per pass over a row

// Dequantise segment `part` (0..7) of super-block `blk`: w[0..15] are the
// weights 64c + 16(part&1) + i of sub-block 2c, w[16..31] those 32 further on
// (sub-block 2c+1), with c = part >> 1.
__device__ __forceinline__ void dequant_segment(const uint8_t* __restrict__ blk, int part, float* w) {
  const uint4 hdr = __ldg(reinterpret_cast<const uint4*>(blk));
  const uint4 qv = __ldg(reinterpret_cast<const uint4*>(blk + 16 + part * 16));
  const float d = __half2float(__ushort_as_half((unsigned short)(hdr.x & 0xFFFF)));
  const float dmin = __half2float(__ushort_as_half((unsigned short)(hdr.x >> 16)));
  uint8_t sb[12];
  const uint32_t words[3] = {hdr.y, hdr.z, hdr.w};
#pragma unroll
  for (int i = 0; i < 12; ++i) sb[i] = (uint8_t)(words[i >> 2] >> (8 * (i & 3)));
  const int c = part >> 1;
  int sc0, m0, sc1, m1;
  q4k_scale_min(sb, 2 * c, sc0, m0);
  q4k_scale_min(sb, 2 * c + 1, sc1, m1);
  const float s0 = d * (float)sc0, n0 = dmin * (float)m0;
  const float s1 = d * (float)sc1, n1 = dmin * (float)m1;
  const uint32_t q[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t byte = (q[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    w[i] = fmaf(s0, (float)(byte & 15u), -n0);
    w[16 + i] = fmaf(s1, (float)(byte >> 4), -n1);
  }
}

// 16 consecutive bf16 -> fp32
__device__ __forceinline__ void load16_bf16(const __nv_bfloat16* __restrict__ p, float* v) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p + 8));
  const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16lo(u[i]);
    v[2 * i + 1] = bf16hi(u[i]);
  }
}

__device__ __forceinline__ void load16_f32(const float* __restrict__ p, float* v) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p) + i);
    v[4 * i] = a.x;
    v[4 * i + 1] = a.y;
    v[4 * i + 2] = a.z;
    v[4 * i + 3] = a.w;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// gate/up + SwiGLU:  h[r, i] = silu(W_g[i] . x_t) * (W_u[i] . x_t)
__global__ void __launch_bounds__(kRowsPerBlock * 32)
gate_up_simt_kernel(const uint8_t* const* __restrict__ wptr, const __nv_bfloat16* __restrict__ x,
                    int H, int I, int nbh, int kS, int tiles, const int* __restrict__ act,
                    const int* __restrict__ n_act, const int* __restrict__ counts,
                    const int* __restrict__ offsets, const int* __restrict__ perm,
                    float* __restrict__ h, int I_pad) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = *n_act * tiles;
  const size_t row_bytes = (size_t)nbh * kQBytes;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int a = unit / tiles, tile = unit - a * tiles;
    const int e = act[a];
    const int c = counts[e], r0 = offsets[e];
    const int row = tile * kRowsPerBlock + warp;
    if (row >= I) continue;
    const uint8_t* grow = wptr[3 * e + 0] + row * row_bytes;
    const uint8_t* urow = wptr[3 * e + 1] + row * row_bytes;
    for (int tc = 0; tc < c; tc += kTokChunk) {
      const int nt = min(kTokChunk, c - tc);
      const __nv_bfloat16* xr[kTokChunk];
#pragma unroll
      for (int i = 0; i < kTokChunk; ++i)
        xr[i] = x + (size_t)(perm[r0 + tc + min(i, nt - 1)] / kS) * H;
      float ag[kTokChunk], au[kTokChunk];
#pragma unroll
      for (int i = 0; i < kTokChunk; ++i) ag[i] = au[i] = 0.f;
      for (int seg = lane; seg < nbh * 8; seg += 32) {
        const int b = seg >> 3, part = seg & 7;
        float wg[32], wu[32];
        dequant_segment(grow + b * kQBytes, part, wg);
        dequant_segment(urow + b * kQBytes, part, wu);
        const int xo = b * kQK + (part >> 1) * 64 + (part & 1) * 16;
#pragma unroll
        for (int i = 0; i < kTokChunk; ++i) {
          if (i < nt) {
            float xv[32];
            load16_bf16(xr[i] + xo, xv);
            load16_bf16(xr[i] + xo + 32, xv + 16);
            float sg = 0.f, su = 0.f;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              sg = fmaf(wg[q], xv[q], sg);
              su = fmaf(wu[q], xv[q], su);
            }
            ag[i] += sg;
            au[i] += su;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kTokChunk; ++i) {
        const float g = warp_sum(ag[i]);
        const float u = warp_sum(au[i]);
        if (lane == 0 && i < nt) h[(size_t)(r0 + tc + i) * I_pad + row] = silu_f(g) * u;
      }
    }
  }
}

// down:  y[r, o] = W_d[o] . h[r]
__global__ void __launch_bounds__(kRowsPerBlock * 32)
down_simt_kernel(const uint8_t* const* __restrict__ wptr, const float* __restrict__ h, int H,
                 int nbi, int I_pad, int tiles, const int* __restrict__ act,
                 const int* __restrict__ n_act, const int* __restrict__ counts,
                 const int* __restrict__ offsets, float* __restrict__ y) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = *n_act * tiles;
  const size_t row_bytes = (size_t)nbi * kQBytes;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int a = unit / tiles, tile = unit - a * tiles;
    const int e = act[a];
    const int c = counts[e], r0 = offsets[e];
    const int row = tile * kRowsPerBlock + warp;
    if (row >= H) continue;
    const uint8_t* drow = wptr[3 * e + 2] + row * row_bytes;
    for (int tc = 0; tc < c; tc += kTokChunk) {
      const int nt = min(kTokChunk, c - tc);
      float acc[kTokChunk];
#pragma unroll
      for (int i = 0; i < kTokChunk; ++i) acc[i] = 0.f;
      for (int seg = lane; seg < nbi * 8; seg += 32) {
        const int b = seg >> 3, part = seg & 7;
        float wd[32];
        dequant_segment(drow + b * kQBytes, part, wd);
        const int xo = b * kQK + (part >> 1) * 64 + (part & 1) * 16;
#pragma unroll
        for (int i = 0; i < kTokChunk; ++i) {
          if (i < nt) {
            const float* hr = h + (size_t)(r0 + tc + i) * I_pad;
            float hv[32];
            load16_f32(hr + xo, hv);
            load16_f32(hr + xo + 32, hv + 16);
            float s = 0.f;
#pragma unroll
            for (int q = 0; q < 32; ++q) s = fmaf(wd[q], hv[q], s);
            acc[i] += s;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kTokChunk; ++i) {
        const float v = warp_sum(acc[i]);
        if (lane == 0 && i < nt) y[(size_t)(r0 + tc + i) * H + row] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_gate_up_simt(const uint8_t* const* wptr, const __nv_bfloat16* x, const Shape& s,
                                const Work& wk, cudaStream_t st) {
  const int tiles = (s.I + kRowsPerBlock - 1) / kRowsPerBlock;
  gate_up_simt_kernel<<<s.n_sm * 8, kRowsPerBlock * 32, 0, st>>>(wptr, x, s.H, s.I, s.nbh, s.k + s.S, tiles,
                                                                wk.act, wk.n_act, wk.counts, wk.offsets,
                                                                wk.perm, wk.h, s.I_pad);
  return cudaGetLastError();
}

cudaError_t launch_down_simt(const uint8_t* const* wptr, const Shape& s, const Work& wk, cudaStream_t st) {
  const int tiles = (s.H + kRowsPerBlock - 1) / kRowsPerBlock;
  down_simt_kernel<<<s.n_sm * 8, kRowsPerBlock * 32, 0, st>>>(wptr, wk.h, s.H, s.nbi, s.I_pad, tiles, wk.act,
                                                             wk.n_act, wk.counts, wk.offsets, wk.y);
  return cudaGetLastError();
}

}  // namespace moe
