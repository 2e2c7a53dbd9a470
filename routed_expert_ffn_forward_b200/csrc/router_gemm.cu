// Router logits for T > 4 tokens on the tensor cores.
//
// l[t, e] = x[t, :] . W[e, :] with x bf16 and W fp32.  W is held as three
// bf16 planes W = W0 + W1 + W2 (each plane the bf16 rounding of what the
// previous ones leave), which carries all 24 bits of W's significand, so every
// product of bf16 x with a plane is exact.
//
// The tensor cores' fp32 accumulation loses precision over long chains of
// MMAs, so K is taken in chunks of 256: each chunk accumulates in tensor
// memory (W0 products in one accumulator, W1 + W2 products in another), and
// the epilogue adds the chunk sums to fp32 registers in chunk order with
// ordinary round-to-nearest adds.  Two TMEM buffers let the next chunk's MMAs
// run while the epilogue drains the previous one.
//
// CTA tile: 128 tokens (MMA M) x 128 experts (MMA N) over one K range (split
// K, to fill the GPU); each split writes its sums to its own slice of `part`,
// and the top-k kernel adds the slices in split order, then the bias -- a
// fixed order, so the logits do not depend on scheduling.
//
//   warp 0     TMA producer: x tile (128 x 64, 128B-swizzled) and the three
//              W-plane tiles of each 64-wide K step
//   warp 1     TMEM allocation (512 columns); one thread issues tcgen05.mma
//              (kind::f16 with bf16 operands, M128 N<=128 K16, 3 per K16)
//   warps 2-9  epilogue: a warp owns 32 tokens (TMEM lane quarter warp % 4)
//              x 64 experts, chunk sums accumulated in registers
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kRM = 128, kRN = 128;
constexpr int kRStages = 3;
constexpr int kRChunk = 4;                           // 64-wide K steps per TMEM accumulation chain
constexpr int kRTile = 128 * 64 * 2;                 // 16 KB: one 128 x 64 bf16 tile
constexpr int kRStageBytes = 4 * kRTile;             // x tile + 3 W-plane tiles
constexpr int kREpiWarps = 8;
constexpr int kRThreads = (2 + kREpiWarps) * 32;
constexpr size_t kRSmem = 1024 + (size_t)kRStages * kRStageBytes + 8 * (2 * kRStages + 5) + 16;
static_assert(kRSmem <= 227 * 1024, "router GEMM shared memory");

__global__ void __launch_bounds__(kRThreads, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                       RouterGemmArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kRStages * kRStageBytes);
  uint64_t* empty = full + kRStages;
  uint64_t* acc_full = empty + kRStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile of this CTA: (token tile, expert tile, split)
  const int tiles_e = (a.E + kRN - 1) / kRN;
  const int split = blockIdx.x % a.nsplit;
  const int te = (blockIdx.x / a.nsplit) % tiles_e;
  const int tt = blockIdx.x / (a.nsplit * tiles_e);
  const int t0 = tt * kRM, e0 = te * kRN;
  const int ne = min(kRN, a.E - e0);
  const int kk0 = split * a.nk_split;
  const int nchunks = (a.nk_split + kRChunk - 1) / kRChunk;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&acc_full[i], 1);
      ptx::mbar_init(&acc_empty[i], kREpiWarps);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_barrier_init();
  }
  if (warp == 1) ptx::tmem_alloc(s_tmem, 512);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, last_ph = 0, ph = 0;
      int s = 0;
      for (int kk = 0; kk < a.nk_split; ++kk) {
        if (!ptx::mbar_wait(&empty[s], ph ^ 1u)) {
          atomicOr(a.err, 512u);
          break;
        }
        uint8_t* st = sm + s * kRStageBytes;
        const int kx = (kk0 + kk) * 64;
        ptx::mbar_arrive_expect_tx(&full[s], kRStageBytes);
        ptx::tma_load_2d(st, &xmap, kx, t0, &full[s]);
#pragma unroll
        for (int p = 0; p < 3; ++p) ptx::tma_load_2d(st + (1 + p) * kRTile, &wmap, kx, p * a.E + e0, &full[s]);
        issued |= 1u << s;
        last_ph = (last_ph & ~(1u << s)) | (ph << s);
        if (++s == kRStages) { s = 0; ph ^= 1u; }
      }
      for (int i = 0; i < kRStages; ++i)
        if ((issued >> i) & 1u) ptx::mbar_wait(&full[i], (last_ph >> i) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = ptx::umma_idesc_bf16(kRM, (ne + 15) & ~15);
      uint32_t ph = 0;
      int s = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int b = c & 1;
        if (!ptx::mbar_wait(&acc_empty[b], ((c >> 1) & 1) ^ 1u)) {
          atomicOr(a.err, 512u);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_hi = tmem + (uint32_t)(b * 2 * kRN), d_lo = d_hi + kRN;
        bool ok = true;
        const int kend = min(a.nk_split, (c + 1) * kRChunk);
        for (int kk = c * kRChunk; kk < kend; ++kk) {
          if (!ptx::mbar_wait(&full[s], ph)) {
            atomicOr(a.err, 512u);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t base = ptx::smem_u32(sm + s * kRStageBytes);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t ad = ptx::umma_desc_sw128(base + 32 * k16);
            const bool first = kk == c * kRChunk && k16 == 0;
            ptx::umma_f16(d_hi, ad, ptx::umma_desc_sw128(base + kRTile + 32 * k16), idesc, !first);
            ptx::umma_f16(d_lo, ad, ptx::umma_desc_sw128(base + 2 * kRTile + 32 * k16), idesc, !first);
            ptx::umma_f16(d_lo, ad, ptx::umma_desc_sw128(base + 3 * kRTile + 32 * k16), idesc, true);
          }
          ptx::umma_commit(&empty[s]);
          if (++s == kRStages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        ptx::umma_commit(&acc_full[b]);
      }
      ptx::umma_commit(drain);
      if (!ptx::mbar_wait(drain, 0)) atomicOr(a.err, 512u);
    }
  } else {
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;            // experts half*64 .. +63 of the tile
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int b = c & 1;
      ok = ptx::mbar_wait(&acc_full[b], (c >> 1) & 1);
      __syncwarp();
      if (!ok) {
        atomicOr(a.err, 512u);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * 2 * kRN + half * 64);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float vh[32], vl[32];
        ptx::tmem_ld32(tb + 32 * h, vh);
        ptx::tmem_ld32(tb + kRN + 32 * h, vl);
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[32 * h + i] += vh[i] + vl[i];
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[b]);
    }
    const int t = t0 + q * 32 + lane;
    const int cbase = half * 64;
    if (ok && t < a.T) {
      float* dst = a.part + (size_t)split * a.split_stride + (size_t)t * a.E + e0 + cbase;
#pragma unroll
      for (int i = 0; i < 64; ++i)
        if (cbase + i < ne) dst[i] = acc[i];
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// W (fp32 [E, H]) -> three bf16 planes [3][E][H] with W ~= P0 + P1 + P2.
__global__ void split_router_kernel(const float* __restrict__ W, size_t n, __nv_bfloat16* __restrict__ planes) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float w = W[i];
    const __nv_bfloat16 p0 = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(p0);
    const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(p1);
    planes[i] = p0;
    planes[n + i] = p1;
    planes[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

}  // namespace

int router_gemm_splits(int T, int E, int H, int n_sm) {
  const int tiles = ((T + kRM - 1) / kRM) * ((E + kRN - 1) / kRN);
  const int nk = H / 64;
  int ns = 1;
  for (int d = 1; d <= nk; ++d)
    if (nk % d == 0 && tiles * d <= n_sm) ns = d;
  return ns;
}

size_t router_part_floats(int T_cap, int E, int n_sm) {
  return (size_t)std::max(T_cap, kRM * n_sm) * (size_t)E;
}

cudaError_t launch_split_router(const float* W, int E, int H, __nv_bfloat16* planes, cudaStream_t st) {
  const size_t n = (size_t)E * H;
  split_router_kernel<<<(unsigned)std::min<size_t>((n + 255) / 256, 4096), 256, 0, st>>>(W, n, planes);
  return cudaGetLastError();
}

cudaError_t launch_router_gemm(const CUtensorMap& xmap, const CUtensorMap& wmap, const RouterGemmArgs& a,
                               cudaStream_t st) {
  static uint64_t attr_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!(attr_done & (1ull << (dev & 63)))) {
    e = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRSmem);
    if (e != cudaSuccess) return e;
    attr_done |= 1ull << (dev & 63);
  }
  const int tiles = ((a.T + kRM - 1) / kRM) * ((a.E + kRN - 1) / kRN);
  router_gemm_kernel<<<tiles * a.nsplit, kRThreads, kRSmem, st>>>(xmap, wmap, a);
  return cudaGetLastError();
}

}  // namespace moe
