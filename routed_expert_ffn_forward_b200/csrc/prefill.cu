// Prefill path (T > 4): grouped GEMMs on the 5th-generation tensor cores
// (tcgen05.mma, fp32 accumulators in tensor memory) over Q4_K weights.
//
// A work unit is (tile, feature block): a tile is up to 256 consecutive rows
// of one expert in the expert-sorted order, a feature block 256 weight rows
// (gate/up: 128 gate rows + the same 128 up rows; down: 256 output rows).
// The weights are the A operand as two M = 128 halves, the tile's activation
// rows the B operand (N <= 256), so one dequantisation of a weight tile
// serves up to 256 rows and the two accumulators fill all 512 TMEM columns.
// K advances in steps of 32 (one Q4_K sub-block) through a 4-deep ring of
// 64B-swizzled A/B stages.
//
//   warp 0      producer of raw Q4_K tiles (2-D TMA, 128 rows x 1 super-block,
//               both A halves, two super-blocks in flight)
//   warp 1      producer of activation tiles (2-D TMA, 64B-swizzled fp16,
//               256 rows x 32 columns)
//   warp 2      TMEM allocation; one thread issues tcgen05.mma M128 N<=256 K16
//               and tcgen05.commit
//   warps 3-10  dequantise Q4_K to fp16 straight into the UMMA 64B-swizzled
//               K-major layout: warps 3-6 the first A half, 7-10 the second,
//               one weight row per thread
//   warps 11-18 epilogue: tcgen05.ld of the accumulators (a warp reads the TMEM
//               lane quarter warp % 4; two warps per quarter split the columns),
//               SwiGLU with the fast exp and divide intrinsics (relative error
//               ~1e-6, far below the fp16 rounding of the operands)
//
// Numerics: activations are fp16 scaled per row by a power of two (largest
// magnitude in [2^14, 2^15), 1/scale kept in `rinv`); weights are fp16 scaled
// per weight row by 2^k (sub-block scale and min rounded to fp16, one rounding
// per weight), k <= 8 chosen on the host from the row's blocks so that every
// intermediate stays below 60000 (`wexp`); products accumulate in fp32 and the
// epilogue undoes both scales exactly (powers of two).
//
// K order: within every group of four K elements both operands are stored in
// the order (0, 2, 1, 3), so two quant nibbles of one 32-bit word become one
// fp16x2 register without byte shuffles; the dot product is unchanged.
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kGM = 128;                       // rows of one A half (MMA M)
constexpr int kGN = 256;                       // activation rows per tile (max MMA N)
constexpr int kRawBytes = kGM * kQBytes;       // one A half, one super-block: 18432
constexpr int kABytes = kGM * 32 * 2;          // one A half, 32 K as fp16: 8192
constexpr int kBBytes = kGN * 32 * 2;          // 256 rows x 32 K as fp16: 16384
constexpr int kNR = 2;                         // raw super-block stages
constexpr int kNS = 4;                         // A/B stages (32 K each); even, a chunk fills two
constexpr int kDeqWarps = 8;
constexpr int kEpiWarps = 8;
constexpr int kFirstDeq = 3, kFirstEpi = kFirstDeq + kDeqWarps;
constexpr int kGemmThreads = (kFirstEpi + kEpiWarps) * 32;  // 608

constexpr size_t kSmemRaw = (size_t)kNR * 2 * kRawBytes;
constexpr size_t kSmemA = (size_t)kNS * 2 * kABytes;
constexpr size_t kSmemB = (size_t)kNS * kBBytes;
constexpr size_t kSmemBar = 8 * (2 * kNR + 3 * kNS + 2 + 1) + 16;
constexpr size_t kGemmSmem = 1024 + kSmemRaw + kSmemA + kSmemB + kSmemBar;
static_assert(kGemmSmem <= 227 * 1024, "GEMM shared memory");

// fp16x2 scale pair (s_lo, s_hi) = 2^k * d * (sc_2c, sc_2c+1) and min pair
// (nm_lo, nm_hi) = -2^k * dmin * (m_2c, m_2c+1) of chunk c of a Q4_K block
// whose first 16 bytes are `hdr` (fp16 d, fp16 dmin, 12 scale bytes).  All
// in fp16 arithmetic: the 6-bit fields become fp16 integers through the 1024
// exponent trick, and d * sc rounds once, as a float product converted to
// fp16 would.  `d2s`/`nm2s` are (2^k d, 2^k d) and (-2^k dmin, -2^k dmin).
__device__ __forceinline__ void chunk_scales(uint4 hdr, int c, __half2 d2s, __half2 nm2s, __half2& s2, __half2& nm2) {
  const uint32_t sh = 16u * (uint32_t)(c & 1);
  const uint32_t s0 = hdr.y >> sh, s1 = hdr.z >> sh, s2w = hdr.w >> sh;
  uint32_t vsc, vm;
  if (c < 2) {
    vsc = s0 & 0x3F3Fu;
    vm = s1 & 0x3F3Fu;
  } else {
    vsc = (s2w & 0x0F0Fu) | ((s0 >> 2) & 0x3030u);
    vm = ((s2w >> 4) & 0x0F0Fu) | ((s1 >> 2) & 0x3030u);
  }
  // bytes (f0, f1) -> fp16x2 (1024 + f0, 1024 + f1)
  const uint32_t tsc = __byte_perm(vsc, 0x64u, 0x4140u), tm = __byte_perm(vm, 0x64u, 0x4140u);
  const __half2 k1024 = __float2half2_rn(1024.f);
  const __half2 sc = __hsub2(*reinterpret_cast<const __half2*>(&tsc), k1024);
  const __half2 mm = __hsub2(*reinterpret_cast<const __half2*>(&tm), k1024);
  s2 = __hmul2(d2s, sc);
  nm2 = __hmul2(nm2s, mm);
}

// fp16x2 (o + a, o + b) -> (a * s - m, b * s - m), `off` = (o, o), `nm` = -m
__device__ __forceinline__ uint32_t deq2(uint32_t t, __half2 off, __half2 s, __half2 nm) {
  const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&t), off);
  const __half2 v = __hfma2(q, s, nm);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 2^e as a float, exactly, for -126 <= e <= 127
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }
// 2^e as an fp16 pair, exactly, for -14 <= e <= 15
__device__ __forceinline__ __half2 pow2h2(int e) {
  const uint32_t b = (uint32_t)(15 + e) << 10;
  const uint32_t v = b | (b << 16);
  return *reinterpret_cast<const __half2*>(&v);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* raw) {
  const uint32_t pad = (1024u - (ptx::smem_u32(raw) & 1023u)) & 1023u;
  return raw + pad;
}

// Epilogue of unit u, run by the epilogue warps: warp w reads TMEM lane
// quarter w % 4 and the 32-column chunks (w - first epilogue warp) / 4 + 2j.
// Returns false (error flag set) if the accumulators never became ready.
template <int kMode>
__device__ __forceinline__ bool gemm_epilogue(const GemmArgs& a, uint32_t tmem, uint64_t* acc_full,
                                              uint64_t* acc_empty, int u, uint32_t& fph, int wk, int warp,
                                              int lane) {
  const int4 tl = __ldcg(a.tiles + u / a.ft);
  const int f = u % a.ft;
  const int q = warp & 3;                      // TMEM lane quarter this warp may read
  const int sub = wk >> 2;                     // 0..kEpiWarps/4-1
  const int mrow = q * 32 + lane;              // row of the A halves
  const bool ok = ptx::mbar_wait_sleep(acc_full, fph, 200);
  __syncwarp();
  if (!ok) {
    atomicOr(a.err, 128u);
    return false;
  }
  fph ^= 1u;
  ptx::tc_fence_after();
  const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
  const int pair0 = tl.w + tl.y;
  // 2^-k of the weight rows this thread's accumulator lanes belong to
  const int8_t* wx = a.wexp + (size_t)in_range(tl.x, a.n_ex, a.err) * a.wexp_stride;
  float s0, s1;
  if (kMode == 0) {
    const int feat = min(f * kGM + mrow, a.out_rows - 1);
    s0 = pow2f(-__ldg(wx + feat));
    s1 = pow2f(-__ldg(wx + a.out_rows + feat));
  } else {
    const int orow = f * 2 * kGM + mrow;
    s0 = pow2f(-__ldg(wx + a.wexp_down + orow));
    s1 = pow2f(-__ldg(wx + a.wexp_down + orow + kGM));
  }
  for (int c0 = 32 * sub; c0 < tl.z; c0 += 32 * (kEpiWarps / 4)) {
    const int nc = min(32, tl.z - c0);
    // lane i holds the inverse scale of column c0 + i
    const float my_inv = __ldg(a.rinv + pair0 + c0 + min(lane, nc - 1));
    uint32_t r0[32], r1[32];
    ptx::tmem_ld32x2(tq + c0, tq + kGN + c0, r0, r1);
    if (kMode == 0) {
      const int feat = f * kGM + mrow;
      const bool frow = feat < a.out_rows;
      float* outp = a.out + (size_t)(pair0 + c0) * a.out_ld + feat;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float inv = __shfl_sync(0xffffffffu, my_inv, i);
        const float g = __uint_as_float(r0[i]) * (inv * s0), up = __uint_as_float(r1[i]) * (inv * s1);
        const float hv = __fdividef(g, 1.f + __expf(-g)) * up;   // silu(g) * up
        if (i < nc && frow) outp[(size_t)i * a.out_ld] = hv;
      }
    } else {
      const int orow = f * 2 * kGM + mrow;
      float* outp = a.out + (size_t)(pair0 + c0) * a.out_ld + orow;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float inv = __shfl_sync(0xffffffffu, my_inv, i);
        if (i < nc) {
          outp[(size_t)i * a.out_ld] = __uint_as_float(r0[i]) * (inv * s0);
          outp[(size_t)i * a.out_ld + kGM] = __uint_as_float(r1[i]) * (inv * s1);
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive(acc_empty);
  return true;
}

// kMode 0: gate/up, out = h (fp32 [P, ld]) = silu(g) * u.
// kMode 1: down,    out = y (fp32 [P, ld]).
template <int kMode>
__global__ void __launch_bounds__(kGemmThreads, 1) q4k_gemm_kernel(const __grid_constant__ CUtensorMap bmap,
                                                                    const GemmArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* s_rawbuf = sm;                       // [kNR][2][kRawBytes]
  uint8_t* s_a = s_rawbuf + kSmemRaw;           // [kNS][2][kABytes]
  uint8_t* s_b = s_a + kSmemA;                  // [kNS][kBBytes]
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(s_b + kSmemB);
  uint64_t* raw_empty = raw_full + kNR;
  uint64_t* a_full = raw_empty + kNR;
  uint64_t* b_full = a_full + kNS;
  uint64_t* ab_empty = b_full + kNS;
  uint64_t* acc_full = ab_empty + kNS;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNR; ++i) {
      ptx::mbar_init(&raw_full[i], 1);
      ptx::mbar_init(&raw_empty[i], kDeqWarps);
    }
    for (int i = 0; i < kNS; ++i) {
      ptx::mbar_init(&a_full[i], kDeqWarps);
      ptx::mbar_init(&b_full[i], 1);
      ptx::mbar_init(&ab_empty[i], 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, kEpiWarps);
    ptx::mbar_init(drain, 1);
    ptx::fence_barrier_init();
  }
  if (warp == 2) ptx::tmem_alloc(s_tmem, 512);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  ptx::pdl_wait();  // tiles, activations and scales of the previous kernels
  ptx::pdl_launch_dependents();

  const int ft = a.ft;
  const int n_units = __ldcg(a.n_tiles) * ft;

  if (warp == 0) {
    // ------------------------------------------------------------ raw weight tiles
    if (lane == 0) {
      int rs = 0;
      uint32_t rph = 0, issued = 0, last_ph = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int4 tl = __ldcg(a.tiles + u / ft);  // (expert, n0, count, r0)
        const int f = u % ft;
        const int ex = in_range(tl.x, a.n_ex, a.err);
        const CUtensorMap* wm = a.wmaps + kMapsPerSlot * in_range(__ldcg(a.slot_of + ex), a.n_slots, a.err) + 3;
        const CUtensorMap* m0 = kMode == 0 ? wm : wm + 2;
        const CUtensorMap* m1 = kMode == 0 ? wm + 1 : wm + 2;
        const int y0 = kMode == 0 ? f * kGM : f * 2 * kGM;
        const int y1 = kMode == 0 ? f * kGM : f * 2 * kGM + kGM;
        for (int kb = 0; kb < a.nkb; ++kb) {
          if (!ptx::mbar_wait_sleep(&raw_empty[rs], rph ^ 1u, 100)) {
            atomicOr(a.err, 16u);
            goto raw_drain;
          }
          ptx::mbar_arrive_expect_tx(&raw_full[rs], 2 * kRawBytes);
          ptx::tma_load_w(s_rawbuf + (2 * rs) * kRawBytes, m0, kb, y0, &raw_full[rs]);
          ptx::tma_load_w(s_rawbuf + (2 * rs + 1) * kRawBytes, m1, kb, y1, &raw_full[rs]);
          issued |= 1u << rs;
          last_ph = (last_ph & ~(1u << rs)) | (rph << rs);
          if (++rs == kNR) { rs = 0; rph ^= 1u; }
        }
      }
    raw_drain:
      // never leave with a copy into shared memory in flight
      for (int i = 0; i < kNR; ++i)
        if ((issued >> i) & 1u) ptx::mbar_wait(&raw_full[i], (last_ph >> i) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ activation tiles
    if (lane == 0) {
      int bs = 0;
      uint32_t bph = 0, issued = 0, last_ph = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int4 tl = __ldcg(a.tiles + u / ft);
        const int row = tl.w + tl.y;
        for (int ks = 0; ks < a.nkb * 8; ++ks) {
          if (!ptx::mbar_wait_sleep(&ab_empty[bs], bph ^ 1u, 50)) {
            atomicOr(a.err, 16u);
            goto b_drain;
          }
          ptx::mbar_arrive_expect_tx(&b_full[bs], kBBytes);
          ptx::tma_load_2d(s_b + bs * kBBytes, &bmap, ks * 32, row, &b_full[bs]);
          issued |= 1u << bs;
          last_ph = (last_ph & ~(1u << bs)) | (bph << bs);
          if (++bs == kNS) { bs = 0; bph ^= 1u; }
        }
      }
    b_drain:
      for (int i = 0; i < kNS; ++i)
        if ((issued >> i) & 1u) ptx::mbar_wait(&b_full[i], (last_ph >> i) & 1u);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int as = 0;
      uint32_t aph = 0, eph = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int4 tl = __ldcg(a.tiles + u / ft);
        const uint32_t idesc = ptx::umma_idesc_f16(kGM, min(kGN, (tl.z + 15) & ~15));
        if (!ptx::mbar_wait_sleep(acc_empty, eph ^ 1u, 100)) {
          atomicOr(a.err, 32u);
          break;
        }
        eph ^= 1u;
        ptx::tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < a.nkb * 8; ++ks) {
          if (!ptx::mbar_wait(&a_full[as], aph) || !ptx::mbar_wait(&b_full[as], aph)) {
            atomicOr(a.err, 32u);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(s_a + (2 * as) * kABytes);
          const uint32_t b0 = ptx::smem_u32(s_b + as * kBBytes);
#pragma unroll
          for (int k16 = 0; k16 < 2; ++k16) {
            const uint64_t bd = ptx::umma_desc_sw64(b0 + 32 * k16);
            const bool acc = (ks | k16) != 0;
            ptx::umma_f16(tmem, ptx::umma_desc_sw64(a0 + 32 * k16), bd, idesc, acc);
            ptx::umma_f16(tmem + kGN, ptx::umma_desc_sw64(a0 + kABytes + 32 * k16), bd, idesc, acc);
          }
          ptx::umma_commit(&ab_empty[as]);
          if (++as == kNS) { as = 0; aph ^= 1u; }
        }
        if (!ok) break;
        ptx::umma_commit(acc_full);
      }
      // wait for every MMA this thread issued before TMEM is released
      ptx::umma_commit(drain);
      if (!ptx::mbar_wait(drain, 0)) atomicOr(a.err, 32u);
    }
  } else if (warp < kFirstEpi) {
    // ------------------------------------------------------------ dequantisers
    const int m = (warp - kFirstDeq) >> 2;                    // A half
    const int r = ((warp - kFirstDeq) & 3) * 32 + lane;       // weight row of the half, 0..127
    const uint32_t sw = (uint32_t)((r >> 1) & 3);             // 64B swizzle of row r
    const __half2 off_lo = __float2half2_rn(1024.f), off_hi = __float2half2_rn(64.f);
    const __half2 kNeg2 = __float2half2_rn(-1.f);
    int rs = 0, as = 0;
    uint32_t rph = 0, aph = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      // this thread's weight row and its power-of-two scale 2^k
      const int ex = in_range(__ldcg(a.tiles + u / a.ft).x, a.n_ex, a.err), f = u % a.ft;
      const int8_t* wx = a.wexp + (size_t)ex * a.wexp_stride;
      const int wrow = kMode == 0 ? min(f * kGM + r, a.out_rows - 1) + m * a.out_rows
                                  : a.wexp_down + f * 2 * kGM + m * kGM + r;
      const __half2 wsc2 = pow2h2(__ldg(wx + wrow));
      const __half2 nwsc2 = __hmul2(wsc2, kNeg2);
      for (int kb = 0; kb < a.nkb; ++kb) {
        if (!ptx::mbar_wait(&raw_full[rs], rph)) {
          atomicOr(a.err, 64u);
          goto done;
        }
        const uint8_t* row = s_rawbuf + (2 * rs + m) * kRawBytes + r * kQBytes;
        const uint4 hdr = *reinterpret_cast<const uint4*>(row);
        // (d, d) and (dmin, dmin) scaled by the row's 2^k (exact)
        const uint32_t dd = __byte_perm(hdr.x, 0u, 0x1010u), mm = __byte_perm(hdr.x, 0u, 0x3232u);
        const __half2 d2 = *reinterpret_cast<const __half2*>(&dd), dm2 = *reinterpret_cast<const __half2*>(&mm);
        const __half2 d2s = __hmul2(d2, wsc2), nm2s = __hmul2(dm2, nwsc2);
        for (int c = 0; c < 4; ++c) {
          // chunk c: 32 quant bytes; low nibbles are sub-block 2c, high nibbles 2c+1
          const uint4 qa = *reinterpret_cast<const uint4*>(row + 16 + 32 * c);
          const uint4 qb = *reinterpret_cast<const uint4*>(row + 32 + 32 * c);
          const uint32_t w[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
          __half2 s2, nm2;
          chunk_scales(hdr, c, d2s, nm2s, s2, nm2);
#pragma unroll
          for (int nib = 0; nib < 2; ++nib) {
            if (!ptx::mbar_wait(&ab_empty[as], aph ^ 1u)) {
              atomicOr(a.err, 64u);
              goto done;
            }
            const __half2 sc = nib ? __high2half2(s2) : __low2half2(s2);
            const __half2 nm = nib ? __high2half2(nm2) : __low2half2(nm2);
            const __half2 off = nib ? off_hi : off_lo;
            // low nibbles as 1024 + q (mask 0x000F), high nibbles as 64 + q (mask 0x00F0)
            const uint32_t mask = nib ? 0x00F000F0u : 0x000F000Fu;
            const uint32_t magic = nib ? 0x54005400u : 0x64006400u;
            uint8_t* arow = s_a + (2 * as + m) * kABytes + r * 64;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t w0 = w[2 * j], w1 = w[2 * j + 1];
              uint4 o;
              o.x = deq2((w0 & mask) | magic, off, sc, nm);
              o.y = deq2(((w0 >> 8) & mask) | magic, off, sc, nm);
              o.z = deq2((w1 & mask) | magic, off, sc, nm);
              o.w = deq2(((w1 >> 8) & mask) | magic, off, sc, nm);
              *reinterpret_cast<uint4*>(arow + ((j ^ sw) << 4)) = o;
            }
            ptx::fence_proxy_async();  // generic-proxy stores -> visible to the tensor cores
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&a_full[as]);
            if (++as == kNS) { as = 0; aph ^= 1u; }
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&raw_empty[rs]);
        if (++rs == kNR) { rs = 0; rph ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    uint32_t fph = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x)
      if (!gemm_epilogue<kMode>(a, tmem, acc_full, acc_empty, u, fph, warp - kFirstEpi, warp, lane)) goto done;
  }
done:
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ============================================================================ few-row tiles
// Tiles of at most kMtMaxRows activation rows (experts with few rows, and the
// last partial tile of the others) stream their weights through warp-level
// fp16 MMAs (mma.sync m16n8k16, fp32 accumulate) instead of the tensor-memory
// GEMM above.  The weights are dequantised in registers straight into MMA
// fragments -- the same fp16 values as the dequantisers above, 2^k row scale
// included -- so a weight tile costs its HBM read and about 1.6 instructions
// per weight whatever its row count, with no shared-memory round trip.
//
// Work unit: (tile, feature block), claimed from a counter -- gate/up 128
// features (128 gate rows + the same 128 up rows), down 256 output rows.  A
// stage is one super-block along K: the unit's 256 weight rows (two 2-D TMA
// boxes of 128 rows) and the tile's activation rows (a bulk copy of 256 fp16
// per row; rows kMtXPitch bytes apart so that the fragment loads of eight rows
// fall on distinct banks).
//
// Warp w owns 16 weight rows as one MMA M tile and all of K -- gate/up: rows
// 0-7 are the gate rows of features 8w..8w+7 and rows 8-15 their up rows, so a
// thread holds g and u of the same (feature, token) and applies SwiGLU in
// registers; down: output rows 16w..16w+15 -- against every activation row of
// the tile as up to kMtMaxRows / 8 MMA N tiles.  The producer warp issues a
// stage's activation rows one per lane.
//
// K order: the thread at quad position c takes, from each 16-weight half of a
// 32-weight run, the weights 4c..4c+3: nibbles (0, 2) of its quant word form
// one fp16 pair and (1, 3) the other, which is the order (0, 2, 1, 3) in which
// the activations are stored within every group of four.
constexpr int kMtWarps = 16;
constexpr int kMtThreads = (kMtWarps + 1) * 32;          // + one producer warp
constexpr int kMtWBytes = 2 * kRawBytes;                 // 256 weight rows x 1 super-block
constexpr int kMtXPitch = 2 * kQK + 32;                  // one activation row's 256 fp16, padded
// Two builds: tiles of at most 32 rows with 4 stages, at most 64 with 3
template <int kRows>
struct MtCfg {
  static constexpr int kStages = kRows <= 32 ? 4 : 3;
  static constexpr int kStageBytes = kMtWBytes + kRows * kMtXPitch;
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 32 * kStages;
  static_assert(kSmem <= 227 * 1024, "few-row kernel shared memory");
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned");
};

struct MtRows {
  int boxA, boxB, rowA, rowB;   // the 128-row box and row in it of M-tile rows g and g + 8
};

// One work unit of the few-row kernel for one consumer warp: nkb stages of
// MMAs into NT N tiles, then the epilogue.  Returns false if a stage never
// arrived (error flag set).
template <int kMode, int kRows, int NT>
__device__ __forceinline__ bool mt_unit(const GemmArgs& a, const uint8_t* sm, uint64_t* full, uint64_t* empty,
                                        int& stage, uint32_t& phase, const int4 tl, int f, int warp, int lane,
                                        const MtRows& rw) {
  const int g = lane >> 2, c4 = lane & 3;
  const uint32_t offA = (uint32_t)(rw.boxA * kRawBytes + rw.rowA * kQBytes);
  const uint32_t offB = (uint32_t)(rw.boxB * kRawBytes + rw.rowB * kQBytes);
  const __half2 off_lo = __float2half2_rn(1024.f), off_hi = __float2half2_rn(64.f);
  const __half2 kNeg2 = __float2half2_rn(-1.f);
  const int ex = in_range(tl.x, a.n_ex, a.err);
  using C = MtCfg<kRows>;
  const int cnt = min(tl.z, kRows);
  // weight rows of this thread and their 2^k scales
  const int8_t* wx = a.wexp + (size_t)ex * a.wexp_stride;
  int wrA, wrB, oA, oB;   // wexp rows; output columns
  if (kMode == 0) {
    oA = oB = f * kGM + 8 * warp + g;
    const int fr = min(oA, a.out_rows - 1);
    wrA = fr;
    wrB = a.out_rows + fr;
  } else {
    oA = f * 2 * kGM + rw.boxA * kGM + rw.rowA;
    oB = f * 2 * kGM + rw.boxB * kGM + rw.rowB;
    wrA = a.wexp_down + oA;
    wrB = a.wexp_down + oB;
  }
  const int kA = __ldg(wx + wrA), kB = __ldg(wx + wrB);
  const __half2 wsA = pow2h2(kA), wsB = pow2h2(kB);
  const __half2 nwsA = __hmul2(wsA, kNeg2), nwsB = __hmul2(wsB, kNeg2);
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  for (int kb = 0; kb < a.nkb; ++kb) {
    if (kb > 0 && !ptx::mbar_wait(&full[stage], phase)) {
      atomicOr(a.err, 64u);
      return false;
    }
    const uint32_t st = ptx::smem_u32(sm) + (uint32_t)(stage * C::kStageBytes);
    const uint32_t rA = st + offA, rB = st + offB;
    const uint32_t xs = st + kMtWBytes + g * kMtXPitch + 8 * c4;   // token row g of N tile 0
    const uint4 hA = ptx::lds_v4(rA), hB = ptx::lds_v4(rB);
    __half2 d2sA, nm2sA, d2sB, nm2sB;
    {
      const uint32_t dA = __byte_perm(hA.x, 0u, 0x1010u), mA = __byte_perm(hA.x, 0u, 0x3232u);
      const uint32_t dB = __byte_perm(hB.x, 0u, 0x1010u), mB = __byte_perm(hB.x, 0u, 0x3232u);
      d2sA = __hmul2(*reinterpret_cast<const __half2*>(&dA), wsA);
      nm2sA = __hmul2(*reinterpret_cast<const __half2*>(&mA), nwsA);
      d2sB = __hmul2(*reinterpret_cast<const __half2*>(&dB), wsB);
      nm2sB = __hmul2(*reinterpret_cast<const __half2*>(&mB), nwsB);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      __half2 sA2, nmA2, sB2, nmB2;
      chunk_scales(hA, c, d2sA, nm2sA, sA2, nmA2);
      chunk_scales(hB, c, d2sB, nm2sB, sB2, nmB2);
      const uint32_t qA = rA + 16 + 32 * c + 4 * c4, qB = rB + 16 + 32 * c + 4 * c4;
      const uint32_t wA[2] = {ptx::lds_u32(qA), ptx::lds_u32(qA + 16)};
      const uint32_t wB[2] = {ptx::lds_u32(qB), ptx::lds_u32(qB + 16)};
#pragma unroll
      for (int nib = 0; nib < 2; ++nib) {   // run 2c (low nibbles), run 2c + 1 (high nibbles)
        const __half2 sa = nib ? __high2half2(sA2) : __low2half2(sA2);
        const __half2 na = nib ? __high2half2(nmA2) : __low2half2(nmA2);
        const __half2 sb = nib ? __high2half2(sB2) : __low2half2(sB2);
        const __half2 nb = nib ? __high2half2(nmB2) : __low2half2(nmB2);
        const __half2 off = nib ? off_hi : off_lo;
        const uint32_t mask = nib ? 0x00F000F0u : 0x000F000Fu;
        const uint32_t magic = nib ? 0x54005400u : 0x64006400u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {   // weights 16h + 4c4 .. +3 of the run
          const uint32_t wa = wA[h], wb = wB[h];
          uint32_t af[4];
          af[0] = deq2((wa & mask) | magic, off, sa, na);          // row g,     nibbles 0, 2
          af[1] = deq2((wb & mask) | magic, off, sb, nb);          // row g + 8
          af[2] = deq2(((wa >> 8) & mask) | magic, off, sa, na);   // row g,     nibbles 1, 3
          af[3] = deq2(((wb >> 8) & mask) | magic, off, sb, nb);
          const uint32_t xk = xs + 2 * (64 * c + 32 * nib + 16 * h);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const uint2 bv = ptx::lds_v2(xk + j * 8 * kMtXPitch);
            ptx::mma_f16(acc[j], af, bv.x, bv.y);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[stage]);
    if (++stage == C::kStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
  // epilogue: undo the row's 2^k and the activation row's scale
  const int prow0 = tl.w + tl.y;
  const float sA = pow2f(-kA), sB = pow2f(-kB);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 8 * j + 2 * c4 + e;
      if (n < cnt) {
        const int prow = prow0 + n;
        const float inv = __ldg(a.rinv + prow);
        float* orow = a.out + (size_t)prow * a.out_ld;
        if (kMode == 0) {
          if (oA < a.out_rows) {
            const float gv = acc[j][e] * (inv * sA), up = acc[j][2 + e] * (inv * sB);
            orow[oA] = __fdividef(gv, 1.f + __expf(-gv)) * up;   // silu(g) * u
          }
        } else {
          orow[oA] = acc[j][e] * (inv * sA);
          orow[oB] = acc[j][2 + e] * (inv * sB);
        }
      }
    }
  }
  return true;
}

template <int kMode, int kRows>
__global__ void __launch_bounds__(kMtThreads, 1) q4k_mt_kernel(const GemmArgs a) {
  using C = MtCfg<kRows>;
  constexpr int kMtStages = C::kStages, kMtStageBytes = C::kStageBytes;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kMtStages * kMtStageBytes);
  uint64_t* empty = full + kMtStages;
  int* s_unit = reinterpret_cast<int*>(empty + kMtStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMtStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kMtWarps);
    }
    ptx::fence_barrier_init();
  }
  __syncthreads();
  ptx::pdl_wait();  // tiles, counters and activation rows of the previous kernels
  ptx::pdl_launch_dependents();
  const int ft = a.ft, nkb = a.nkb;
  const int n_units = __ldcg(a.n_tiles) * ft;

  if (warp == kMtWarps) {
    // ------------------------------------------------------------ producer
    // lane 0 claims units, waits for free stages and issues the weight
    // boxes; every lane issues some of the stage's activation-row copies
    int stage = 0;
    uint32_t phase = 0;
    ptx::IssueLog log;
    bool ok = true;
    while (ok) {
      int u = 0;
      if (lane == 0) u = (int)atomicAdd(a.next, 1u);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u >= n_units) break;
      const int4 tl = __ldcg(a.tiles + u / ft);   // (expert, n0, count, r0)
      const int f = u % ft;
      const int cnt = min(tl.z, kRows);
      const __half* xr = a.bsrc + (size_t)in_range(tl.w + tl.y, a.n_rows, a.err) * a.b_ld;
      for (int kb = 0; kb < nkb; ++kb) {
        int free = 1;
        if (lane == 0) free = ptx::mbar_wait(&empty[stage], phase ^ 1u) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, free, 0)) {
          if (lane == 0) atomicOr(a.err, 16u);
          ok = false;
          break;
        }
        uint8_t* dst = sm + stage * kMtStageBytes;
        if (lane == 0) {
          const int ex = in_range(tl.x, a.n_ex, a.err);
          const CUtensorMap* wm = a.wmaps + kMapsPerSlot * in_range(__ldcg(a.slot_of + ex), a.n_slots, a.err) + 3;
          const CUtensorMap* m0 = kMode == 0 ? wm : wm + 2;
          const CUtensorMap* m1 = kMode == 0 ? wm + 1 : wm + 2;
          const int y0 = kMode == 0 ? f * kGM : f * 2 * kGM;
          const int y1 = kMode == 0 ? f * kGM : f * 2 * kGM + kGM;
          s_unit[stage] = u;
          ptx::mbar_arrive_expect_tx(&full[stage], (uint32_t)(kMtWBytes + cnt * 2 * kQK));
          ptx::tma_load_w(dst, m0, kb, y0, &full[stage]);
          ptx::tma_load_w(dst + kRawBytes, m1, kb, y1, &full[stage]);
        }
        __syncwarp();   // the expected bytes are set before any row copy can complete
        for (int n = lane; n < cnt; n += 32)
          ptx::bulk_load(dst + kMtWBytes + n * kMtXPitch, xr + (size_t)n * a.b_ld + kb * kQK, 2 * kQK,
                         &full[stage]);
        log.note(stage, phase);
        if (++stage == kMtStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (lane == 0) {
      if (ok) {
        // end of work: a stage with unit -1 and no bytes (its earlier issue
        // was consumed, so it leaves the drain list)
        if (ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
          s_unit[stage] = -1;
          log.issued &= ~(1u << stage);
          ptx::mbar_arrive(&full[stage]);
        } else {
          atomicOr(a.err, 16u);
        }
      }
      // never leave with a copy into shared memory in flight
      log.drain(full, kMtStages);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2;
  // this warp's rows: (box, row in box) of M-tile rows g and g + 8
  MtRows rw;
  rw.boxA = kMode == 0 ? 0 : warp >> 3;
  rw.boxB = kMode == 0 ? 1 : warp >> 3;
  rw.rowA = kMode == 0 ? 8 * warp + g : 16 * (warp & 7) + g;
  rw.rowB = kMode == 0 ? rw.rowA : rw.rowA + 8;
  int stage = 0;
  uint32_t phase = 0;
  while (true) {
    bool ok = ptx::mbar_wait(&full[stage], phase);
    const int u = ok ? s_unit[stage] : -1;
    if (!ok) {
      atomicOr(a.err, 64u);
      break;
    }
    if (u < 0) break;
    const int4 tl = __ldcg(a.tiles + u / ft);
    const int f = u % ft;
    const int nt = (min(tl.z, kRows) + 7) >> 3;
    // one instantiation per N-tile count: no MMA is issued for an empty N tile
    switch (nt) {
      case 1: ok = mt_unit<kMode, kRows, (1 <= kRows / 8 ? 1 : kRows / 8)>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
      case 2: ok = mt_unit<kMode, kRows, (2 <= kRows / 8 ? 2 : kRows / 8)>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
      case 3: ok = mt_unit<kMode, kRows, (3 <= kRows / 8 ? 3 : kRows / 8)>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
      case 4: ok = mt_unit<kMode, kRows, (4 <= kRows / 8 ? 4 : kRows / 8)>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
      case 5: ok = mt_unit<kMode, kRows, (5 <= kRows / 8 ? 5 : kRows / 8)>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
      case 6: ok = mt_unit<kMode, kRows, (6 <= kRows / 8 ? 6 : kRows / 8)>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
      case 7: ok = mt_unit<kMode, kRows, (7 <= kRows / 8 ? 7 : kRows / 8)>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
      default: ok = mt_unit<kMode, kRows, kRows / 8>(a, sm, full, empty, stage, phase, tl, f, warp, lane, rw); break;
    }
    if (!ok) break;
  }
}

// ---------------------------------------------------------------- helper kernels
// Tiles: each expert with more than `small_rows` rows, in chunks of kGN rows:
// (expert, n0, count, r0).  Experts with 1..small_rows rows go to `small`
// (for the decode kernels, which stream their weights once without
// dequantising them).  With mt_rows > 0, an expert with at most mt_rows rows
// becomes one few-row tile, and so does the last partial chunk of a larger
// expert when it has at most mt_rows rows.  The few-row tiles are listed by
// their MMA N-tile count (rows / 8, rounded up), largest first, in expert
// order within a count: their units are claimed in list order, so the
// longest run first.  The unit counters of the few-row kernels are zeroed
// here.  One block of 1024 threads; experts are taken 1024 at a time with
// block scans (GEMM tiles, small experts) and warp ballots (few-row tiles).
struct TileCls {
  int e, c, r0, nt, sm, mt, nb;   // expert, rows, first row, GEMM tiles, small, few-row tile, its N tiles
};
__device__ __forceinline__ TileCls classify(int i, int na, const int* act, const int* counts, const int* offsets,
                                            int small_rows, int mt_rows, int ep_rank, int ep_world) {
  TileCls t{0, 0, 0, 0, 0, 0, 0};
  if (i >= na) return t;
  t.e = __ldcg(act + i);
  t.c = __ldcg(counts + t.e);
  t.r0 = __ldcg(offsets + t.e);
  t.sm = t.c <= small_rows ? 1 : 0;
  if (!t.sm) {
    t.nt = (t.c + kGN - 1) / kGN;
    const int last = t.c - (t.nt - 1) * kGN;   // rows of the last chunk
    if (last <= mt_rows) {
      t.mt = 1;
      t.nb = (last + 7) >> 3;
      --t.nt;
    }
  }
  if (!ep_owned(t.e, ep_rank, ep_world)) t.sm = t.nt = t.mt = t.nb = 0;   // another rank's expert
  return t;
}

__global__ void __launch_bounds__(1024) build_tiles_kernel(const int* __restrict__ act, const int* __restrict__ n_act,
                                                           const int* __restrict__ counts,
                                                           const int* __restrict__ offsets, int4* __restrict__ tiles,
                                                           int* __restrict__ n_tiles, int small_rows,
                                                           int* __restrict__ small, int* __restrict__ n_small,
                                                           int mt_rows, int4* __restrict__ mtiles,
                                                           int* __restrict__ n_mtiles, unsigned* __restrict__ mt_next,
                                                           int ep_rank, int ep_world) {
  constexpr int kNB = kMtMaxRows / 8 + 1;   // N-tile counts 0..8 (0: not a few-row tile)
  __shared__ int s_warp[32];
  __shared__ int s_bw[kNB][32];             // per count, per warp: tiles, then their first position
  __shared__ int s_base[kNB];               // per count: first position in the list (all chunks)
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();   // the next kernel waits for this one's end before reading
  const int na = __ldcg(n_act);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  if (threadIdx.x < kNB) s_base[threadIdx.x] = 0;
  __syncthreads();
  // pass 1: GEMM tiles, small experts, and the number of few-row tiles per N-tile count
  int base = 0, sbase = 0;
  for (int c0 = 0; c0 < na; c0 += blockDim.x) {
    const TileCls t = classify(c0 + threadIdx.x, na, act, counts, offsets, small_rows, mt_rows, ep_rank, ep_world);
    int tot, stot;
    const int pos = base + block_exclusive_scan_1024(t.nt, &tot, s_warp);
    __syncthreads();
    const int spos = sbase + block_exclusive_scan_1024(t.sm, &stot, s_warp);
    for (int j = 0; j < t.nt; ++j) tiles[pos + j] = make_int4(t.e, j * kGN, min(kGN, t.c - j * kGN), t.r0);
    if (t.sm) small[spos] = t.e;
    if (t.mt) atomicAdd(&s_base[t.nb], 1);   // counts: the order of the adds does not matter
    base += tot;
    sbase += stot;
    __syncthreads();
  }
  // first position of each count, largest count first
  if (threadIdx.x == 0) {
    int run = 0;
    for (int b = kNB - 1; b >= 1; --b) {
      const int n = s_base[b];
      s_base[b] = run;
      run += n;
    }
    *n_tiles = base;
    *n_small = sbase;
    *n_mtiles = run;
    mt_next[0] = 0u;
    mt_next[1] = 0u;
  }
  __syncthreads();
  if (mt_rows == 0) return;
  // pass 2: positions of the few-row tiles (rank within their count: warp
  // ballots, then a prefix over the warps of the chunk)
  for (int c0 = 0; c0 < na; c0 += blockDim.x) {
    const TileCls t = classify(c0 + threadIdx.x, na, act, counts, offsets, small_rows, mt_rows, ep_rank, ep_world);
    int rank = 0;
#pragma unroll
    for (int b = 1; b < kNB; ++b) {
      const uint32_t m = __ballot_sync(0xffffffffu, t.mt && t.nb == b);
      if (t.mt && t.nb == b) rank = __popc(m & lt);
      if (lane == 0) s_bw[b][warp] = __popc(m);
    }
    __syncthreads();
    if (warp >= 1 && warp < kNB) {   // warp b: exclusive prefix of count b over the chunk's warps
      const int b = warp;
      const int v = lane < (int)(blockDim.x >> 5) ? s_bw[b][lane] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      s_bw[b][lane] = s_base[b] + incl - v;
      __syncwarp();
      if (lane == 31) s_base[b] += incl;   // the next chunk continues after this one
    }
    __syncthreads();
    if (t.mt) mtiles[s_bw[t.nb][warp] + rank] = make_int4(t.e, t.nt * kGN, t.c - t.nt * kGN, t.r0);
    __syncthreads();
  }
}

// x (bf16 [T, H]) as 16-bit fixed point per 32-element run for the decode
// kernels: one warp per run.
__global__ void __launch_bounds__(256) quant_x_kernel(const __nv_bfloat16* __restrict__ x, int T, int H,
                                                       int8_t* __restrict__ xq, size_t plane, float2* __restrict__ xsc) {
  ptx::pdl_wait();
  const int runs = H / 32;
  const int run = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (run >= T * runs) return;
  const int t = run / runs, r = run - t * runs;
  const size_t o = (size_t)t * H + r * 32 + lane;
  float2 rsc;
  int8_t hi;
  uint8_t lo;
  quant_run16(__bfloat162float(x[o]), hi, lo, rsc);
  xq[o] = hi;
  reinterpret_cast<uint8_t*>(xq + plane)[o] = lo;
  if (lane == 0) xsc[run] = rsc;
}

// Power of two p with max * p in [2^14, 2^15) (1 for max == 0 or not finite); *inv = 1/p.
__device__ __forceinline__ float row_scale(float mx, float* inv) {
  int e = 0;
  if (mx > 0.f && mx < 3.0e38f) e = (int)((__float_as_uint(mx) >> 23) & 0xFFu) - 127;
  e = max(-110, min(110, e));
  *inv = __uint_as_float((uint32_t)(127 - 14 + e) << 23);
  return __uint_as_float((uint32_t)(127 + 14 - e) << 23);
}

// 4 floats -> 4 fp16 in the order (0, 2, 1, 3)
__device__ __forceinline__ uint2 pack4_swz(float a0, float a1, float a2, float a3) {
  const __half2 p = __floats2half2_rn(a0, a2), q = __floats2half2_rn(a1, a3);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&p), *reinterpret_cast<const uint32_t*>(&q));
}

constexpr int kRowWarps = 8;

// Row r of the expert-sorted order: token perm[r] / kS of x as scaled fp16
// (x16[r, :]), rinv[r] = 1/scale.  One warp per row, two passes over the
// token's row (the maximum by a warp reduction, then the conversion; x is
// read from L2 both times).  A block per row with a block barrier ran at
// 3.8 TB/s of read + write traffic at config 3.
__global__ void __launch_bounds__(kRowWarps * 32) gather_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                                   const int* __restrict__ perm, int kS, int H,
                                                                   int P, __half* __restrict__ x16,
                                                                   float* __restrict__ rinv) {
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (r >= P) return;
  const uint2* src = reinterpret_cast<const uint2*>(x + (size_t)(__ldg(perm + r) / kS) * H);
  const int nv = H / 4;
  float m = 0.f;
#pragma unroll 4
  for (int c = lane; c < nv; c += 32) {
    const uint2 v = __ldg(src + c);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))), fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float inv;
  const float sc = row_scale(m, &inv);
  uint2* dst = reinterpret_cast<uint2*>(x16 + (size_t)r * H);
#pragma unroll 4
  for (int c = lane; c < nv; c += 32) {
    const uint2 v = __ldg(src + c);
    dst[c] = pack4_swz(bf16lo(v.x) * sc, bf16hi(v.x) * sc, bf16lo(v.y) * sc, bf16hi(v.y) * sc);
  }
  if (lane == 0) rinv[r] = inv;
}

// h (fp32 [P, I_pad], columns >= I unwritten) -> fp16 h16 scaled by the power
// of two that puts the row's largest magnitude in [2^14, 2^15), padding
// zeroed, K order (0, 2, 1, 3); hinv[r] = 1/scale.  One warp per row, two
// passes over it: the maximum (a warp reduction, no block barrier), then
// the conversion (the row is still in L1/L2).  A block per row left each
// block with two loads per thread and a block barrier: 1.5 TB/s at config 3.
__device__ __forceinline__ float4 h_quad(const float4* src, int c, int I) {
  float4 f = __ldcg(src + c);
  const int i = 4 * c;
  if (i + 3 >= I) {
    f.x = i < I ? f.x : 0.f;
    f.y = i + 1 < I ? f.y : 0.f;
    f.z = i + 2 < I ? f.z : 0.f;
    f.w = 0.f;
  }
  return f;
}
constexpr int kConvWarps = 8;
__global__ void __launch_bounds__(kConvWarps * 32) convert_h_kernel(const float* __restrict__ h, int I, int I_pad,
                                                                    int P, __half* __restrict__ h16,
                                                                    float* __restrict__ hinv) {
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kConvWarps + (threadIdx.x >> 5);
  if (r >= P) return;
  const float4* src = reinterpret_cast<const float4*>(h + (size_t)r * I_pad);
  const int nv = I_pad / 4;
  float m = 0.f;
#pragma unroll 4
  for (int c = lane; c < nv; c += 32) {
    const float4 f = h_quad(src, c, I);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float inv;
  const float sc = row_scale(m, &inv);
  uint2* dst = reinterpret_cast<uint2*>(h16 + (size_t)r * I_pad);
#pragma unroll 4
  for (int c = lane; c < nv; c += 32) {
    const float4 f = h_quad(src, c, I);
    dst[c] = pack4_swz(f.x * sc, f.y * sc, f.z * sc, f.w * sc);
  }
  if (lane == 0) hinv[r] = inv;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace

size_t prefill_gemm_smem() { return kGemmSmem; }

size_t prefill_max_tiles(int n_experts_total, size_t pairs) { return (size_t)n_experts_total + pairs / kGN + 1; }

cudaError_t launch_build_tiles(const Work& wk, int small_rows, int mt_rows, cudaStream_t st, int ep_rank,
                               int ep_world) {
  if (mt_rows < 0 || mt_rows > kMtMaxRows) return cudaErrorInvalidValue;
  return launch_pdl(build_tiles_kernel, dim3(1), dim3(1024), 0, st, (const int*)wk.act, (const int*)wk.n_act,
                    (const int*)wk.counts, (const int*)wk.offsets, wk.tiles, wk.n_tiles, small_rows, wk.act1,
                    wk.n_act1, mt_rows, wk.mtiles, wk.n_mtiles, wk.mt_next, ep_rank, ep_world);
}

cudaError_t launch_quant_x(const __nv_bfloat16* x, const Work& wk, int T, int H, cudaStream_t st) {
  const int runs = T * (H / 32);
  return launch_pdl(quant_x_kernel, dim3((runs + 7) / 8), dim3(256), 0, st, x, T, H, wk.xq, wk.xq_plane, wk.xsc);
}

cudaError_t launch_gather_rows(const __nv_bfloat16* x, const Work& wk, int P, int kS, int H, cudaStream_t st) {
  if (H % 4 || P <= 0) return cudaErrorInvalidValue;
  return launch_pdl(gather_rows_kernel, dim3((P + kRowWarps - 1) / kRowWarps), dim3(kRowWarps * 32), 0, st, x,
                    (const int*)wk.perm, kS, H, P, wk.x16, wk.rinv);
}

cudaError_t launch_convert_h(const Work& wk, int P, int I, int I_pad, cudaStream_t st) {
  if (P <= 0) return cudaSuccess;
  return launch_pdl(convert_h_kernel, dim3((P + kConvWarps - 1) / kConvWarps), dim3(kConvWarps * 32), 0, st,
                    (const float*)wk.h, I, I_pad, P, wk.h16, wk.hinv);
}

cudaError_t launch_prefill_mt(int mode, const GemmArgs& a, int n_sm, cudaStream_t st, int max_rows) {
  static uint64_t attr_done[4] = {0, 0, 0, 0};  // per (mode, build), one bit per device
  if (max_rows < 1 || max_rows > kMtMaxRows) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  const bool wide = max_rows > 32;
  const int v = (mode & 1) * 2 + (wide ? 1 : 0);
  void (*kern)(const GemmArgs) = wide ? (mode == 0 ? q4k_mt_kernel<0, 64> : q4k_mt_kernel<1, 64>)
                                      : (mode == 0 ? q4k_mt_kernel<0, 32> : q4k_mt_kernel<1, 32>);
  const size_t smem = wide ? MtCfg<64>::kSmem : MtCfg<32>::kSmem;
  if (!(attr_done[v] & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[v] |= bit;
  }
  return launch_pdl(kern, dim3(n_sm), dim3(kMtThreads), smem, st, a);
}

cudaError_t launch_prefill_gemm(int mode, const CUtensorMap& bmap, const GemmArgs& a, int n_sm, cudaStream_t st) {
  static uint64_t attr_done[2] = {0, 0};  // per mode, one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  auto kern = mode == 0 ? q4k_gemm_kernel<0> : q4k_gemm_kernel<1>;
  if (!(attr_done[mode & 1] & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
    if (e != cudaSuccess) return e;
    attr_done[mode & 1] |= bit;
  }
  return launch_pdl(kern, dim3(n_sm), dim3(kGemmThreads), kGemmSmem, st, bmap, a);
}

}  // namespace moe
