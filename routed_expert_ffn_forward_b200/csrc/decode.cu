// Decode-path expert kernels for experts with few rows (1..kD1MaxTok tokens):
// gate/up + SwiGLU, then down.  (The weighted combine follows as its own
// kernel, chained with programmatic dependent launch.)
//
// Both kernels stream raw Q4_K tiles (64 weight rows x a few super-blocks) from
// HBM into a ring of shared-memory stages with 2-D TMA loads issued by one
// producer thread, and sixteen consumer warps turn them into dot products on
// the warp tensor-core integer MMA (m16n8k32, u8 x s8/u8, exact s32
// accumulate) without ever materialising dequantised weights:
//
//  * A fragment = four 4-bit quants as bytes: masking a 32-bit quant word with
//    0x0F0F0F0F gives four low nibbles, one shift more the four high ones.
//  * B fragment = the activations as 16-bit fixed point per 32-element run
//    (x = (256*hi + lo) * 2^-s, hi signed and lo unsigned bytes, s chosen per
//    run so its largest value lands in [2^13, 2^14)), laid out
//    block-diagonally: column n of B holds sub-block n of the super-block and
//    zeros elsewhere.  A super-block's MMAs leave, in thread (g, c), the exact
//    integer sums sum_i q_i * x_i of sub-blocks 2c, 2c+1 of its rows g and g+8
//    -- the rows and sub-blocks whose scales that thread decodes.
//  * Epilogue per (row, sub-block), in fp32:
//      acc += d*sc * 2^-s * (256*C_hi + C_lo) - dmin*m * X
//    with X the run's sum of the represented activations: the Q4_K value
//    d*sc*q - dmin*m applied exactly (up to fp32 rounding), weights never rounded.
//
// Thread (g, c) owns weight rows g and g+8 of its warp's 16 rows and quant
// chunk c (bytes 32c..32c+31, sub-blocks 2c and 2c+1) of a super-block.  Each
// stage's super-blocks are split across warps; partial sums meet in shared
// memory at the end of a work unit (active expert, 64-row tile).  Persistent
// CTAs walk the units.  Kernels are chained with programmatic dependent launch
// and wait (griddepcontrol.wait) before reading a predecessor's outputs.
#include "moe_internal.h"
#include "ptx.cuh"
#include "q4k_decode.cuh"

namespace moe {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kConsumerThreads = kConsumerWarps * 32;

// gate/up: stage = 64 rows x 2 super-blocks of gate and of up
constexpr int kGuSB = 2;
constexpr int kGuStages = 5;
constexpr int kGuTileBytes = kTileRows * kGuSB * kQBytes;  // 18432
constexpr int kGuStageBytes = 2 * kGuTileBytes;             // 36864
// Without x staged per CTA, a stage also carries the stage's slice of each of
// the unit's tokens' activations: hi bytes, lo bytes (kGuSB x 256 each) and
// run scales (kGuSB x 8 float2).
constexpr int kXSliceBytes = kGuSB * (2 * kQK + 8 * 8);   // 1152
template <int kMaxTok, bool kStageX>
__host__ __device__ constexpr int gu_stage_stride() {
  return kGuStageBytes + (kStageX ? 0 : kMaxTok * kXSliceBytes);
}
// down: stage = 64 rows x 4 super-blocks
constexpr int kDnSB = 4;
constexpr int kDnStages = 4;
constexpr int kDnStageBytes = kTileRows * kDnSB * kQBytes;  // 36864

// One row's block header and quant chunk c (32 bytes).  A stage holds its
// super-blocks one after another, each as 64 rows 144 bytes apart (the
// tile-major weight layout), so the rows g of an 8-lane phase start 4 banks
// apart and their 16-byte pieces never share a bank.
__device__ __forceinline__ void load_row_block(const uint8_t* blk, int c, uint4& hdr, uint32_t* q) {
  hdr = *reinterpret_cast<const uint4*>(blk);
  const uint4 lo = *reinterpret_cast<const uint4*>(blk + 16 + 32 * c);
  const uint4 hi = *reinterpret_cast<const uint4*>(blk + 32 + 32 * c);
  q[0] = lo.x; q[1] = lo.y; q[2] = lo.z; q[3] = lo.w;
  q[4] = hi.x; q[5] = hi.y; q[6] = hi.z; q[7] = hi.w;
}


// One super-block of one warp's 16 rows against one activation vector.
//  ahi/alo: the super-block's 256 activations, high (s8) and low (u8) bytes
//           (shared memory; zero: 32 zero bytes of shared memory)
//  sc:      (2^-s, X) of runs 2c and 2c+1 of the super-block
// Lane (g, c) supplies B only if g == 2c (low positions of its chunk) or
// g == 2c+1 (high positions).  The same registers feed the low-nibble MMA,
// whose column 2c sees exactly lane (2c, c), and the high-nibble MMA, whose
// column 2c+1 sees lane (2c+1, c); the other column of each is never read.
// Four chains of four MMAs (low/high nibbles x high/low activation bytes).
__device__ __forceinline__ void sb_dot(const uint32_t* q, const uint32_t* q8, const RowScales& rs,
                                       const RowScales& rs8, const uint8_t* ahi, const uint8_t* alo,
                                       const uint8_t* zero, float4 sc, int g, int c, float& acc, float& acc8) {
  const bool own = (g >> 1) == c;
  const int off = 64 * c + 32 * (g & 1);
  const uint4* ph = reinterpret_cast<const uint4*>(own ? ahi + off : zero);
  const uint4* pl = reinterpret_cast<const uint4*>(own ? alo + off : zero);
  const uint4 bh0 = ph[0], bh1 = ph[1], bl0 = pl[0], bl1 = pl[1];
  const uint32_t Bh0[4] = {bh0.x, bh0.y, bh0.z, bh0.w}, Bh1[4] = {bh1.x, bh1.y, bh1.z, bh1.w};
  const uint32_t Bl0[4] = {bl0.x, bl0.y, bl0.z, bl0.w}, Bl1[4] = {bl1.x, bl1.y, bl1.z, bl1.w};
  int Clh[4], Cll[4], Chh[4], Chl[4];
#pragma unroll
  for (int mi = 0; mi < 4; ++mi) {
    const uint32_t alow[4] = {q[mi] & 0x0F0F0F0Fu, q8[mi] & 0x0F0F0F0Fu, q[mi + 4] & 0x0F0F0F0Fu,
                              q8[mi + 4] & 0x0F0F0F0Fu};
    const uint32_t ahigh[4] = {(q[mi] >> 4) & 0x0F0F0F0Fu, (q8[mi] >> 4) & 0x0F0F0F0Fu,
                               (q[mi + 4] >> 4) & 0x0F0F0F0Fu, (q8[mi + 4] >> 4) & 0x0F0F0F0Fu};
    if (mi == 0) {
      ptx::mma_u8<true, true>(Clh, alow, Bh0[mi], Bh1[mi]);
      ptx::mma_u8<false, true>(Cll, alow, Bl0[mi], Bl1[mi]);
      ptx::mma_u8<true, true>(Chh, ahigh, Bh0[mi], Bh1[mi]);
      ptx::mma_u8<false, true>(Chl, ahigh, Bl0[mi], Bl1[mi]);
    } else {
      ptx::mma_u8<true, false>(Clh, alow, Bh0[mi], Bh1[mi]);
      ptx::mma_u8<false, false>(Cll, alow, Bl0[mi], Bl1[mi]);
      ptx::mma_u8<true, false>(Chh, ahigh, Bh0[mi], Bh1[mi]);
      ptx::mma_u8<false, false>(Chl, ahigh, Bl0[mi], Bl1[mi]);
    }
  }
  // sum q*x of each (row, sub-block): 256*C_hi + C_lo, exact in int32 and fp32
  const float vlo = (float)(Clh[0] * 256 + Cll[0]), vhi = (float)(Chh[1] * 256 + Chl[1]);
  const float vlo8 = (float)(Clh[2] * 256 + Cll[2]), vhi8 = (float)(Chh[3] * 256 + Chl[3]);
  acc += rs.s_lo * sc.x * vlo + rs.s_hi * sc.z * vhi - (rs.m_lo * sc.y + rs.m_hi * sc.w);
  acc8 += rs8.s_lo * sc.x * vlo8 + rs8.s_hi * sc.z * vhi8 - (rs8.m_lo * sc.y + rs8.m_hi * sc.w);
}

__device__ __forceinline__ void flag_error(unsigned* err, unsigned bit) { atomicOr(err, bit); }

// Dynamic shared memory rounded up to a 1024-byte boundary (TMA destinations
// must be aligned); the launch asks for 1024 bytes of slack.
__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw) {
  const uint32_t pad = (1024u - (ptx::smem_u32(raw) & 1023u)) & 1023u;
  return raw + pad;
}

// ============================================================================ gate/up
// kMaxTok: the most rows (tokens) an expert may have in this launch.  With
// kStageX, x (all tokens) is copied to shared memory once per CTA; without,
// the producer bulk-copies each stage's slice of the unit's tokens' x next to
// the stage's weights.
template <int kMaxTok, bool kStageX>
__global__ void __launch_bounds__(kThreads, 1) gate_up_d1_kernel(DecodeArgs a) {
  constexpr int kStride = gu_stage_stride<kMaxTok, kStageX>();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGuStages * kStride);
  uint64_t* empty = full + kGuStages;
  float* s_part = reinterpret_cast<float*>(empty + kGuStages);  // [kp 2][mat 2][64][kMaxTok]
  int& s_abort = *reinterpret_cast<int*>(s_part + 4 * kTileRows * kMaxTok);
  uint8_t* s_zero = reinterpret_cast<uint8_t*>(&s_abort) + 16;  // 32 zero bytes
  uint8_t* s_x = s_zero + 32;                                   // staged x: hi, lo, then run scales
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < kGuStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kConsumerWarps);
    }
    ptx::fence_barrier_init();
  }
  if (threadIdx.x < 8) reinterpret_cast<uint32_t*>(s_zero)[threadIdx.x] = 0u;
  __syncthreads();
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();

  const int tiles = (a.I + kTileRows - 1) / kTileRows;
  const int n_units = __ldcg(a.n_act) * tiles;
  const int n_st = (a.nbh + kGuSB - 1) / kGuSB;
  const int runs = a.H / 32;

  if (warp == kConsumerWarps) {  // producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      ptx::IssueLog log;
      for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
        const int ai = unit / tiles, rt = unit - ai * tiles;
        const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
        const CUtensorMap* mg = a.tmaps + kMapsPerSlot * in_range(__ldcg(a.slot_of + e), a.n_slots, a.err);
        int cnt = 0, tok[kMaxTok];
        if (!kStageX) {
          cnt = __ldcg(a.counts + e);
          const int r0 = in_range(__ldcg(a.offsets + e), a.n_rows, a.err);
#pragma unroll
          for (int t = 0; t < kMaxTok; ++t)
            tok[t] = t < cnt ? in_range(__ldcg(a.perm + in_range(r0 + t, a.n_rows, a.err)) / a.kS, a.T, a.err) : 0;
        }
        for (int st = 0; st < n_st; ++st) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
            flag_error(a.err, 1u);
            log.drain(full, kGuStages);
            return;
          }
          const int nsb = min(kGuSB, a.nbh - st * kGuSB);  // super-blocks of x this stage needs
          ptx::mbar_arrive_expect_tx(&full[stage], kGuStageBytes + (uint32_t)(cnt * nsb * (2 * kQK + 64)));
          uint8_t* dst = stages + stage * kStride;
          ptx::tma_load_w(dst, mg, st * kGuSB, rt * kTileRows, &full[stage]);
          ptx::tma_load_w(dst + kGuTileBytes, mg + 1, st * kGuSB, rt * kTileRows, &full[stage]);
          if (!kStageX) {
#pragma unroll
            for (int t = 0; t < kMaxTok; ++t) {
              if (t < cnt) {
                uint8_t* xs = dst + kGuStageBytes + t * kXSliceBytes;
                const size_t xo = (size_t)tok[t] * a.H + (size_t)st * kGuSB * kQK;
                ptx::bulk_load(xs, a.xq + xo, (uint32_t)(nsb * kQK), &full[stage]);
                ptx::bulk_load(xs + kGuSB * kQK, a.xq + a.xq_plane + xo, (uint32_t)(nsb * kQK), &full[stage]);
                ptx::bulk_load(xs + 2 * kGuSB * kQK, a.xsc + (size_t)tok[t] * runs + (size_t)st * kGuSB * 8,
                               (uint32_t)(nsb * 64), &full[stage]);
              }
            }
          }
          log.note(stage, phase);
          if (++stage == kGuStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      log.drain(full, kGuStages);
    }
    return;
  }

  // staged x: [T][H] hi bytes, [T][H] lo bytes, [T][runs] run scales
  const size_t xbytes = (size_t)a.T * a.H;
  if (kStageX) {
    const uint4* src_h = reinterpret_cast<const uint4*>(a.xq);
    const uint4* src_l = reinterpret_cast<const uint4*>(a.xq + a.xq_plane);
    uint4* dh = reinterpret_cast<uint4*>(s_x);
    uint4* dl = reinterpret_cast<uint4*>(s_x + xbytes);
    for (int i = threadIdx.x; i < (int)(xbytes / 16); i += kConsumerThreads) {
      dh[i] = __ldcg(src_h + i);
      dl[i] = __ldcg(src_l + i);
    }
    float2* dsc = reinterpret_cast<float2*>(s_x + 2 * xbytes);
    for (int i = threadIdx.x; i < a.T * runs; i += kConsumerThreads) dsc[i] = __ldcg(a.xsc + i);
    ptx::named_barrier_sync(1, kConsumerThreads);
  }
  const uint8_t* xh_base = s_x;
  const uint8_t* xl_base = s_x + xbytes;
  const float2* xsc_base = reinterpret_cast<const float2*>(s_x + 2 * xbytes);
  const uint8_t* zero = s_zero;

  // consumers: warp w takes matrix (w>>2)&1 (gate, up), rows 16*(w&3).., and
  // super-block w>>3 of every stage
  const int mat = (warp >> 2) & 1, rbase = (warp & 3) * 16, kp = warp >> 3;
  const int g = lane >> 2, c = lane & 3;
  const int pitch = kQBytes;                      // rows of one super-block
  int stage = 0;
  uint32_t phase = 0;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int ai = unit / tiles, rt = unit - ai * tiles;
    const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
    const int cnt = __ldcg(a.counts + e), r0 = in_range(__ldcg(a.offsets + e), a.n_rows, a.err);
    int tok[kMaxTok];
    if (kStageX) {
#pragma unroll
      for (int t = 0; t < kMaxTok; ++t)
        tok[t] = t < cnt ? in_range(__ldcg(a.perm + in_range(r0 + t, a.n_rows, a.err)) / a.kS, a.T, a.err) : 0;
    }
    float acc[kMaxTok], acc8[kMaxTok];
#pragma unroll
    for (int t = 0; t < kMaxTok; ++t) acc[t] = acc8[t] = 0.f;
    bool ok = true;
    for (int st = 0; st < n_st; ++st) {
      if (!ptx::mbar_wait(&full[stage], phase)) {
        flag_error(a.err, 2u);
        ok = false;
        break;
      }
      const int kb = st * kGuSB + kp;
      if (kb < a.nbh) {
        const uint8_t* sbase = stages + stage * kStride;
        const uint8_t* blk = sbase + mat * kGuTileBytes + kp * kTileRows * kQBytes + (rbase + g) * pitch;
        uint4 h0, h8;
        uint32_t q[8], q8[8];
        load_row_block(blk, c, h0, q);
        load_row_block(blk + 8 * pitch, c, h8, q8);
        const RowScales rs = decode_scales(h0, c), rs8 = decode_scales(h8, c);
#pragma unroll
        for (int t = 0; t < kMaxTok; ++t) {
          if (t < cnt) {
            if (kStageX) {
              const size_t xo = (size_t)tok[t] * a.H + kb * kQK;
              const float4 sc = reinterpret_cast<const float4*>(xsc_base + (size_t)tok[t] * runs + kb * 8)[c];
              sb_dot(q, q8, rs, rs8, xh_base + xo, xl_base + xo, zero, sc, g, c, acc[t], acc8[t]);
            } else {
              // the token's slice in this stage: hi, lo, run scales
              const uint8_t* xs = sbase + kGuStageBytes + t * kXSliceBytes;
              const float4 sc = reinterpret_cast<const float4*>(xs + 2 * kGuSB * kQK + kp * 64)[c];
              sb_dot(q, q8, rs, rs8, xs + kp * kQK, xs + kGuSB * kQK + kp * kQK, zero, sc, g, c, acc[t], acc8[t]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[stage]);
      if (++stage == kGuStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // a warp that gave up on a wait sets the flag before the barrier; every
    // consumer warp reaches it (all waits are bounded) and they stop together
    if (!ok) s_abort = 1;
    ptx::named_barrier_sync(1, kConsumerThreads);  // also: the previous unit's SwiGLU reads are done
    if (s_abort) return;
#pragma unroll
    for (int t = 0; t < kMaxTok; ++t) {  // the quad's four threads hold disjoint sub-blocks
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 1);
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 2);
      acc8[t] += __shfl_xor_sync(0xffffffffu, acc8[t], 1);
      acc8[t] += __shfl_xor_sync(0xffffffffu, acc8[t], 2);
    }
    if (c == 0) {
      float* p = s_part + ((kp * 2 + mat) * kTileRows + rbase + g) * kMaxTok;
#pragma unroll
      for (int t = 0; t < kMaxTok; ++t) {
        p[t] = acc[t];
        p[8 * kMaxTok + t] = acc8[t];
      }
    }
    ptx::named_barrier_sync(1, kConsumerThreads);
    // SwiGLU, 16-bit fixed point per run, and run scales: one warp per (token, run)
    for (int job = warp; job < 2 * cnt; job += kConsumerWarps) {
      const int t = job >> 1, run = job & 1;
      const int f = run * 32 + lane;
      const float gv = s_part[(0 * kTileRows + f) * kMaxTok + t] + s_part[(2 * kTileRows + f) * kMaxTok + t];
      const float uv = s_part[(1 * kTileRows + f) * kMaxTok + t] + s_part[(3 * kTileRows + f) * kMaxTok + t];
      float2 rsc;
      int8_t hh;
      uint8_t hl;
      quant_run16(silu_f(gv) * uv, hh, hl, rsc);
      const int feat0 = rt * kTileRows + run * 32;
      const size_t o = (size_t)(r0 + t) * a.I_pad + feat0 + lane;
      a.hq[o] = hh;
      reinterpret_cast<uint8_t*>(a.hq + a.hq_plane)[o] = hl;
      if (lane == 0) a.hsc[(size_t)(r0 + t) * (a.I_pad / 32) + feat0 / 32] = rsc;
    }
  }
}

// ============================================================================ down
// The producer also copies each unit's activations (h of the expert's rows:
// both byte planes and the run scales) into one of two shared-memory slots,
// so they arrive with the weights instead of being fetched from L2 by every warp.
template <int kMaxTok>
__global__ void __launch_bounds__(kThreads, 1) down_d1_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDnStages * kDnStageBytes);
  uint64_t* empty = full + kDnStages;
  uint64_t* afull = empty + kDnStages;  // activation slots
  uint64_t* aempty = afull + 2;
  float* s_part = reinterpret_cast<float*>(aempty + 2);  // [kp 4][64][kMaxTok]
  int& s_abort = *reinterpret_cast<int*>(s_part + 4 * kTileRows * kMaxTok);
  uint8_t* s_zero = reinterpret_cast<uint8_t*>(&s_abort) + 16;  // 32 zero bytes
  uint8_t* s_act = s_zero + 32;                                 // 2 slots of a.act_slot_bytes
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hruns = a.I_pad / 32;
  const uint32_t plane_bytes = (uint32_t)(kMaxTok * a.I_pad);  // per slot: hi plane, lo plane, scales
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < kDnStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kConsumerWarps);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&afull[s], 1);
      ptx::mbar_init(&aempty[s], kConsumerWarps);
    }
    ptx::fence_barrier_init();
  }
  if (threadIdx.x < 8) reinterpret_cast<uint32_t*>(s_zero)[threadIdx.x] = 0u;
  __syncthreads();
  // The routing (act lists, counts) comes from two kernels back; the kernel in
  // between waited for it before letting this one launch, so it is complete.
  const int tiles = a.H / kTileRows;
  const int n_units = __ldcg(a.n_act) * tiles;
  const int n_st = (a.nbi + kDnSB - 1) / kDnSB;

  if (warp == kConsumerWarps) {
    if (lane == 0) {
      int stage = 0, slot = 0;
      uint32_t phase = 0, aphase = 0;
      bool waited = false;
      ptx::IssueLog log, alog;
      for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
        const int ai = unit / tiles, rt = unit - ai * tiles;
        const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
        const CUtensorMap* md = a.tmaps + kMapsPerSlot * in_range(__ldcg(a.slot_of + e), a.n_slots, a.err) + 2;
        // weights first: they do not depend on the gate/up kernel
        for (int st = 0; st < n_st; ++st) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
            flag_error(a.err, 4u);
            if (!waited) ptx::pdl_wait();
            log.drain(full, kDnStages);
            alog.drain(afull, 2);
            return;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], kDnStageBytes);
          ptx::tma_load_w(stages + stage * kDnStageBytes, md, st * kDnSB, rt * kTileRows, &full[stage]);
          log.note(stage, phase);
          if (++stage == kDnStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        // then the unit's activations, written by the gate/up kernel
        if (!waited) {
          ptx::pdl_wait();
          waited = true;
        }
        if (!ptx::mbar_wait(&aempty[slot], aphase ^ 1u)) {
          flag_error(a.err, 4u);
          log.drain(full, kDnStages);
          alog.drain(afull, 2);
          return;
        }
        const int cnt = __ldcg(a.counts + e), r0 = in_range(__ldcg(a.offsets + e), a.n_rows, a.err);
        const uint32_t nb = (uint32_t)(cnt * a.I_pad);
        const uint32_t sb = (uint32_t)(cnt * hruns * 8);
        uint8_t* dst = s_act + slot * a.act_slot_bytes;
        ptx::mbar_arrive_expect_tx(&afull[slot], 2 * nb + sb);
        const size_t ho = (size_t)r0 * a.I_pad;
        ptx::bulk_load(dst, a.hq + ho, nb, &afull[slot]);
        ptx::bulk_load(dst + plane_bytes, a.hq + a.hq_plane + ho, nb, &afull[slot]);
        ptx::bulk_load(dst + 2 * plane_bytes, a.hsc + (size_t)r0 * hruns, sb, &afull[slot]);
        alog.note(slot, aphase);
        if (++slot == 2) {
          slot = 0;
          aphase ^= 1u;
        }
      }
      if (!waited) ptx::pdl_wait();
      log.drain(full, kDnStages);
      alog.drain(afull, 2);
    } else {
      ptx::pdl_wait();
    }
    return;
  }
  ptx::pdl_wait();  // hq / hsc come from the gate/up kernel
  ptx::pdl_launch_dependents();

  // consumers: warp w takes rows 16*(w&3).. and super-block w>>2 of every stage
  const int rbase = (warp & 3) * 16, kp = warp >> 2;
  const int g = lane >> 2, c = lane & 3;
  const int pitch = kQBytes;                      // rows of one super-block
  int stage = 0, slot = 0;
  uint32_t phase = 0, aphase = 0;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int ai = unit / tiles, rt = unit - ai * tiles;
    const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
    const int cnt = __ldcg(a.counts + e), r0 = in_range(__ldcg(a.offsets + e), a.n_rows, a.err);
    float acc[kMaxTok], acc8[kMaxTok];
#pragma unroll
    for (int t = 0; t < kMaxTok; ++t) acc[t] = acc8[t] = 0.f;
    bool ok = ptx::mbar_wait(&afull[slot], aphase);
    if (!ok) flag_error(a.err, 8u);
    const uint8_t* act = s_act + slot * a.act_slot_bytes;
    const float2* asc = reinterpret_cast<const float2*>(act + 2 * plane_bytes);
    for (int st = 0; st < n_st && ok; ++st) {
      if (!ptx::mbar_wait(&full[stage], phase)) {
        flag_error(a.err, 8u);
        ok = false;
        break;
      }
      const int kb = st * kDnSB + kp;
      if (kb < a.nbi) {
        const uint8_t* blk = stages + stage * kDnStageBytes + kp * kTileRows * kQBytes + (rbase + g) * pitch;
        uint4 h0, h8;
        uint32_t q[8], q8[8];
        load_row_block(blk, c, h0, q);
        load_row_block(blk + 8 * pitch, c, h8, q8);
        const RowScales rs = decode_scales(h0, c), rs8 = decode_scales(h8, c);
#pragma unroll
        for (int t = 0; t < kMaxTok; ++t) {
          if (t < cnt) {
            const int ho = t * a.I_pad + kb * kQK;
            const float4 sc = reinterpret_cast<const float4*>(asc + t * hruns + kb * 8)[c];
            sb_dot(q, q8, rs, rs8, act + ho, act + plane_bytes + ho, s_zero, sc, g, c, acc[t], acc8[t]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[stage]);
      if (++stage == kDnStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&aempty[slot]);
    if (++slot == 2) {
      slot = 0;
      aphase ^= 1u;
    }
    if (!ok) s_abort = 1;
    ptx::named_barrier_sync(1, kConsumerThreads);  // also: the previous unit's reads of s_part are done
    if (s_abort) return;
#pragma unroll
    for (int t = 0; t < kMaxTok; ++t) {
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 1);
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 2);
      acc8[t] += __shfl_xor_sync(0xffffffffu, acc8[t], 1);
      acc8[t] += __shfl_xor_sync(0xffffffffu, acc8[t], 2);
    }
    if (c == 0) {
      float* p = s_part + (kp * kTileRows + rbase + g) * kMaxTok;
#pragma unroll
      for (int t = 0; t < kMaxTok; ++t) {
        p[t] = acc[t];
        p[8 * kMaxTok + t] = acc8[t];
      }
    }
    ptx::named_barrier_sync(1, kConsumerThreads);
    // the four K-parts of each row, summed in a fixed order, to y
    for (int i = threadIdx.x; i < kTileRows * cnt; i += kConsumerThreads) {
      const int t = i / kTileRows, row = i - t * kTileRows;
      float v = 0.f;
#pragma unroll
      for (int part = 0; part < 4; ++part) v += s_part[(part * kTileRows + row) * kMaxTok + t];
      a.y[(size_t)(r0 + t) * a.H + rt * kTileRows + row] = v;
    }
  }
}

}  // namespace

// Shared memory of the decode kernels (bytes, with 1024 of alignment slack).
// x_stage_bytes > 0: x staged once per CTA (the max_tok = 1 kernel); 0: each
// stage carries max_tok tokens' x slices.
size_t gate_up_d1_smem(int max_tok, size_t x_stage_bytes) {
  const size_t stride = kGuStageBytes + (x_stage_bytes ? 0 : (size_t)max_tok * kXSliceBytes);
  return 1024 + (size_t)kGuStages * stride + 2 * kGuStages * 8 + 4 * kTileRows * max_tok * 4 + 16 + 32 +
         x_stage_bytes;
}
size_t down_d1_smem(int max_tok, size_t act_slot_bytes) {
  return 1024 + (size_t)kDnStages * kDnStageBytes + 2 * kDnStages * 8 + 4 * 8 + 4 * kTileRows * max_tok * 4 + 16 +
         32 + 2 * act_slot_bytes;
}

static bool attr_done(uint64_t* mask) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (*mask & bit) return true;
  *mask |= bit;
  return false;
}

static cudaError_t launch_pdl(const void* fn, int grid, int threads, size_t smem, cudaStream_t st, DecodeArgs* args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* params[1] = {args};
  return cudaLaunchKernelExC(&cfg, fn, params);
}

template <typename K>
static cudaError_t launch_with_smem(K kernel, uint64_t* mask, size_t smem, int n_sm, cudaStream_t st,
                                    const DecodeArgs& a) {
  if (!attr_done(mask)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDecodeSmem);
    if (e != cudaSuccess) return e;
  }
  DecodeArgs args = a;
  return launch_pdl(reinterpret_cast<const void*>(kernel), n_sm, kThreads, smem, st, &args);
}

cudaError_t launch_gate_up_d1(const DecodeArgs& a, int max_tok, int n_sm, cudaStream_t st) {
  static uint64_t m1 = 0, m4 = 0;
  if (max_tok == 1 && a.stage_x) {
    const size_t xs = 2 * (size_t)a.T * a.H + (size_t)a.T * (a.H / 32) * 8;
    return launch_with_smem(gate_up_d1_kernel<1, true>, &m1, gate_up_d1_smem(1, xs), n_sm, st, a);
  }
  return launch_with_smem(gate_up_d1_kernel<kD1MaxTok, false>, &m4, gate_up_d1_smem(kD1MaxTok, 0), n_sm, st, a);
}

cudaError_t launch_down_d1(const DecodeArgs& a, int max_tok, int n_sm, cudaStream_t st) {
  static uint64_t m1 = 0, m4 = 0;
  if (max_tok == 1) return launch_with_smem(down_d1_kernel<1>, &m1, down_d1_smem(1, a.act_slot_bytes), n_sm, st, a);
  return launch_with_smem(down_d1_kernel<kD1MaxTok>, &m4, down_d1_smem(kD1MaxTok, a.act_slot_bytes), n_sm, st, a);
}

}  // namespace moe
