// Single-token decode (T = 1) expert kernels: gate/up + SwiGLU, then down, as
// GEMVs over the raw Q4_K bytes with byte dot products (dp4a).
//
// One thread owns one weight row of a 128-row tile and a fixed part of each
// super-block; a stage is one 128-row x 1 (gate/up: of each matrix) or 2
// (down) super-block tile streamed by 2-D TMA into a shared-memory ring.  For
// a 32-bit quant word w (four quants of sub-block 2c in its low nibbles and
// four of sub-block 2c+1 in its high nibbles) the thread forms
//   lo = w & 0x0F0F0F0F,  hi = w & 0xF0F0F0F0  (16 x the high quants)
// and accumulates dp4a(lo, x_hi) and dp4a(lo, x_lo) (and the same for hi),
// where the activations are 16-bit fixed point per 32-element run,
// x = (256*x_hi + x_lo) * 2^-s (x_hi signed, x_lo unsigned bytes), so the
// integer sums are exact.  Per (row, sub-block) the fp32 epilogue adds
//   d*sc * 2^-s * (256*C_hi + C_lo) - dmin*m * X
// (X the run's sum of the represented activations; the 1/16 of the high
// nibbles is folded into the scale, exactly): the Q4_K weight value
// d*sc*q - dmin*m applied exactly up to fp32 rounding -- the same arithmetic as
// the multi-token decode kernels, with fewer instructions per weight.
//
// A thread takes one chunk of two rows, so each activation load serves two
// rows and the two rows' integer chains run side by side.
// gate/up: unit = (expert, 128 rows); warp w handles chunk w>>2 of every
// super-block for row 32*(w&3)+lane of both matrices; at the unit's end the
// four chunk parts meet in shared memory (fixed order), and gate rows meet up
// rows for SwiGLU, written as h in the same fixed-point form.
// down: unit = (expert, 128 output rows); warp w handles rows 32*(w&1)+lane
// and +64, super-block w>>3 of each stage's two and chunk (w>>1)&3; the eight
// parts of a row meet in shared memory in a fixed order.
#include "moe_internal.h"
#include "ptx.cuh"
#include "gemv_dot.cuh"
#include "q4k_decode.cuh"

namespace moe {
namespace {

constexpr int kGvRows = 128;                    // rows per unit (one TMA box)
constexpr int kGvConsumerWarps = 16;
constexpr int kGvThreads = (kGvConsumerWarps + 1) * 32;
constexpr int kGvConsumers = kGvConsumerWarps * 32;
constexpr int kGvBox = kGvRows * kQBytes;       // one 128-row x 1 super-block box: 18432
constexpr int kGvStageBytes = 2 * kGvBox;       // gate/up: gate + up; down: two super-blocks
constexpr int kGvStages = 4;

__device__ __forceinline__ uint8_t* gv_aligned(uint8_t* raw) {
  const uint32_t pad = (1024u - (ptx::smem_u32(raw) & 1023u)) & 1023u;
  return raw + pad;
}

// ============================================================================ gate/up
__global__ void __launch_bounds__(kGvThreads, 1) gemv_gate_up_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = gv_aligned(smem_raw);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGvStages * kGvStageBytes);
  uint64_t* empty = full + kGvStages;
  float* s_part = reinterpret_cast<float*>(empty + kGvStages);   // [2 mats][4 chunks][128]
  int& s_abort = *reinterpret_cast<int*>(s_part + 8 * kGvRows);
  uint8_t* s_x = reinterpret_cast<uint8_t*>(&s_abort) + 16;      // x: hi plane, lo plane, run scales
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < kGvStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kGvConsumerWarps);
    }
    ptx::fence_barrier_init();
  }
  __syncthreads();
  ptx::pdl_wait();  // routing and the fixed-point x come from the route kernel
  ptx::pdl_launch_dependents();

  const int tiles = (a.I + kGvRows - 1) / kGvRows;
  const int n_units = __ldcg(a.n_act) * tiles;
  const int H = a.H, runs = H / 32;

  if (warp == kGvConsumerWarps) {  // producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      ptx::IssueLog log;
      for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
        const int ai = unit / tiles, rt = unit - ai * tiles;
        const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
        const CUtensorMap* m = a.tmaps + kMapsPerSlot * in_range(__ldcg(a.slot_of + e), a.n_slots, a.err) + 3;
        for (int kb = 0; kb < a.nbh; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
            atomicOr(a.err, 1u);
            log.drain(full, kGvStages);
            return;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], kGvStageBytes);
          uint8_t* dst = stages + stage * kGvStageBytes;
          ptx::tma_load_w(dst, m, kb, rt * kGvRows, &full[stage]);
          ptx::tma_load_w(dst + kGvBox, m + 1, kb, rt * kGvRows, &full[stage]);
          log.note(stage, phase);
          if (++stage == kGvStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      log.drain(full, kGvStages);
    }
    return;
  }

  // x of the token, staged once: hi plane, lo plane, run scales
  {
    const uint4* src_h = reinterpret_cast<const uint4*>(a.xq);
    const uint4* src_l = reinterpret_cast<const uint4*>(a.xq + a.xq_plane);
    uint4* dh = reinterpret_cast<uint4*>(s_x);
    uint4* dl = reinterpret_cast<uint4*>(s_x + H);
    for (int i = threadIdx.x; i < H / 16; i += kGvConsumers) {
      dh[i] = __ldcg(src_h + i);
      dl[i] = __ldcg(src_l + i);
    }
    float2* dsc = reinterpret_cast<float2*>(s_x + 2 * H);
    for (int i = threadIdx.x; i < runs; i += kGvConsumers) dsc[i] = __ldcg(a.xsc + i);
    ptx::named_barrier_sync(1, kGvConsumers);
  }
  const uint8_t* xh = s_x;
  const uint8_t* xl = s_x + H;
  const float2* xsc = reinterpret_cast<const float2*>(s_x + 2 * H);

  // warp w: chunk c = w >> 2 of every super-block, row 32*(w&3)+lane of both
  // matrices (the chunk's activations serve the gate row and the up row)
  const int c = warp >> 2, row = (warp & 3) * 32 + lane;
  int stage = 0;
  uint32_t phase = 0;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int ai = unit / tiles, rt = unit - ai * tiles;
    const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
    const int r0 = in_range(__ldcg(a.offsets + e), a.n_rows, a.err);
    float acc[2] = {0.f, 0.f};  // gate, up
    bool ok = true;
    for (int kb = 0; kb < a.nbh; ++kb) {
      if (!ptx::mbar_wait(&full[stage], phase)) {
        atomicOr(a.err, 2u);
        ok = false;
        break;
      }
      const uint8_t* bg = stages + stage * kGvStageBytes + row * kQBytes;
      const uint8_t* const blk[2] = {bg, bg + kGvBox};
      gv_chunk_rows<2>(blk, c, xh + kb * kQK, xl + kb * kQK, xsc + kb * 8, acc);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[stage]);
      if (++stage == kGvStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // a warp that gave up on a wait sets the flag before the barrier; every
    // consumer warp reaches it (all waits are bounded) and they stop together
    if (!ok) s_abort = 1;
    ptx::named_barrier_sync(1, kGvConsumers);  // also: the previous unit's SwiGLU reads are done
    if (s_abort) return;
    s_part[c * kGvRows + row] = acc[0];
    s_part[(4 + c) * kGvRows + row] = acc[1];
    ptx::named_barrier_sync(1, kGvConsumers);
    // SwiGLU (chunk parts summed in a fixed order), 16-bit fixed point per run:
    // warps 0-3 own features 32*w .. 32*w+31 of the tile
    if (warp < 4) {
      const int f = warp * 32 + lane;
      const float* pg = s_part + f;
      const float* pu = s_part + 4 * kGvRows + f;
      const float g = ((pg[0] + pg[kGvRows]) + pg[2 * kGvRows]) + pg[3 * kGvRows];
      const float u = ((pu[0] + pu[kGvRows]) + pu[2 * kGvRows]) + pu[3 * kGvRows];
      float2 rsc;
      int8_t hh;
      uint8_t hl;
      quant_run16(silu_f(g) * u, hh, hl, rsc);
      const int feat = rt * kGvRows + f;
      const size_t o = (size_t)r0 * a.I_pad + feat;
      a.hq[o] = hh;
      reinterpret_cast<uint8_t*>(a.hq + a.hq_plane)[o] = hl;
      if (lane == 0) a.hsc[(size_t)r0 * (a.I_pad / 32) + feat / 32] = rsc;
    }
  }
}

// ============================================================================ down
// The producer also copies each unit's activations (h of the expert's token:
// both byte planes and the run scales) into one of two shared-memory slots.
// It issues the first unit's weights before waiting for the gate/up kernel.
__global__ void __launch_bounds__(kGvThreads, 1) gemv_down_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = gv_aligned(smem_raw);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGvStages * kGvStageBytes);
  uint64_t* empty = full + kGvStages;
  uint64_t* afull = empty + kGvStages;  // activation slots
  uint64_t* aempty = afull + 2;
  float* s_part = reinterpret_cast<float*>(aempty + 2);  // [8 parts][128]
  int& s_abort = *reinterpret_cast<int*>(s_part + 8 * kGvRows);
  uint8_t* s_act = reinterpret_cast<uint8_t*>(&s_abort) + 16;  // 2 slots of act_slot_bytes
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int I_pad = a.I_pad, hruns = I_pad / 32;
  const size_t slot_bytes = a.act_slot_bytes;   // 2 * I_pad + hruns * 8
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < kGvStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kGvConsumerWarps);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&afull[s], 1);
      ptx::mbar_init(&aempty[s], kGvConsumerWarps);
    }
    ptx::fence_barrier_init();
  }
  __syncthreads();
  // The routing comes from two kernels back; the kernel in between waited for
  // it before letting this one launch, so it is complete.
  const int tiles = a.H / kGvRows;
  const int n_units = __ldcg(a.n_act) * tiles;
  const int n_st = (a.nbi + 1) / 2;

  if (warp == kGvConsumerWarps) {
    if (lane == 0) {
      int stage = 0, slot = 0;
      uint32_t phase = 0, aphase = 0;
      bool waited = false;
      ptx::IssueLog log, alog;
      // The unit's activations (h of the expert's token, written by the
      // gate/up kernel: both byte planes and the run scales) go to a slot.
      auto load_act = [&](int e) -> bool {
        if (!ptx::mbar_wait(&aempty[slot], aphase ^ 1u)) return false;
        const int r0 = in_range(__ldcg(a.offsets + e), a.n_rows, a.err);
        uint8_t* dst = s_act + slot * slot_bytes;
        ptx::mbar_arrive_expect_tx(&afull[slot], (uint32_t)(2 * I_pad + hruns * 8));
        ptx::bulk_load(dst, a.hq + (size_t)r0 * I_pad, (uint32_t)I_pad, &afull[slot]);
        ptx::bulk_load(dst + I_pad, a.hq + a.hq_plane + (size_t)r0 * I_pad, (uint32_t)I_pad, &afull[slot]);
        ptx::bulk_load(dst + 2 * I_pad, a.hsc + (size_t)r0 * hruns, (uint32_t)(hruns * 8), &afull[slot]);
        alog.note(slot, aphase);
        if (++slot == 2) {
          slot = 0;
          aphase ^= 1u;
        }
        return true;
      };
      for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
        const int ai = unit / tiles, rt = unit - ai * tiles;
        const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
        const CUtensorMap* md = a.tmaps + kMapsPerSlot * in_range(__ldcg(a.slot_of + e), a.n_slots, a.err) + 5;
        // Once the gate/up kernel is complete, a unit's activations are issued
        // before its weights, so they never hold up the unit's first stage.
        if (waited && !load_act(e)) {
          atomicOr(a.err, 4u);
          log.drain(full, kGvStages);
          alog.drain(afull, 2);
          return;
        }
        // the first unit's weights do not depend on the gate/up kernel: they
        // are issued before waiting for it
        for (int st = 0; st < n_st; ++st) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u)) {
            atomicOr(a.err, 4u);
            if (!waited) ptx::pdl_wait();
            log.drain(full, kGvStages);
            alog.drain(afull, 2);
            return;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], kGvStageBytes);
          uint8_t* dst = stages + stage * kGvStageBytes;
          // a second box past the last super-block reads zeros (never used)
          ptx::tma_load_w(dst, md, 2 * st, rt * kGvRows, &full[stage]);
          ptx::tma_load_w(dst + kGvBox, md, 2 * st + 1, rt * kGvRows, &full[stage]);
          log.note(stage, phase);
          if (++stage == kGvStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!waited) {
          ptx::pdl_wait();
          waited = true;
          if (!load_act(e)) {
            atomicOr(a.err, 4u);
            log.drain(full, kGvStages);
            alog.drain(afull, 2);
            return;
          }
        }
      }
      if (!waited) ptx::pdl_wait();
      log.drain(full, kGvStages);
      alog.drain(afull, 2);
    } else {
      ptx::pdl_wait();
    }
    return;
  }
  ptx::pdl_wait();  // hq / hsc come from the gate/up kernel
  ptx::pdl_launch_dependents();

  // consumers: warp w takes part p = w >> 1 of each stage -- super-block
  // p >> 2 of the stage's two, chunk p & 3 -- for rows 32*(w&1)+lane and
  // 64 rows further (the chunk's activations serve both rows)
  const int row = (warp & 1) * 32 + lane, part = warp >> 1;
  const int sbi = part >> 2, c = part & 3;
  int stage = 0, slot = 0;
  uint32_t phase = 0, aphase = 0;
  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int ai = unit / tiles, rt = unit - ai * tiles;
    const int e = in_range(__ldcg(a.act + ai), a.n_ex, a.err);
    const int r0 = in_range(__ldcg(a.offsets + e), a.n_rows, a.err);
    float acc[2] = {0.f, 0.f};  // rows row, row + 64
    bool ok = ptx::mbar_wait(&afull[slot], aphase);
    if (!ok) atomicOr(a.err, 8u);
    const uint8_t* act = s_act + slot * slot_bytes;
    const float2* asc = reinterpret_cast<const float2*>(act + 2 * I_pad);
    for (int st = 0; st < n_st && ok; ++st) {
      if (!ptx::mbar_wait(&full[stage], phase)) {
        atomicOr(a.err, 8u);
        ok = false;
        break;
      }
      const int kb = 2 * st + sbi;
      if (kb < a.nbi) {
        const uint8_t* b0 = stages + stage * kGvStageBytes + sbi * kGvBox + row * kQBytes;
        const uint8_t* const blk[2] = {b0, b0 + 64 * kQBytes};
        gv_chunk_rows<2>(blk, c, act + kb * kQK, act + I_pad + kb * kQK, asc + kb * 8, acc);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[stage]);
      if (++stage == kGvStages) {
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
    ptx::named_barrier_sync(1, kGvConsumers);  // also: the previous unit's reads of s_part are done
    if (s_abort) return;
    s_part[part * kGvRows + row] = acc[0];
    s_part[part * kGvRows + row + 64] = acc[1];
    ptx::named_barrier_sync(1, kGvConsumers);
    // the eight parts of each row, summed in a fixed order, to y
    if (warp < 4) {
      const int r = warp * 32 + lane;
      float v = s_part[r];
#pragma unroll
      for (int p = 1; p < 8; ++p) v += s_part[p * kGvRows + r];
      a.y[(size_t)r0 * a.H + rt * kGvRows + r] = v;
    }
  }
}

template <typename K>
cudaError_t gv_launch(K kernel, uint64_t* mask, size_t smem, int n_sm, cudaStream_t st, const DecodeArgs& a) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (smem > kMaxDecodeSmem) return cudaErrorInvalidValue;
  if (!(*mask & bit)) {  // once per device, for the largest size any shape may need
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDecodeSmem);
    if (e != cudaSuccess) return e;
    *mask |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace

size_t gemv_gate_up_smem(int H) {
  return 1024 + (size_t)kGvStages * kGvStageBytes + 2 * kGvStages * 8 + 8 * kGvRows * 4 + 16 + 2 * (size_t)H +
         (size_t)(H / 32) * 8;
}
size_t gemv_down_smem(size_t act_slot_bytes) {
  return 1024 + (size_t)kGvStages * kGvStageBytes + 2 * kGvStages * 8 + 4 * 8 + 8 * kGvRows * 4 + 16 +
         2 * act_slot_bytes;
}

cudaError_t launch_gemv_gate_up(const DecodeArgs& a, int n_sm, cudaStream_t st) {
  static uint64_t mask = 0;
  return gv_launch(gemv_gate_up_kernel, &mask, gemv_gate_up_smem(a.H), n_sm, st, a);
}

cudaError_t launch_gemv_down(const DecodeArgs& a, int n_sm, cudaStream_t st) {
  static uint64_t mask = 0;
  return gv_launch(gemv_down_kernel, &mask, gemv_down_smem(a.act_slot_bytes), n_sm, st, a);
}

}  // namespace moe
