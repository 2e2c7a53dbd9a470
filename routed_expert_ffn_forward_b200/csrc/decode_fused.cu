// Single-token decode (T = 1) as one persistent kernel: router, top-k and
// gating, gate/up + SwiGLU, down and the weighted combine, with no kernel
// boundary between the steps.
//
// One CTA per SM (16 consumer warps + 1 TMA producer warp).  Steps meet
// through counters in global memory instead of kernel boundaries, so the
// weight stream never drains between them:
//
//  1. Router.  Each CTA computes the logits of experts blockIdx.x,
//     blockIdx.x + grid, ... (256 threads per expert row; the constant router
//     weights are loaded before the kernel waits for its predecessor), then
//     arrives on a grid-wide barrier.  Every CTA needs the routing, and after
//     the barrier each one runs the same top-k + gating over the E logits
//     itself (identical inputs and code, so identical results), which costs
//     one warp a few hundred cycles and saves a second barrier.
//  2. Gate/up + SwiGLU.  Unit = (expert j of the token's k + S, 128 weight
//     rows), the shared experts first: they need no routing, so their CTAs
//     stream weights from the first cycle, overlapping the router.  A unit
//     writes its 128 features of h_j (16-bit fixed point per 32-element run)
//     and adds one to ready[j] (release).
//  3. Down.  Unit = (expert j, 64 output rows), claimed dynamically from a
//     counter (shared experts first), so units balance across SMs.  The
//     producer issues the unit's weights at once and bulk-copies h_j into
//     shared memory once ready[j] counts every gate/up unit of j (acquire).
//     The unit writes its 64 rows of y_j (fp32) and adds one to done[tile].
//  4. Combine.  The unit that completes a 64-row output tile (done[tile]
//     reaches k + S) sums the tile's y rows in the fixed order j = 0..k-1
//     (weighted), then the shared experts, rounds to bf16 and writes out:
//     no atomics on the data, the same order every run (LayerStoRm README,
//     "Notes": a deterministic expert combine).
//
// The dot products are those of the single-token GEMVs (exact integer dp4a
// sums of the raw Q4_K nibbles against fixed-point activations, fp32
// epilogue per sub-block; see gemv_dot.cuh).
//
// Every wait is bounded (2 s): an mbarrier, the grid barrier, a readiness
// counter.  A CTA that gives up sets an error bit that moe_check reports; the
// producer drains every copy it issued before the CTA exits.  The grid
// barrier assumes every CTA is resident at once: the grid is one CTA per SM
// and the shared-memory footprint admits one CTA per SM.
#include "gemv_dot.cuh"
#include "moe_internal.h"
#include "ptx.cuh"
#include "qdot.cuh"
#include "topk.cuh"

namespace moe {
namespace {

constexpr int kFzWarps = 16;                       // consumer warps
constexpr int kFzThreads = (kFzWarps + 1) * 32;
constexpr int kFzConsumers = kFzWarps * 32;
constexpr int kFzGuRows = 64;                      // gate/up unit: weight rows of gate and of up
constexpr int kFzDnRows = 64;                      // down unit: output rows
constexpr int kFzDnSb = 4;                         // 256-weight groups per down stage
constexpr int kFzStages = kFusedMaxStages;         // at most; a stage is 256 x the group size (Q4_K: 36,864 B)
constexpr uint64_t kFzLimitNs = 2000000000ull;

// error bits (moe_check): which wait gave up
constexpr unsigned kErrFzProducer = 1u << 10, kErrFzConsumer = 1u << 11, kErrFzGrid = 1u << 12,
                   kErrFzReady = 1u << 13;

// global sync words (FusedArgs::sync)
// sync words: [4..5] launch counter (64-bit; every CTA adds 1 at its start
// and it is never reset, so a CTA of launch L reads a value in
// [L·grid, (L+1)·grid)).  Per launch parity s = L & 1: [8+s] routed gate/up
// unit claims, [10+s] down-unit claims, [12+s] finished down units,
// [16+64s+j] finished gate/up units of pick j; launch L zeroes parity
// s ^ 1 for launch L + 1 (launch L - 1, its last user, has completed).
// [kSyncLogits..] the logits, each a 64-bit word (L + 1, fp32 bits): a
// reader knows a logit is this launch's without any barrier or fence.
constexpr int kSyncEpoch = 4, kSyncGu = 8, kSyncNext = 10, kSyncDone = 12, kSyncReady = 16, kSyncLogits = 256;
static_assert(kSyncLogits + 2 * 1024 <= kSyncWords, "sync words hold 1024 tagged logits");

// Shared-memory layout (offsets from the 1024-aligned base).
struct FzLayout {
  uint32_t bars, unit, ids, w, flags, part, xh, xl, xsc, uni, total;
  __host__ __device__ FzLayout(int H, size_t act_slot, int ring_bytes) {
    auto up16 = [](uint32_t v) { return (v + 15u) & ~15u; };
    bars = (uint32_t)ring_bytes;                      // full[S] empty[S] afull[2] aempty[2] route[1]
    unit = bars + (2 * kFzStages + 5) * 8;            // int [kFzStages]
    ids = up16(unit + kFzStages * 4);                 // int [40]
    w = ids + 40 * 4;                                 // float [40]
    flags = up16(w + 40 * 4);                         // int [4], then the u64 launch index (8-byte aligned)
    part = up16(flags + 24);                          // float [2][1024]
    xh = part + 2048 * 4;                             // u8 [H]
    xl = xh + (uint32_t)H;                            // u8 [H]
    xsc = xl + (uint32_t)H;                           // float2 [H/32]
    uni = up16(xsc + (uint32_t)(H / 32) * 8);         // bf16 x [H] | act slots [2][act_slot]
    const uint32_t u1 = (uint32_t)H * 2, u2 = 2 * (uint32_t)act_slot;
    total = up16(uni + (u1 > u2 ? u1 : u2));
  }
};

__device__ __forceinline__ uint8_t* fz_aligned(uint8_t* raw) {
  const uint32_t pad = (1024u - (ptx::smem_u32(raw) & 1023u)) & 1023u;
  return raw + pad;
}

// Spin (one thread) until *p >= v (acquire, 64-bit); false after `lim` ns.
__device__ __forceinline__ bool spin_until_ge64(const uint64_t* p, uint64_t v, uint64_t lim) {
  if (ptx::ld_acquire_gpu_u64(p) >= v) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (ptx::ld_acquire_gpu_u64(p) < v) {
    __nanosleep(32);
    if (ptx::globaltimer() - t0 > lim) return false;
  }
  return true;
}
// Spin (one thread) until *p >= v (acquire); false after `lim` ns.
__device__ __forceinline__ bool spin_until_ge(const uint32_t* p, uint32_t v, uint64_t lim) {
  if (ptx::ld_acquire_gpu(p) >= v) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (ptx::ld_acquire_gpu(p) < v) {
    __nanosleep(32);
    if (ptx::globaltimer() - t0 > lim) return false;
  }
  return true;
}

template <int PL>
__global__ void __launch_bounds__(kFzThreads, 1) decode1_fused_kernel(const FusedArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* sm = fz_aligned(smem_raw);
  const int H = a.H, E = a.E, k = a.k, S = a.S, kS = k + S;
  const FzLayout lay(H, a.act_slot_bytes, a.stages * a.stage_bytes);
  const int n_stages = a.stages, stage_bytes = a.stage_bytes;
  const int gu_box = kFzGuRows * a.sbb_gu, dn_box = kFzDnRows * a.sbb_d;   // bytes of one box
  uint8_t* ring = sm;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + lay.bars);
  uint64_t* empty = full + kFzStages;
  uint64_t* afull = empty + kFzStages;
  uint64_t* aempty = afull + 2;
  uint64_t* route_ready = aempty + 2;
  int* s_unit = reinterpret_cast<int*>(sm + lay.unit);
  int* s_ids = reinterpret_cast<int*>(sm + lay.ids);
  float* s_w = reinterpret_cast<float*>(sm + lay.w);
  volatile int* s_flag = reinterpret_cast<volatile int*>(sm + lay.flags);  // [0] abort [3] owned picks
  // this launch's index L (launch counter / grid)
  uint64_t& s_epoch = *reinterpret_cast<uint64_t*>(sm + lay.flags + 16);
  float* s_part = reinterpret_cast<float*>(sm + lay.part);
  uint8_t* s_xh = sm + lay.xh;
  uint8_t* s_xl = sm + lay.xl;
  float2* s_xsc = reinterpret_cast<float2*>(sm + lay.xsc);
  uint8_t* s_uni = sm + lay.uni;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gu_tiles = (a.I + kFzGuRows - 1) / kFzGuRows;
  const int n_gu = kS * gu_tiles, n_gu_sh = S * gu_tiles;   // units: the shared experts' first
  const int n_gst = (a.nbh + 1) / 2;                        // stages per gate/up unit
  const int dn_tiles = H / kFzDnRows;
  const int n_dn = kS * dn_tiles;
  const int n_dst = (a.nbi + kFzDnSb - 1) / kFzDnSb;  // stages per down unit
  uint32_t* sync = a.sync;
  // limit of every wait but the final drain (a test hook may shorten it)
  const uint64_t lim = a.wait_ns ? a.wait_ns : kFzLimitNs;

  if (threadIdx.x == 0) {
    for (int s = 0; s < n_stages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kFzWarps);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&afull[s], 1);
      ptx::mbar_init(&aempty[s], kFzWarps);
    }
    ptx::mbar_init(route_ready, 1);
    s_flag[0] = 0;
    s_flag[1] = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------------ producer
  if (warp == kFzWarps) {
    if (lane != 0) return;
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_par = 0;  // per stage: a copy was issued, its phase parity
    int aslot = 0;
    uint32_t aphase = 0, a_issued = 0, a_last = 0;
    bool routed = false, ok = true;
    // in streaming mode the expert -> slot table comes from the previous kernel
    if (!a.early) ptx::pdl_wait();
    auto expert_of = [&](int j) { return in_range(j < k ? s_ids[j] : E + (j - k), E + S, a.err); };
    auto next_stage = [&]() {
      if (++stage == n_stages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    // the image of pick j's expert (tile-major: 64-row tiles one after another, each
    // tile its groups one after another, a group 64 rows x its group bytes)
    auto image_of = [&](int j) {
      return a.warena + a.wstride * (size_t)in_range(__ldcg(a.slot_of + expert_of(j)), a.n_slots, a.err);
    };
    // the stages of gate/up unit u: per stage two super-blocks (columns) of the
    // unit's 64 gate rows and 64 up rows.  In the tile-major image those are
    // one contiguous run per matrix, so each is one bulk copy.
    auto issue_gu = [&](int u) -> bool {
      const int jj = u / gu_tiles, rt = u - jj * gu_tiles;
      const int j = jj < S ? k + jj : jj - S;
      const uint8_t* wg = image_of(j) + (size_t)rt * a.nbh * gu_box;   // tile rt of gate
      const uint8_t* wu = wg + a.gate_bytes;                            // tile rt of up
      for (int st = 0; st < n_gst; ++st) {
        if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, lim)) return false;
        const uint32_t run = (uint32_t)(min(2, a.nbh - 2 * st) * gu_box);
        s_unit[stage] = u;
        ptx::mbar_arrive_expect_tx(&full[stage], 2u * run);
        uint8_t* dst = ring + stage * stage_bytes;
        ptx::bulk_load(dst, wg + (size_t)2 * st * gu_box, run, &full[stage]);
        ptx::bulk_load(dst + 2 * gu_box, wu + (size_t)2 * st * gu_box, run, &full[stage]);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        next_stage();
      }
      return true;
    };
    // gate/up: the shared experts' units statically (blockIdx.x, + grid, ...:
    // they need no routing), then the routed ones claimed from a counter that
    // CTA 0 zeroed before the grid barrier, once route_ready fires
    for (int u = blockIdx.x; u < n_gu_sh && ok; u += gridDim.x) {
      if (!ep_owned(E + u / gu_tiles, a.ep_rank, a.ep_world)) continue;   // another rank's expert
      ok = issue_gu(u);
    }
    if (ok) {
      ok = ptx::mbar_wait_sleep(route_ready, 0, 64, lim);
      routed = ok;
    }
    // this launch's counters (s_epoch was set before route_ready fired)
    const int par = (int)(s_epoch & 1u);
    uint32_t* const ctr_gu = sync + kSyncGu + par;
    uint32_t* const ctr_next = sync + kSyncNext + par;
    const uint32_t* const ready = sync + kSyncReady + 64 * par;
    while (ok) {
      const int u = n_gu_sh + (int)atomicAdd(ctr_gu, 1u);
      if (u >= n_gu) break;
      const int j = u / gu_tiles - S;
      if (!ep_owned(expert_of(j), a.ep_rank, a.ep_world)) continue;
      ok = issue_gu(u);
    }
    // down: units claimed from a counter that CTA 0 zeroed before the grid
    // barrier; a down unit's code in s_unit is n_gu + its index
    while (ok) {
      if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, lim)) {
        ok = false;
        break;
      }
      const int u = (int)atomicAdd(ctr_next, 1u);
      if (u >= n_dn) {
        // end of work.  The stage is empty, so its last copy has landed and
        // been read; its arrival below completes one more phase of full[stage],
        // so the final drain must not wait for that copy's phase again (the
        // parity would match the phase after next and never complete).
        s_unit[stage] = -1;
        issued &= ~(1u << stage);
        ptx::mbar_arrive(&full[stage]);
        break;
      }
      const int jj = u / dn_tiles, rt = u - jj * dn_tiles;
      const int j = jj < S ? k + jj : jj - S;
      if (!ep_owned(expert_of(j), a.ep_rank, a.ep_world)) continue;   // the slot stays free for the next claim
      // tile rt of down: per stage up to kFzDnSb groups, one contiguous run
      const uint8_t* wd = image_of(j) + 2 * a.gate_bytes + (size_t)rt * a.nbi * dn_box;
      for (int st = 0; st < n_dst; ++st) {
        if (st > 0 && !ptx::mbar_wait(&empty[stage], phase ^ 1u, lim)) {
          ok = false;
          break;
        }
        const uint32_t run = (uint32_t)(min(kFzDnSb, a.nbi - st * kFzDnSb) * dn_box);
        s_unit[stage] = n_gu + u;
        ptx::mbar_arrive_expect_tx(&full[stage], run);
        ptx::bulk_load(ring + stage * stage_bytes, wd + (size_t)st * kFzDnSb * dn_box, run, &full[stage]);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        next_stage();
      }
      if (!ok) break;
      // h_j, once every gate/up unit of expert j has published its features
      if (!ptx::mbar_wait(&aempty[aslot], aphase ^ 1u, lim)) {
        ok = false;
        break;
      }
      if (!spin_until_ge(ready + j, (uint32_t)gu_tiles, lim)) {
        atomicOr(a.err, kErrFzReady);
        ok = false;
        break;
      }
      ptx::fence_proxy_async_global();  // generic-proxy writes of h, read below by the bulk copy
      const int I_pad = a.I_pad, hruns = I_pad / 32;
      uint8_t* adst = s_uni + aslot * a.act_slot_bytes;
      ptx::mbar_arrive_expect_tx(&afull[aslot], (uint32_t)(2 * I_pad + hruns * 8));
      ptx::bulk_load(adst, a.hq + (size_t)j * I_pad, (uint32_t)I_pad, &afull[aslot]);
      ptx::bulk_load(adst + I_pad, a.hq + a.hq_plane + (size_t)j * I_pad, (uint32_t)I_pad, &afull[aslot]);
      ptx::bulk_load(adst + 2 * I_pad, a.hsc + (size_t)j * hruns, (uint32_t)(hruns * 8), &afull[aslot]);
      a_issued |= 1u << aslot;
      a_last = (a_last & ~(1u << aslot)) | (aphase << aslot);
      if (++aslot == 2) {
        aslot = 0;
        aphase ^= 1u;
      }
    }
    if (!ok) atomicOr(a.err, kErrFzProducer);
    // never leave with a copy into shared memory in flight
    for (int s = 0; s < n_stages; ++s)
      if ((issued >> s) & 1u) ptx::mbar_wait(&full[s], (last_par >> s) & 1u);
    for (int s = 0; s < 2; ++s)
      if ((a_issued >> s) & 1u) ptx::mbar_wait(&afull[s], (a_last >> s) & 1u);
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int tid = threadIdx.x;
  // every consumer warp reaches every cbar() (all waits are bounded and every
  // decision to stop is taken from s_flag right after one), so none is left
  // waiting on a named barrier
  auto cbar = [] {
    __syncwarp();
    ptx::named_barrier_sync(1, kFzConsumers);
  };
  auto fail = [&](unsigned bit) {
    atomicOr(a.err, bit);
    s_flag[0] = 1;
  };

  // (1) router logits: two expert rows at a time (warps 0-7 and 8-15); a
  // thread takes the float4 pieces ht + 256 i of its row, 8 per pass, all
  // loaded before any arithmetic
  {
    const int half = warp >> 3, ht = tid & 255;
    const int nq = H / 4;                                 // float4 pieces per row
    constexpr int kPieces = 8;
    __nv_bfloat16* s_x = reinterpret_cast<__nv_bfloat16*>(s_uni);
    const uint2* xv = reinterpret_cast<const uint2*>(s_x);
    // this CTA's count on the launch counter, taken first so that its round
    // trip overlaps the router's loads
    unsigned long long launch_ctr = 0;
    if (tid == 0) launch_ctr = atomicAdd(reinterpret_cast<unsigned long long*>(sync + kSyncEpoch), 1ull);
    bool first = true;
    for (int e0 = blockIdx.x; e0 < E; e0 += 2 * gridDim.x) {
      const int e = e0 + half * gridDim.x;
      const float4* wrow = reinterpret_cast<const float4*>(a.W + (size_t)min(e, E - 1) * H);
      float acc = 0.f;
      for (int base = 0; base < nq; base += kPieces * 256) {
        float4 w4[kPieces];
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int q = base + ht + 256 * i;
          if (e < E && q < nq) w4[i] = __ldg(wrow + q);
        }
        if (first) {
          // x comes from the previous kernel (or the caller): wait, then stage
          // it; the constant router weights above are already in flight
          ptx::pdl_wait();
          const uint4* src = reinterpret_cast<const uint4*>(a.x);
          for (int i = tid; i < H / 8; i += kFzConsumers) reinterpret_cast<uint4*>(s_x)[i] = __ldcg(src + i);
          if (tid == 0) s_epoch = launch_ctr / gridDim.x;
          cbar();
          first = false;
        }
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int q = base + ht + 256 * i;
          if (e < E && q < nq) {
            const uint2 v = xv[q];
            acc = fmaf(w4[i].x, bf16lo(v.x), acc);
            acc = fmaf(w4[i].y, bf16hi(v.x), acc);
            acc = fmaf(w4[i].z, bf16lo(v.y), acc);
            acc = fmaf(w4[i].w, bf16hi(v.y), acc);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) s_part[warp] = acc;
      cbar();
      if ((warp & 7) == 0 && lane == 0 && e < E) {
        float v = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) v += s_part[half * 8 + w8];
        const float lv = v + (a.b ? a.b[e] : 0.f);
        a.logits[e] = lv;
        ptx::st_relaxed_gpu_u64(reinterpret_cast<uint64_t*>(sync + kSyncLogits) + e,
                                ((uint64_t)(uint32_t)(s_epoch + 1u) << 32) | __float_as_uint(lv));
      }
      cbar();
    }
    if (first) {  // no expert row here: still wait for x
      ptx::pdl_wait();
      const uint4* src = reinterpret_cast<const uint4*>(a.x);
      for (int i = tid; i < H / 8; i += kFzConsumers) reinterpret_cast<uint4*>(s_x)[i] = __ldcg(src + i);
      if (tid == 0) s_epoch = launch_ctr / gridDim.x;
      cbar();
    }
    // CTA 0 zeroes the other parity's counters for the next launch (the
    // previous launch, their last user, is complete: this is after the wait
    // for the previous kernel)
    if (blockIdx.x == 0) {
      const int nx = (int)((s_epoch & 1u) ^ 1u);
      if (tid == 0) {
        sync[kSyncGu + nx] = 0u;
        sync[kSyncNext + nx] = 0u;
        sync[kSyncDone + nx] = 0u;
      }
      for (int i = tid; i < kS; i += kFzConsumers) sync[kSyncReady + 64 * nx + i] = 0u;
    }
  }

  // (2) x as 16-bit fixed point per 32-element run (each CTA its own copy),
  // by warps w0 .. 15: all of them before this CTA's shared-expert units,
  // else warps 1-15 while warp 0 polls the logits
  int n_sh = 0;   // this CTA's shared gate/up units (the producer skips the same ones)
  for (int u = blockIdx.x; u < n_gu_sh; u += gridDim.x) n_sh += ep_owned(E + u / gu_tiles, a.ep_rank, a.ep_world);
  auto quant_x = [&](int w0) {
    const __nv_bfloat16* s_x = reinterpret_cast<const __nv_bfloat16*>(s_uni);
    for (int run = warp - w0; run < H / 32; run += kFzWarps - w0) {
      float2 rsc;
      int8_t xh;
      uint8_t xl;
      quant_run16(__bfloat162float(s_x[run * 32 + lane]), xh, xl, rsc);
      s_xh[run * 32 + lane] = (uint8_t)xh;
      s_xl[run * 32 + lane] = xl;
      if (lane == 0) s_xsc[run] = rsc;
    }
  };
  if (n_sh > 0) {
    quant_x(0);
    cbar();
  }

  // the routing: every CTA selects from the E logits itself, after the barrier
  bool routed = false;
  auto route = [&]() {
    bool got = false;
    // warps 0-1 may still be reading the last unit's partials in s_part,
    // which warp 0 is about to reuse for the logits
    cbar();
    if (warp == 0) {
      // every logit of this launch, polled until all carry its tag (+ hold,
      // a test hook that makes the wait run out), copied to shared memory
      const uint32_t want = (uint32_t)(s_epoch + 1u + (uint64_t)a.hold);
      const uint64_t* lg = reinterpret_cast<const uint64_t*>(sync + kSyncLogits);
      float* s_lg = s_part;   // free: every consumer warp has passed the barrier above
      const uint64_t t0 = ptx::globaltimer();
      while (true) {
        bool mine = true;
        for (int e = lane; e < E; e += 32) {
          const uint64_t v = ptx::ld_relaxed_gpu_u64(lg + e);
          mine &= (uint32_t)(v >> 32) == want;
          s_lg[e] = __uint_as_float((uint32_t)v);
        }
        if (__all_sync(0xffffffffu, mine)) {
          got = true;
          break;
        }
        if (ptx::globaltimer() - t0 > lim) break;
      }
      if (!got && lane == 0) fail(kErrFzGrid);
      __syncwarp();
    } else if (n_sh == 0) {
      quant_x(1);
    }
    if (got) {
      warp_topk_gate<PL, false>(s_part, E, k, a.gating, a.forced, s_ids, s_w);
      __syncwarp();
      if (lane < S) {
        s_ids[k + lane] = E + lane;
        s_w[k + lane] = 1.f;
      }
      if (blockIdx.x == 0 && lane < k) {
        a.ids[lane] = s_ids[lane];
        a.w[lane] = s_w[lane];
      }
      __syncwarp();
      // contributions each output tile waits for: the experts this rank owns
      int own = 0;
      for (int q = 0; q < kS; ++q) own += ep_owned(s_ids[q], a.ep_rank, a.ep_world);
      if (lane == 0) s_flag[3] = own;
      if (lane == 0) ptx::mbar_arrive(route_ready);
    }
    cbar();
    routed = true;
  };

  int stage = 0;
  uint32_t phase = 0;
  auto next_stage = [&]() {
    if (++stage == n_stages) {
      stage = 0;
      phase ^= 1u;
    }
  };

  // (3) gate/up + SwiGLU units and (4) down units, in the order the producer
  // issues them: this CTA's shared-expert gate/up units, then routed gate/up
  // units and down units as claimed.  The routing is needed from the first
  // unit after the shared ones on.
  {
    const int g_row = (warp & 1) * 32 + lane, g_sb = (warp >> 1) & 1, g_c = warp >> 2;   // gate/up: row, column, chunk
    const int r0 = lane, sb = warp >> 2, c = warp & 3;                                    // down: rows r0, r0 + 32
    const int I_pad = a.I_pad;
    int aslot = 0, buf = 0, seen = 0;
    uint32_t aphase = 0;
    while (true) {
      if (seen++ == n_sh && !routed) {
        route();
        if (s_flag[0]) return;
      }
      bool ok = ptx::mbar_wait(&full[stage], phase, lim);
      const int u = ok ? s_unit[stage] : -1;   // -1 from the producer: end of work
      if (!ok) fail(kErrFzConsumer);
      if (u < 0) {
        cbar();
        if (s_flag[0]) return;
        break;
      }
      if (u < n_gu) {
        // ---- gate/up unit: 64 features of pick j
        const int jj = u / gu_tiles, rt = u - jj * gu_tiles;
        const int j = jj < S ? k + jj : jj - S;
        float acc[2] = {0.f, 0.f};   // gate row, up row
        for (int st = 0; st < n_gst; ++st) {
          if (st > 0 && !ptx::mbar_wait(&full[stage], phase, lim)) {
            ok = false;
            break;
          }
          const int kb = 2 * st + g_sb;
          if (kb < a.nbh) {
            const uint8_t* bg = ring + stage * stage_bytes + g_sb * gu_box + g_row * a.sbb_gu;
            const uint8_t* const blk[2] = {bg, bg + 2 * gu_box};
            const uint8_t *xh = s_xh + kb * kQK, *xl = s_xl + kb * kQK;
            const float2* xs = s_xsc + kb * 8;
            switch (a.qgu) {   // uniform across the CTA
              case kQ5_K: q_chunk_rows<kQ5_K, 2>(blk, g_c, xh, xl, xs, acc); break;
              case kQ6_K: q_chunk_rows<kQ6_K, 2>(blk, g_c, xh, xl, xs, acc); break;
              case kQ8_0: q_chunk_rows<kQ8_0, 2>(blk, g_c, xh, xl, xs, acc); break;
              case kMXFP4: q_chunk_rows<kMXFP4, 2>(blk, g_c, xh, xl, xs, acc); break;
              default: q_chunk_rows<kQ4_K, 2>(blk, g_c, xh, xl, xs, acc); break;
            }
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&empty[stage]);
          next_stage();
        }
        if (!ok) fail(kErrFzConsumer);
        // the unit's partial sums go to the buffer the unit before last used
        // (double-buffered like the down units'), so the two warps that run
        // the SwiGLU may lag the others by a unit
        float* sp = s_part + buf * (kFzWarps * kFzDnRows);
        sp[(g_sb * 4 + g_c) * kFzGuRows + g_row] = acc[0];
        sp[(8 + g_sb * 4 + g_c) * kFzGuRows + g_row] = acc[1];
        cbar();                          // every warp, every unit: the partials are complete
        if (s_flag[0]) return;
        // SwiGLU (the 8 parts of each row summed in a fixed order) -> h_j,
        // warps 0-1; then one thread publishes the features (release,
        // cumulative over the two warps' stores; the ready counters are
        // zeroed before the routing)
        if (warp < 2) {
          const int f = warp * 32 + lane;
          float g = sp[f], up = sp[8 * kFzGuRows + f];
#pragma unroll
          for (int p = 1; p < 8; ++p) {
            g += sp[p * kFzGuRows + f];
            up += sp[(8 + p) * kFzGuRows + f];
          }
          float2 rsc;
          int8_t hh;
          uint8_t hl;
          quant_run16(silu_f(g) * up, hh, hl, rsc);
          const int feat = rt * kFzGuRows + f;
          const size_t o = (size_t)j * I_pad + feat;
          a.hq[o] = hh;
          reinterpret_cast<uint8_t*>(a.hq + a.hq_plane)[o] = hl;
          if (lane == 0) a.hsc[(size_t)j * (I_pad / 32) + feat / 32] = rsc;
          ptx::named_barrier_sync(2, 64);
          if (tid == 0) {
            ptx::fence_proxy_async_global();
            ptx::red_add_release_gpu(sync + kSyncReady + 64 * (int)(s_epoch & 1u) + j, 1u);
          }
        }
        buf ^= 1;
        continue;
      }
      // ---- down unit: 64 output rows of pick j.  Its 64 rows of y_j are
      // published with one release add to the count of finished units, which
      // no thread waits on; the unit partials are double-buffered, so the two
      // warps that reduce them may lag the others by a unit.
      const int v = u - n_gu;
      const int jj = v / dn_tiles, rt = v - jj * dn_tiles;
      const int j = jj < S ? k + jj : jj - S;
      float acc[2] = {0.f, 0.f};
      ok = ptx::mbar_wait(&afull[aslot], aphase, lim);
      const uint8_t* act = s_uni + aslot * a.act_slot_bytes;
      const float2* asc = reinterpret_cast<const float2*>(act + 2 * I_pad);
      for (int st = 0; st < n_dst && ok; ++st) {
        if (st > 0 && !ptx::mbar_wait(&full[stage], phase, lim)) {
          ok = false;
          break;
        }
        const int kb = st * kFzDnSb + sb;
        if (kb < a.nbi) {
          const uint8_t* b0 = ring + stage * stage_bytes + sb * dn_box + r0 * a.sbb_d;
          const uint8_t* const blk[2] = {b0, b0 + 32 * a.sbb_d};
          const uint8_t *xh = act + kb * kQK, *xl = act + I_pad + kb * kQK;
          const float2* xs = asc + kb * 8;
          switch (a.qd) {   // uniform across the CTA
            case kQ5_K: q_chunk_rows<kQ5_K, 2>(blk, c, xh, xl, xs, acc); break;
            case kQ6_K: q_chunk_rows<kQ6_K, 2>(blk, c, xh, xl, xs, acc); break;
            case kQ8_0: q_chunk_rows<kQ8_0, 2>(blk, c, xh, xl, xs, acc); break;
            case kMXFP4: q_chunk_rows<kMXFP4, 2>(blk, c, xh, xl, xs, acc); break;
            default: q_chunk_rows<kQ4_K, 2>(blk, c, xh, xl, xs, acc); break;
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[stage]);
        next_stage();
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&aempty[aslot]);
      if (++aslot == 2) {
        aslot = 0;
        aphase ^= 1u;
      }
      if (!ok) fail(kErrFzConsumer);
      float* sp = s_part + buf * (kFzWarps * kFzDnRows);
      sp[warp * kFzDnRows + r0] = acc[0];
      sp[warp * kFzDnRows + r0 + 32] = acc[1];
      cbar();                          // every warp, every unit: the partials are complete
      if (s_flag[0]) return;
      if (warp < 2) {
        // the 16 parts of each row, in a fixed order, to y_j; then one thread
        // publishes the unit (release: cumulative over the two warps' stores)
        const int r = warp * 32 + lane;
        float yv = sp[r];
#pragma unroll
        for (int p = 1; p < kFzWarps; ++p) yv += sp[p * kFzDnRows + r];
        a.y[(size_t)j * H + rt * kFzDnRows + r] = yv;
        ptx::named_barrier_sync(2, 64);
        if (tid == 0) ptx::red_add_release_gpu(sync + kSyncDone + (int)(s_epoch & 1u), 1u);
      }
      buf ^= 1;
    }

    // (5) combine: out = sum over the picks this rank owns (all of them
    // without expert parallelism) of w_j y_j, then the shared experts, in
    // that fixed order; CTA c takes outputs c*512 .. c*512+511, + grid*512, ...
    if (tid == 0) {
      const uint32_t want = (uint32_t)(s_flag[3] * dn_tiles);
      if (!spin_until_ge(sync + kSyncDone + (int)(s_epoch & 1u), want, lim)) fail(kErrFzReady);
    }
    cbar();
    if (s_flag[0]) return;
    for (int o = blockIdx.x * kFzConsumers + tid; o < H; o += gridDim.x * kFzConsumers) {
      float acc2 = 0.f;
      for (int q = 0; q < k; ++q)
        if (ep_owned(s_ids[q], a.ep_rank, a.ep_world)) acc2 = fmaf(s_w[q], __ldcg(a.y + (size_t)q * H + o), acc2);
      for (int q = k; q < kS; ++q)
        if (ep_owned(E + (q - k), a.ep_rank, a.ep_world)) acc2 += __ldcg(a.y + (size_t)q * H + o);
      if (a.partial)
        a.partial[o] = acc2;
      else
        a.out[o] = __float2bfloat16_rn(acc2);
    }
  }
  ptx::pdl_launch_dependents();
}

}  // namespace

size_t decode1_fused_smem(int H, size_t act_slot_bytes, int ring_bytes) {
  return 1024 + FzLayout(H, act_slot_bytes, ring_bytes).total;
}

cudaError_t launch_decode1_fused(const FusedArgs& a, int n_sm, cudaStream_t st) {
  static uint64_t attr_done[2] = {0, 0};
  const size_t smem = decode1_fused_smem(a.H, a.act_slot_bytes, a.stages * a.stage_bytes);
  if (smem > kMaxDecodeSmem || a.T != 1 || a.k + a.S > 40 || a.H % kFzDnRows || a.H > 16384 || a.E > 1024 ||
      a.stages < 2 || a.stages > kFzStages || a.stage_bytes < 256 * std::max(a.sbb_gu, a.sbb_d))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  const bool small_e = a.E <= 256;
  auto kern = small_e ? decode1_fused_kernel<8> : decode1_fused_kernel<32>;
  uint64_t& done = attr_done[small_e ? 0 : 1];
  if (!(done & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDecodeSmem);
    if (e != cudaSuccess) return e;
    done |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(kFzThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace moe
