// Internal declarations shared by the host runtime and the kernel files of
// libmoe.so.  Nothing here is part of the C ABI (include/moe.h).
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace moe {

// GGUF block types (GGML type ids)
constexpr int kQ8_0 = 8, kQ4_K = 12, kQ5_K = 13, kQ6_K = 14, kMXFP4 = 39;
// Device bytes of one group of 256 weights of type q, as the kernels read
// them: the GGUF bytes, except that Q6_K blocks (210 bytes) are padded to 224
// and MXFP4 blocks (17 bytes, 32 weights) are grouped eight at a time into
// 144, so that every group starts on a 16-byte boundary.  0: not supported.
__host__ __device__ constexpr int dev_sb_bytes(int q) {
  return q == kQ4_K ? 144 : q == kQ5_K ? 176 : q == kQ6_K ? 224 : q == kQ8_0 ? 272 : q == kMXFP4 ? 144 : 0;
}
// Host (GGUF) block geometry: weights and bytes per block.
constexpr int host_block_elems(int q) { return q == kQ8_0 || q == kMXFP4 ? 32 : 256; }
constexpr int host_block_bytes(int q) {
  return q == kQ4_K ? 144 : q == kQ5_K ? 176 : q == kQ6_K ? 210 : q == kQ8_0 ? 34 : q == kMXFP4 ? 17 : 0;
}

constexpr int kQK = 256;        // weights per Q4_K super-block
constexpr int kQBytes = 144;    // bytes per Q4_K super-block
constexpr int kD1MaxTok = 4;    // experts with <= this many rows use the per-sub-block decode kernels
constexpr int kTileRows = 64;   // weight rows per decode work unit

// Pointers to one layer's per-call scratch (device memory owned by the layer).
struct Work {
  float* logits;      // [T, E]
  int* ids;           // [T, k]
  float* w;           // [T, k]
  int* forced;        // [T, k] forced ids staged for moe_forward_routed
  int* counts;        // [E+S]
  int* offsets;       // [E+S+1]
  int* perm;          // [P] row r of the expert-sorted order -> pair t*(k+S)+j
  int* inv;           // [P] pair -> row r
  int* act;           // [E+S] experts with at least one row, ascending
  int* n_act;         // [1]
  unsigned* ticket;   // [1] last-block-done counter of the permutation kernel
  float* h;           // [P, I_pad] SwiGLU activations, padded columns are zero
  float* y;           // [P, H] expert outputs
  // decode path: activations as 16-bit fixed point per 32-element run,
  // x = (256*hi + lo) * 2^-s, in two byte planes (hi s8, then lo u8), with
  // (2^-s, sum of the represented values) per run
  int8_t* xq;         // [2][T_cap, H]
  size_t xq_plane;    // T_cap * H
  float2* xsc;        // [T, H/32]
  int8_t* hq;         // [2][P_cap, I_pad] SwiGLU output
  size_t hq_plane;    // P_cap * I_pad
  float2* hsc;        // [P, I_pad/32]
  int* act1;          // experts with 1..kD1MaxTok rows
  int* n_act1;
  int* act2;          // experts with more rows
  int* n_act2;
  unsigned* err;      // device-side error flags (timeouts)
  // prefill path (tensor-core GEMMs)
  int4* tiles;        // [max tiles] (expert, n0, count, r0): up to 256 rows of one expert
  int* n_tiles;
  int4* mtiles;       // [E+S] few-row tiles (expert, n0, count <= kMtMaxRows, r0)
  int* n_mtiles;
  unsigned* mt_next;  // [2] unit counters of the few-row kernels (gate/up, down)
  __half* x16;        // [P_cap, H] activations of each row, fp16 scaled by 1/rinv, K order (0,2,1,3)
  float* rinv;        // [P]
  __half* h16;        // [P_cap, I_pad] SwiGLU output, fp16 scaled by 1/hinv, same K order
  float* hinv;        // [P]
  float* rpart;       // router partial logits [splits][T][E]
  unsigned* sync;     // [kSyncWords] launch counter, step counters and tagged logits of the one-token kernel
};
constexpr int kSyncWords = 2304;   // counters, then 1024 tagged 64-bit logits

struct RouteArgs {
  const __nv_bfloat16* x;
  const float* W;
  const float* b;
  const int* forced;   // device [T, k] or null
  int T, H, E, k, S, gating;
  float* logits;
  int *ids;
  float* w;
  int *counts, *offsets, *perm, *inv;
  int *act1, *n_act1, *act2, *n_act2, *n_act;
  int8_t* xq;
  size_t xq_plane;
  float2* xsc;
  unsigned* ticket;
  int ep_rank, ep_world;  // expert parallelism: only experts e % ep_world == ep_rank get work
};
cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st);

// Expert parallelism: expert e (shared experts numbered E..E+S-1) belongs to
// rank e % world.  With world <= 1 every expert is owned.
__host__ __device__ inline bool ep_owned(int e, int rank, int world) { return world <= 1 || e % world == rank; }
// Copy `bytes` (a multiple of 16, both addresses 16-byte aligned) from mapped
// host memory `src` (its device address) to device memory `dst`; the next
// kernel may be launched as its programmatic dependent.
cudaError_t launch_stage_in(const void* src, void* dst, size_t bytes, cudaStream_t st);

// Arguments of the decode expert kernels.
struct DecodeArgs {
  const CUtensorMap* tmaps;  // [slots][kMapsPerSlot] maps of gate, up, down (4-D, 8-byte elements)
  const int* slot_of;        // [E+S] expert -> slot
  const int* act;            // experts this kernel handles
  const int* n_act;
  const int *counts, *offsets, *perm, *inv;
  const float* w;
  int kS, T, k, S;
  int H, I, I_pad, nbh, nbi;
  const int8_t* xq;
  size_t xq_plane;
  const float2* xsc;
  int8_t* hq;
  size_t hq_plane;
  float2* hsc;
  float* y;
  __nv_bfloat16* out;
  unsigned* err;
  int stage_x;            // gate/up: copy x (all T tokens) to shared memory once per CTA
  size_t act_slot_bytes;  // down: bytes of one activation slot (2 * max_tok * I_pad + scales)
  int n_ex, n_slots, n_rows;  // bounds of expert ids (E+S), cache slots, rows (T(k+S)); debug builds
};
constexpr size_t kMaxDecodeSmem = 227 * 1024;
// max_tok: 1 (every expert has one row, T == 1) or kD1MaxTok
cudaError_t launch_gate_up_d1(const DecodeArgs& a, int max_tok, int n_sm, cudaStream_t st);
cudaError_t launch_down_d1(const DecodeArgs& a, int max_tok, int n_sm, cudaStream_t st);
size_t gate_up_d1_smem(int max_tok, size_t x_stage_bytes);
size_t down_d1_smem(int max_tok, size_t act_slot_bytes);
// T = 1: GEMV kernels on byte dot products (128-row units); act_slot_bytes of
// one token's h (2 * I_pad + I_pad / 32 * 8)
cudaError_t launch_gemv_gate_up(const DecodeArgs& a, int n_sm, cudaStream_t st);
cudaError_t launch_gemv_down(const DecodeArgs& a, int n_sm, cudaStream_t st);
size_t gemv_gate_up_smem(int H);
size_t gemv_down_smem(size_t act_slot_bytes);

// T = 1 as one persistent kernel: router, top-k, gate/up + SwiGLU, down and
// combine (one CTA per SM; steps meet through counters in `sync`).
struct FusedArgs {
  const uint8_t* warena;     // expert images (tile-major gate, up, down), slot s at warena + s * wstride
  size_t wstride, gate_bytes;  // bytes from one slot to the next; of one gate (= up) matrix
  const int* slot_of;        // [E+S] expert -> slot
  const __nv_bfloat16* x;    // [H]
  const float* W;            // router [E, H]
  const float* b;            // router bias [E] or null
  const int* forced;         // device [k] or null
  int T, H, I, I_pad, E, k, S, nbh, nbi, gating;
  float* logits;             // [E]
  int* ids;                  // [k]
  float* w;                  // [k]
  int8_t* hq;                // h of expert j (j = 0..k+S-1) at row j: [2][rows][I_pad]
  size_t hq_plane;
  float2* hsc;               // [rows][I_pad / 32]
  float* y;                  // [k+S, H]
  __nv_bfloat16* out;        // [H]
  unsigned* sync;            // kSyncWords, zero before the first launch
  unsigned* err;
  size_t act_slot_bytes;     // 2 * I_pad + I_pad / 32 * 8
  int early;                 // weights and slot table constant: stream them before the predecessor ends
  uint64_t wait_ns;          // limit of the bounded waits (0: the default 2 s); test hook
  int hold;                  // > 0: the grid barrier waits for that many arrivals more (test hook)
  int n_slots;               // bound of cache slots (debug builds)
  int qgu, qd;               // GGUF block types of gate/up and of down
  int sbb_gu, sbb_d;         // their device bytes per 256-weight group
  int stages, stage_bytes;   // weight ring: stages x (256 x the larger group size)
  int ep_rank, ep_world;     // expert parallelism: work only for owned experts
  float* partial;            // non-null: write the owned experts' unrounded sum here instead of out
};
size_t decode1_fused_smem(int H, size_t act_slot_bytes, int ring_bytes);
constexpr int kFusedMaxStages = 5;
// Weight-ring geometry of the single-token kernel for these group sizes: as
// many stages (2 .. kFusedMaxStages, at most 180 KB) as fit in shared memory
// beside the kernel's other arrays for this H and activation slot size.
inline void decode1_ring(int sbb_gu, int sbb_d, int H, size_t act_slot_bytes, int* stages, int* stage_bytes) {
  *stage_bytes = 256 * std::max(sbb_gu, sbb_d);
  int n = std::max(2, std::min(kFusedMaxStages, 184320 / *stage_bytes));
  while (n > 2 && decode1_fused_smem(H, act_slot_bytes, n * *stage_bytes) > kMaxDecodeSmem) --n;
  *stages = n;
}
cudaError_t launch_decode1_fused(const FusedArgs& a, int n_sm, cudaStream_t st);

// Tensor maps of one expert's matrices at `base` (tile-major), kMapsPerSlot of
// them: [0..2] gate, up, down with boxes of 64 rows x 2 (gate/up) or 4 (down)
// groups (decode kernels); [3..5] gate, up, down with boxes of 128 rows x 1
// group (single-token GEMVs, prefill GEMMs and the few-row kernel).  The
// fused single-token kernel reads the images with plain bulk copies.
constexpr int kMapsPerSlot = 6;
struct Shape;
cudaError_t encode_expert_maps(CUtensorMap* maps, const uint8_t* base, const Shape& s);
// Weight matrices live in device memory tile-major (tiles of kWTile rows; see
// tmap.cu): bytes of a matrix of `rows` rows of drow device bytes.
constexpr int kWTile = 64;
inline size_t tiled_matrix_bytes(int rows, size_t drow) { return (size_t)((rows + kWTile - 1) / kWTile) * kWTile * drow; }
// Upload one matrix: its GGUF host rows into `staging` (row-major device
// rows, copy_matrix_h2d), then a kernel rewrites them tile-major into `dst`;
// both on `st`, so `staging` is free again once `st` has reached the next
// upload.  drow = nb * sbb.
cudaError_t upload_matrix(uint8_t* dst, const uint8_t* src, int rows, int q, size_t hrow, size_t drow, int nb,
                          int sbb, uint8_t* staging, cudaStream_t st);
// The second half of upload_matrix alone: row-major device rows in `staging`
// rewritten tile-major into `dst` on `st`.
cudaError_t launch_retile(const uint8_t* staging, uint8_t* dst, int rows, int nb, int sbb, cudaStream_t st);
// Copy one weight matrix of `rows` rows from its GGUF host bytes into the
// device layout of its type (dev_sb_bytes), asynchronously on `st`.
cudaError_t copy_matrix_h2d(uint8_t* dst, const uint8_t* src, int rows, int q, size_t hrow, size_t drow,
                            cudaStream_t st);
// 2-D map over a row-major 16-bit matrix [rows, cols] (fp16 or bf16) with
// 128B-swizzled boxes of box_rows rows x 64 columns (cols a multiple of 64).
cudaError_t encode_sw128_16(CUtensorMap* map, const void* base, bool bf16, size_t rows, int cols, int box_rows);
// box_cols 64 (128B swizzle) or 32 (64B swizzle)
cudaError_t encode_swz_16(CUtensorMap* map, const void* base, bool bf16, size_t rows, int cols, int box_rows,
                          int box_cols);
// B operands of the prefill GEMMs: boxes of 256 rows x 32 columns, 64B swizzle
inline cudaError_t encode_act16(CUtensorMap* map, const __half* base, size_t rows, int cols) {
  return encode_swz_16(map, base, false, rows, cols, 256, 32);
}

// Router logits on the tensor cores (T > 4): partial sums per K split.
struct RouterGemmArgs {
  int T, E;
  int nsplit, nk_split;     // K splits; 64-wide K steps per split
  float* part;              // [nsplit][T][E]
  size_t split_stride;      // floats between splits
  unsigned* err;
};
int router_gemm_splits(int T, int E, int H, int n_sm);
size_t router_part_floats(int T_cap, int E, int n_sm);
cudaError_t launch_split_router(const float* W, int E, int H, __nv_bfloat16* planes, cudaStream_t st);
cudaError_t launch_router_gemm(const CUtensorMap& xmap, const CUtensorMap& wmap, const RouterGemmArgs& a,
                               cudaStream_t st);

// Prefill GEMMs (tcgen05): mode 0 gate/up -> h, mode 1 down -> y.
struct GemmArgs {
  const CUtensorMap* wmaps;  // [slots][kMapsPerSlot]
  const int* slot_of;        // [E+S] expert -> slot
  const int4* tiles;
  const int* n_tiles;
  int ft;                    // feature blocks per tile: ceil(I/128) (mode 0), H/256 (mode 1)
  int nkb;                   // super-blocks along K: H/256 (mode 0), I_pad/256 (mode 1)
  const float* rinv;         // [P] inverse activation scale of each row
  float* out;                // h [P, I_pad] or y [P, H]
  int out_ld, out_rows;      // row pitch (floats); features stored (mode 0: I)
  // per expert, per weight row: the exponent k of the 2^k scale applied to
  // the dequantised fp16 weights (gate rows [0, I), up rows [I, 2I), down
  // rows [2I, 2I + H)); wexp_stride = 2I + H, wexp_down = 2I
  const int8_t* wexp;
  int wexp_stride, wexp_down;
  unsigned* err;
  int n_ex, n_slots;         // bounds of expert ids and cache slots (debug builds)
  // few-row kernel (launch_prefill_mt): its activation rows, fp16 [P, b_ld]
  // in the GEMM's K order, and its unit counter (zeroed by build_tiles)
  const __half* bsrc;
  int b_ld;
  unsigned* next;
  int n_rows;                // activation rows P (debug builds)
};
constexpr int kMtMaxRows = 64;   // most activation rows of a few-row tile (builds for 32 and 64)
// The default row limit: 64 for batches of at most kMtWideMaxT tokens (their
// experts have a few to a few dozen rows), 32 above (there the 3-stage build
// slows the many small tiles more than it gains on the 33-64-row ones).
constexpr int kMtWideMaxT = 256;
inline int default_few_rows(int T) { return T <= kMtWideMaxT ? 64 : 32; }
size_t prefill_gemm_smem();
size_t prefill_max_tiles(int n_experts_total, size_t pairs);
// GEMM tiles of up to 256 rows for the experts with more than small_rows rows
// (the others are listed in act1); with mt_rows > 0, an expert with at most
// mt_rows rows, and the last partial tile of a larger one when it has at most
// mt_rows rows, become few-row tiles (mtiles) instead.
cudaError_t launch_build_tiles(const Work& wk, int small_rows, int mt_rows, cudaStream_t st, int ep_rank = 0,
                               int ep_world = 1);
cudaError_t launch_quant_x(const __nv_bfloat16* x, const Work& wk, int T, int H, cudaStream_t st);
cudaError_t launch_gather_rows(const __nv_bfloat16* x, const Work& wk, int P, int kS, int H, cudaStream_t st);
cudaError_t launch_convert_h(const Work& wk, int P, int I, int I_pad, cudaStream_t st);
cudaError_t launch_prefill_gemm(int mode, const CUtensorMap& bmap, const GemmArgs& a, int n_sm, cudaStream_t st);
// The few-row tiles (a.tiles / a.n_tiles = the mtiles list) of mode 0 (gate/up)
// or 1 (down), same outputs as the GEMM.
cudaError_t launch_prefill_mt(int mode, const GemmArgs& a, int n_sm, cudaStream_t st, int max_rows);
size_t route_decode_smem(int H, int T, int E, int k, int S);

struct Shape {
  int H, I, E, k, S;
  int nbh;    // super-blocks per gate/up row  = H / 256
  int nbi;    // super-blocks per down row     = ceil(I / 256)
  int I_pad;  // nbi * 256
  int n_sm;   // streaming multiprocessors of the device
  int qgu, qd;            // GGUF block types of gate and up (shared), and of down
  int sbb_gu, sbb_d;      // device bytes per 256-weight group (dev_sb_bytes)
  size_t hrow_gu, hrow_d; // host (GGUF) bytes per row
  size_t drow_gu, drow_d; // device bytes per row: nbh * sbb_gu, nbi * sbb_d
};

// ---- kernels (one launch helper per kernel; all enqueue on `st`) ----------
cudaError_t launch_router_logits(const __nv_bfloat16* x, const float* W, const float* b,
                                 float* logits, int T, int H, int E, cudaStream_t st);
// Top-k + gating.  With `part` (nsplit slices of partial logits, split_stride
// floats apart) the logits are first summed in split order, the bias added and
// the result written to `logits`.
cudaError_t launch_topk(float* logits, int T, int E, int k, int gating,
                        const int* forced, int* ids, float* w, cudaStream_t st,
                        const float* part = nullptr, int nsplit = 0, size_t split_stride = 0,
                        const float* bias = nullptr);
cudaError_t launch_permute(const int* ids, int T, const Shape& s, const Work& wk, cudaStream_t st);
// Weighted combine of each token's pairs in the fixed order.  With
// `partial` (fp32 [T, H]) only the pairs whose expert this rank owns are
// summed and the sum is written unrounded there instead of to `out`.
cudaError_t launch_combine(const Work& wk, int T, const Shape& s, __nv_bfloat16* out, cudaStream_t st,
                           bool pdl = false, float* partial = nullptr, int ep_rank = 0, int ep_world = 1);
// out[t, h] = bf16_rne(sum over r = 0..world-1, in that order, of partials[r][t][h])
cudaError_t launch_combine_partials(const float* partials, __nv_bfloat16* out, int T, int H, int world,
                                    cudaStream_t st);

// Streaming cache: point experts at their cache slots (the slot_of table the
// kernels index tensor maps with).
struct SlotUpdate {
  static constexpr int kMax = 64;
  int n;
  int expert[kMax];
  int slot[kMax];
};
cudaError_t launch_set_slots(int* slot_of, const SlotUpdate& u, cudaStream_t st);

// Exponents k (<= 8) of the power-of-two weight scales of the prefill GEMMs,
// one per weight row of one Q4_K matrix of `rows` rows x `nb` super-blocks:
// the largest k with 2^k * max over the row's blocks of (|d|*945 + |dmin|*63)
// below 60000, so that no fp16 intermediate of the dequantisation overflows.
void q4k_row_exponents(const uint8_t* q4k, int rows, int nb, int8_t* out);

// Set / clear the thread-local message returned by moe_last_error().
int report_error(int status, const char* msg);
void clear_error();

// ---- device helpers -------------------------------------------------------
// Debug builds (-DMOE_DEBUG_BOUNDS, libmoe_debug.so) check every index that a
// kernel reads from memory before it addresses memory with it: an expert id,
// a cache slot, a row offset or a permutation entry.  A bad one sets
// kErrBoundsBit in the layer's error word (moe_check reports it) and is
// replaced by 0, so the access stays in bounds.  Release builds skip the check.
constexpr unsigned kErrBoundsBit = 1u << 20;
#ifdef __CUDACC__
#ifdef MOE_DEBUG_BOUNDS
__device__ __forceinline__ int in_range(int v, int n, unsigned* err) {
  if ((unsigned)v < (unsigned)n) return v;
  atomicOr(err, kErrBoundsBit);
  return 0;
}
#else
__device__ __forceinline__ int in_range(int v, int, unsigned*) { return v; }
#endif
#endif

#ifdef __CUDACC__
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// 6-bit scale and min of sub-block j from the 12 packed scale bytes
// (GGUF k-quant layout: sub-blocks 0..3 use the low 6 bits of bytes j and j+4;
// sub-blocks 4..7 take nibbles of byte j+4 plus the top 2 bits of bytes j-4 / j).
__device__ __forceinline__ void q4k_scale_min(const uint8_t* sb, int j, int& sc, int& m) {
  if (j < 4) {
    sc = sb[j] & 63;
    m = sb[j + 4] & 63;
  } else {
    sc = (sb[j + 4] & 0x0F) | ((sb[j - 4] >> 6) << 4);
    m = (sb[j + 4] >> 4) | ((sb[j] >> 6) << 4);
  }
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// Called by a full warp with one value per lane (a 32-element run): writes
// this lane's value as 16-bit fixed point x ~ (256*hi + lo) * 2^-s, with s
// chosen so the run's largest magnitude lands in [2^13, 2^14), and returns in
// run_sc (2^-s, sum of the represented values) of the run.
__device__ __forceinline__ void quant_run16(float v, int8_t& hi, uint8_t& lo, float2& run_sc) {
  float m = fabsf(v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int e = 0;
  if (m > 0.f && m < 3.0e38f) e = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;
  e = max(-100, min(100, e));
  const float scale = __uint_as_float((uint32_t)(127 + 13 - e) << 23);
  const float inv = __uint_as_float((uint32_t)(127 - 13 + e) << 23);
  const int xi = __float2int_rn(v * scale);  // |xi| <= 2^14
  hi = (int8_t)(xi >> 8);
  lo = (uint8_t)(xi & 0xFF);
  int s = xi;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  run_sc = make_float2(inv, (float)s * inv);
}

// Exclusive scan of one int per thread over a block of any size <= 1024;
// returns the prefix and writes the block total.  s_warp: 32 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int* total, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
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
    if (lane < nw) s_warp[lane] = wv;
  }
  __syncthreads();
  const int before = warp ? s_warp[warp - 1] : 0;
  *total = s_warp[nw - 1];
  __syncthreads();
  return before + incl - v;
}
#endif

}  // namespace moe
