/*
 * moe.h -- C ABI of libmoe.so: the routed mixture-of-experts FFN layer on B200.
 *
 * The layer (LayerStoRm README, "TL;DR"): each token activates only a few of
 * the layer's experts, picked by a router; the full expert set lives in pinned
 * host RAM and the GPU's memory is a cache in front of it, with the activated
 * experts streamed in and overlapped with compute.  Weights are GGUF Q4_K
 * ("Get a model": UD-Q4_K_XL GGUF weights); the architecture is the
 * DeepSeek-V3 MoE ("References"): routed experts plus always-on shared experts.
 *
 * One forward computes, for every token t of x[T,H]:
 *   l[e]   = sum_h x[t,h] * Wr[e,h] + b[e]                       router logits
 *   S_t    = the top_k largest l[e] (ties to the lower index)      top-k routing
 *   w_j    = softmax(l[S_t])_j             (MOE_GATE_SOFTMAX_TOPK)
 *          = sig(l_j) / sum sig(l[S_t])    (MOE_GATE_SIGMOID_RENORM)
 *   y_e    = W_d,e ( silu(W_g,e x) * (W_u,e x) )                  SwiGLU expert
 *   out[t] = bf16_rne( sum_j w_j y_(S_t[j]) + sum_s y_(shared s) ) combine
 * The combine runs in a fixed order with no atomics, so results are identical
 * run to run (the pages' "Notes": a deterministic expert-parallel combine).
 *
 * Conventions for every call:
 *  - Every call returns a moe_status and never aborts.  On failure
 *    moe_last_error() returns a message (thread-local, valid until the next
 *    call on that thread).  A CUDA error maps to MOE_ERR_CUDA.
 *  - "device pointer" means memory of the GPU that was current when the layer
 *    was created; calls must be made with that GPU current.  "host pointer"
 *    means CPU memory.  A `stream` argument is a cudaStream_t passed as void*
 *    (NULL = the legacy default stream).
 *  - Calls on one layer are not thread-safe; calls on different layers are.
 *
 * Q4_K weight layout (public GGUF k-quant format): a matrix of R rows and C
 * input columns is R rows of ceil(C/256) consecutive 144-byte super-blocks.
 * A super-block holds 256 weights: fp16 d, fp16 dmin, 12 bytes packing eight
 * 6-bit scales and mins, and 128 bytes of 4-bit quants; weight = d*sc*q - dmin*m.
 * When C is not a multiple of 256 the last block of each row is padded; the
 * padded weights are read but multiply zeros and never contribute.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_layer* moe_layer_t; /* opaque, owned by the library */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,     /* bad shape, null pointer, wrong memory kind */
  MOE_ERR_UNSUPPORTED = -2,     /* a quant type or size this build cannot run */
  MOE_ERR_OOM = -3,             /* device or pinned allocation failed */
  MOE_ERR_CUDA = -4,            /* a CUDA runtime call failed */
  MOE_ERR_CACHE_TOO_SMALL = -5, /* one call needs more experts than cache slots */
  MOE_ERR_NOT_READY = -6        /* router or experts not set yet */
} moe_status;

/* GGUF block types (GGML type ids).  Q4_K runs every path; the others run
 * each token through the single-token kernel (see moe_layer_create_mixed). */
typedef enum {
  MOE_Q8_0 = 8,   /* 32 weights: fp16 scale, 32 signed bytes */
  MOE_Q4_K = 12,  /* 256 weights: fp16 d, dmin, 6-bit scales/mins, 4-bit quants */
  MOE_Q5_K = 13,  /* as Q4_K with a fifth quant bit */
  MOE_Q6_K = 14,  /* 256 weights: 6-bit quants, 16 signed 8-bit scales, fp16 d */
  MOE_MXFP4 = 39  /* 32 weights: E8M0 power-of-two scale, FP4 E2M1 values */
} moe_quant;

typedef enum {
  MOE_GATE_SOFTMAX_TOPK = 0,  /* softmax over the top_k selected logits */
  MOE_GATE_SIGMOID_RENORM = 1 /* sigmoid of the selected logits, renormalised to 1 */
} moe_gating;

typedef struct {
  uint64_t forwards;        /* moe_forward* calls that launched work */
  uint64_t tokens;          /* sum of T over those calls */
  uint64_t decode_calls;    /* calls that took the decode path (T <= 4) */
  uint64_t prefill_calls;   /* calls that took the prefill path (T > 4) */
  uint64_t cache_hits;      /* streamed experts found in the cache */
  uint64_t cache_misses;    /* streamed experts fetched on demand */
  uint64_t prefetches;      /* experts fetched by moe_prefetch */
  uint64_t evictions;       /* cache slots reused for another expert */
  uint64_t h2d_bytes;       /* bytes copied host -> device into the cache */
  uint64_t cache_slots;     /* slots of the streaming cache (0: none) */
  uint64_t slot_bytes;      /* bytes per cache slot */
  uint64_t launches;        /* kernels launched by the library */
} moe_stats;

/* Per-kernel device time of profiled forwards, summed (milliseconds, from CUDA
 * events recorded on the forward's stream right before and after each kernel). */
enum {
  MOE_K_ROUTER = 0,  /* router logits */
  MOE_K_TOPK = 1,    /* top-k + gating */
  MOE_K_PERMUTE = 2, /* counting-sort permutation */
  MOE_K_GATE_UP = 3, /* gate/up projections + SwiGLU */
  MOE_K_DOWN = 4,    /* down projection */
  MOE_K_COMBINE = 5, /* weighted combine */
  MOE_K_PREP = 6,    /* prefill only: activation rows and SwiGLU output to scaled fp16 */
  MOE_K_SMALL = 7,   /* prefill only: decode kernels for experts with <= 4 rows (few-row tiles off) */
  MOE_K_FORWARD = 8, /* whole forward, first kernel start to last kernel end */
  MOE_K_FUSED = 9,   /* decode of one token as one kernel (router through combine) */
  MOE_K_FEW_GATE_UP = 10, /* prefill only: gate/up + SwiGLU of the few-row tiles (moe_set_few_row_tiles) */
  MOE_K_FEW_DOWN = 11,    /* prefill only: down projection of the few-row tiles */
  MOE_K_COUNT = 12
};
typedef struct {
  uint64_t forwards;             /* forwards profiled */
  double ms[MOE_K_COUNT];        /* summed device time per MOE_K_* */
  uint64_t launches[MOE_K_COUNT];/* launches per MOE_K_* */
} moe_profile;

/* Bytes one expert (gate + up + down, all of type `quant`) occupies in device
 * memory, i.e. one cache slot: its GGUF bytes, except that Q6_K blocks are
 * padded from 210 to 224 bytes and MXFP4 blocks grouped eight at a time from
 * 136 into 144 bytes (16-byte aligned groups for the copy engines), and each
 * matrix's rows are padded with zero rows to a multiple of 64 (the device
 * layout is tile-major: 64-row tiles, stored group after group).  0 on bad
 * args.  Source: LayerStoRm README, "Get a model" (GGUF weights). */
size_t moe_expert_bytes(int hidden, int inter, moe_quant quant);

/* Create a layer on the current GPU.
 * hidden: H, multiple of 256, <= 16384.  inter: I, >= 1, <= 16384 (any value;
 * the down rows are padded to whole super-blocks).  n_experts: E, 1..1024.
 * top_k: 1..min(32, E).  n_shared: S, 0..8 always-on experts (weight 1).
 * quant must be MOE_Q4_K.  *out receives the handle.
 * Errors: INVALID_ARG (shape out of range, out == NULL), UNSUPPORTED (quant),
 * CUDA/OOM (small device allocations).
 * Source: LayerStoRm README, "References" (DeepSeek-V3 MoE: routed experts,
 * top-k routing, always-on shared experts) and "Get a model" (Q4_K). */
moe_status moe_layer_create(int hidden, int inter, int n_experts, int top_k,
                            int n_shared, moe_quant quant, moe_layer_t* out);

/* Create a layer whose gate and up weights are of one GGUF block type and
 * down weights of another, as in UD-Q*_K_XL files that mix block types per
 * tensor.  moe_layer_create(..., q, out) equals this with q for both.  A
 * layer with both types Q4_K takes every path of moe_forward; any other
 * layer runs each token through the single-token kernel (one launch per
 * token, in order, on the forward's stream), so its throughput at T tokens is
 * T times the single-token time.  Types Q8_0 and MXFP4 for the down weights
 * need inter to be a multiple of 256.  The host pointers of moe_set_experts
 * hold GGUF rows of these types (rows of ceil(cols / block) blocks).
 * Errors: as moe_layer_create; UNSUPPORTED for another type.
 * Source: LayerStoRm README, "Get a model" (UD-Q4_K_XL GGUF files) and
 * "License and attributions" (GGUF and MXFP4 decode paths). */
moe_status moe_layer_create_mixed(int hidden, int inter, int n_experts, int top_k, int n_shared,
                                  moe_quant quant_gate_up, moe_quant quant_down, moe_layer_t* out);

/* Destroy a layer: waits for the layer's outstanding work (its last forward
 * and its internal copy stream), frees its device memory (cudaFree itself may
 * wait for the GPU) and drops its experts from the shared cache.  NULL is a
 * no-op.  No counterpart on the pages (resource management). */
moe_status moe_layer_destroy(moe_layer_t layer);

/* Router weights: W fp32 [E, H] row-major and bias fp32 [E] (NULL = zero),
 * host or device pointers; both are copied, so the caller keeps ownership.
 * The bias is added to the logits and used for both selection and weights.
 * Source: LayerStoRm README, "TL;DR" (the router picks each token's few
 * experts); the gating functions are the plainest readings of the pages'
 * DeepSeek-V3 reference ("References"). */
moe_status moe_set_router(moe_layer_t layer, const float* W, const float* bias,
                          moe_gating gating);

/* Expert weights: three arrays of E+S host pointers (routed experts 0..E-1,
 * then the shared ones), each to one Q4_K matrix: gate [I, H], up [I, H],
 * down [H, I].  The memory must be pinned (cudaHostAlloc/cudaHostRegister) and
 * stay valid and unchanged until the layer is destroyed: it is borrowed, not
 * copied, and cache misses are copied from it later.  In resident mode (see
 * moe_set_cache_bytes) every expert is uploaded to device memory here, and the
 * call returns when the upload is done.
 * The call also scans every weight row's block scales once (host threads) to
 * choose the power-of-two scale of the prefill path's fp16 dequantisation.
 * Errors: INVALID_ARG (NULL entry or a pointer that is not pinned host memory),
 * OOM (resident copy does not fit).
 * Source: LayerStoRm README, "TL;DR" and "Requirements" (the whole expert set
 * pinned in host RAM, the GPU holding what is needed). */
moe_status moe_set_experts(moe_layer_t layer, const void* const* gate,
                           const void* const* up, const void* const* down);

/* Device memory budget for experts, shared by every layer on this GPU.
 * SIZE_MAX (the default) = resident mode: each layer keeps all its experts in
 * device memory, forwards never wait on the host and can be captured in a CUDA
 * graph.  Any other value = streaming mode for layers registered afterwards:
 * floor(bytes / slot_bytes) slots form an LRU cache in front of pinned host
 * RAM; misses are copied with cudaMemcpyAsync on an internal copy-engine
 * stream and compute waits on per-slot events.  Changing the budget empties
 * the streaming cache (it waits for the GPU first).
 * Source: LayerStoRm README, "TL;DR" (GPU memory as a cache of experts,
 * streamed in and overlapped with compute); rebasdaily LayerStoRm explainer
 * (the host link as the final bottleneck). */
moe_status moe_set_cache_bytes(size_t bytes);

typedef enum {
  MOE_CACHE_LRU = 0, /* evict the least recently used expert (default) */
  MOE_CACHE_LFU = 1  /* evict the least frequently used expert, least recent among equals */
} moe_cache_policy;

/* Replacement policy of the streaming cache (process-wide; takes effect at
 * the next miss, keeps the cached experts).  MOE_CACHE_LFU counts, for every
 * (layer, expert) seen, its arrivals: forwards of its layer that used it when
 * the layer's previous forward did not (prefetches excluded), halving all
 * counts after every 64 x slots arrivals so that popularity ages.  A miss
 * takes an empty slot if there is one, else evicts, preferably among experts
 * neither prefetched (moe_prefetch) for their layer's next forward nor used by
 * their layer's previous forward, the one with the fewest arrivals (the least
 * recently used among equals).  An expert a layer keeps
 * using stays; among the rest the popular ones stay where LRU would let
 * one-off experts push them out.
 * Errors: INVALID_ARG for an unknown policy.
 * Source: glm-flash-lite project page, "How it works" (experts kept in tiers
 * ranked by how often they are used); LayerStoRm README, "Status and
 * limitations" (cache and prefetch policy as active work). */
moe_status moe_set_cache_policy(int policy);

/* Prefill path (T > 4), process-wide, read at each forward: an expert with at
 * most max_rows rows, and the last partial 256-row tile of a larger expert
 * when it has at most max_rows rows, runs on the few-row kernel (warp-level
 * fp16 MMAs, Q4_K dequantised in registers: one pass over the weights at the
 * HBM rate, whatever the row count) instead of the tensor-memory GEMM, whose
 * cost per tile is its dequantisation of all 256 weight rows of every feature
 * block, whatever the row count.  Both compute the same fp16 products with
 * fp32 accumulation; the rounding order differs.  0 = off: all tiles on the
 * GEMM and experts with <= 4 rows on the decode kernels.
 * With T <= max_rows every expert is a single few-row tile and the GEMM
 * kernels are not launched.
 * Up to 32 rows the kernel keeps 4 stages in flight, above 3.  -1 (the
 * default) = 64 for batches of at most 256 tokens, 32 above (measured: at
 * T = 64, 0.55 ms with 64 against 0.58 with 32; at T = 4096, 5.6 ms with 32
 * against 5.9 with 64).  Errors: INVALID_ARG outside -1..64.
 * Source: LayerStoRm README, "Notes" (decode and prefill throughput measured
 * on the boot-verified configuration: both paths are the product). */
moe_status moe_set_few_row_tiles(int max_rows);

/* Forward: x bf16 [T, H] and out bf16 [T, H], device pointers, row-major.
 * T >= 0 (T = 0 returns at once).  T <= 4 takes the decode path (fused router,
 * expert kernels straight from the Q4_K bytes: byte dot products for T = 1,
 * the integer tensor MMA for 2..4), larger T the prefill path (router and the
 * projections of experts with more than 4 rows as tcgen05 grouped GEMMs; the
 * Q4_K weights are dequantised to fp16 in shared memory under a power-of-two
 * scale per weight row that moe_set_experts derives from the row's blocks, so
 * any finite Q4_K block is in range; experts with at most 4 rows take the
 * decode kernels).  Work is enqueued on `stream`; in resident mode the call does not
 * wait for the GPU, except that the first forward at a T larger than any
 * before on this layer allocates its per-call scratch, waiting for the
 * layer's previous forward first.  On the decode path the first kernel is launched as a
 * programmatic dependent of the stream's previous work: it waits for that
 * work before it reads x or writes anything.
 * In streaming mode the call reads the routing back to the host (one stream
 * synchronisation) to resolve cache misses before the expert kernels are
 * launched.  out must not overlap x.
 * Source: LayerStoRm README, "TL;DR" (router, activated experts, combine) and
 * "Notes" (a deterministic expert combine). */
moe_status moe_forward(moe_layer_t layer, const void* x, void* out, int T, void* stream);

/* Forward with the routing given: forced_ids int32 [T, top_k] on the HOST
 * (validated: every id in 0..E-1).  The gate weights are the gating function
 * of the router logits at these ids.  In streaming mode no synchronisation is
 * needed: the cache is resolved from the host ids before anything launches.
 * No counterpart on the pages: a test and benchmark hook that replays a
 * routing trace. */
moe_status moe_forward_routed(moe_layer_t layer, const void* x, void* out, int T,
                              const int32_t* forced_ids, void* stream);

/* Forward on HOST buffers: x (host, bf16 [T, H]) in, moe_forward, out (host,
 * bf16 [T, H]) back, all on `stream`; returns once the work is enqueued
 * (synchronise the stream before reading out).  With T <= 4 and pinned
 * buffers (16-byte aligned) the kernels read x and write out in host memory
 * in place; otherwise x and out are copied through device buffers (pinned
 * buffers make those copies asynchronous).  No counterpart on the pages: the
 * end-to-end entry for callers that hold activations in host memory. */
moe_status moe_forward_host(moe_layer_t layer, const void* x_host, void* out_host,
                            int T, void* stream);

/* Routing of the last forward: ids int32 [T, top_k] and weights fp32
 * [T, top_k] (either may be NULL), copied on `stream` to device or host
 * memory.  ids[t] are ordered by decreasing logit.  No counterpart on the
 * pages (inspection). */
moe_status moe_get_routing(moe_layer_t layer, int32_t* ids, float* weights, void* stream);

/* Router logits of the last forward, fp32 [T, E], copied on `stream`.  No
 * counterpart on the pages (inspection). */
moe_status moe_get_logits(moe_layer_t layer, float* logits, void* stream);

/* Streaming mode: start fetching the given experts (host array of n ids in
 * 0..E+S-1) into the cache now, on the copy stream, so a later forward finds
 * them ready.  A no-op for resident layers and for experts already cached.
 * Source: LayerStoRm README, "Status and limitations" (predictive prefetch)
 * and "References" (PreScope, SP-MoE: prefetching the next layer's experts). */
moe_status moe_prefetch(moe_layer_t layer, const int32_t* ids, int n);

/* Wait for the layer's own outstanding work (its last forward, on whatever
 * stream it ran, and its internal copy stream; other work on the GPU is not
 * waited for), then report whether one of the layer's kernels gave up on a
 * bounded wait (a shared-memory pipeline barrier that did not complete
 * within its time limit; the kernel then stops early and its output is
 * invalid).  Returns MOE_ERR_CUDA with a message in that case and clears the
 * record; MOE_OK otherwise.  No counterpart on the pages (failure detection). */
moe_status moe_check(moe_layer_t layer);

/* Counters of all layers (moe_stats), process-wide; reset keeps the cache
 * geometry.  No counterpart on the pages (metrics). */
moe_status moe_get_stats(moe_stats* out);
moe_status moe_reset_stats(void);

/* Profiling (global, off by default): when on, every forward records CUDA
 * events around each of its kernels.  moe_get_profile waits for the recorded
 * events, adds their times into *out and forgets them; moe_reset_profile
 * drops recorded events without waiting.  No counterpart on the pages
 * (tracing). */
moe_status moe_set_profiling(int enable);
moe_status moe_get_profile(moe_profile* out);
moe_status moe_reset_profile(void);

/* Router step only (logits, top-k, gating), for callers that cannot allocate
 * device memory: their device memory belongs to another allocator (a
 * framework's caching allocator or an arena reserved at start-up), or they run
 * on a latency-critical path that cannot take cudaMalloc's implicit
 * synchronisation, so they cannot create a moe_layer.  The pages have no
 * counterpart to this call.
 * x bf16 [T, H] (16-byte aligned), W fp32 [E, H] (16-byte aligned), bias fp32
 * [E] or NULL: device pointers.  ids int32 [T, top_k] and weights fp32
 * [T, top_k]: device outputs, same meaning as in moe_get_routing.  bias, ids
 * and weights must be 4-byte aligned.  A misaligned pointer is rejected with
 * MOE_ERR_INVALID_ARG before anything is launched.  Work is enqueued on
 * `stream`.
 * Allocates nothing: the [T, E] logits scratch is a fixed array inside the
 * library of 65536 floats (256 KiB, held on every GPU that loads the library
 * until the process exits), so T * E must be <= 65536 (MOE_ERR_UNSUPPORTED
 * otherwise).  The first call on a GPU looks up the array's device address
 * and caches it with the current context; a call in a new context (after
 * cudaDeviceReset) looks it up again.  Make the first call on each GPU, and
 * the first after a reset, outside stream capture: inside capture it returns
 * MOE_ERR_NOT_READY.  All calls on a GPU share the array and it keeps the last
 * call's contents: calls whose kernels may overlap on the GPU (different
 * streams without ordering) race on it.  H: multiple of 256; E <= 1024;
 * top_k <= min(32, E). */
moe_status moe_route_noalloc(const void* x, const float* W, const float* bias, int T, int H, int E,
                             int top_k, moe_gating gating, int32_t* ids, float* weights,
                             void* stream);

/* Expert parallelism (LayerStoRm README, "Notes": experts split across GPUs,
 * with a deterministic expert-parallel combine).  Expert e of the layer
 * (shared experts numbered E..E+S-1) belongs to rank e % world; after this
 * call the layer fetches, caches and computes only its own experts.  Every
 * rank runs the whole router.  world = 1 (the default) owns everything.
 * Errors: INVALID_ARG unless 0 <= rank < world <= 1024. */
moe_status moe_set_expert_parallel(moe_layer_t layer, int rank, int world);

/* The layer's share of a forward: partial fp32 [T, H] (device, 16-byte
 * aligned) = for every token, the sum over the token's experts that this rank
 * owns, in the fixed combine order (weighted routed experts j = 0..k-1, then
 * the shared ones), not rounded.  A token with none of this rank's experts
 * gets zeros.  Otherwise as moe_forward. */
moe_status moe_forward_partial(moe_layer_t layer, const void* x, float* partial, int T, void* stream);

/* out bf16 [T, H] = bf16_rne(sum over r = 0..world-1, in rank order, of
 * partials[r]), with partials fp32 [world][T][H] (device): the ranks'
 * moe_forward_partial results gathered in rank order (an all-gather of T*H*4
 * bytes per rank).  The same bits on every rank and every run. */
moe_status moe_combine_partials(const float* partials, void* out, int T, int H, int world, void* stream);

/* Test hooks for failure detection (process-wide, off by default), read by
 * the single-token kernel at each launch.  wait_limit_ns: limit of its bounded
 * waits (0 = the default 2 s); the final wait for its own copies in flight
 * keeps the default.  hold_barrier > 0: its wait for the router's logits
 * (the one point where every CTA waits for all the others) looks for the
 * logits of a launch that many launches ahead, so the wait runs out and the
 * kernel returns with an error that moe_check reports (which also resets the
 * kernel's step counters, so the next forward runs normally).  No GPU fault is
 * involved: the kernel's CTAs give up and exit.  No counterpart on the pages
 * (failure detection). */
moe_status moe_set_test_hooks(uint64_t wait_limit_ns, int hold_barrier);

/* Message of the last failed call on this thread ("" if none). */
const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
