// Host runtime of libmoe.so: the C ABI of include/moe.h.
//
// A layer owns its router weights (fp32, and as three bf16 planes for the
// tensor-core router), TMA tensor maps over every slot its experts can occupy,
// a device table expert -> slot, and per-call scratch.  Experts live either in
// a per-layer resident copy
// (cache budget SIZE_MAX) or in the device-wide streaming cache: an arena of
// fixed-size slots with a host-side LRU, filled from pinned host RAM by
// cudaMemcpyAsync on an internal copy-engine stream (LayerStoRm README,
// "TL;DR": GPU memory is a cache in front of the expert set pinned in host RAM,
// activated experts are streamed in, overlapped with compute).
//
// Ordering without host waits: a slot's `ready` event is recorded on the copy
// stream after its fill, and compute waits on it; a slot's `used` event is
// recorded on the compute stream after the kernels that read it, and a later
// fill of that slot waits on it before overwriting.
#include <algorithm>
#include <cstdarg>
#include <thread>
#include <cstdio>
#include <cstring>
#include <list>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/moe.h"
#include "moe_internal.h"

using namespace moe;

namespace {

thread_local std::string g_err;

// NVTX range for the duration of a scope: the host-side steps of a forward
// (routing read-back, cache resolution, launches) show up on a timeline
// under a profiler; without one a push/pop costs a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

moe_status fail(moe_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

// On failure the runtime's last-error record is read (and so cleared), so a
// failed launch is reported once and not again by the next call's check.
#define CUDA_TRY(call)                                                                       \
  do {                                                                                       \
    cudaError_t e_ = (call);                                                                 \
    if (e_ != cudaSuccess) {                                                                 \
      (void)cudaGetLastError();                                                              \
      return fail(e_ == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA, "%s: %s", #call, \
                  cudaGetErrorString(e_));                                                   \
    }                                                                                        \
  } while (0)

#define MOE_TRY(call)               \
  do {                              \
    moe_status s_ = (call);         \
    if (s_ != MOE_OK) return s_;    \
  } while (0)

constexpr int kMaxTokens = 32768;

std::mutex g_mu;            // guards the cache, the stats and the budget
moe_stats g_stats{};
size_t g_cache_bytes = SIZE_MAX;
int g_cache_policy = MOE_CACHE_LRU;
uint64_t g_hook_wait_ns = 0;  // moe_set_test_hooks
int g_hook_hold = 0;
int g_mt_rows = -1;   // moe_set_few_row_tiles (-1: default_few_rows(T))
uint32_t g_next_layer_id = 1;

struct Slot {
  uint64_t key = UINT64_MAX;  // (layer id << 32) | expert, UINT64_MAX = empty
  cudaEvent_t ready = nullptr;
  cudaEvent_t used = nullptr;
  bool ready_rec = false, used_rec = false;
  uint64_t epoch = 0;         // last forward that needs this slot
  std::list<int>::iterator lru;
};

struct Cache {
  int device = -1;
  size_t slot_bytes = 0;
  int n_slots = 0;
  uint8_t* arena = nullptr;
  // Uploads: the copy engine writes a matrix's host rows into staging[b] on
  // `copy` while the previous matrix is retiled from staging[b ^ 1] into its
  // slot on `retile`; events keep each buffer's two users in order.
  uint8_t* staging[2] = {nullptr, nullptr};   // slot_bytes each
  cudaStream_t retile = nullptr;
  cudaEvent_t copied[2] = {nullptr, nullptr}, retiled[2] = {nullptr, nullptr};
  bool retiled_rec[2] = {false, false};
  uint64_t uploads = 0;
  std::vector<Slot> slots;
  std::list<int> lru;  // front = most recently used
  std::unordered_map<uint64_t, int> where;
  cudaStream_t copy = nullptr;
  uint64_t epoch = 0;
  uint64_t gen = 0;  // changes whenever the arena is (re)allocated
  // MOE_CACHE_LFU bookkeeping for every (layer, expert) key seen, cached or
  // not: how often it entered use (used by a forward of its layer after not
  // being used by that layer's previous forward), and the layer's forward
  // index at its last use, and the forward a prefetch fetched it for.  Arrival
  // counts halve every kAgeEvery * n_slots arrivals, so that old popularity
  // fades.
  struct Use {
    uint32_t arrivals = 0;
    uint64_t last_fwd = 0;
    uint64_t prefetched_for = 0;
  };
  std::unordered_map<uint64_t, Use> use;
  std::unordered_map<uint32_t, uint64_t> layer_fwds;  // layer id -> forwards resolved so far
  uint64_t arrivals = 0;
};
constexpr uint64_t kAgeEvery = 64;
Cache* g_cache = nullptr;
uint64_t g_cache_gen = 0;

// Profiling: events recorded around each kernel launch of a forward, in launch
// order, each range attributed to one MOE_K_* step; resolved by moe_get_profile.
constexpr int kProfRanges = 16;              // launches per forward at most
struct ProfRec {
  int n = 0;
  int kid[kProfRanges];
  cudaEvent_t ev[2 * kProfRanges];
};
bool g_profiling = false;
std::vector<ProfRec> g_prof_pending;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void cache_free(Cache* c) {
  if (!c) return;
  for (auto& s : c->slots) {
    if (s.ready) cudaEventDestroy(s.ready);
    if (s.used) cudaEventDestroy(s.used);
  }
  if (c->arena) cudaFree(c->arena);
  for (int b = 0; b < 2; ++b) {
    if (c->staging[b]) cudaFree(c->staging[b]);
    if (c->copied[b]) cudaEventDestroy(c->copied[b]);
    if (c->retiled[b]) cudaEventDestroy(c->retiled[b]);
  }
  if (c->copy) cudaStreamDestroy(c->copy);
  if (c->retile) cudaStreamDestroy(c->retile);
  delete c;
}

}  // namespace

// Error reporting for entry points defined in other files of the library.
int moe::report_error(int status, const char* msg) {
  g_err = msg;
  return status;
}
void moe::clear_error() { g_err.clear(); }

struct moe_layer {
  uint32_t id = 0;
  int device = 0;
  Shape s{};
  size_t gate_bytes = 0, down_bytes = 0, expert_bytes = 0;  // device bytes (a cache slot: expert_bytes)
  size_t host_expert_bytes = 0;                              // GGUF bytes of one expert in host memory
  moe_gating gating = MOE_GATE_SIGMOID_RENORM;
  bool router_set = false, experts_set = false, resident = false;
  float* d_W = nullptr;
  float* d_b = nullptr;
  __nv_bfloat16* d_Wp = nullptr;        // router weight as three bf16 planes [3][E][H]
  CUtensorMap wp_map{};                 // over d_Wp, for the tensor-core router
  std::vector<const uint8_t*> host;     // (E+S)*3 borrowed pinned pointers
  uint8_t* d_resident = nullptr;        // resident copy of all experts
  int8_t* d_wexp = nullptr;             // [E+S][2I + H] prefill weight-scale exponents per weight row
  CUtensorMap* d_tmaps = nullptr;       // [slots][kMapsPerSlot] TMA maps (resident: one slot per expert)
  size_t n_tmap_slots = 0;
  const uint8_t* w_arena = nullptr;     // the images the maps cover: slot i at w_arena + i * w_stride
  size_t w_stride = 0;
  int* d_slot_of = nullptr;             // [E+S] expert -> slot of d_tmaps
  uint64_t cache_gen = 0;               // streaming: cache arena the maps point into
  cudaStream_t copy = nullptr;          // resident uploads
  int ep_rank = 0, ep_world = 1;        // expert parallelism: the experts e % ep_world == ep_rank
  // scratch
  int T_cap = 0;
  void* scratch = nullptr;
  Work wk{};
  __nv_bfloat16* xbuf = nullptr;
  __nv_bfloat16* obuf = nullptr;
  int32_t* h_ids = nullptr;             // pinned, for reading routing back
  unsigned* h_err = nullptr;            // pinned word for reading the error flags back
  cudaEvent_t done = nullptr;           // recorded on the stream at the end of every forward
  bool done_rec = false;
  int last_T = 0;
  CUtensorMap x16_map{}, h16_map{};     // B operands of the prefill GEMMs (over the scratch)
};

namespace {

moe_status check_device(const moe_layer* L) {
  int dev = -1;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev != L->device)
    return fail(MOE_ERR_INVALID_ARG, "layer lives on device %d but device %d is current", L->device, dev);
  return MOE_OK;
}

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// Wait for the layer's own outstanding work: its last forward (on whatever
// stream it ran) and its copy stream.  Other work on the device is not waited for.
moe_status wait_layer(moe_layer* L) {
  if (L->done && L->done_rec) CUDA_TRY(cudaEventSynchronize(L->done));
  if (L->copy) CUDA_TRY(cudaStreamSynchronize(L->copy));
  return MOE_OK;
}

// Grow the per-call scratch to hold T tokens (power of two, at least 64).
// The old scratch may still be read by the layer's last forward, so that is
// waited for before it is freed; the new one is zeroed on `st`, ahead of the
// forward that needs it.
moe_status ensure_scratch(moe_layer* L, int T, cudaStream_t st) {
  if (T <= L->T_cap) return MOE_OK;
  int cap = 64;
  while (cap < T) cap <<= 1;
  const Shape& s = L->s;
  const size_t P = (size_t)cap * (s.k + s.S);
  const size_t ES = (size_t)(s.E + s.S);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
  const size_t o_logits = take((size_t)cap * s.E * 4), o_ids = take((size_t)cap * s.k * 4),
               o_w = take((size_t)cap * s.k * 4), o_forced = take((size_t)cap * s.k * 4),
               o_counts = take(ES * 4), o_offsets = take((ES + 1) * 4), o_perm = take(P * 4),
               o_inv = take(P * 4), o_act = take(ES * 4), o_nact = take(4), o_ticket = take(4),
               o_h = take(P * s.I_pad * 4), o_y = take(P * s.H * 4),
               o_x = take((size_t)cap * s.H * 2), o_o = take((size_t)cap * s.H * 2),
               o_xq = take((size_t)cap * s.H * 2), o_xsc = take((size_t)cap * (s.H / 32) * 8),
               o_hq = take(P * s.I_pad * 2), o_hsc = take(P * (s.I_pad / 32) * 8), o_act1 = take(ES * 4),
               o_act2 = take(ES * 4), o_nact1 = take(4), o_nact2 = take(4),
               o_err = take(4), o_tiles = take(prefill_max_tiles((int)ES, P) * 16), o_ntiles = take(4),
               o_mtiles = take(ES * 16), o_nmtiles = take(4), o_mtnext = take(8),
               o_x16 = take(P * s.H * 2), o_rinv = take(P * 4), o_h16 = take(P * s.I_pad * 2), o_hinv = take(P * 4),
               o_rpart = take(router_part_floats(cap, s.E, s.n_sm) * 4), o_sync = take(kSyncWords * 4);
  if (L->scratch) {
    MOE_TRY(wait_layer(L));
    cudaFree(L->scratch);
    L->scratch = nullptr;
    L->T_cap = 0;
  }
  if (L->h_ids) {
    cudaFreeHost(L->h_ids);
    L->h_ids = nullptr;
  }
  CUDA_TRY(cudaMalloc(&L->scratch, off));
  CUDA_TRY(cudaMallocHost(&L->h_ids, (size_t)cap * s.k * 4));
  uint8_t* b = static_cast<uint8_t*>(L->scratch);
  L->wk.logits = reinterpret_cast<float*>(b + o_logits);
  L->wk.ids = reinterpret_cast<int*>(b + o_ids);
  L->wk.w = reinterpret_cast<float*>(b + o_w);
  L->wk.forced = reinterpret_cast<int*>(b + o_forced);
  L->wk.counts = reinterpret_cast<int*>(b + o_counts);
  L->wk.offsets = reinterpret_cast<int*>(b + o_offsets);
  L->wk.perm = reinterpret_cast<int*>(b + o_perm);
  L->wk.inv = reinterpret_cast<int*>(b + o_inv);
  L->wk.act = reinterpret_cast<int*>(b + o_act);
  L->wk.n_act = reinterpret_cast<int*>(b + o_nact);
  L->wk.ticket = reinterpret_cast<unsigned*>(b + o_ticket);
  L->wk.h = reinterpret_cast<float*>(b + o_h);
  L->wk.y = reinterpret_cast<float*>(b + o_y);
  L->xbuf = reinterpret_cast<__nv_bfloat16*>(b + o_x);
  L->obuf = reinterpret_cast<__nv_bfloat16*>(b + o_o);
  L->wk.xq = reinterpret_cast<int8_t*>(b + o_xq);
  L->wk.xq_plane = (size_t)cap * s.H;
  L->wk.xsc = reinterpret_cast<float2*>(b + o_xsc);
  L->wk.hq = reinterpret_cast<int8_t*>(b + o_hq);
  L->wk.hq_plane = P * s.I_pad;
  L->wk.hsc = reinterpret_cast<float2*>(b + o_hsc);
  L->wk.act1 = reinterpret_cast<int*>(b + o_act1);
  L->wk.act2 = reinterpret_cast<int*>(b + o_act2);
  L->wk.n_act1 = reinterpret_cast<int*>(b + o_nact1);
  L->wk.n_act2 = reinterpret_cast<int*>(b + o_nact2);
  L->wk.err = reinterpret_cast<unsigned*>(b + o_err);
  L->wk.tiles = reinterpret_cast<int4*>(b + o_tiles);
  L->wk.n_tiles = reinterpret_cast<int*>(b + o_ntiles);
  L->wk.mtiles = reinterpret_cast<int4*>(b + o_mtiles);
  L->wk.n_mtiles = reinterpret_cast<int*>(b + o_nmtiles);
  L->wk.mt_next = reinterpret_cast<unsigned*>(b + o_mtnext);
  L->wk.x16 = reinterpret_cast<__half*>(b + o_x16);
  L->wk.rinv = reinterpret_cast<float*>(b + o_rinv);
  L->wk.h16 = reinterpret_cast<__half*>(b + o_h16);
  L->wk.hinv = reinterpret_cast<float*>(b + o_hinv);
  L->wk.rpart = reinterpret_cast<float*>(b + o_rpart);
  L->wk.sync = reinterpret_cast<unsigned*>(b + o_sync);
  if (encode_act16(&L->x16_map, L->wk.x16, P, s.H) != cudaSuccess ||
      encode_act16(&L->h16_map, L->wk.h16, P, s.I_pad) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the activation maps");
  // zero everything once, ahead of the forward on its stream: the ticket
  // and the error word must start at 0
  CUDA_TRY(cudaMemsetAsync(L->scratch, 0, off, st));
  CUDA_TRY(cudaEventRecord(L->done, st));
  L->done_rec = true;
  L->T_cap = cap;
  return MOE_OK;
}

// Build (or rebuild) the streaming cache so its slots hold `slot_bytes`.
// Caller holds g_mu.
moe_status ensure_cache(int device, size_t slot_bytes) {
  if (g_cache && g_cache->device == device && g_cache->slot_bytes >= slot_bytes) return MOE_OK;
  if (g_cache) {
    CUDA_TRY(cudaDeviceSynchronize());
    cache_free(g_cache);
    g_cache = nullptr;
    g_stats.cache_slots = 0;
    g_stats.slot_bytes = 0;
  }
  if (g_cache_bytes == SIZE_MAX) return fail(MOE_ERR_INVALID_ARG, "no streaming budget set");
  const size_t n = g_cache_bytes / slot_bytes;
  if (n == 0)
    return fail(MOE_ERR_CACHE_TOO_SMALL, "cache budget %zu B holds no %zu-byte expert", g_cache_bytes,
                slot_bytes);
  Cache* c = new Cache();
  c->device = device;
  c->slot_bytes = slot_bytes;
  c->n_slots = (int)n;
  cudaError_t e = cudaMalloc(&c->arena, n * slot_bytes);
  for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
    e = cudaMalloc(&c->staging[b], slot_bytes);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->copied[b], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->retiled[b], cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    cache_free(c);
    return fail(MOE_ERR_OOM, "cache arena of %zu slots x %zu B: %s", n, slot_bytes, cudaGetErrorString(e));
  }
  e = cudaStreamCreateWithFlags(&c->copy, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->retile, cudaStreamNonBlocking);
  c->slots.resize(n);
  for (size_t i = 0; i < n && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&c->slots[i].ready, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->slots[i].used, cudaEventDisableTiming);
    c->slots[i].lru = c->lru.insert(c->lru.end(), (int)i);
  }
  if (e != cudaSuccess) {
    cache_free(c);
    return fail(MOE_ERR_CUDA, "cache setup: %s", cudaGetErrorString(e));
  }
  c->gen = ++g_cache_gen;
  g_cache = c;
  g_stats.cache_slots = n;
  g_stats.slot_bytes = slot_bytes;
  return MOE_OK;
}

uint64_t slot_key(const moe_layer* L, int e) { return ((uint64_t)L->id << 32) | (uint32_t)e; }

// Make sure expert e of L is in the cache (or on its way there).  Returns the
// slot.  `pin_epoch` != 0 marks the slot as needed by the current forward so
// that later misses of the same forward cannot evict it.  Caller holds g_mu.
moe_status cache_fetch(moe_layer* L, int e, uint64_t pin_epoch, bool prefetch, int* slot_out) {
  Cache* c = g_cache;
  const uint64_t key = slot_key(L, e);
  auto it = c->where.find(key);
  int s;
  if (!prefetch && g_cache_policy == MOE_CACHE_LFU) {
    const uint64_t f = c->layer_fwds[L->id];
    Cache::Use& u = c->use[key];
    if (u.last_fwd == 0 || f - u.last_fwd > 1) {
      u.arrivals++;
      if (++c->arrivals % (kAgeEvery * (uint64_t)c->n_slots) == 0)
        for (auto& kv : c->use) kv.second.arrivals >>= 1;
    }
    u.last_fwd = f;
  }
  if (prefetch && g_cache_policy == MOE_CACHE_LFU) c->use[key].prefetched_for = c->layer_fwds[L->id] + 1;
  if (it != c->where.end()) {
    s = it->second;
    if (!prefetch) g_stats.cache_hits++;
  } else {
    // victim, among the slots not needed by the current forward: LRU takes
    // the least recently used.  LFU takes an empty slot if there is one, else
    // keeps experts prefetched for their layer's next forward, then those used
    // by their layer's previous forward, and among the rest takes the one that
    // entered use least often; the least recently used among equals
    int victim = -1;
    uint64_t best = UINT64_MAX;
    for (auto r = c->lru.rbegin(); r != c->lru.rend(); ++r) {
      if (c->slots[*r].epoch != c->epoch || c->epoch == 0) {
        const uint64_t k2 = c->slots[*r].key;
        if (g_cache_policy != MOE_CACHE_LFU || k2 == UINT64_MAX) {
          victim = *r;
          break;
        }
        const Cache::Use& u = c->use[k2];
        const uint64_t lf = c->layer_fwds[(uint32_t)(k2 >> 32)];
        const bool recent = u.last_fwd != 0 && lf - u.last_fwd < 2;
        const bool pending = u.prefetched_for > lf;   // that forward has not run yet
        const uint64_t score = ((uint64_t)pending << 33) | ((uint64_t)recent << 32) | u.arrivals;
        if (score < best) {
          best = score;
          victim = *r;
        }
      }
    }
    if (victim < 0)
      return fail(MOE_ERR_CACHE_TOO_SMALL, "one forward needs more than the %d cache slots", c->n_slots);
    s = victim;
    NvtxRange nv(prefetch ? "moe.prefetch_copy" : "moe.miss_copy");
    Slot& sl = c->slots[s];
    if (sl.key != UINT64_MAX) {
      c->where.erase(sl.key);
      g_stats.evictions++;
    }
    // the slot's last reader has finished before the retile writes it
    if (sl.used_rec) CUDA_TRY(cudaStreamWaitEvent(c->retile, sl.used, 0));
    uint8_t* dst = c->arena + (size_t)s * c->slot_bytes;
    const uint8_t* const* hp = &L->host[3 * (size_t)e];
    const Shape& sh = L->s;
    const size_t off[3] = {0, L->gate_bytes, 2 * L->gate_bytes};
    const int rows[3] = {sh.I, sh.I, sh.H}, q[3] = {sh.qgu, sh.qgu, sh.qd};
    const int nb[3] = {sh.nbh, sh.nbh, sh.nbi}, sbb[3] = {sh.sbb_gu, sh.sbb_gu, sh.sbb_d};
    const size_t hrow[3] = {sh.hrow_gu, sh.hrow_gu, sh.hrow_d}, drow[3] = {sh.drow_gu, sh.drow_gu, sh.drow_d};
    for (int m = 0; m < 3; ++m) {
      const int b = (int)(c->uploads++ & 1u);
      if (c->retiled_rec[b]) CUDA_TRY(cudaStreamWaitEvent(c->copy, c->retiled[b], 0));   // staging[b] read
      CUDA_TRY(copy_matrix_h2d(c->staging[b], hp[m], rows[m], q[m], hrow[m], drow[m], c->copy));
      CUDA_TRY(cudaEventRecord(c->copied[b], c->copy));
      CUDA_TRY(cudaStreamWaitEvent(c->retile, c->copied[b], 0));
      CUDA_TRY(launch_retile(c->staging[b], dst + off[m], rows[m], nb[m], sbb[m], c->retile));
      CUDA_TRY(cudaEventRecord(c->retiled[b], c->retile));
      c->retiled_rec[b] = true;
    }
    CUDA_TRY(cudaEventRecord(sl.ready, c->retile));
    sl.ready_rec = true;
    sl.key = key;
    c->where[key] = s;
    g_stats.h2d_bytes += L->host_expert_bytes;
    if (prefetch)
      g_stats.prefetches++;
    else
      g_stats.cache_misses++;
  }
  Slot& sl = c->slots[s];
  c->lru.erase(sl.lru);
  sl.lru = c->lru.insert(c->lru.begin(), s);
  if (pin_epoch) sl.epoch = pin_epoch;
  *slot_out = s;
  return MOE_OK;
}

// TMA maps for every slot the layer's experts can occupy: `n_slots` expert
// images `stride` bytes apart from `arena`.
moe_status build_maps(moe_layer* L, const uint8_t* arena, size_t stride, size_t n_slots) {
  std::vector<CUtensorMap> maps(kMapsPerSlot * n_slots);
  for (size_t i = 0; i < n_slots; ++i) {
    if (encode_expert_maps(&maps[kMapsPerSlot * i], arena + i * stride, L->s) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for slot %zu", i);
  }
  if (L->n_tmap_slots < n_slots) {
    if (L->d_tmaps) {
      CUDA_TRY(cudaDeviceSynchronize());
      cudaFree(L->d_tmaps);
      L->d_tmaps = nullptr;
      L->n_tmap_slots = 0;
    }
    CUDA_TRY(cudaMalloc(&L->d_tmaps, sizeof(CUtensorMap) * maps.size()));
    L->n_tmap_slots = n_slots;
  }
  CUDA_TRY(cudaMemcpy(L->d_tmaps, maps.data(), sizeof(CUtensorMap) * maps.size(), cudaMemcpyHostToDevice));
  L->w_arena = arena;
  L->w_stride = stride;
  return MOE_OK;
}

// Streaming layers: point the maps at the current cache arena.  Caller holds g_mu.
moe_status refresh_stream_maps(moe_layer* L) {
  if (L->cache_gen == g_cache->gen) return MOE_OK;
  MOE_TRY(build_maps(L, g_cache->arena, g_cache->slot_bytes, (size_t)g_cache->n_slots));
  L->cache_gen = g_cache->gen;
  return MOE_OK;
}

// Streaming: bring every expert a forward needs into the cache, make `st`
// wait for their fills and point the device table at their slots.
// Caller holds g_mu until the `used` events of these slots are recorded.
moe_status resolve_experts(moe_layer* L, const int32_t* ids, int n, cudaStream_t st,
                           std::vector<int>* used_slots) {
  NvtxRange nv("moe.resolve_experts");
  const Shape& s = L->s;
  std::vector<char> need(s.E + s.S, 0);
  for (int i = 0; i < n; ++i) need[ids[i]] = 1;
  for (int j = 0; j < s.S; ++j) need[s.E + j] = 1;
  for (int e = 0; e < s.E + s.S; ++e)
    if (!ep_owned(e, L->ep_rank, L->ep_world)) need[e] = 0;   // another rank's expert
  MOE_TRY(ensure_cache(L->device, L->expert_bytes));
  MOE_TRY(refresh_stream_maps(L));
  Cache* c = g_cache;
  c->epoch++;
  c->layer_fwds[L->id]++;
  SlotUpdate u{};
  for (int e = 0; e < s.E + s.S; ++e) {
    if (!need[e]) continue;
    int slot;
    MOE_TRY(cache_fetch(L, e, c->epoch, false, &slot));
    if (c->slots[slot].ready_rec) CUDA_TRY(cudaStreamWaitEvent(st, c->slots[slot].ready, 0));
    used_slots->push_back(slot);
    u.expert[u.n] = e;
    u.slot[u.n] = slot;
    if (++u.n == SlotUpdate::kMax) {
      CUDA_TRY(launch_set_slots(L->d_slot_of, u, st));
      g_stats.launches++;
      u.n = 0;
    }
  }
  if (u.n) {
    CUDA_TRY(launch_set_slots(L->d_slot_of, u, st));
    g_stats.launches++;
  }
  return MOE_OK;
}

// `partial` (fp32 [T, H]): write the unrounded sum over the experts this
// layer owns there instead of the bf16 output (expert parallelism).
moe_status forward_impl(moe_layer* L, const void* x, void* out, int T, const int32_t* forced,
                        cudaStream_t st, float* partial = nullptr) {
  NvtxRange nv(T == 1 ? "moe.forward T=1" : T <= kD1MaxTok ? "moe.forward decode" : "moe.forward prefill");
  if (!L) return fail(MOE_ERR_INVALID_ARG, "null layer");
  if (T < 0 || T > kMaxTokens) return fail(MOE_ERR_INVALID_ARG, "T=%d outside 0..%d", T, kMaxTokens);
  if (T > 0 && (!x || !out)) return fail(MOE_ERR_INVALID_ARG, "null x or out");
  if (!L->router_set) return fail(MOE_ERR_NOT_READY, "router not set");
  if (!L->experts_set) return fail(MOE_ERR_NOT_READY, "experts not set");
  MOE_TRY(check_device(L));
  const Shape& s = L->s;
  if (forced) {
    for (int i = 0; i < T * s.k; ++i)
      if (forced[i] < 0 || forced[i] >= s.E)
        return fail(MOE_ERR_INVALID_ARG, "forced id %d at %d outside 0..%d", forced[i], i, s.E - 1);
  }
  if (T == 0) return MOE_OK;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MOE_ERR_INVALID_ARG, "x and out must be 16-byte aligned");
  MOE_TRY(ensure_scratch(L, T, st));
  const Work& wk = L->wk;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  // one kernel launch, optionally bracketed by profiling events
  ProfRec pr{};
  bool prof;
  uint64_t hook_wait_ns;
  int hook_hold, mt_rows;
  {
    std::lock_guard<std::mutex> lk0(g_mu);
    prof = g_profiling;
    hook_wait_ns = g_hook_wait_ns;
    hook_hold = g_hook_hold;
    mt_rows = g_mt_rows < 0 ? default_few_rows(T) : g_mt_rows;
    if (prof)
      for (int i = 0; i < 2 * kProfRanges; ++i) pr.ev[i] = prof_event();
  }
  int n_launch = 0;
#define MOE_KERNEL(k_id, call)                                          \
  do {                                                                  \
    const bool rec_ = prof && pr.n < kProfRanges;                       \
    if (rec_) CUDA_TRY(cudaEventRecord(pr.ev[2 * pr.n], st));           \
    CUDA_TRY(call);                                                     \
    if (rec_) {                                                         \
      CUDA_TRY(cudaEventRecord(pr.ev[2 * pr.n + 1], st));               \
      pr.kid[pr.n++] = (k_id);                                          \
    }                                                                   \
    ++n_launch;                                                         \
  } while (0)
  // decode path (few tokens): kernels specialised for one row per expert when
  // T == 1; activation slots of the down kernel must fit in shared memory
  const int max_tok = T == 1 ? 1 : kD1MaxTok;
  const size_t act_slot = (size_t)max_tok * (2 * (size_t)s.I_pad + (size_t)(s.I_pad / 32) * 8);
  const size_t x_stage = 2 * (size_t)T * s.H + (size_t)T * (s.H / 32) * 8;
  const bool stage_x = max_tok == 1 && gate_up_d1_smem(1, x_stage) <= kMaxDecodeSmem;
  const bool fast = T <= kD1MaxTok && down_d1_smem(max_tok, act_slot) <= kMaxDecodeSmem;
  if (forced)
    CUDA_TRY(cudaMemcpyAsync(wk.forced, forced, (size_t)T * s.k * 4, cudaMemcpyHostToDevice, st));
  // One token: the whole forward as one persistent kernel, when the experts
  // are resident or the routing is given (a streamed forward that routes on
  // the GPU must read the routing back before its experts can be fetched).
  // Layers with other block types than Q4_K run every token this way.
  const size_t act1 = 2 * (size_t)s.I_pad + (size_t)(s.I_pad / 32) * 8;
  int ring_stages = 0, ring_stage_bytes = 0;
  decode1_ring(s.sbb_gu, s.sbb_d, s.H, act1, &ring_stages, &ring_stage_bytes);
  const bool fused_ok = s.k + s.S <= 40 && s.H % 64 == 0 &&
                        decode1_fused_smem(s.H, act1, ring_stages * ring_stage_bytes) <= kMaxDecodeSmem;
  const bool q4k = s.qgu == kQ4_K && s.qd == kQ4_K;
  if (!q4k && !fused_ok)
    return fail(MOE_ERR_UNSUPPORTED, "block types %d/%d need the single-token kernel, which this shape does not fit",
                s.qgu, s.qd);
  if ((T == 1 && (L->resident || forced) && fused_ok) || !q4k) {
    std::unique_lock<std::mutex> lk(g_mu, std::defer_lock);
    std::vector<int> used;
    const int* dev_forced = forced ? wk.forced : nullptr;
    if (!L->resident) {
      const int32_t* hid = forced;
      if (!hid) {
        // route on the GPU first, read the picks back, then run the tokens
        // with those picks as their routing
        if (T <= kD1MaxTok) {
          RouteArgs ra{xb, L->d_W, L->d_b, nullptr, T, s.H, s.E, s.k, s.S, (int)L->gating, wk.logits, wk.ids, wk.w,
                       wk.counts, wk.offsets, wk.perm, wk.inv, wk.act1, wk.n_act1, wk.act2, wk.n_act2, wk.n_act,
                       wk.xq, wk.xq_plane, wk.xsc, wk.ticket, L->ep_rank, L->ep_world};
          MOE_KERNEL(MOE_K_ROUTER, launch_route_decode(ra, st));
        } else {
          CUtensorMap xmap;
          if (encode_sw128_16(&xmap, xb, true, (size_t)T, s.H, 128) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
          RouterGemmArgs rg{};
          rg.T = T;
          rg.E = s.E;
          rg.nsplit = router_gemm_splits(T, s.E, s.H, s.n_sm);
          rg.nk_split = s.H / 64 / rg.nsplit;
          rg.part = wk.rpart;
          rg.split_stride = (size_t)T * s.E;
          rg.err = wk.err;
          MOE_KERNEL(MOE_K_ROUTER, launch_router_gemm(xmap, L->wp_map, rg, st));
          MOE_KERNEL(MOE_K_TOPK, launch_topk(wk.logits, T, s.E, s.k, (int)L->gating, nullptr, wk.ids, wk.w, st,
                                             wk.rpart, rg.nsplit, rg.split_stride, L->d_b));
        }
        CUDA_TRY(cudaMemcpyAsync(L->h_ids, wk.ids, (size_t)T * s.k * 4, cudaMemcpyDeviceToHost, st));
        CUDA_TRY(cudaStreamSynchronize(st));
        hid = L->h_ids;
        CUDA_TRY(cudaMemcpyAsync(wk.forced, wk.ids, (size_t)T * s.k * 4, cudaMemcpyDeviceToDevice, st));
        dev_forced = wk.forced;
      }
      lk.lock();
      MOE_TRY(resolve_experts(L, hid, T * s.k, st, &used));
    }
    FusedArgs fa{};
    fa.warena = L->w_arena;
    fa.wstride = L->w_stride;
    fa.gate_bytes = L->gate_bytes;
    fa.slot_of = L->d_slot_of;
    fa.W = L->d_W;
    fa.b = L->d_b;
    fa.T = 1;
    fa.H = s.H;
    fa.I = s.I;
    fa.I_pad = s.I_pad;
    fa.E = s.E;
    fa.k = s.k;
    fa.S = s.S;
    fa.nbh = s.nbh;
    fa.nbi = s.nbi;
    fa.gating = (int)L->gating;
    fa.hq = wk.hq;
    fa.hq_plane = wk.hq_plane;
    fa.hsc = wk.hsc;
    fa.y = wk.y;
    fa.sync = wk.sync;
    fa.err = wk.err;
    fa.act_slot_bytes = act1;
    fa.early = L->resident ? 1 : 0;
    fa.n_slots = (int)L->n_tmap_slots;
    fa.wait_ns = hook_wait_ns;
    fa.hold = hook_hold;
    fa.qgu = s.qgu;
    fa.qd = s.qd;
    fa.sbb_gu = s.sbb_gu;
    fa.sbb_d = s.sbb_d;
    fa.stages = ring_stages;
    fa.stage_bytes = ring_stage_bytes;
    fa.ep_rank = L->ep_rank;
    fa.ep_world = L->ep_world;
    // one launch per token, in order (each reuses the kernel's scratch rows)
    for (int t = 0; t < T; ++t) {
      fa.x = xb + (size_t)t * s.H;
      fa.out = static_cast<__nv_bfloat16*>(out) + (size_t)t * s.H;
      fa.partial = partial ? partial + (size_t)t * s.H : nullptr;
      fa.forced = dev_forced ? dev_forced + (size_t)t * s.k : nullptr;
      fa.logits = wk.logits + (size_t)t * s.E;
      fa.ids = wk.ids + (size_t)t * s.k;
      fa.w = wk.w + (size_t)t * s.k;
      MOE_KERNEL(MOE_K_FUSED, launch_decode1_fused(fa, s.n_sm, st));
    }
    CUDA_TRY(cudaEventRecord(L->done, st));
    L->done_rec = true;
    if (!lk.owns_lock()) lk.lock();
    if (prof) g_prof_pending.push_back(pr);
    g_stats.launches += (uint64_t)n_launch;
    for (int slot : used) {
      CUDA_TRY(cudaEventRecord(g_cache->slots[slot].used, st));
      g_cache->slots[slot].used_rec = true;
    }
    g_stats.forwards++;
    g_stats.tokens += (uint64_t)T;
    g_stats.decode_calls++;
    L->last_T = T;
    return MOE_OK;
  }
  if (fast) {
    RouteArgs ra{xb, L->d_W, L->d_b, forced ? wk.forced : nullptr, T, s.H, s.E, s.k, s.S, (int)L->gating,
                 wk.logits, wk.ids, wk.w, wk.counts, wk.offsets, wk.perm, wk.inv, wk.act1, wk.n_act1, wk.act2,
                 wk.n_act2, wk.n_act, wk.xq, wk.xq_plane, wk.xsc, wk.ticket, L->ep_rank, L->ep_world};
    MOE_KERNEL(MOE_K_ROUTER, launch_route_decode(ra, st));
  } else {
    // router on the tensor cores: split-K partial logits, summed in split order by top-k
    CUtensorMap xmap;
    if (encode_sw128_16(&xmap, xb, true, (size_t)T, s.H, 128) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
    RouterGemmArgs rg{};
    rg.T = T;
    rg.E = s.E;
    rg.nsplit = router_gemm_splits(T, s.E, s.H, s.n_sm);
    rg.nk_split = s.H / 64 / rg.nsplit;
    rg.part = wk.rpart;
    rg.split_stride = (size_t)T * s.E;
    rg.err = wk.err;
    MOE_KERNEL(MOE_K_ROUTER, launch_router_gemm(xmap, L->wp_map, rg, st));
    MOE_KERNEL(MOE_K_TOPK, launch_topk(wk.logits, T, s.E, s.k, (int)L->gating, forced ? wk.forced : nullptr,
                                       wk.ids, wk.w, st, wk.rpart, rg.nsplit, rg.split_stride, L->d_b));
  }
  // Streaming: the cache lock is held from resolving the experts until the
  // slots' `used` events are recorded, so no other forward can evict a slot
  // between this forward's fill-wait and its last read.
  std::unique_lock<std::mutex> lk(g_mu, std::defer_lock);
  std::vector<int> used;
  if (!L->resident) {
    const int32_t* hid = forced;
    if (!hid) {
      CUDA_TRY(cudaMemcpyAsync(L->h_ids, wk.ids, (size_t)T * s.k * 4, cudaMemcpyDeviceToHost, st));
      CUDA_TRY(cudaStreamSynchronize(st));
      hid = L->h_ids;
    }
    lk.lock();
    MOE_TRY(resolve_experts(L, hid, T * s.k, st, &used));
  }
  // arguments of the per-sub-block decode kernels (all experts on the decode
  // path; on the prefill path the experts with <= kD1MaxTok rows)
  DecodeArgs da{};
  da.tmaps = L->d_tmaps;
  da.slot_of = L->d_slot_of;
  da.act = wk.act1;
  da.n_act = wk.n_act1;
  da.counts = wk.counts;
  da.offsets = wk.offsets;
  da.perm = wk.perm;
  da.inv = wk.inv;
  da.w = wk.w;
  da.kS = s.k + s.S;
  da.T = T;
  da.k = s.k;
  da.S = s.S;
  da.H = s.H;
  da.I = s.I;
  da.I_pad = s.I_pad;
  da.nbh = s.nbh;
  da.nbi = s.nbi;
  da.xq = wk.xq;
  da.xq_plane = wk.xq_plane;
  da.xsc = wk.xsc;
  da.hq = wk.hq;
  da.hq_plane = wk.hq_plane;
  da.hsc = wk.hsc;
  da.y = wk.y;
  da.out = static_cast<__nv_bfloat16*>(out);
  da.err = wk.err;
  da.stage_x = stage_x ? 1 : 0;
  da.act_slot_bytes = act_slot;
  da.n_ex = s.E + s.S;
  da.n_slots = (int)L->n_tmap_slots;
  da.n_rows = T * (s.k + s.S);
  if (fast) {
    const bool gemv = T == 1 && gemv_gate_up_smem(s.H) <= kMaxDecodeSmem && gemv_down_smem(act_slot) <= kMaxDecodeSmem;
    if (gemv) {
      MOE_KERNEL(MOE_K_GATE_UP, launch_gemv_gate_up(da, s.n_sm, st));
      MOE_KERNEL(MOE_K_DOWN, launch_gemv_down(da, s.n_sm, st));
    } else {
      MOE_KERNEL(MOE_K_GATE_UP, launch_gate_up_d1(da, max_tok, s.n_sm, st));
      MOE_KERNEL(MOE_K_DOWN, launch_down_d1(da, max_tok, s.n_sm, st));
    }
    MOE_KERNEL(MOE_K_COMBINE, launch_combine(wk, T, s, static_cast<__nv_bfloat16*>(out), st, true, partial, L->ep_rank, L->ep_world));
  } else {
    // prefill: tensor-core GEMMs over tiles of up to 256 rows of one expert;
    // experts with <= mt_rows rows, and last partial tiles that small, run on
    // the few-row warp-MMA kernel instead (dequantisation in registers, one
    // weight pass at the HBM rate); with mt_rows == 0, experts with <=
    // kD1MaxTok rows (when their kernels fit) stream through the decode
    // kernels instead, which do not dequantise
    const int kS = s.k + s.S, P = T * kS;
    const bool split_small = mt_rows == 0 && down_d1_smem(kD1MaxTok, act_slot) <= kMaxDecodeSmem;
    // an expert has at most T rows, so with T <= mt_rows every one is a
    // single few-row tile and the GEMM tile lists are empty: skip the GEMMs
    const bool gemms = !(mt_rows > 0 && T <= mt_rows);
    MOE_KERNEL(MOE_K_PERMUTE, launch_permute(wk.ids, T, s, wk, st));
    MOE_KERNEL(MOE_K_PERMUTE,
               launch_build_tiles(wk, split_small ? kD1MaxTok : 0, mt_rows, st, L->ep_rank, L->ep_world));
    if (split_small) MOE_KERNEL(MOE_K_PREP, launch_quant_x(xb, wk, T, s.H, st));
    MOE_KERNEL(MOE_K_PREP, launch_gather_rows(xb, wk, P, kS, s.H, st));
    GemmArgs ga{};
    ga.wmaps = L->d_tmaps;
    ga.slot_of = L->d_slot_of;
    ga.tiles = wk.tiles;
    ga.n_tiles = wk.n_tiles;
    ga.ft = (s.I + 127) / 128;
    ga.nkb = s.nbh;
    ga.rinv = wk.rinv;
    ga.out = wk.h;
    ga.out_ld = s.I_pad;
    ga.out_rows = s.I;
    ga.wexp = L->d_wexp;
    ga.wexp_stride = 2 * s.I + s.H;
    ga.wexp_down = 2 * s.I;
    ga.err = wk.err;
    ga.n_ex = s.E + s.S;
    ga.n_slots = (int)L->n_tmap_slots;
    ga.n_rows = P;
    if (gemms) MOE_KERNEL(MOE_K_GATE_UP, launch_prefill_gemm(0, L->x16_map, ga, s.n_sm, st));
    GemmArgs gm = ga;   // the few-row tiles
    gm.tiles = wk.mtiles;
    gm.n_tiles = wk.n_mtiles;
    gm.bsrc = wk.x16;
    gm.b_ld = s.H;
    gm.next = wk.mt_next;
    if (mt_rows) MOE_KERNEL(MOE_K_FEW_GATE_UP, launch_prefill_mt(0, gm, s.n_sm, st, mt_rows));
    if (split_small) MOE_KERNEL(MOE_K_SMALL, launch_gate_up_d1(da, kD1MaxTok, s.n_sm, st));
    MOE_KERNEL(MOE_K_PREP, launch_convert_h(wk, P, s.I, s.I_pad, st));
    ga.ft = s.H / 256;
    ga.nkb = s.nbi;
    ga.rinv = wk.hinv;
    ga.out = wk.y;
    ga.out_ld = s.H;
    ga.out_rows = s.H;
    if (gemms) MOE_KERNEL(MOE_K_DOWN, launch_prefill_gemm(1, L->h16_map, ga, s.n_sm, st));
    gm.ft = ga.ft;
    gm.nkb = ga.nkb;
    gm.rinv = ga.rinv;
    gm.out = ga.out;
    gm.out_ld = ga.out_ld;
    gm.out_rows = ga.out_rows;
    gm.bsrc = wk.h16;
    gm.b_ld = s.I_pad;
    gm.next = wk.mt_next + 1;
    if (mt_rows) MOE_KERNEL(MOE_K_FEW_DOWN, launch_prefill_mt(1, gm, s.n_sm, st, mt_rows));
    if (split_small) MOE_KERNEL(MOE_K_SMALL, launch_down_d1(da, kD1MaxTok, s.n_sm, st));
    MOE_KERNEL(MOE_K_COMBINE, launch_combine(wk, T, s, static_cast<__nv_bfloat16*>(out), st, true, partial, L->ep_rank, L->ep_world));
  }
#undef MOE_KERNEL
  CUDA_TRY(cudaEventRecord(L->done, st));
  L->done_rec = true;
  {
    if (!lk.owns_lock()) lk.lock();
    if (prof) g_prof_pending.push_back(pr);
    g_stats.launches += (uint64_t)n_launch;
    if (!used.empty() && g_cache) {
      for (int slot : used) {
        CUDA_TRY(cudaEventRecord(g_cache->slots[slot].used, st));
        g_cache->slots[slot].used_rec = true;
      }
    }
    g_stats.forwards++;
    g_stats.tokens += (uint64_t)T;
    if (fast)
      g_stats.decode_calls++;
    else
      g_stats.prefill_calls++;
  }
  L->last_T = T;
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_expert_bytes(int hidden, int inter, moe_quant quant) {
  const int q = (int)quant;
  if (!dev_sb_bytes(q) || hidden <= 0 || inter <= 0 || hidden % kQK) return 0;
  if (host_block_elems(q) != kQK && inter % kQK) return 0;
  const size_t nbh = hidden / kQK, nbi = (inter + kQK - 1) / kQK;
  return 2 * tiled_matrix_bytes(inter, nbh * dev_sb_bytes(q)) + tiled_matrix_bytes(hidden, nbi * dev_sb_bytes(q));
}

moe_status moe_layer_create(int hidden, int inter, int n_experts, int top_k, int n_shared,
                            moe_quant quant, moe_layer_t* out) {
  return moe_layer_create_mixed(hidden, inter, n_experts, top_k, n_shared, quant, quant, out);
}

moe_status moe_layer_create_mixed(int hidden, int inter, int n_experts, int top_k, int n_shared,
                                  moe_quant quant_gate_up, moe_quant quant_down, moe_layer_t* out) {
  g_err.clear();
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  const int qgu = (int)quant_gate_up, qd = (int)quant_down;
  if (!dev_sb_bytes(qgu) || !dev_sb_bytes(qd))
    return fail(MOE_ERR_UNSUPPORTED, "quant types %d, %d (supported: Q8_0=8, Q4_K=12, Q5_K=13, Q6_K=14, MXFP4=39)",
                qgu, qd);
  if (host_block_elems(qd) != kQK && inter % kQK)
    return fail(MOE_ERR_UNSUPPORTED, "inter=%d must be a multiple of 256 for down weights of type %d", inter, qd);
  if (hidden <= 0 || hidden > 16384 || hidden % kQK)
    return fail(MOE_ERR_INVALID_ARG, "hidden=%d must be a multiple of 256 in 256..16384", hidden);
  if (inter <= 0 || inter > 16384) return fail(MOE_ERR_INVALID_ARG, "inter=%d outside 1..16384", inter);
  if (n_experts <= 0 || n_experts > 1024)
    return fail(MOE_ERR_INVALID_ARG, "n_experts=%d outside 1..1024", n_experts);
  if (top_k <= 0 || top_k > 32 || top_k > n_experts)
    return fail(MOE_ERR_INVALID_ARG, "top_k=%d outside 1..min(32, E)", top_k);
  if (n_shared < 0 || n_shared > 8) return fail(MOE_ERR_INVALID_ARG, "n_shared=%d outside 0..8", n_shared);
  moe_layer* L = new moe_layer();
  Shape& s = L->s;
  s.H = hidden;
  s.I = inter;
  s.E = n_experts;
  s.k = top_k;
  s.S = n_shared;
  s.nbh = hidden / kQK;
  s.nbi = (inter + kQK - 1) / kQK;
  s.I_pad = s.nbi * kQK;
  s.qgu = qgu;
  s.qd = qd;
  s.sbb_gu = dev_sb_bytes(qgu);
  s.sbb_d = dev_sb_bytes(qd);
  s.hrow_gu = (size_t)((hidden + host_block_elems(qgu) - 1) / host_block_elems(qgu)) * host_block_bytes(qgu);
  s.hrow_d = (size_t)((inter + host_block_elems(qd) - 1) / host_block_elems(qd)) * host_block_bytes(qd);
  s.drow_gu = (size_t)s.nbh * s.sbb_gu;
  s.drow_d = (size_t)s.nbi * s.sbb_d;
  L->gate_bytes = tiled_matrix_bytes(inter, s.drow_gu);
  L->down_bytes = tiled_matrix_bytes(hidden, s.drow_d);
  L->expert_bytes = 2 * L->gate_bytes + L->down_bytes;
  L->host_expert_bytes = 2 * (size_t)inter * s.hrow_gu + (size_t)hidden * s.hrow_d;
  cudaError_t e = cudaGetDevice(&L->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&s.n_sm, cudaDevAttrMultiProcessorCount, L->device);
  if (e == cudaSuccess) e = cudaMalloc(&L->d_slot_of, sizeof(int) * (size_t)(s.E + s.S));
  if (e == cudaSuccess) e = cudaMemset(L->d_slot_of, 0, sizeof(int) * (size_t)(s.E + s.S));
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->copy, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->done, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaMallocHost(&L->h_err, sizeof(unsigned));
  if (e != cudaSuccess) {
    moe_layer_destroy(L);
    return fail(e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA, "layer setup: %s",
                cudaGetErrorString(e));
  }
  {
    std::lock_guard<std::mutex> lk(g_mu);
    L->id = g_next_layer_id++;
  }
  *out = L;
  return MOE_OK;
}

moe_status moe_layer_destroy(moe_layer_t L) {
  g_err.clear();
  if (!L) return MOE_OK;
  // the layer's own work only; cudaFree below may still wait for the device
  // as the CUDA runtime requires
  if (wait_layer(L) != MOE_OK) (void)cudaGetLastError();
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_cache) {
      for (int e = 0; e < L->s.E + L->s.S; ++e) {
        auto it = g_cache->where.find(slot_key(L, e));
        if (it != g_cache->where.end()) {
          g_cache->slots[it->second].key = UINT64_MAX;
          g_cache->where.erase(it);
        }
      }
    }
  }
  if (L->d_W) cudaFree(L->d_W);
  if (L->d_b) cudaFree(L->d_b);
  if (L->d_Wp) cudaFree(L->d_Wp);
  if (L->d_resident) cudaFree(L->d_resident);
  if (L->d_wexp) cudaFree(L->d_wexp);
  if (L->d_tmaps) cudaFree(L->d_tmaps);
  if (L->d_slot_of) cudaFree(L->d_slot_of);
  if (L->scratch) cudaFree(L->scratch);
  if (L->h_ids) cudaFreeHost(L->h_ids);
  if (L->h_err) cudaFreeHost(L->h_err);
  if (L->done) cudaEventDestroy(L->done);
  if (L->copy) cudaStreamDestroy(L->copy);
  delete L;
  return MOE_OK;
}

moe_status moe_set_router(moe_layer_t L, const float* W, const float* bias, moe_gating gating) {
  g_err.clear();
  if (!L || !W) return fail(MOE_ERR_INVALID_ARG, "null layer or W");
  if (gating != MOE_GATE_SOFTMAX_TOPK && gating != MOE_GATE_SIGMOID_RENORM)
    return fail(MOE_ERR_INVALID_ARG, "gating=%d", (int)gating);
  MOE_TRY(check_device(L));
  const size_t wb = (size_t)L->s.E * L->s.H * sizeof(float);
  if (!L->d_W) CUDA_TRY(cudaMalloc(&L->d_W, wb));
  CUDA_TRY(cudaMemcpy(L->d_W, W, wb, cudaMemcpyDefault));
  if (bias) {
    if (!L->d_b) CUDA_TRY(cudaMalloc(&L->d_b, (size_t)L->s.E * sizeof(float)));
    CUDA_TRY(cudaMemcpy(L->d_b, bias, (size_t)L->s.E * sizeof(float), cudaMemcpyDefault));
  } else if (L->d_b) {
    cudaFree(L->d_b);
    L->d_b = nullptr;
  }
  // bf16 planes of W for the tensor-core router (T > 4)
  if (!L->d_Wp) CUDA_TRY(cudaMalloc(&L->d_Wp, 3 * (size_t)L->s.E * L->s.H * sizeof(__nv_bfloat16)));
  CUDA_TRY(launch_split_router(L->d_W, L->s.E, L->s.H, L->d_Wp, L->copy));
  CUDA_TRY(cudaStreamSynchronize(L->copy));
  if (encode_sw128_16(&L->wp_map, L->d_Wp, true, 3 * (size_t)L->s.E, L->s.H, 128) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the router planes");
  L->gating = gating;
  L->router_set = true;
  return MOE_OK;
}

moe_status moe_set_experts(moe_layer_t L, const void* const* gate, const void* const* up,
                           const void* const* down) {
  g_err.clear();
  if (!L || !gate || !up || !down) return fail(MOE_ERR_INVALID_ARG, "null argument");
  MOE_TRY(check_device(L));
  NvtxRange nv("moe.set_experts");
  const int n = L->s.E + L->s.S;
  std::vector<const uint8_t*> host(3 * (size_t)n);
  for (int e = 0; e < n; ++e) {
    const void* p[3] = {gate[e], up[e], down[e]};
    for (int m = 0; m < 3; ++m) {
      if (!p[m]) return fail(MOE_ERR_INVALID_ARG, "expert %d matrix %d is NULL", e, m);
      cudaPointerAttributes a{};
      cudaError_t err = cudaPointerGetAttributes(&a, p[m]);
      if (err != cudaSuccess || a.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        return fail(MOE_ERR_INVALID_ARG, "expert %d matrix %d is not pinned host memory", e, m);
      }
      host[3 * (size_t)e + m] = static_cast<const uint8_t*>(p[m]);
    }
  }
  // power-of-two scales of the prefill GEMMs' fp16 weights, one per weight
  // row, from the host bytes (several threads: a layer is gigabytes)
  const int stride = 2 * L->s.I + L->s.H;
  std::vector<int8_t> wexp((size_t)n * stride);
  {
    const int nth = (int)std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
    std::vector<std::thread> pool;
    for (int t = 0; t < nth; ++t)
      pool.emplace_back([&, t] {
        for (int e = t; e < n; e += nth) {
          int8_t* o = wexp.data() + (size_t)e * stride;
          if (L->s.qgu == kQ4_K) {
            q4k_row_exponents(host[3 * (size_t)e], L->s.I, L->s.nbh, o);
            q4k_row_exponents(host[3 * (size_t)e + 1], L->s.I, L->s.nbh, o + L->s.I);
          }
          if (L->s.qd == kQ4_K) q4k_row_exponents(host[3 * (size_t)e + 2], L->s.H, L->s.nbi, o + 2 * L->s.I);
        }
      });
    for (auto& th : pool) th.join();
  }
  if (!L->d_wexp) CUDA_TRY(cudaMalloc(&L->d_wexp, wexp.size()));
  CUDA_TRY(cudaMemcpy(L->d_wexp, wexp.data(), wexp.size(), cudaMemcpyHostToDevice));
  size_t budget;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    budget = g_cache_bytes;
  }
  L->host = std::move(host);
  L->experts_set = false;
  if (budget == SIZE_MAX) {
    // resident: one device copy of every expert, uploaded now
    if (!L->d_resident) CUDA_TRY(cudaMalloc(&L->d_resident, (size_t)n * L->expert_bytes));
    uint8_t* staging = nullptr;   // one matrix before retiling, freed once the uploads are done
    CUDA_TRY(cudaMalloc(&staging, std::max(L->gate_bytes, L->down_bytes)));
    cudaError_t ue = cudaSuccess;
    for (int e = 0; e < n && ue == cudaSuccess; ++e) {
      uint8_t* dst = L->d_resident + (size_t)e * L->expert_bytes;
      const size_t off[3] = {0, L->gate_bytes, 2 * L->gate_bytes};
      const int rows[3] = {L->s.I, L->s.I, L->s.H}, q[3] = {L->s.qgu, L->s.qgu, L->s.qd};
      const int nb[3] = {L->s.nbh, L->s.nbh, L->s.nbi}, sbb[3] = {L->s.sbb_gu, L->s.sbb_gu, L->s.sbb_d};
      const size_t hrow[3] = {L->s.hrow_gu, L->s.hrow_gu, L->s.hrow_d}, drow[3] = {L->s.drow_gu, L->s.drow_gu, L->s.drow_d};
      for (int m = 0; m < 3 && ue == cudaSuccess; ++m)
        ue = upload_matrix(dst + off[m], L->host[3 * (size_t)e + m], rows[m], q[m], hrow[m], drow[m], nb[m], sbb[m],
                           staging, L->copy);
    }
    const cudaError_t se = cudaStreamSynchronize(L->copy);
    cudaFree(staging);
    CUDA_TRY(ue);
    CUDA_TRY(se);
    MOE_TRY(build_maps(L, L->d_resident, L->expert_bytes, (size_t)n));
    std::vector<int> ident(n);
    for (int e = 0; e < n; ++e) ident[e] = e;
    CUDA_TRY(cudaMemcpy(L->d_slot_of, ident.data(), sizeof(int) * n, cudaMemcpyHostToDevice));
    L->resident = true;
  } else {
    if (L->d_resident) {
      CUDA_TRY(cudaDeviceSynchronize());
      cudaFree(L->d_resident);
      L->d_resident = nullptr;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    MOE_TRY(ensure_cache(L->device, L->expert_bytes));
    L->cache_gen = 0;
    MOE_TRY(refresh_stream_maps(L));
    L->resident = false;
  }
  L->experts_set = true;
  return MOE_OK;
}

moe_status moe_set_cache_bytes(size_t bytes) {
  g_err.clear();
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_cache) {
    CUDA_TRY(cudaDeviceSynchronize());
    cache_free(g_cache);
    g_cache = nullptr;
    g_stats.cache_slots = 0;
    g_stats.slot_bytes = 0;
  }
  g_cache_bytes = bytes;
  return MOE_OK;
}

moe_status moe_set_test_hooks(uint64_t wait_limit_ns, int hold_barrier) {
  g_err.clear();
  if (hold_barrier < 0) return fail(MOE_ERR_INVALID_ARG, "hold_barrier=%d", hold_barrier);
  std::lock_guard<std::mutex> lk(g_mu);
  g_hook_wait_ns = wait_limit_ns;
  g_hook_hold = hold_barrier;
  return MOE_OK;
}

moe_status moe_set_few_row_tiles(int max_rows) {
  g_err.clear();
  if (max_rows < -1 || max_rows > kMtMaxRows)
    return fail(MOE_ERR_INVALID_ARG, "max_rows=%d outside -1..%d", max_rows, kMtMaxRows);
  std::lock_guard<std::mutex> lk(g_mu);
  g_mt_rows = max_rows;
  return MOE_OK;
}

moe_status moe_set_cache_policy(int policy) {
  g_err.clear();
  if (policy != MOE_CACHE_LRU && policy != MOE_CACHE_LFU) return fail(MOE_ERR_INVALID_ARG, "policy=%d", policy);
  std::lock_guard<std::mutex> lk(g_mu);
  g_cache_policy = policy;
  return MOE_OK;
}

moe_status moe_forward(moe_layer_t L, const void* x, void* out, int T, void* stream) {
  g_err.clear();
  return forward_impl(L, x, out, T, nullptr, static_cast<cudaStream_t>(stream));
}

moe_status moe_forward_routed(moe_layer_t L, const void* x, void* out, int T, const int32_t* forced_ids,
                              void* stream) {
  g_err.clear();
  if (T > 0 && !forced_ids) return fail(MOE_ERR_INVALID_ARG, "forced_ids is NULL");
  return forward_impl(L, x, out, T, forced_ids, static_cast<cudaStream_t>(stream));
}

// Device address of a pinned host buffer that kernels may access in place,
// or null (pageable memory, or not mapped for the current device).
static void* mapped_device_ptr(const void* p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

moe_status moe_set_expert_parallel(moe_layer_t L, int rank, int world) {
  g_err.clear();
  if (!L) return fail(MOE_ERR_INVALID_ARG, "null layer");
  if (world < 1 || world > 1024 || rank < 0 || rank >= world)
    return fail(MOE_ERR_INVALID_ARG, "rank=%d world=%d", rank, world);
  L->ep_rank = rank;
  L->ep_world = world;
  return MOE_OK;
}

moe_status moe_forward_partial(moe_layer_t L, const void* x, float* partial, int T, void* stream) {
  g_err.clear();
  if (T > 0 && !partial) return fail(MOE_ERR_INVALID_ARG, "null partial");
  if (reinterpret_cast<uintptr_t>(partial) & 15) return fail(MOE_ERR_INVALID_ARG, "partial must be 16-byte aligned");
  // out is not written in this mode; pass the partial buffer for the checks
  return forward_impl(L, x, partial, T, nullptr, static_cast<cudaStream_t>(stream), partial);
}

moe_status moe_combine_partials(const float* partials, void* out, int T, int H, int world, void* stream) {
  g_err.clear();
  if (T < 0 || H <= 0 || H % 4 || world < 1) return fail(MOE_ERR_INVALID_ARG, "T=%d H=%d world=%d", T, H, world);
  if (T == 0) return MOE_OK;
  if (!partials || !out) return fail(MOE_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(partials) & 15) || (reinterpret_cast<uintptr_t>(out) & 7))
    return fail(MOE_ERR_INVALID_ARG, "partials must be 16-byte and out 8-byte aligned");
  CUDA_TRY(launch_combine_partials(partials, static_cast<__nv_bfloat16*>(out), T, H, world,
                                   static_cast<cudaStream_t>(stream)));
  std::lock_guard<std::mutex> lk(g_mu);
  g_stats.launches++;
  return MOE_OK;
}

moe_status moe_forward_host(moe_layer_t L, const void* x_host, void* out_host, int T, void* stream) {
  g_err.clear();
  if (!L) return fail(MOE_ERR_INVALID_ARG, "null layer");
  if (T < 0 || T > kMaxTokens) return fail(MOE_ERR_INVALID_ARG, "T=%d outside 0..%d", T, kMaxTokens);
  if (T == 0) return MOE_OK;
  if (!x_host || !out_host) return fail(MOE_ERR_INVALID_ARG, "null x or out");
  MOE_TRY(check_device(L));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_TRY(ensure_scratch(L, T, st));
  const size_t bytes = (size_t)T * L->s.H * 2;
  // Decode path with pinned (mapped) host buffers: the kernels read x from
  // and write out to host memory in place -- x by a staging kernel that the
  // route kernel overlaps, out by the combine kernel.  Otherwise the buffers
  // are copied through device memory.
  const void* x_dev = T <= kD1MaxTok ? mapped_device_ptr(x_host) : nullptr;
  void* o_dev = T <= kD1MaxTok ? mapped_device_ptr(out_host) : nullptr;
  if (reinterpret_cast<uintptr_t>(o_dev) & 15u) o_dev = nullptr;
  if (x_dev && launch_stage_in(x_dev, L->xbuf, bytes, st) == cudaSuccess) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_stats.launches += 1;
  } else {
    cudaGetLastError();  // an unaligned buffer takes the copy
    CUDA_TRY(cudaMemcpyAsync(L->xbuf, x_host, bytes, cudaMemcpyHostToDevice, st));
  }
  MOE_TRY(forward_impl(L, L->xbuf, o_dev ? o_dev : L->obuf, T, nullptr, st));
  if (!o_dev) CUDA_TRY(cudaMemcpyAsync(out_host, L->obuf, bytes, cudaMemcpyDeviceToHost, st));
  return MOE_OK;
}

moe_status moe_get_routing(moe_layer_t L, int32_t* ids, float* weights, void* stream) {
  g_err.clear();
  if (!L) return fail(MOE_ERR_INVALID_ARG, "null layer");
  if (L->last_T == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = (size_t)L->last_T * L->s.k * 4;
  if (ids) CUDA_TRY(cudaMemcpyAsync(ids, L->wk.ids, n, cudaMemcpyDefault, st));
  if (weights) CUDA_TRY(cudaMemcpyAsync(weights, L->wk.w, n, cudaMemcpyDefault, st));
  return MOE_OK;
}

moe_status moe_get_logits(moe_layer_t L, float* logits, void* stream) {
  g_err.clear();
  if (!L || !logits) return fail(MOE_ERR_INVALID_ARG, "null argument");
  if (L->last_T == 0) return MOE_OK;
  CUDA_TRY(cudaMemcpyAsync(logits, L->wk.logits, (size_t)L->last_T * L->s.E * 4, cudaMemcpyDefault,
                           static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_prefetch(moe_layer_t L, const int32_t* ids, int n) {
  g_err.clear();
  if (!L || (n > 0 && !ids) || n < 0) return fail(MOE_ERR_INVALID_ARG, "bad argument");
  if (!L->experts_set) return fail(MOE_ERR_NOT_READY, "experts not set");
  if (L->resident || n == 0) return MOE_OK;
  MOE_TRY(check_device(L));
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= L->s.E + L->s.S)
      return fail(MOE_ERR_INVALID_ARG, "prefetch id %d outside 0..%d", ids[i], L->s.E + L->s.S - 1);
  std::lock_guard<std::mutex> lk(g_mu);
  MOE_TRY(ensure_cache(L->device, L->expert_bytes));
  for (int i = 0; i < n; ++i) {
    if (!ep_owned(ids[i], L->ep_rank, L->ep_world)) continue;   // another rank's expert
    int slot;
    MOE_TRY(cache_fetch(L, ids[i], 0, true, &slot));
  }
  return MOE_OK;
}

moe_status moe_check(moe_layer_t L) {
  g_err.clear();
  if (!L) return fail(MOE_ERR_INVALID_ARG, "null layer");
  MOE_TRY(check_device(L));
  MOE_TRY(wait_layer(L));
  if (!L->scratch) return MOE_OK;
  CUDA_TRY(cudaMemcpyAsync(L->h_err, L->wk.err, sizeof(unsigned), cudaMemcpyDeviceToHost, L->copy));
  CUDA_TRY(cudaStreamSynchronize(L->copy));
  const unsigned flags = *L->h_err;
  if (flags) {
    // a kernel that gave up may have left its step counters half-way: start
    // them from zero again (not the launch counter, words 4-5, which stays a
    // multiple of the grid: every CTA of every launch adds 1 at its start)
    CUDA_TRY(cudaMemsetAsync(L->wk.sync + 8, 0, (kSyncWords - 8) * sizeof(unsigned), L->copy));
    CUDA_TRY(cudaMemsetAsync(L->wk.err, 0, sizeof(unsigned), L->copy));
    CUDA_TRY(cudaStreamSynchronize(L->copy));
    if (flags & kErrBoundsBit)
      return fail(MOE_ERR_CUDA, "an index a kernel read from memory was out of range (flags 0x%x)", flags);
    return fail(MOE_ERR_CUDA, "a kernel of this layer gave up waiting (flags 0x%x)", flags);
  }
  return MOE_OK;
}

moe_status moe_get_stats(moe_stats* out) {
  g_err.clear();
  if (!out) return fail(MOE_ERR_INVALID_ARG, "null out");
  std::lock_guard<std::mutex> lk(g_mu);
  *out = g_stats;
  return MOE_OK;
}

moe_status moe_reset_stats(void) {
  g_err.clear();
  std::lock_guard<std::mutex> lk(g_mu);
  const uint64_t slots = g_stats.cache_slots, sb = g_stats.slot_bytes;
  g_stats = moe_stats{};
  g_stats.cache_slots = slots;
  g_stats.slot_bytes = sb;
  return MOE_OK;
}

moe_status moe_set_profiling(int enable) {
  g_err.clear();
  std::lock_guard<std::mutex> lk(g_mu);
  g_profiling = enable != 0;
  return MOE_OK;
}

moe_status moe_get_profile(moe_profile* out) {
  g_err.clear();
  if (!out) return fail(MOE_ERR_INVALID_ARG, "null out");
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    recs.swap(g_prof_pending);
  }
  moe_status st = MOE_OK;
  for (auto& r : recs) {
    for (int i = 0; i < r.n; ++i) {
      float ms = 0.f;
      cudaError_t e = cudaEventSynchronize(r.ev[2 * i + 1]);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.ev[2 * i], r.ev[2 * i + 1]);
      if (e != cudaSuccess) {
        st = fail(MOE_ERR_CUDA, "profile events: %s", cudaGetErrorString(e));
        continue;
      }
      out->ms[r.kid[i]] += ms;
      out->launches[r.kid[i]]++;
    }
    if (r.n > 0) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, r.ev[0], r.ev[2 * r.n - 1]) == cudaSuccess) {
        out->ms[MOE_K_FORWARD] += ms;
        out->launches[MOE_K_FORWARD]++;
      }
      out->forwards++;
    }
  }
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& r : recs)
    for (auto e : r.ev) g_prof_pool.push_back(e);
  return st;
}

moe_status moe_reset_profile(void) {
  g_err.clear();
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& r : g_prof_pending)
    for (auto e : r.ev) g_prof_pool.push_back(e);
  g_prof_pending.clear();
  return MOE_OK;
}

const char* moe_last_error(void) { return g_err.c_str(); }

}  // extern "C"
