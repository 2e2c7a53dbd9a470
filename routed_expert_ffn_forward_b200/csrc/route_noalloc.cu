// moe_route_noalloc: the router step (logits, top-k, gating) for callers that
// cannot allocate device memory.
//
// Who needs it: a caller whose device memory is entirely owned by another
// allocator (a framework's caching allocator or a fixed arena carved out at
// start-up), or one on a latency-critical path that cannot afford the implicit
// device synchronisation of cudaMalloc/cudaFree, cannot create a moe_layer,
// because a layer allocates its own weights and scratch.  This entry point
// needs nothing but the caller's buffers: its only scratch, the [T, E] fp32
// logits, lives in a fixed-size array in the library's own device memory.
//
// The scratch array is shared by every call on a device and keeps the last
// call's contents.  Nothing in it needs to start at zero: the logits kernel
// writes every element the top-k kernel reads.  Calls whose kernels overlap
// on the GPU (different streams, no ordering between them) race on it.
#include <cstdio>
#include <mutex>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace {

// Largest T * E one call may use: 65536 fp32 logits = 256 KiB per device.
constexpr int kNoAllocMaxLogits = 65536;

static __device__ __align__(256) float g_noalloc_logits[kNoAllocMaxLogits];

// The array's device address, looked up once per device and context: a
// context that was destroyed and created again (cudaDeviceReset) loads the
// library's module afresh, so the address is looked up again for it.
constexpr int kMaxDevices = 64;
struct ScratchAddr {
  CUcontext ctx = nullptr;
  float* ptr = nullptr;
};
std::mutex g_noalloc_mu;
ScratchAddr g_noalloc_addr[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

moe_status fail(moe_status st, const char* msg) { return (moe_status)moe::report_error(st, msg); }

}  // namespace

extern "C" moe_status moe_route_noalloc(const void* x, const float* W, const float* bias, int T, int H,
                                        int E, int top_k, moe_gating gating, int32_t* ids,
                                        float* weights, void* stream) {
  moe::clear_error();
  char msg[256];
  if (T < 0 || H <= 0 || H % moe::kQK || E <= 0 || E > 1024 || top_k <= 0 || top_k > 32 || top_k > E) {
    snprintf(msg, sizeof msg, "bad shape T=%d H=%d E=%d top_k=%d (H multiple of 256, E <= 1024, top_k <= min(32, E))",
             T, H, E, top_k);
    return fail(MOE_ERR_INVALID_ARG, msg);
  }
  if (gating != MOE_GATE_SOFTMAX_TOPK && gating != MOE_GATE_SIGMOID_RENORM) return fail(MOE_ERR_INVALID_ARG, "bad gating");
  if ((long long)T * E > kNoAllocMaxLogits) {
    snprintf(msg, sizeof msg, "T*E = %lld exceeds the fixed scratch of %d logits", (long long)T * E,
             kNoAllocMaxLogits);
    return fail(MOE_ERR_UNSUPPORTED, msg);
  }
  if (T == 0) return MOE_OK;
  if (!x || !W || !ids || !weights) return fail(MOE_ERR_INVALID_ARG, "null pointer");
  // the logits kernel reads x and W in 16-byte vectors; bias, ids and weights
  // are read or written one 4-byte element at a time
  if (reinterpret_cast<uintptr_t>(x) & 15) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(W) & 15) return fail(MOE_ERR_INVALID_ARG, "W must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(bias) | reinterpret_cast<uintptr_t>(ids) | reinterpret_cast<uintptr_t>(weights)) & 3)
    return fail(MOE_ERR_INVALID_ARG, "bias, ids and weights must be 4-byte aligned");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "cudaGetDevice: %s", cudaGetErrorString(e));
    return fail(MOE_ERR_CUDA, msg);
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof msg, "device index %d >= %d", dev, kMaxDevices);
    return fail(MOE_ERR_UNSUPPORTED, msg);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scratch;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    CUcontext ctx = nullptr;
    CtxGetCurrentFn get_ctx = ctx_get_current();
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuCtxGetCurrent failed");
    ScratchAddr& sa = g_noalloc_addr[dev];
    if (!sa.ptr || sa.ctx != ctx) {
      // first call on this device (or in a new context): look up the device
      // address of the array; the host-side symbol is only a stand-in.  The
      // lookup may load the module, which a capturing stream does not allow.
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone)
        return fail(MOE_ERR_NOT_READY,
                    "the first call on this device must not be inside stream capture (it looks up the scratch address)");
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_logits);
      if (e != cudaSuccess) {
        (void)cudaGetLastError();
        snprintf(msg, sizeof msg, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        return fail(MOE_ERR_CUDA, msg);
      }
      // the lookup may have made the primary context current for the first time
      if (get_ctx(&ctx) != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuCtxGetCurrent failed");
      sa.ptr = static_cast<float*>(p);
      sa.ctx = ctx;
    }
    scratch = sa.ptr;
  }
  e = moe::launch_router_logits(static_cast<const __nv_bfloat16*>(x), W, bias, scratch, T, H, E, st);
  if (e == cudaSuccess) e = moe::launch_topk(scratch, T, E, top_k, (int)gating, nullptr, ids, weights, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    snprintf(msg, sizeof msg, "kernel launch: %s", cudaGetErrorString(e));
    return fail(MOE_ERR_CUDA, msg);
  }
  return MOE_OK;
}
