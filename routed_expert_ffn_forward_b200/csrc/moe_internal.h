// Internal declarations shared by the host runtime and the kernel files of
// libmoe.so.  Nothing here is part of the C ABI (include/moe.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace moe {

constexpr int kQK = 256;        // weights per Q4_K super-block
constexpr int kQBytes = 144;    // bytes per Q4_K super-block
constexpr int kDecodeMaxT = 64; // T <= this takes the decode path

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
};

struct Shape {
  int H, I, E, k, S;
  int nbh;    // super-blocks per gate/up row  = H / 256
  int nbi;    // super-blocks per down row     = ceil(I / 256)
  int I_pad;  // nbi * 256
  int n_sm;   // streaming multiprocessors of the device
};

// ---- kernels (one launch helper per kernel; all enqueue on `st`) ----------
cudaError_t launch_router_logits(const __nv_bfloat16* x, const float* W, const float* b,
                                 float* logits, int T, int H, int E, cudaStream_t st);
cudaError_t launch_topk(const float* logits, int T, int E, int k, int gating,
                        const int* forced, int* ids, float* w, cudaStream_t st);
cudaError_t launch_permute(const int* ids, int T, const Shape& s, const Work& wk, cudaStream_t st);
cudaError_t launch_gate_up_simt(const uint8_t* const* wptr, const __nv_bfloat16* x, const Shape& s,
                                const Work& wk, cudaStream_t st);
cudaError_t launch_down_simt(const uint8_t* const* wptr, const Shape& s, const Work& wk, cudaStream_t st);
cudaError_t launch_combine(const Work& wk, int T, const Shape& s, __nv_bfloat16* out, cudaStream_t st);

// Streaming cache: point experts at their cache slots (device pointer table).
struct PtrUpdate {
  static constexpr int kMax = 64;
  int n;
  int expert[kMax];
  const uint8_t* base[kMax];
};
cudaError_t launch_set_ptrs(const uint8_t** table, const PtrUpdate& u, size_t gate_bytes,
                            cudaStream_t st);

// Set / clear the thread-local message returned by moe_last_error().
int report_error(int status, const char* msg);
void clear_error();

// ---- device helpers -------------------------------------------------------
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
#endif

}  // namespace moe
