// Tensor maps (TMA descriptors) over Q4_K expert matrices.
//
// A matrix of R rows and nb super-blocks per row is viewed as a 2-D array of
// 8-byte elements, nb*18 wide and R high (row pitch nb*144 bytes, a multiple
// of 16).  A box is 64 rows by SB super-blocks (SB*18 elements, SB*144 bytes);
// boxes past the last row or block read zeros, which decode to zero weights.
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

cudaError_t encode_q4k(CUtensorMap* m, const uint8_t* base, int rows, int nb, int box_blocks) {
  EncodeFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)nb * 18, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)nb * kQBytes};
  const cuuint32_t box[2] = {(cuuint32_t)box_blocks * 18, (cuuint32_t)kTileRows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t encode_expert_maps(CUtensorMap* maps3, const uint8_t* base, int H, int I) {
  const int nbh = H / kQK, nbi = (I + kQK - 1) / kQK;
  const size_t gate_bytes = (size_t)I * nbh * kQBytes;
  cudaError_t e = encode_q4k(&maps3[0], base, I, nbh, 2);
  if (e == cudaSuccess) e = encode_q4k(&maps3[1], base + gate_bytes, I, nbh, 2);
  if (e == cudaSuccess) e = encode_q4k(&maps3[2], base + 2 * gate_bytes, H, nbi, 4);
  return e;
}

}  // namespace moe
