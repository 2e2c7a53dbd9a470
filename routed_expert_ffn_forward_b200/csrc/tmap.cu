// Tensor maps (TMA descriptors) over Q4_K expert matrices.
//
// A matrix of R rows and nb super-blocks per row is viewed as a 2-D array of
// 8-byte elements, nb*18 wide and R high (row pitch nb*144 bytes, a multiple
// of 16).  A box is 64 or 128 rows by SB super-blocks (SB*18 elements, SB*144
// bytes); boxes past the last row or block read zeros, which decode to zero
// weights.  16-bit operand matrices of the tensor-core GEMMs (activations,
// router planes) use 128-byte-swizzled boxes of 64 columns.
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

cudaError_t encode_q4k(CUtensorMap* m, const uint8_t* base, int rows, int nb, int box_blocks, int box_rows) {
  EncodeFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)nb * 18, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)nb * kQBytes};
  const cuuint32_t box[2] = {(cuuint32_t)box_blocks * 18, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t encode_expert_maps(CUtensorMap* maps, const uint8_t* base, int H, int I) {
  const int nbh = H / kQK, nbi = (I + kQK - 1) / kQK;
  const size_t gate_bytes = (size_t)I * nbh * kQBytes;
  const uint8_t* mats[3] = {base, base + gate_bytes, base + 2 * gate_bytes};
  const int rows[3] = {I, I, H}, nb[3] = {nbh, nbh, nbi};
  cudaError_t e = cudaSuccess;
  for (int m = 0; m < 3 && e == cudaSuccess; ++m) e = encode_q4k(&maps[m], mats[m], rows[m], nb[m], m < 2 ? 2 : 4, kTileRows);
  for (int m = 0; m < 3 && e == cudaSuccess; ++m) e = encode_q4k(&maps[3 + m], mats[m], rows[m], nb[m], 1, 128);
  return e;
}

cudaError_t encode_sw128_16(CUtensorMap* map, const void* base, bool bf16, size_t rows, int cols, int box_rows) {
  return encode_swz_16(map, base, bf16, rows, cols, box_rows, 64);
}

cudaError_t encode_swz_16(CUtensorMap* map, const void* base, bool bf16, size_t rows, int cols, int box_rows,
                          int box_cols) {
  EncodeFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if ((box_cols != 64 && box_cols != 32) || cols % box_cols || rows == 0 || box_rows <= 0 || box_rows > 256)
    return cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace moe
