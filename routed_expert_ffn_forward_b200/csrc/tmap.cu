// Tensor maps (TMA descriptors) over the expert weight matrices.
//
// A matrix of R rows and nb groups of 256 weights per row (sbb device bytes
// per group: 144 for Q4_K, see dev_sb_bytes) is viewed as a 2-D array of
// 8-byte elements, nb*sbb/8 wide and R high (row pitch nb*sbb bytes, a
// multiple of 16).  A box is 64 or 128 rows by a few groups; boxes past the
// last row or group read zeros, which decode to zero weights.  16-bit operand matrices of the tensor-core GEMMs (activations,
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

// Matrix of `rows` rows of nb groups of `sbb` bytes (a multiple of 16), boxes
// of box_rows rows x box_blocks groups.
cudaError_t encode_q4k(CUtensorMap* m, const uint8_t* base, int rows, int nb, int box_blocks, int box_rows,
                       int sbb = kQBytes) {
  EncodeFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const int el = sbb / 8;   // 8-byte elements per group
  const cuuint64_t dims[2] = {(cuuint64_t)nb * el, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)nb * sbb};
  const cuuint32_t box[2] = {(cuuint32_t)(box_blocks * el), (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t encode_expert_maps(CUtensorMap* maps, const uint8_t* base, const Shape& s) {
  const int H = s.H, I = s.I, nbh = s.nbh, nbi = s.nbi;
  const size_t gate_bytes = (size_t)I * s.drow_gu;
  const uint8_t* mats[3] = {base, base + gate_bytes, base + 2 * gate_bytes};
  const int rows[3] = {I, I, H}, nb[3] = {nbh, nbh, nbi}, sbb[3] = {s.sbb_gu, s.sbb_gu, s.sbb_d};
  cudaError_t e = cudaSuccess;
  for (int m = 0; m < 3 && e == cudaSuccess; ++m)
    e = encode_q4k(&maps[m], mats[m], rows[m], nb[m], m < 2 ? 2 : 4, kTileRows, sbb[m]);
  for (int m = 0; m < 3 && e == cudaSuccess; ++m) e = encode_q4k(&maps[3 + m], mats[m], rows[m], nb[m], 1, 128, sbb[m]);
  if (e == cudaSuccess) e = encode_q4k(&maps[6], mats[2], rows[2], nb[2], 1, 64, sbb[2]);
  for (int m = 0; m < 2 && e == cudaSuccess; ++m) e = encode_q4k(&maps[7 + m], mats[m], rows[m], nb[m], 1, 64, sbb[m]);
  return e;
}

cudaError_t copy_matrix_h2d(uint8_t* dst, const uint8_t* src, int rows, int q, size_t hrow, size_t drow,
                            cudaStream_t st) {
  if (hrow == drow) return cudaMemcpyAsync(dst, src, (size_t)rows * hrow, cudaMemcpyHostToDevice, st);
  // each GGUF block (Q6_K, 210 bytes) or group of eight (MXFP4, 136 bytes)
  // into its 16-byte-aligned device slot
  const size_t hb = q == kQ6_K ? 210 : q == kMXFP4 ? 136 : 0;
  const size_t db = (size_t)dev_sb_bytes(q);
  if (!hb || hrow % hb || drow % db || hrow / hb != drow / db) return cudaErrorInvalidValue;
  return cudaMemcpy2DAsync(dst, db, src, hb, hb, (size_t)rows * (hrow / hb), cudaMemcpyHostToDevice, st);
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
