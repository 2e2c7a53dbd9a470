// Tensor maps (TMA descriptors) over the expert weight matrices, and their
// upload.
//
// In device memory a matrix of R rows and nb groups of 256 weights per row
// (sbb bytes per group: 144 for Q4_K, see dev_sb_bytes) is stored tile-major:
// for every tile of 64 rows, group after group, the tile's 64 rows of that
// group (64*sbb contiguous bytes); the rows of the last tile past R are
// zeros.  A kernel's box -- 64 or 128 rows by one or a few groups -- is then
// one to four contiguous runs of 9 KB or more instead of 64 to 128 pieces of
// sbb bytes a row pitch apart, which the DRAM streams markedly faster (a
// probe of 148 MB through the same TMA ring: 3.8 TB/s in row pieces, 4.3 TB/s
// contiguous; 4.4 against 5.7 TB/s over 594 MB).  The map is 4-D over 8-byte
// elements: (sbb/8, 64 rows, nb groups, R/64 tiles); a box (sbb/8, 64, k, t)
// lands in shared memory as [t][k][64 rows][sbb]: for one group, rows in
// order; for k groups, group after group.  Boxes past the last tile read
// zeros.  16-bit operand matrices of the tensor-core GEMMs (activations,
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

// Tile-major matrix of `rows` rows of nb groups of `sbb` bytes (a multiple of
// 16), boxes of box_rows (64 or 128) rows x box_blocks groups.
cudaError_t encode_q4k(CUtensorMap* m, const uint8_t* base, int rows, int nb, int box_blocks, int box_rows,
                       int sbb = kQBytes) {
  EncodeFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (box_rows % kWTile || sbb % 16) return cudaErrorInvalidValue;
  const int el = sbb / 8;   // 8-byte elements per group
  const cuuint64_t tiles = (cuuint64_t)((rows + kWTile - 1) / kWTile);
  const cuuint64_t dims[4] = {(cuuint64_t)el, (cuuint64_t)kWTile, (cuuint64_t)nb, tiles};
  const cuuint64_t strides[3] = {(cuuint64_t)sbb, (cuuint64_t)kWTile * sbb, (cuuint64_t)nb * kWTile * sbb};
  const cuuint32_t box[4] = {(cuuint32_t)el, (cuuint32_t)kWTile, (cuuint32_t)box_blocks,
                             (cuuint32_t)(box_rows / kWTile)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 4, const_cast<uint8_t*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t encode_expert_maps(CUtensorMap* maps, const uint8_t* base, const Shape& s) {
  const int H = s.H, I = s.I, nbh = s.nbh, nbi = s.nbi;
  const size_t gate_bytes = tiled_matrix_bytes(I, s.drow_gu);
  const uint8_t* mats[3] = {base, base + gate_bytes, base + 2 * gate_bytes};
  const int rows[3] = {I, I, H}, nb[3] = {nbh, nbh, nbi}, sbb[3] = {s.sbb_gu, s.sbb_gu, s.sbb_d};
  cudaError_t e = cudaSuccess;
  for (int m = 0; m < 3 && e == cudaSuccess; ++m)
    e = encode_q4k(&maps[m], mats[m], rows[m], nb[m], m < 2 ? 2 : 4, kTileRows, sbb[m]);
  for (int m = 0; m < 3 && e == cudaSuccess; ++m) e = encode_q4k(&maps[3 + m], mats[m], rows[m], nb[m], 1, 128, sbb[m]);
  return e;
}

namespace {

// Row-major device rows (rows x nb groups of sbb bytes) -> tile-major, the
// rows of the last tile past `rows` zeroed.  Block b copies group b % nb of
// tile b / nb.
__global__ void __launch_bounds__(256) retile_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int rows,
                                                     int nb, int sbb) {
  const int tile = blockIdx.x / nb, g = blockIdx.x - tile * nb;
  const int v = sbb / 16;                         // 16-byte vectors per group
  uint4* out = dst + (size_t)blockIdx.x * kWTile * v;
  for (int i = threadIdx.x; i < kWTile * v; i += blockDim.x) {
    const int r = tile * kWTile + i / v, c = i - (i / v) * v;
    out[i] = r < rows ? src[((size_t)r * nb + g) * v + c] : make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

cudaError_t launch_retile(const uint8_t* staging, uint8_t* dst, int rows, int nb, int sbb, cudaStream_t st) {
  if (sbb % 16 || rows <= 0 || nb <= 0) return cudaErrorInvalidValue;
  const int tiles = (rows + kWTile - 1) / kWTile;
  retile_kernel<<<tiles * nb, 256, 0, st>>>(reinterpret_cast<const uint4*>(staging), reinterpret_cast<uint4*>(dst),
                                            rows, nb, sbb);
  return cudaGetLastError();
}

cudaError_t upload_matrix(uint8_t* dst, const uint8_t* src, int rows, int q, size_t hrow, size_t drow, int nb,
                          int sbb, uint8_t* staging, cudaStream_t st) {
  if (drow != (size_t)nb * sbb) return cudaErrorInvalidValue;
  cudaError_t e = copy_matrix_h2d(staging, src, rows, q, hrow, drow, st);
  return e == cudaSuccess ? launch_retile(staging, dst, rows, nb, sbb, st) : e;
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
