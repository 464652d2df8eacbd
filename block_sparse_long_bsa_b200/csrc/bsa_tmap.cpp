// Host-side TMA tensor-map encoding shared by the kernels' launchers.
#include "bsa_tmap.h"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <string>

#include "bsa_internal.h"

namespace bsa {
namespace tmap {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
int g_encode_status = BSA_OK;
std::string g_encode_msg;

int encode_tiled(CUtensorMap* m, const void* ptr, cuuint32_t rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")");
  return BSA_OK;
}

}  // namespace

int get_encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q{};
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
      g_encode_status = BSA_ERR_CUDA;
      g_encode_msg = std::string("cuTensorMapEncodeTiled unavailable: ") + cudaGetErrorString(e);
      return;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode_status != BSA_OK) return set_error(g_encode_status, g_encode_msg);
  return BSA_OK;
}

int encode_rows(CUtensorMap* m, const void* ptr, int slices, int n, int d, int rows) {
  const cuuint64_t row = cuuint64_t(d) * 2, slice = cuuint64_t(n) * row;
  if (d == 128) {
    const cuuint64_t dims[4] = {64, cuuint64_t(n), 2, cuuint64_t(slices)};
    const cuuint64_t str[3] = {row, 128, slice};
    const cuuint32_t box[4] = {64, cuuint32_t(rows), 2, 1};
    return encode_tiled(m, ptr, 4, dims, str, box);
  }
  const cuuint64_t dims[3] = {64, cuuint64_t(n), cuuint64_t(slices)};
  const cuuint64_t str[2] = {row, slice};
  const cuuint32_t box[3] = {64, cuuint32_t(rows), 1};
  return encode_tiled(m, ptr, 3, dims, str, box);
}

int encode_q(CUtensorMap* m, const void* ptr, int heads, int n, int d, int blk) {
  const cuuint64_t row = cuuint64_t(d) * 2, slice = cuuint64_t(n) * row;
  if (d == 128 && blk == 64) {
    const cuuint64_t dims[4] = {64, cuuint64_t(n), cuuint64_t(heads), 2};
    const cuuint64_t str[3] = {row, slice, 128};
    const cuuint32_t box[4] = {64, 64, 2, 2};
    return encode_tiled(m, ptr, 4, dims, str, box);
  }
  if (d == 128) return encode_rows(m, ptr, heads, n, d, 128);
  const cuuint64_t dims[3] = {64, cuuint64_t(n), cuuint64_t(heads)};
  const cuuint64_t str[2] = {row, slice};
  const cuuint32_t box[3] = {64, cuuint32_t(blk), cuuint32_t(blk == 64 ? 2 : 1)};
  return encode_tiled(m, ptr, 3, dims, str, box);
}

int encode_atoms(CUtensorMap* m, const void* ptr, int slices, int n, int d, int rows) {
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(n), cuuint64_t(slices)};
  const cuuint64_t str[2] = {cuuint64_t(d) * 2, cuuint64_t(n) * cuuint64_t(d) * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(rows), 1};
  return encode_tiled(m, ptr, 3, dims, str, box);
}

int encode_o(CUtensorMap* m, const void* ptr, int heads, int n, int d) {
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(n), cuuint64_t(heads)};
  const cuuint64_t str[2] = {cuuint64_t(d) * 2, cuuint64_t(n) * cuuint64_t(d) * 2};
  const cuuint32_t box[3] = {64, 32, 1};
  return encode_tiled(m, ptr, 3, dims, str, box);
}

}  // namespace tmap
}  // namespace bsa
