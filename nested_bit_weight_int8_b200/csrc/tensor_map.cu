// Host-side encoding of 2-D TMA tensor maps (through the driver entry point,
// so the library does not link libcuda directly), with a small cache keyed by
// (address, shape, box): a map only encodes where and how to read, so a cached
// map stays valid for any data later written at the same address.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <tuple>

#include "mq_internal.h"

namespace mq {
namespace {

std::mutex g_tm_mutex;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::map<std::tuple<const void*, uint64_t, uint64_t, uint32_t, uint32_t, int, int>, CUtensorMap> g_maps;

cudaError_t load_encoder() {
  if (g_encode) return cudaSuccess;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return e;
  if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

}  // namespace

cudaError_t encode_map_2d(CUtensorMap* out, const void* base, uint64_t rows, uint64_t row_elems,
                          uint32_t box_inner, uint32_t box_rows, int elem_bytes, int swizzle_bytes) {
  if (swizzle_bytes != 0 && swizzle_bytes != 32 && swizzle_bytes != 64 && swizzle_bytes != 128)
    return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lk(g_tm_mutex);
  auto key = std::make_tuple(base, rows, row_elems, box_inner, box_rows, elem_bytes, swizzle_bytes);
  auto it = g_maps.find(key);
  if (it != g_maps.end()) {
    *out = it->second;
    return cudaSuccess;
  }
  cudaError_t e = load_encoder();
  if (e != cudaSuccess) return e;
  CUtensorMap m;
  const cuuint64_t dims[2] = {row_elems, rows};
  const cuuint64_t strides[1] = {row_elems * static_cast<cuuint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = g_encode(&m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                        : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                        : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps.emplace(key, m);
  *out = m;
  return cudaSuccess;
}

}  // namespace mq
