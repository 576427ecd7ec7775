// TMA tensor-map encoding (see tma_host.h).
#include <mutex>

#include "tma_host.h"

namespace tpa {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

}  // namespace

namespace {

cudaError_t encode_uncached(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                            uint32_t box_rows, int swizzle_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (swizzle_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  if (swizzle_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  if (swizzle_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The last kMapCache descriptions encoded on this host thread.  A map depends only on these
// arguments (an address range and its tiling), so a hit is the map the driver would return.
constexpr int kMapCache = 32;
struct MapEntry {
  const void* base;
  uint64_t inner, rows;
  uint32_t box_inner, box_rows;
  int swizzle;
  bool valid;
  CUtensorMap map;
};
thread_local MapEntry t_maps[kMapCache];
thread_local int t_next = 0;

}  // namespace

cudaError_t encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                           uint32_t box_rows, int swizzle_bytes) {
  for (const MapEntry& e : t_maps) {
    if (e.valid && e.base == base && e.inner == inner && e.rows == rows && e.box_inner == box_inner &&
        e.box_rows == box_rows && e.swizzle == swizzle_bytes) {
      *map = e.map;
      return cudaSuccess;
    }
  }
  const cudaError_t r = encode_uncached(map, base, inner, rows, box_inner, box_rows, swizzle_bytes);
  if (r != cudaSuccess) return r;
  MapEntry& e = t_maps[t_next];
  t_next = (t_next + 1) % kMapCache;
  e = MapEntry{base, inner, rows, box_inner, box_rows, swizzle_bytes, true, *map};
  return cudaSuccess;
}

}  // namespace tpa
