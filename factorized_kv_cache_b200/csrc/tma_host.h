// Host-side TMA tensor-map encoding through the driver entry point (no link
// against libcuda): 2-D row-major bf16 tiles.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

namespace tpa {

// rows x inner bf16 elements, row pitch inner*2 bytes; box = box_rows x box_inner;
// swizzle_bytes in {0, 32, 64, 128}.  Returns cudaErrorInvalidValue when the
// driver rejects the description.  Recently encoded maps are kept per host
// thread and returned without a driver call.
cudaError_t encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                           uint32_t box_rows, int swizzle_bytes);

}  // namespace tpa
