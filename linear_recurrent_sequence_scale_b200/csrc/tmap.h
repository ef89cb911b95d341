// Host-side creation of TMA tensor maps (driver entry point looked up at run
// time through the CUDA runtime, so the library does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ret {

// 3-D bf16 tensor [d2][d1][d0] (d0 contiguous), 128-byte swizzle, box
// {box0, box1, 1}; out-of-range elements read as zero.  Returns cudaSuccess
// or an error code (cudaErrorInvalidValue when the driver rejects the map).
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint32_t box0, uint32_t box1);

}  // namespace ret
