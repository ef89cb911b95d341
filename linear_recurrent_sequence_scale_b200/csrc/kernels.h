// Internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ret {

cudaError_t launch_step(const void* q, const void* k, const void* v, const float* gammas,
                        float* state, void* o, int B, int H, int dk, int dv, int dtype,
                        float eps, cudaStream_t st);

size_t simt_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk);

cudaError_t launch_simt_chunkwise(const void* q, const void* k, const void* v,
                                  const float* gammas, int chunk, const float* state_in,
                                  float* state_out, void* o, int B, int H, int N, int dk, int dv,
                                  int dtype, float eps, void* ws, cudaStream_t st);

cudaError_t launch_simt_parallel(const void* q, const void* k, const void* v, const float* gammas,
                                 void* o, int B, int H, int N, int dk, int dv, int dtype,
                                 float eps, cudaStream_t st);

}  // namespace ret
