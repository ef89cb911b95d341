// Chunkwise retention for callers that cannot allocate device memory.
//
// Some callers of this library own no allocator: a plugin inside a host
// runtime that has already reserved all device memory in its own pool and
// gives plugins no way to ask for more, or a latency-critical loop where a
// cudaMalloc/cudaFree (which can synchronise the whole device) is not
// acceptable.  ret_chunkwise needs scratch space for the per-chunk states;
// this entry point takes it from a fixed array compiled into the library
// instead of from the caller.
//
// The array lives in device memory of every GPU that loads the library, for
// as long as the process runs.  Its device address is looked up on the first
// call made with that device current, and kept once the lookup succeeds (a
// failed lookup, say inside a stream capture, is retried on the next call).
// The stream passed in must belong to the current device: the array used is
// the current device's copy.  All calls share the one array, so calls that
// overlap on the GPU (different streams, or different host threads on the
// same device) race on it and must be serialised by the caller.  The array keeps whatever the last call left in
// it; nothing needs to start at zero, because the chunkwise kernels write
// every state slot before they read it.
#include <cuda_runtime.h>

#include <mutex>

#include "retention.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[RET_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Per device: the array's device address once a lookup has succeeded (null
// until then).  A failed lookup is not remembered, so a later call retries it.
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu[kMaxDevices];

// This device's copy of the array (the current device), or null if the
// runtime could not give its address.
void* scratch_for(int dev) {
  std::lock_guard<std::mutex> lock(g_scratch_mu[dev]);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int ret_chunkwise_noalloc(const void* q, const void* k, const void* v,
                                     const float* gammas, int chunk, const float* state_in,
                                     float* state_out, void* o, int B, int H, int N, int dk,
                                     int dv, int dtype, float gn_eps, void* stream) {
  // Size check first: it needs no device and gives the clearest error.
  const size_t need = ret_chunkwise_workspace(B, H, N, dk, dv, chunk, dtype);
  if (need > RET_NOALLOC_SCRATCH_BYTES) return RET_EWORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RET_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return RET_EUNSUPPORTED;
  // Host code may not use the array's name as an address: ask the runtime
  // for this device's copy (with the device current; cached once found).
  void* scratch = scratch_for(dev);
  if (!scratch) return RET_ECUDA;
  return ret_chunkwise(q, k, v, gammas, chunk, state_in, state_out, o, B, H, N, dk, dv, dtype,
                       gn_eps, scratch, RET_NOALLOC_SCRATCH_BYTES, stream);
}
