// State prefix for a sequence split into spans held by different GPUs.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations, Chunkwise Recurrent: the state carried from one chunk to the next
// is R_i = gamma^L R_{i-1} + (the chunk's own contribution).  Applied to spans
// of a sequence, with S_local(g) the end state of span g computed from a zero
// state and N_g its length,
//     S_in(0) = S0,   S_in(g + 1) = gamma^(N_g) S_in(g) + S_local(g),
// so the state entering span r is
//     S_in(r) = gamma^(N_0 + ... + N_(r-1)) S0
//             + sum over g < r of gamma^(N_(g+1) + ... + N_(r-1)) S_local(g).
// One thread per four state elements walks g = 0 .. r-1 in order; the work is
// a read of r + 1 states and a write of one, bound by HBM.
#include "common.cuh"
#include "kernels.h"

namespace ret {

struct Spans {
  int n[kMaxSpans];
};

__global__ void state_combine_kernel(const float4* __restrict__ locals, Spans spans, int r,
                                     const float* __restrict__ gammas,
                                     const float4* __restrict__ state0, float4* __restrict__ out,
                                     int H, size_t per_head4, size_t total4) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total4;
       e += (size_t)gridDim.x * blockDim.x) {
    const int h = static_cast<int>((e / per_head4) % H);
    const float lg = log2f(gammas[h]);
    float4 acc = state0 ? state0[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < r; ++g) {
      const float d = gpow(lg, spans.n[g]);
      const float4 s = locals[(size_t)g * total4 + e];
      acc.x = fmaf(d, acc.x, s.x);
      acc.y = fmaf(d, acc.y, s.y);
      acc.z = fmaf(d, acc.z, s.z);
      acc.w = fmaf(d, acc.w, s.w);
    }
    out[e] = acc;
  }
}

cudaError_t launch_state_combine(const float* locals, const int* spans, int r,
                                 const float* gammas, const float* state0, float* out, int B,
                                 int H, int dk, int dv, cudaStream_t st) {
  Spans sp = {};
  for (int g = 0; g < r; ++g) sp.n[g] = spans[g];
  const size_t per_head4 = (size_t)dk * dv / 4;
  const size_t total4 = (size_t)B * H * per_head4;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const size_t want = (total4 + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < (size_t)nsm * 8 ? want : (size_t)nsm * 8);
  state_combine_kernel<<<grid, 256, 0, st>>>(
      reinterpret_cast<const float4*>(locals), sp, r, gammas,
      reinterpret_cast<const float4*>(state0), reinterpret_cast<float4*>(out), H, per_head4,
      total4);
  return cudaPeekAtLastError();
}

}  // namespace ret
