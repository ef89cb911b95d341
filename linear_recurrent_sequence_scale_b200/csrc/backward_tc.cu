// Chunkwise backward for bf16 inputs, as three calls of the forward chunkwise
// form (which runs on the tensor cores where the shapes fit).
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations, Recurrent Form: S_n = gamma S_{n-1} + k_n^T v_n, o_n = q_n S_n,
// S_{-1} = S_in, S_out = S_{N-1}.  With G_n = dL/dS_n,
//     G_n = q_n^T dO_n + gamma G_{n+1},   G_{N-1} = q_{N-1}^T dO_{N-1} + dS_out,
//     dq_n = dO_n S_n^T,   dk_n = v_n G_n^T,   dv_n = k_n G_n,   dS_in = gamma G_0.
// Written out, each gradient is the retention operation again:
//   dq_n = sum_{m<=n} gamma^(n-m) (dO_n . v_m) k_m + gamma^(n+1) dO_n S_in^T
//        = the forward with (q, k, v) = (dO, V, K) and incoming state S_in^T;
//   in reversed time n' = N-1-n (rows of every tensor reversed),
//   dk'_n' = sum_{j'<=n'} gamma^(n'-j') (v'_n' . dO'_j') q'_j' + gamma^n' v'_n' dS_out^T
//        = the forward with (V', dO', Q') and incoming state dS_out^T / gamma;
//   dv'_n' = the forward with (K', Q', dO') and incoming state dS_out / gamma,
//   whose final state is G_0, so dS_in = gamma G_0.
// (The forward's incoming state decays by gamma^(n'+1), the final-state
// gradient by gamma^n', hence the division; for gamma = 0 only the last
// token sees dS_out, and a small pass adds v_{N-1} dS_out^T and
// k_{N-1} dS_out there.)
// The kernels here only move data: reverse the rows of a tensor, transpose
// and scale a float32 state, and that gamma = 0 correction.
#include "common.cuh"
#include "kernels.h"

namespace ret {
namespace bwdtc {

constexpr int kThreads = 256;

// dst[bh][N-1-n] = src[bh][n] for rows of d bf16 (d a multiple of 8), in
// 16-byte pieces.  In place (dst == src) each thread swaps a row pair.
__global__ void reverse_rows(const uint4* __restrict__ src, uint4* __restrict__ dst, int N,
                             int pieces, long long total) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const int c = static_cast<int>(t % pieces);
  const long long rest = t / pieces;
  const int n = static_cast<int>(rest % N);
  const long long bh = rest / N;
  const uint4* s = src + (bh * N) * pieces;
  uint4* d = dst + (bh * N) * pieces;
  if (src == dst) {
    if (2 * n >= N - 1) return;  // the upper half and the middle row
    const uint4 a = s[static_cast<long long>(n) * pieces + c];
    const uint4 b = s[static_cast<long long>(N - 1 - n) * pieces + c];
    d[static_cast<long long>(n) * pieces + c] = b;
    d[static_cast<long long>(N - 1 - n) * pieces + c] = a;
  } else {
    d[static_cast<long long>(N - 1 - n) * pieces + c] = s[static_cast<long long>(n) * pieces + c];
  }
}

// out[bh] = f(in[bh]) for [R][C] float32 states: transposed (out [C][R]) or
// not, times 1 / gamma_h (0 when gamma_h = 0) when inv_gamma, else times
// gamma_h when by_gamma, else as is.
__global__ void prep_state(const float* __restrict__ in, float* __restrict__ out,
                           const float* __restrict__ gammas, int H, int R, int C, int transpose,
                           int inv_gamma, int by_gamma, long long total) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const long long plane = static_cast<long long>(R) * C;
  const long long bh = t / plane;
  const int e = static_cast<int>(t - bh * plane);
  const int r = e / C, c = e - r * C;
  const float g = gammas[bh % H];
  float x = in[t];
  if (inv_gamma) x = g > 0.f ? x / g : 0.f;
  if (by_gamma) x *= g;
  out[bh * plane + (transpose ? static_cast<long long>(c) * R + r : e)] = x;
}

// For heads with gamma = 0 the final-state gradient reaches the last token
// only: dk_{N-1} += v_{N-1} dS_out^T and dv_{N-1} += k_{N-1} dS_out (bf16
// rows read, corrected in float32, rounded once).  One CTA per (b, h).
__global__ void gamma_zero_last_token(const __nv_bfloat16* __restrict__ k,
                                      const __nv_bfloat16* __restrict__ v,
                                      const float* __restrict__ ds, const float* __restrict__ gammas,
                                      __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                                      int H, int N, int DK, int DV) {
  const int bh = blockIdx.x;
  if (gammas[bh % H] != 0.f) return;
  const size_t last = static_cast<size_t>(bh) * N + (N - 1);
  const float* S = ds + static_cast<size_t>(bh) * DK * DV;
  for (int a = threadIdx.x; a < DK; a += blockDim.x) {  // dk_a += sum_b S[a][b] v_b
    float acc = 0.f;
    for (int b = 0; b < DV; ++b) acc = fmaf(S[static_cast<size_t>(a) * DV + b],
                                            __bfloat162float(v[last * DV + b]), acc);
    dk[last * DK + a] = __float2bfloat16_rn(__bfloat162float(dk[last * DK + a]) + acc);
  }
  for (int b = threadIdx.x; b < DV; b += blockDim.x) {  // dv_b += sum_a k_a S[a][b]
    float acc = 0.f;
    for (int a = 0; a < DK; ++a) acc = fmaf(__bfloat162float(k[last * DK + a]),
                                            S[static_cast<size_t>(a) * DV + b], acc);
    dv[last * DV + b] = __float2bfloat16_rn(__bfloat162float(dv[last * DV + b]) + acc);
  }
}

int blocks_for(long long n) { return static_cast<int>((n + kThreads - 1) / kThreads); }

}  // namespace bwdtc

cudaError_t launch_reverse_rows(const void* src, void* dst, int BH, int N, int d, cudaStream_t st) {
  const int pieces = d / 8;
  const long long total = static_cast<long long>(BH) * N * pieces;
  if (total == 0) return cudaSuccess;
  bwdtc::reverse_rows<<<bwdtc::blocks_for(total), bwdtc::kThreads, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), N, pieces, total);
  return cudaPeekAtLastError();
}

cudaError_t launch_prep_state(const float* in, float* out, const float* gammas, int BH, int H,
                              int R, int C, int transpose, int inv_gamma, int by_gamma,
                              cudaStream_t st) {
  const long long total = static_cast<long long>(BH) * R * C;
  bwdtc::prep_state<<<bwdtc::blocks_for(total), bwdtc::kThreads, 0, st>>>(
      in, out, gammas, H, R, C, transpose, inv_gamma, by_gamma, total);
  return cudaPeekAtLastError();
}

cudaError_t launch_gamma_zero_last_token(const void* k, const void* v, const float* ds,
                                         const float* gammas, void* dk, void* dv, int BH, int H,
                                         int N, int DK, int DV, cudaStream_t st) {
  bwdtc::gamma_zero_last_token<<<BH, 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), ds, gammas,
      static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), H, N, DK, DV);
  return cudaPeekAtLastError();
}

}  // namespace ret
