// Float32 CUDA-core kernels for the chunkwise and parallel forms.
//
// These serve float32 inputs, whose 1e-5 tolerance rules out bf16/tf32
// tensor-core operands.  Two kernels:
//
//  simt_state_scan  - per (b, h, 64x64 state tile): walks the chunks in order,
//                     stores the state entering each chunk (R_{i-1}) to the
//                     workspace, then applies
//                     R_i = gamma^L R_{i-1} + K_[i]^T (V_[i] (.) zeta).
//  simt_chunk_out   - per (b, h, 16-row query tile inside one chunk):
//                     O = (Q K^T (.) D) V + (Q (.) xi) R_{i-1}, then the
//                     optional GroupNorm over d_v.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations (Parallel Form, Chunkwise Recurrent).  xi_j = gamma^(j+1) and
// zeta_j = gamma^(L-1-j) for in-chunk position j of a chunk of length L.  The
// parallel form is the single-chunk case (chunk = N) without a state.
#include "common.cuh"
#include "kernels.h"

namespace ret {

constexpr int SC_T = 64;   // state tile edge
constexpr int SC_J = 32;   // tokens staged per step

template <typename T>
__global__ void __launch_bounds__(256)
simt_state_scan(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ gammas,
                int chunk, const float* state_in, float* state_out, float* __restrict__ rws,
                int H, int N, int dk, int dv) {
  __shared__ float ks[SC_J][SC_T];
  __shared__ float vs[SC_J][SC_T];
  const int bh = blockIdx.z;
  const int h = bh % H;
  const int r0 = blockIdx.y * SC_T;
  const int c0 = blockIdx.x * SC_T;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const float lg = log2f(gammas[h]);
  const int nc = cdiv(N, chunk);

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
      acc[i][j] = (state_in && r < dk && c < dv) ? state_in[((size_t)bh * dk + r) * dv + c] : 0.f;
    }

  for (int ci = 0; ci < nc; ++ci) {
    if (rws) {
      float* R = rws + ((size_t)bh * nc + ci) * dk * dv;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
          if (r < dk && c < dv) R[(size_t)r * dv + c] = acc[i][j];
        }
    }
    const int s = ci * chunk;
    const int L = min(chunk, N - s);
    const float gL = gpow(lg, L);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= gL;
    for (int j0 = 0; j0 < L; j0 += SC_J) {
      __syncthreads();
      for (int e = tid; e < SC_J * SC_T; e += 256) {
        const int jj = e / SC_T, x = e % SC_T;
        const int j = j0 + jj;
        const size_t tok = (size_t)bh * N + s + j;
        float kv = 0.f, vv = 0.f;
        if (j < L) {
          if (r0 + x < dk) kv = Elem<T>::ld(k + tok * dk + r0 + x);
          if (c0 + x < dv) vv = Elem<T>::ld(v + tok * dv + c0 + x) * gpow(lg, L - 1 - j);
        }
        ks[jj][x] = kv;
        vs[jj][x] = vv;
      }
      __syncthreads();
#pragma unroll 4
      for (int jj = 0; jj < SC_J; ++jj) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = ks[jj][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = vs[jj][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
    }
  }
  if (state_out) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
        if (r < dk && c < dv) state_out[((size_t)bh * dk + r) * dv + c] = acc[i][j];
      }
  }
}

constexpr int CO_M = 16;    // query rows per CTA
constexpr int CO_K = 16;    // keys (or state rows) staged per step
constexpr int CO_U = 32;    // max columns per thread: dv <= 16 * CO_U = 512

template <typename T, bool GN>
__global__ void __launch_bounds__(256)
simt_chunk_out(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
               const float* __restrict__ gammas, int chunk, const float* __restrict__ rws,
               const T* __restrict__ gate, T* __restrict__ o, int H, int N, int dk, int dv,
               float eps) {
  extern __shared__ float sm[];
  const int ldq = dk + 1;
  float* qs = sm;                        // [CO_M][dk+1]
  float* ks = qs + CO_M * ldq;           // [CO_K][dk+1]
  float* vs = ks + CO_K * ldq;           // [CO_K][dv]   (V rows, then R rows)
  float* ps = vs + CO_K * dv;            // [CO_M][CO_K+1]
  float* red = ps + CO_M * (CO_K + 1);   // [16][CO_M]

  const int bh = blockIdx.y;
  const int h = bh % H;
  const int tpc = cdiv(chunk, CO_M);
  const int ci = blockIdx.x / tpc;
  const int ti = blockIdx.x % tpc;
  const int cs = ci * chunk;
  const int n0 = cs + ti * CO_M;
  const int ce = min(N, cs + chunk);
  if (n0 >= ce) return;
  const int nrows = min(CO_M, ce - n0);
  const int nc = cdiv(N, chunk);
  const int tid = threadIdx.x;
  const int row = tid & 15;
  const int cgp = tid >> 4;
  const float lg = log2f(gammas[h]);

  for (int e = tid; e < CO_M * dk; e += 256) {
    const int r = e / dk, x = e % dk;
    qs[r * ldq + x] = r < nrows ? Elem<T>::ld(q + ((size_t)bh * N + n0 + r) * dk + x) : 0.f;
  }

  float acc[CO_U];
#pragma unroll
  for (int u = 0; u < CO_U; ++u) acc[u] = 0.f;

  const int kend = n0 + nrows;  // keys past the last query row contribute nothing
  for (int m0 = cs; m0 < kend; m0 += CO_K) {
    __syncthreads();
    for (int e = tid; e < CO_K * dk; e += 256) {
      const int r = e / dk, x = e % dk;
      ks[r * ldq + x] = (m0 + r < kend) ? Elem<T>::ld(k + ((size_t)bh * N + m0 + r) * dk + x) : 0.f;
    }
    for (int e = tid; e < CO_K * dv; e += 256) {
      const int r = e / dv, x = e % dv;
      vs[r * dv + x] = (m0 + r < kend) ? Elem<T>::ld(v + ((size_t)bh * N + m0 + r) * dv + x) : 0.f;
    }
    __syncthreads();
    {
      const int sr = tid >> 4, sk = tid & 15;
      const int n = n0 + sr, m = m0 + sk;
      float dot = 0.f;
      for (int x = 0; x < dk; ++x) dot = fmaf(qs[sr * ldq + x], ks[sk * ldq + x], dot);
      const float d = (m <= n && sr < nrows) ? gpow(lg, n - m) : 0.f;
      ps[sr * (CO_K + 1) + sk] = dot * d;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < CO_K; ++kk) {
      const float p = ps[row * (CO_K + 1) + kk];
#pragma unroll
      for (int u = 0; u < CO_U; ++u) {
        const int c = cgp + 16 * u;
        if (c < dv) acc[u] = fmaf(p, vs[kk * dv + c], acc[u]);
      }
    }
  }

  if (rws) {
    const float* R = rws + ((size_t)bh * nc + ci) * dk * dv;
    const float xi = gpow(lg, n0 + row - cs + 1);
    float acc2[CO_U];
#pragma unroll
    for (int u = 0; u < CO_U; ++u) acc2[u] = 0.f;
    for (int r0 = 0; r0 < dk; r0 += CO_K) {
      __syncthreads();
      for (int e = tid; e < CO_K * dv; e += 256) {
        const int r = e / dv, x = e % dv;
        vs[r * dv + x] = (r0 + r < dk) ? R[(size_t)(r0 + r) * dv + x] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < CO_K; ++kk) {
        const float a = (r0 + kk < dk) ? qs[row * ldq + r0 + kk] : 0.f;
#pragma unroll
        for (int u = 0; u < CO_U; ++u) {
          const int c = cgp + 16 * u;
          if (c < dv) acc2[u] = fmaf(a, vs[kk * dv + c], acc2[u]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < CO_U; ++u) acc[u] = fmaf(xi, acc2[u], acc[u]);
  }

  if constexpr (GN) {
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < CO_U; ++u)
      if (cgp + 16 * u < dv) s += acc[u];
    __syncthreads();
    red[cgp * CO_M + row] = s;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < 16; ++i) tot += red[i * CO_M + row];
    const float mean = tot / static_cast<float>(dv);
    float s2 = 0.f;
#pragma unroll
    for (int u = 0; u < CO_U; ++u)
      if (cgp + 16 * u < dv) {
        acc[u] -= mean;
        s2 = fmaf(acc[u], acc[u], s2);
      }
    __syncthreads();
    red[cgp * CO_M + row] = s2;
    __syncthreads();
    float sq = 0.f;
    for (int i = 0; i < 16; ++i) sq += red[i * CO_M + row];
    const float inv = 1.0f / sqrtf(sq / static_cast<float>(dv) + eps);
#pragma unroll
    for (int u = 0; u < CO_U; ++u) acc[u] *= inv;
  }

  if (row < nrows) {
    T* orow = o + ((size_t)bh * N + n0 + row) * dv;
    const T* grow = gate ? gate + ((size_t)bh * N + n0 + row) * dv : nullptr;
#pragma unroll
    for (int u = 0; u < CO_U; ++u) {
      const int c = cgp + 16 * u;
      if (c < dv) Elem<T>::st(orow + c, grow ? acc[u] * swishf(Elem<T>::ld(grow + c)) : acc[u]);
    }
  }
}

static size_t chunk_out_smem(int dk, int dv) {
  return sizeof(float) * (size_t)(CO_M * (dk + 1) + CO_K * (dk + 1) + CO_K * dv +
                                  CO_M * (CO_K + 1) + 16 * CO_M);
}

size_t simt_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk) {
  const size_t nc = (size_t)cdiv(N, chunk);
  return sizeof(float) * (size_t)B * H * nc * dk * dv;
}

template <typename T, bool GN>
static cudaError_t launch_out(const void* q, const void* k, const void* v, const float* gammas,
                              int chunk, const float* rws, const void* gate, void* o, int B, int H,
                              int N, int dk, int dv, float eps, cudaStream_t st) {
  const size_t smem = chunk_out_smem(dk, dv);
  auto fn = simt_chunk_out<T, GN>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nc = cdiv(N, chunk);
  dim3 grid(nc * cdiv(chunk, CO_M), B * H);
  fn<<<grid, 256, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                              static_cast<const T*>(v), gammas, chunk, rws,
                              static_cast<const T*>(gate), static_cast<T*>(o), H, N, dk, dv, eps);
  return cudaPeekAtLastError();
}

template <typename T>
static cudaError_t simt_states_t(const void* k, const void* v, const float* gammas, int chunk,
                                 const float* state_in, float* state_out, int B, int H, int N,
                                 int dk, int dv, void* ws, cudaStream_t st) {
  dim3 g1(cdiv(dv, SC_T), cdiv(dk, SC_T), B * H);
  simt_state_scan<T><<<g1, 256, 0, st>>>(static_cast<const T*>(k), static_cast<const T*>(v),
                                         gammas, chunk, state_in, state_out,
                                         static_cast<float*>(ws), H, N, dk, dv);
  return cudaPeekAtLastError();
}

template <typename T>
static cudaError_t simt_output_t(const void* q, const void* k, const void* v, const float* gammas,
                                 int chunk, const void* gate, void* o, int B, int H, int N, int dk,
                                 int dv, float eps, const void* ws, cudaStream_t st) {
  const float* rws = static_cast<const float*>(ws);
  if (eps >= 0.f)
    return launch_out<T, true>(q, k, v, gammas, chunk, rws, gate, o, B, H, N, dk, dv, eps, st);
  return launch_out<T, false>(q, k, v, gammas, chunk, rws, gate, o, B, H, N, dk, dv, eps, st);
}

cudaError_t launch_simt_states(const void* k, const void* v, const float* gammas, int chunk,
                               const float* state_in, float* state_out, int B, int H, int N,
                               int dk, int dv, int dtype, void* ws, cudaStream_t st) {
  if (dtype == RET_BF16)
    return simt_states_t<__nv_bfloat16>(k, v, gammas, chunk, state_in, state_out, B, H, N, dk,
                                        dv, ws, st);
  return simt_states_t<float>(k, v, gammas, chunk, state_in, state_out, B, H, N, dk, dv, ws, st);
}

cudaError_t launch_simt_output(const void* q, const void* k, const void* v, const float* gammas,
                               int chunk, const void* gate, void* o, int B, int H, int N, int dk,
                               int dv, int dtype, float eps, const void* ws, cudaStream_t st) {
  if (dtype == RET_BF16)
    return simt_output_t<__nv_bfloat16>(q, k, v, gammas, chunk, gate, o, B, H, N, dk, dv, eps, ws,
                                        st);
  return simt_output_t<float>(q, k, v, gammas, chunk, gate, o, B, H, N, dk, dv, eps, ws, st);
}

cudaError_t launch_simt_parallel(const void* q, const void* k, const void* v, const float* gammas,
                                 const void* gate, void* o, int B, int H, int N, int dk, int dv,
                                 int dtype, float eps, cudaStream_t st) {
  if (dtype == RET_BF16) {
    if (eps >= 0.f)
      return launch_out<__nv_bfloat16, true>(q, k, v, gammas, N, nullptr, gate, o, B, H, N, dk,
                                             dv, eps, st);
    return launch_out<__nv_bfloat16, false>(q, k, v, gammas, N, nullptr, gate, o, B, H, N, dk,
                                            dv, eps, st);
  }
  if (eps >= 0.f)
    return launch_out<float, true>(q, k, v, gammas, N, nullptr, gate, o, B, H, N, dk, dv, eps, st);
  return launch_out<float, false>(q, k, v, gammas, N, nullptr, gate, o, B, H, N, dk, dv, eps, st);
}

}  // namespace ret
