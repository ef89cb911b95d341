// Chunkwise backward: dQ, dK, dV and the gradient of the incoming state, on
// the CUDA cores in float32 (any d_k, d_v up to 512; f32 or bf16 storage).
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations, Chunkwise Recurrent: in chunk i (positions j = 0 .. L-1)
//     O_[i] = (Q K^T (.) D) V + (Q (.) xi) R_{i-1},   xi_j = gamma^(j+1)
//     R_i   = gamma^L R_{i-1} + K^T (V (.) zeta),      zeta_j = gamma^(L-1-j)
// With dO the gradient of O and G_i that of R_i (G of the last chunk = the
// gradient of the final state), the chain rule gives
//     G_{i-1}   = gamma^L G_i + (Q (.) xi)^T dO              (reverse scan)
//     dQ_[i]    = (dO V^T (.) D) K + xi (.) (dO R_{i-1}^T)
//     dK_[i]    = (dO V^T (.) D)^T Q + zeta (.) (V G_i^T)
//     dV_[i]    = (Q K^T (.) D)^T dO + zeta (.) (K G_i)
// and the gradient of the incoming state is G_{-1}.
//   1. state_scan<FWD>: the forward chunk states R_{i-1}, float32
//   2. state_scan<!FWD>: G_i for every chunk, walking the chunks backwards
//   3. chunk_scores: D (.) (dO V^T) and D (.) (Q K^T) per chunk, float32
//   4. chunk_grads: dQ, dK, dV, each one batched product per chunk that adds
//      the cross-chunk term to the in-chunk one.
#include "common.cuh"
#include "kernels.h"

namespace ret {
namespace bwd {

constexpr int ST = 64;  // state tile edge of the scan
constexpr int SJ = 32;  // tokens staged per scan step

// The two chunk-state recurrences of the backward, one 64 x 64 tile of the
// d_k x d_v state per CTA, walking the chunks in order:
//   FWD    slot i = R_{i-1} (the state entering chunk i), starting from
//          state_in:   R_i = gamma^L R_{i-1} + K_[i]^T (V_[i] (.) zeta)
//   !FWD   slot i = G_i (the gradient of the state leaving chunk i), from
//          the last chunk down, starting from d_state_out:
//          G_{i-1} = gamma^L G_i + (Q_[i] (.) xi)^T dO_[i];  G_{-1} is written
//          to `last` (the gradient of state_in) when it is not null.
// a is K (FWD) or Q, [.., N, dk]; b is V (FWD) or dO, [.., N, dv].
template <typename T, bool FWD>
__global__ void __launch_bounds__(256, 4)
state_scan(const T* __restrict__ a, const T* __restrict__ b, const float* __restrict__ gammas,
           int chunk, const float* __restrict__ first, float* __restrict__ last,
           float* __restrict__ slots, int H, int N, int dk, int dv) {
  __shared__ float as[SJ][ST];
  __shared__ float bs[SJ][ST];
  const int bh = blockIdx.z;
  const float lg = log2f(gammas[bh % H]);
  const int r0 = blockIdx.y * ST;
  const int c0 = blockIdx.x * ST;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const int nc = cdiv(N, chunk);

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
      acc[i][j] = (first && r < dk && c < dv) ? first[((size_t)bh * dk + r) * dv + c] : 0.f;
    }
  for (int t = 0; t < nc; ++t) {
    const int ci = FWD ? t : nc - 1 - t;
    float* S = slots + ((size_t)bh * nc + ci) * dk * dv;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
        if (r < dk && c < dv) S[(size_t)r * dv + c] = acc[i][j];
      }
    const int s = ci * chunk;
    const int L = min(chunk, N - s);
    const float gL = gpow(lg, L);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= gL;
    for (int j0 = 0; j0 < L; j0 += SJ) {
      __syncthreads();
      for (int e = tid; e < SJ * ST; e += 256) {
        const int jj = e / ST, x = e % ST;
        const int j = j0 + jj;
        const size_t tok = (size_t)bh * N + s + j;
        float av = 0.f, bv = 0.f;
        if (j < L) {
          if (r0 + x < dk) av = Elem<T>::ld(a + tok * dk + r0 + x);
          if (c0 + x < dv)
            bv = Elem<T>::ld(b + tok * dv + c0 + x) * gpow(lg, FWD ? L - 1 - j : j + 1);
        }
        as[jj][x] = av;
        bs[jj][x] = bv;
      }
      __syncthreads();
#pragma unroll 4
      for (int jj = 0; jj < SJ; ++jj) {
        float av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = as[jj][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = bs[jj][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
    }
  }
  if (last) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
        if (r < dk && c < dv) last[((size_t)bh * dk + r) * dv + c] = acc[i][j];
      }
  }
}

// ---- register-tiled products: 64 x 64 results per CTA, 4 x 4 per thread,
// 16-deep slices of both operands through shared memory ----
constexpr int GM = 64, GN_ = 64, GK = 16;

struct Tile {
  float as[GK][GM + 4];
  float bs[GK][GN_ + 4];
};

// acc += A[.., k0 .. k1) B[k0 .. k1), ..] over this CTA's 64 x 64 tile, with
// la(r, k) = A[r][k] and lb(k, c) = B[k][c] (tile-local r, c; both return 0
// outside the operand).  A_KC / B_KC: consecutive k of one r (of one c) are
// adjacent in memory, so consecutive threads load along k; otherwise they
// load along r (along c).
template <bool A_KC, bool B_KC, class LA, class LB>
__device__ __forceinline__ void tile_product(Tile& t, LA la, LB lb, int k0, int k1,
                                             float (&acc)[4][4]) {
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  for (int kb = k0; kb < k1; kb += GK) {
    __syncthreads();
    for (int e = tid; e < GM * GK; e += 256) {
      const int r = A_KC ? e / GK : e % GM;
      const int kk = A_KC ? e % GK : e / GM;
      t.as[kk][r] = kb + kk < k1 ? la(r, kb + kk) : 0.f;
    }
    for (int e = tid; e < GK * GN_; e += 256) {
      const int c = B_KC ? e / GK : e % GN_;
      const int kk = B_KC ? e % GK : e / GN_;
      t.bs[kk][c] = kb + kk < k1 ? lb(kb + kk, c) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = t.as[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = t.bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
}

// Masked scores of one chunk, S[n][m] = D_nm (x_n . y_m) for in-chunk
// positions n, m < L, into a float32 [chunk][chunk] slot per (b, h, chunk):
// P = D (.) (dO V^T) for dQ and dK, and D (.) (Q K^T) for dV.  Only tiles
// on or below the diagonal are computed; nothing reads the others.
// Grid: x = chunk, y = lower-triangular tile pair, z = (b, h).
template <typename T>
__global__ void __launch_bounds__(256)
chunk_scores(const T* __restrict__ x, const T* __restrict__ y, const float* __restrict__ gammas,
             int chunk, float* __restrict__ out, int H, int N, int d) {
  __shared__ Tile t;
  int i = 0;
  while ((i + 1) * (i + 2) / 2 <= (int)blockIdx.y) ++i;
  const int j = blockIdx.y - i * (i + 1) / 2;  // row tile i >= column tile j
  const int ci = blockIdx.x, bh = blockIdx.z;
  const int cs = ci * chunk;
  const int L = min(chunk, N - cs);
  const int r0 = i * GM, c0 = j * GN_;
  if (r0 >= L) return;
  const T* X = x + ((size_t)bh * N + cs) * d;
  const T* Y = y + ((size_t)bh * N + cs) * d;
  float acc[4][4] = {};
  tile_product<true, true>(
      t,
      [&](int r, int k) { return r0 + r < L ? Elem<T>::ld(X + (size_t)(r0 + r) * d + k) : 0.f; },
      [&](int k, int c) { return c0 + c < L ? Elem<T>::ld(Y + (size_t)(c0 + c) * d + k) : 0.f; },
      0, d, acc);
  const float lg = log2f(gammas[bh % H]);
  float* S = out + ((size_t)bh * gridDim.x + ci) * chunk * chunk;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int n = r0 + ty * 4 + a;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int m = c0 + tx * 4 + b;
      if (n < L && m < L) S[(size_t)n * chunk + m] = m <= n ? gpow(lg, n - m) * acc[a][b] : 0.f;
    }
  }
}

// One gradient of one chunk, the in-chunk and the cross-chunk product in one
// accumulation (positions n, m in the chunk, P and S the scores above,
// R = R_{i-1}, G = G_i, both float32 [dk][dv]):
//   MODE 0  dQ[n] = sum_{m<=n} P[n][m] k_m + xi_n   (dO_n R^T)
//   MODE 1  dK[m] = sum_{n>=m} P[n][m] q_n + zeta_m (v_m G^T)
//   MODE 2  dV[m] = sum_{n>=m} S[n][m] dO_n + zeta_m (k_m G)
// b1 holds the rows the scores multiply (k, q, dO), a2 those the state
// multiplies (dO, v, k; a2 rows are d2 wide), out is ncol wide.  Grid: x =
// chunk, y = (64-row tile, 64-column tile), z = (b, h).
template <typename T, int MODE>
__global__ void __launch_bounds__(256)
chunk_grads(const T* __restrict__ b1, const T* __restrict__ a2, const float* __restrict__ scores,
            const float* __restrict__ states, int has_r0, const float* __restrict__ gammas,
            int chunk, T* __restrict__ out, int H, int N, int d2, int ncol, int dk, int dv) {
  __shared__ Tile t;
  __shared__ float rsc[GM];
  const int ctn = cdiv(ncol, GN_);
  const int r0 = (blockIdx.y / ctn) * GM, c0 = (blockIdx.y % ctn) * GN_;
  const int ci = blockIdx.x, bh = blockIdx.z;
  const int cs = ci * chunk;
  const int L = min(chunk, N - cs);
  if (r0 >= L) return;
  const float* P = scores + ((size_t)bh * gridDim.x + ci) * chunk * chunk;
  const T* B1 = b1 + ((size_t)bh * N + cs) * ncol;
  float acc[4][4] = {};
  auto lb1 = [&](int k, int c) {
    return c0 + c < ncol ? Elem<T>::ld(B1 + (size_t)k * ncol + c0 + c) : 0.f;
  };
  if (MODE == 0)
    tile_product<true, false>(
        t, [&](int r, int k) { return r0 + r < L ? P[(size_t)(r0 + r) * chunk + k] : 0.f; }, lb1,
        0, min(L, r0 + GM), acc);
  else
    tile_product<false, false>(
        t, [&](int r, int k) { return r0 + r < L ? P[(size_t)k * chunk + r0 + r] : 0.f; }, lb1,
        r0, L, acc);
  if (MODE != 0 || ci > 0 || has_r0) {
    const float lg = log2f(gammas[bh % H]);
    if (threadIdx.x < GM) {
      const int jj = r0 + threadIdx.x;  // xi_j = gamma^(j+1), zeta_j = gamma^(L-1-j)
      rsc[threadIdx.x] = jj < L ? gpow(lg, MODE == 0 ? jj + 1 : L - 1 - jj) : 0.f;
    }
    const float* St = states + ((size_t)bh * gridDim.x + ci) * dk * dv;
    const T* A2 = a2 + ((size_t)bh * N + cs) * d2;
    auto la = [&](int r, int k) {
      return r0 + r < L ? rsc[r] * Elem<T>::ld(A2 + (size_t)(r0 + r) * d2 + k) : 0.f;
    };
    // rsc is written before the first barrier inside tile_product
    if (MODE == 2)
      tile_product<true, false>(
          t, la, [&](int k, int c) { return c0 + c < ncol ? St[(size_t)k * dv + c0 + c] : 0.f; },
          0, d2, acc);
    else
      tile_product<true, true>(
          t, la, [&](int k, int c) { return c0 + c < ncol ? St[(size_t)(c0 + c) * dv + k] : 0.f; },
          0, d2, acc);
  }
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int n = r0 + ty * 4 + a;
    if (n >= L) continue;
    T* orow = out + ((size_t)bh * N + cs + n) * ncol;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int c = c0 + tx * 4 + b;
      if (c < ncol) Elem<T>::st(orow + c, acc[a][b]);
    }
  }
}

// The chunk length the backward works in.  Every chunk length gives the same
// forward output in exact arithmetic, so the gradients do not depend on it;
// 128 keeps both the [chunk][chunk] scores and the per-chunk states small.
inline int work_chunk(int chunk) { return chunk < 128 ? chunk : 128; }

template <typename T>
cudaError_t backward_t(const void* q, const void* k, const void* v, const float* gammas, int chunk,
                       const float* state_in, const void* dout, const float* d_state_out,
                       void* dq, void* dk_, void* dv_, float* d_state_in, int B, int H, int N,
                       int dk, int dv, void* ws, cudaStream_t st) {
  chunk = work_chunk(chunk);
  const int nc = cdiv(N, chunk);
  const size_t slots = (size_t)B * H * nc;
  float* rws = static_cast<float*>(ws);
  float* gws = rws + slots * dk * dv;
  float* pws = gws + slots * dk * dv;
  float* sws = pws + slots * chunk * chunk;
  const T* Q = static_cast<const T*>(q);
  const T* K = static_cast<const T*>(k);
  const T* V = static_cast<const T*>(v);
  const T* dO = static_cast<const T*>(dout);
  const dim3 g1(cdiv(dv, ST), cdiv(dk, ST), B * H);
  state_scan<T, true><<<g1, 256, 0, st>>>(K, V, gammas, chunk, state_in, nullptr, rws, H, N, dk,
                                          dv);
  state_scan<T, false><<<g1, 256, 0, st>>>(Q, dO, gammas, chunk, d_state_out, d_state_in, gws, H,
                                           N, dk, dv);
  cudaError_t e = cudaPeekAtLastError();
  if (e != cudaSuccess) return e;
  const int nt = cdiv(chunk, GM);
  const dim3 gs(nc, nt * (nt + 1) / 2, B * H);
  chunk_scores<T><<<gs, 256, 0, st>>>(dO, V, gammas, chunk, pws, H, N, dv);
  chunk_scores<T><<<gs, 256, 0, st>>>(Q, K, gammas, chunk, sws, H, N, dk);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  const dim3 gk(nc, nt * cdiv(dk, GN_), B * H), gv(nc, nt * cdiv(dv, GN_), B * H);
  const int has_r0 = state_in != nullptr;
  chunk_grads<T, 0><<<gk, 256, 0, st>>>(K, dO, pws, rws, has_r0, gammas, chunk,
                                        static_cast<T*>(dq), H, N, dv, dk, dk, dv);
  chunk_grads<T, 1><<<gk, 256, 0, st>>>(Q, V, pws, gws, 1, gammas, chunk, static_cast<T*>(dk_), H,
                                        N, dv, dk, dk, dv);
  chunk_grads<T, 2><<<gv, 256, 0, st>>>(dO, K, sws, gws, 1, gammas, chunk, static_cast<T*>(dv_), H,
                                        N, dk, dv, dk, dv);
  return cudaPeekAtLastError();
}

}  // namespace bwd

size_t backward_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk) {
  const int c = bwd::work_chunk(chunk);
  return 2 * sizeof(float) * (size_t)B * H * cdiv(N, c) * ((size_t)dk * dv + (size_t)c * c);
}

cudaError_t launch_chunkwise_backward(const void* q, const void* k, const void* v,
                                      const float* gammas, int chunk, const float* state_in,
                                      const void* dout, const float* d_state_out, void* dq,
                                      void* dk_, void* dv_, float* d_state_in, int B, int H,
                                      int N, int dk, int dv, int dtype, void* ws,
                                      cudaStream_t st) {
  if (dtype == RET_BF16)
    return bwd::backward_t<__nv_bfloat16>(q, k, v, gammas, chunk, state_in, dout, d_state_out, dq,
                                          dk_, dv_, d_state_in, B, H, N, dk, dv, ws, st);
  return bwd::backward_t<float>(q, k, v, gammas, chunk, state_in, dout, d_state_out, dq, dk_, dv_,
                                d_state_in, B, H, N, dk, dv, ws, st);
}

}  // namespace ret
