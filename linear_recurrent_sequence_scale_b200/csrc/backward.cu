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
//   1. the forward chunk states R_{i-1} (the chunkwise states phase, float32)
//   2. grad_scan: G_i for every chunk, walking the chunks backwards
//   3. chunk_grad: per (b, h, chunk, 16 positions) the in-chunk parts of the
//      three row gradients
//   4. cross_chunk_gemm: the cross-chunk parts, one batched GEMM each.
#include "common.cuh"
#include "kernels.h"

namespace ret {
namespace bwd {

constexpr int ST = 64;  // state tile edge of the scan
constexpr int SJ = 32;  // tokens staged per scan step
constexpr int TP = 16;  // positions per gradient tile
constexpr int MAXU = 32;  // columns per thread: d <= 16 * MAXU = 512

// G_i = gradient of the state leaving chunk i, for i = nc-1 down to 0, into
// gws slot i; the gradient of the incoming state at the end.
template <typename T>
__global__ void __launch_bounds__(256)
grad_scan(const T* __restrict__ q, const T* __restrict__ dout, const float* __restrict__ gammas,
          int chunk, const float* __restrict__ d_state_out, float* __restrict__ d_state_in,
          float* __restrict__ gws, int H, int N, int dk, int dv) {
  __shared__ float qs[SJ][ST];
  __shared__ float ds[SJ][ST];
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
      acc[i][j] =
          (d_state_out && r < dk && c < dv) ? d_state_out[((size_t)bh * dk + r) * dv + c] : 0.f;
    }
  for (int ci = nc - 1; ci >= 0; --ci) {
    float* G = gws + ((size_t)bh * nc + ci) * dk * dv;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
        if (r < dk && c < dv) G[(size_t)r * dv + c] = acc[i][j];
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
        float qv = 0.f, dvv = 0.f;
        if (j < L) {
          if (r0 + x < dk) qv = Elem<T>::ld(q + tok * dk + r0 + x);
          if (c0 + x < dv) dvv = Elem<T>::ld(dout + tok * dv + c0 + x) * gpow(lg, j + 1);
        }
        qs[jj][x] = qv;
        ds[jj][x] = dvv;
      }
      __syncthreads();
#pragma unroll 4
      for (int jj = 0; jj < SJ; ++jj) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = qs[jj][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = ds[jj][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
    }
  }
  if (d_state_in) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + j;
        if (r < dk && c < dv) d_state_in[((size_t)bh * dk + r) * dv + c] = acc[i][j];
      }
  }
}

// Rows [n, n + rows) of a [.., N, d] tensor of (b, h) into smem with row
// stride ld (zeros past `rows`).
template <typename T>
__device__ __forceinline__ void stage_rows(float* dst, int ld, const T* src, int bh, int N, int d,
                                           int n, int rows) {
  for (int e = threadIdx.x; e < TP * d; e += 256) {
    const int r = e / d, x = e % d;
    dst[r * ld + x] = r < rows ? Elem<T>::ld(src + ((size_t)bh * N + n + r) * d + x) : 0.f;
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
chunk_grad(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
           const T* __restrict__ dout, const float* __restrict__ gammas, int chunk,
           T* __restrict__ dq, T* __restrict__ dk_, T* __restrict__ dv_, int H, int N, int dk,
           int dv) {
  extern __shared__ float sm[];
  const int lk = dk + 1, lv = dv + 1;
  float* a_v = sm;                 // [TP][dv+1]  tile rows: dO (phase A) / V (phase B)
  float* a_k = a_v + TP * lv;      // [TP][dk+1]  tile rows: K (phase B)
  float* b_v = a_k + TP * lk;      // [TP][dv+1]  other rows: V (A) / dO (B)
  float* b_k = b_v + TP * lv;      // [TP][dk+1]  other rows: K (A) / Q (B)
  float* ps = b_k + TP * lk;       // [TP][TP+1]
  float* ss = ps + TP * (TP + 1);  // [TP][TP+1]

  const int bh = blockIdx.y;
  const float lg = log2f(gammas[bh % H]);
  const int tpc = cdiv(chunk, TP);
  const int ci = blockIdx.x / tpc;
  const int cs = ci * chunk;
  const int p0 = cs + (blockIdx.x % tpc) * TP;
  const int ce = min(N, cs + chunk);
  if (p0 >= ce) return;
  const int rows = min(TP, ce - p0);
  const int tid = threadIdx.x;
  const int t = tid & 15, cg = tid >> 4;  // accumulation: row t, columns cg + 16 x
  const int da = tid >> 4, db = tid & 15;  // dot products: pair (da, db)

  // ---- phase A: dQ rows of this tile ----
  float acc[MAXU];
#pragma unroll
  for (int x = 0; x < MAXU; ++x) acc[x] = 0.f;
  stage_rows(a_v, lv, dout, bh, N, dv, p0, rows);
  for (int m0 = cs; m0 < p0 + rows; m0 += TP) {
    const int mr = min(TP, p0 + rows - m0);
    __syncthreads();
    stage_rows(b_v, lv, v, bh, N, dv, m0, mr);
    stage_rows(b_k, lk, k, bh, N, dk, m0, mr);
    __syncthreads();
    {  // ps[n][m] = D_nm (dO_n . v_m)
      float s = 0.f;
      for (int j = 0; j < dv; ++j) s = fmaf(a_v[da * lv + j], b_v[db * lv + j], s);
      const int n = p0 + da, m = m0 + db;
      ps[da * (TP + 1) + db] = (da < rows && db < mr && m <= n) ? s * gpow(lg, n - m) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int x = 0; x < MAXU; ++x) {
      const int c = cg + 16 * x;
      if (c < dk) {
        float s = acc[x];
        for (int b = 0; b < TP; ++b) s = fmaf(ps[t * (TP + 1) + b], b_k[b * lk + c], s);
        acc[x] = s;
      }
    }
  }
  if (t < rows) {
    const int n = p0 + t;
#pragma unroll
    for (int x = 0; x < MAXU; ++x) {
      const int c = cg + 16 * x;
      if (c < dk) Elem<T>::st(dq + ((size_t)bh * N + n) * dk + c, acc[x]);
    }
  }

  // ---- phase B: dK and dV rows of this tile ----
  float acck[MAXU], accv[MAXU];
#pragma unroll
  for (int x = 0; x < MAXU; ++x) acck[x] = accv[x] = 0.f;
  __syncthreads();
  stage_rows(a_v, lv, v, bh, N, dv, p0, rows);
  stage_rows(a_k, lk, k, bh, N, dk, p0, rows);
  for (int n0 = p0; n0 < ce; n0 += TP) {
    const int nr = min(TP, ce - n0);
    __syncthreads();
    stage_rows(b_v, lv, dout, bh, N, dv, n0, nr);
    stage_rows(b_k, lk, q, bh, N, dk, n0, nr);
    __syncthreads();
    {  // ps[n][m] = D_nm (dO_n . v_m), ss[n][m] = D_nm (q_n . k_m)
      float sp = 0.f, sq = 0.f;
      for (int j = 0; j < dv; ++j) sp = fmaf(b_v[da * lv + j], a_v[db * lv + j], sp);
      for (int j = 0; j < dk; ++j) sq = fmaf(b_k[da * lk + j], a_k[db * lk + j], sq);
      const int n = n0 + da, m = p0 + db;
      const float w = (da < nr && db < rows && n >= m) ? gpow(lg, n - m) : 0.f;
      ps[da * (TP + 1) + db] = sp * w;
      ss[da * (TP + 1) + db] = sq * w;
    }
    __syncthreads();
#pragma unroll
    for (int x = 0; x < MAXU; ++x) {
      const int c = cg + 16 * x;
      if (c < dk) {
        float s = acck[x];
        for (int a = 0; a < TP; ++a) s = fmaf(ps[a * (TP + 1) + t], b_k[a * lk + c], s);
        acck[x] = s;
      }
      if (c < dv) {
        float s = accv[x];
        for (int a = 0; a < TP; ++a) s = fmaf(ss[a * (TP + 1) + t], b_v[a * lv + c], s);
        accv[x] = s;
      }
    }
  }
  if (t < rows) {
    const int m = p0 + t;
#pragma unroll
    for (int x = 0; x < MAXU; ++x) {
      const int c = cg + 16 * x;
      if (c < dk) Elem<T>::st(dk_ + ((size_t)bh * N + m) * dk + c, acck[x]);
      if (c < dv) Elem<T>::st(dv_ + ((size_t)bh * N + m) * dv + c, accv[x]);
    }
  }
}

// Cross-chunk terms as one batched GEMM per (b, h, chunk), added to the
// rows chunk_grad wrote:
//     out[n] += s_n * (A[n] . S')    over the chunk's positions n,
// with S' = S^T (TRANS: dQ += xi (.) dO R_{i-1}^T, dK += zeta (.) V G_i^T) or
// S' = S (dV += zeta (.) K G_i), S a float32 [dk][dv] chunk state.  Tiles of
// 64 rows x 64 columns, 4 x 4 results per thread, 16-deep slices of A and S'
// through shared memory.
constexpr int GM = 64, GN_ = 64, GK = 16;

template <typename T, bool TRANS, bool XI>
__global__ void __launch_bounds__(256)
cross_chunk_gemm(const T* __restrict__ a, const float* __restrict__ states, int has_r0,
                 const float* __restrict__ gammas, int chunk, T* __restrict__ out, int H, int N,
                 int ka, int ncol, int dk, int dv) {
  __shared__ float as[GK][GM + 4];
  __shared__ float bs[GK][GN_ + 4];
  const int nc = cdiv(N, chunk);
  const int rpc = cdiv(chunk, GM);        // row blocks per chunk
  const int ci = blockIdx.y / rpc;
  const int cs = ci * chunk;
  const int r0 = cs + (blockIdx.y % rpc) * GM;
  const int ce = min(N, cs + chunk);
  if (r0 >= ce || (XI && ci == 0 && !has_r0)) return;
  const int bh = blockIdx.z;
  const int c0 = blockIdx.x * GN_;
  const float lg = log2f(gammas[bh % H]);
  const float* S = states + ((size_t)bh * nc + ci) * dk * dv;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < ka; k0 += GK) {
    __syncthreads();
    for (int e = tid; e < GM * GK; e += 256) {  // A rows r0.., columns k0..
      const int r = e / GK, kk = e % GK;
      const int n = r0 + r;
      as[kk][r] = (n < ce && k0 + kk < ka) ? Elem<T>::ld(a + ((size_t)bh * N + n) * ka + k0 + kk)
                                           : 0.f;
    }
    for (int e = tid; e < GK * GN_; e += 256) {  // S' rows k0.., columns c0..
      int kk, c;
      if (TRANS) { c = e / GK; kk = e % GK; } else { kk = e / GN_; c = e % GN_; }
      float x = 0.f;
      if (k0 + kk < ka && c0 + c < ncol)
        x = TRANS ? S[(size_t)(c0 + c) * dv + k0 + kk] : S[(size_t)(k0 + kk) * dv + c0 + c];
      bs[kk][c] = x;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = as[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  const int L = ce - cs;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = r0 + ty * 4 + i;
    if (n >= ce) continue;
    const float sc = XI ? gpow(lg, n - cs + 1) : gpow(lg, L - 1 - (n - cs));
    T* orow = out + ((size_t)bh * N + n) * ncol;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx * 4 + j;
      if (c < ncol) Elem<T>::st(orow + c, Elem<T>::ld(orow + c) + sc * acc[i][j]);
    }
  }
}

template <typename T>
cudaError_t backward_t(const void* q, const void* k, const void* v, const float* gammas, int chunk,
                       const float* state_in, const void* dout, const float* d_state_out,
                       void* dq, void* dk_, void* dv_, float* d_state_in, int B, int H, int N,
                       int dk, int dv, int dtype, void* ws, cudaStream_t st) {
  const int nc = cdiv(N, chunk);
  float* rws = static_cast<float*>(ws);
  float* gws = rws + (size_t)B * H * nc * dk * dv;
  cudaError_t e = launch_simt_states(k, v, gammas, chunk, state_in, nullptr, B, H, N, dk, dv,
                                     dtype, rws, st);
  if (e != cudaSuccess) return e;
  dim3 g1(cdiv(dv, ST), cdiv(dk, ST), B * H);
  grad_scan<T><<<g1, 256, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(dout), gammas,
                                   chunk, d_state_out, d_state_in, gws, H, N, dk, dv);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  const size_t smem =
      sizeof(float) * (size_t)(2 * TP * (dv + 1) + 2 * TP * (dk + 1) + 2 * TP * (TP + 1));
  auto fn = chunk_grad<T>;
  if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  dim3 g2(nc * cdiv(chunk, TP), B * H);
  fn<<<g2, 256, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                            static_cast<const T*>(v), static_cast<const T*>(dout), gammas, chunk,
                            static_cast<T*>(dq),
                            static_cast<T*>(dk_), static_cast<T*>(dv_), H, N, dk, dv);
  if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
  const int rb = nc * cdiv(chunk, GM);
  const dim3 gq(cdiv(dk, GN_), rb, B * H), gv_(cdiv(dv, GN_), rb, B * H);
  cross_chunk_gemm<T, true, true><<<gq, 256, 0, st>>>(
      static_cast<const T*>(dout), rws, state_in != nullptr, gammas, chunk, static_cast<T*>(dq), H,
      N, dv, dk, dk, dv);
  cross_chunk_gemm<T, true, false><<<gq, 256, 0, st>>>(
      static_cast<const T*>(v), gws, 1, gammas, chunk, static_cast<T*>(dk_), H, N, dv, dk, dk, dv);
  cross_chunk_gemm<T, false, false><<<gv_, 256, 0, st>>>(
      static_cast<const T*>(k), gws, 1, gammas, chunk, static_cast<T*>(dv_), H, N, dk, dv, dk, dv);
  return cudaPeekAtLastError();
}

}  // namespace bwd

size_t backward_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk) {
  return 2 * sizeof(float) * (size_t)B * H * cdiv(N, chunk) * dk * dv;
}

cudaError_t launch_chunkwise_backward(const void* q, const void* k, const void* v,
                                      const float* gammas, int chunk, const float* state_in,
                                      const void* dout, const float* d_state_out, void* dq,
                                      void* dk_, void* dv_, float* d_state_in, int B, int H,
                                      int N, int dk, int dv, int dtype, void* ws,
                                      cudaStream_t st) {
  if (dtype == RET_BF16)
    return bwd::backward_t<__nv_bfloat16>(q, k, v, gammas, chunk, state_in, dout, d_state_out, dq,
                                          dk_, dv_, d_state_in, B, H, N, dk, dv, dtype, ws, st);
  return bwd::backward_t<float>(q, k, v, gammas, chunk, state_in, dout, d_state_out, dq, dk_, dv_,
                                d_state_in, B, H, N, dk, dv, dtype, ws, st);
}

}  // namespace ret
