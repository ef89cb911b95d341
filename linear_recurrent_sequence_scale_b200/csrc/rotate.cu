// xPos-style rotation of q or k rows.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", core
// components, item 3: xPos puts relative position into Q and K by a complex
// rotation; "RetNet入門" (Spiral.AI Tech Blog), LEX Transformer paragraph: the
// same term links the recurrent and the parallel forms.  Channels (2c, 2c+1)
// of a row are the real and imaginary parts of z_c; the row at sequence
// position n is multiplied by e^{i n theta_c}:
//     y[2c]   = x[2c] cos(n theta_c) - x[2c+1] sin(n theta_c)
//     y[2c+1] = x[2c] sin(n theta_c) + x[2c+1] cos(n theta_c)
// so that q'_n . k'_m depends on n - m only.
//
// Bound by HBM: every element is read once and written once.  The angle
// depends on (n, c) only, so a thread takes the cos / sin of its V channel
// pairs once, in double precision (n theta reaches 1e6 rad and more, where a
// float32 product would lose the phase), and applies them to the same
// (n, pairs) of up to kRowsPerThread (batch, head) rows, one row at a time
// (kGroup rows would be loaded before any is stored).  More rows in flight
// per thread measured slower: each is a different (batch, head) block 4 MB
// away, so a warp's loads then spread over kGroup DRAM pages at once (8k
// workload, q and k in place: 4 rows 4804 GB/s, 2 rows 5533, 1 row 5748; 32
// rows per thread instead of 16: 5789).  In place (y == x) is safe: every
// element is read and written by the one thread that owns it.
#include "common.cuh"
#include "kernels.h"

namespace ret {
namespace rot {

constexpr int kThreads = 256;
constexpr int kRowsPerThread = 32;  // (batch, head) rows sharing one set of angles
constexpr int kGroup = 1;           // rows loaded together

template <typename T, int V>
struct Pairs {
  float a[2 * V];
  __device__ __forceinline__ void load(const T* p) {
    if constexpr (V % 2 == 0) {
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        const float4 f = Elem<T>::ld4(p + 4 * i);
        a[4 * i] = f.x, a[4 * i + 1] = f.y, a[4 * i + 2] = f.z, a[4 * i + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 2 * V; ++i) a[i] = Elem<T>::ld(p + i);
    }
  }
  __device__ __forceinline__ void store(T* p) const {
    if constexpr (V % 2 == 0) {
#pragma unroll
      for (int i = 0; i < V / 2; ++i)
        Elem<T>::st4(p + 4 * i, make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]));
    } else {
#pragma unroll
      for (int i = 0; i < 2 * V; ++i) Elem<T>::st(p + i, a[i]);
    }
  }
};

// Thread (n, u) of grid.x rotates channel pairs [u V, u V + V) of row n in
// the (batch, head) rows [blockIdx.y R, blockIdx.y R + R), R = rows_per_thread.
template <typename T, int V>
__global__ void __launch_bounds__(kThreads)
rotate_rows(const T* x, T* y, const float* __restrict__ theta, long long pos0, int BH, int N,
            int d, int rows_per_thread) {
  const int U = d / (2 * V);  // thread units per row
  const long long idx = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (idx >= (long long)N * U) return;
  const int n = static_cast<int>(idx / U);
  const int u = static_cast<int>(idx - (long long)n * U);
  float cs[V], sn[V];
  const double pos = static_cast<double>(pos0 + n);
#pragma unroll
  for (int v = 0; v < V; ++v) {
    double s, c;
    sincos(pos * static_cast<double>(theta[u * V + v]), &s, &c);
    cs[v] = static_cast<float>(c);
    sn[v] = static_cast<float>(s);
  }
  const int bh0 = blockIdx.y * rows_per_thread;
  const int bh1 = min(BH, bh0 + rows_per_thread);
  const size_t col = (size_t)u * 2 * V;
  for (int b = bh0; b < bh1; b += kGroup) {
    Pairs<T, V> r[kGroup];
#pragma unroll
    for (int g = 0; g < kGroup; ++g)
      if (b + g < bh1) r[g].load(x + ((size_t)(b + g) * N + n) * d + col);
#pragma unroll
    for (int g = 0; g < kGroup; ++g) {
      if (b + g >= bh1) break;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const float re = r[g].a[2 * v], im = r[g].a[2 * v + 1];
        r[g].a[2 * v] = fmaf(re, cs[v], -im * sn[v]);
        r[g].a[2 * v + 1] = fmaf(re, sn[v], im * cs[v]);
      }
      r[g].store(y + ((size_t)(b + g) * N + n) * d + col);
    }
  }
}

template <typename T>
cudaError_t rotate_t(const void* x, void* y, const float* theta, long long pos0, int BH, int N,
                     int d, cudaStream_t st) {
  // four pairs (eight elements) per thread when rows split into whole
  // 8-element pieces; one pair otherwise
  const bool wide = d % 8 == 0;
  const long long units = (long long)N * (wide ? d / 8 : d / 2);
  const int rpt = BH > kRowsPerThread * 65535 ? cdiv(BH, 65535) : kRowsPerThread;
  const dim3 grid(static_cast<unsigned>((units + kThreads - 1) / kThreads), cdiv(BH, rpt));
  const T* xs = static_cast<const T*>(x);
  T* ys = static_cast<T*>(y);
  if (wide)
    rotate_rows<T, 4><<<grid, kThreads, 0, st>>>(xs, ys, theta, pos0, BH, N, d, rpt);
  else
    rotate_rows<T, 1><<<grid, kThreads, 0, st>>>(xs, ys, theta, pos0, BH, N, d, rpt);
  return cudaPeekAtLastError();
}

}  // namespace rot

cudaError_t launch_rotate(const void* x, void* y, const float* theta, long long pos0, int B,
                          int H, int N, int d, int dtype, cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  if (dtype == RET_BF16)
    return rot::rotate_t<__nv_bfloat16>(x, y, theta, pos0, B * H, N, d, st);
  return rot::rotate_t<float>(x, y, theta, pos0, B * H, N, d, st);
}

}  // namespace ret
