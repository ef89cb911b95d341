// Recurrent decode step: state <- gamma*state + k^T v, o = q state.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations, Recurrent Form.  Per (batch, head) the float32 state is a
// dk x dv row-major matrix; one step reads and writes all of it once, so the
// kernel is bound by HBM bandwidth (about 0.5 flop per byte).
//
// Mapping: a CTA owns STEP_COLS = 128 state columns of one (b, h) and all dk
// rows.  Each warp covers the 128 columns of a row with one 16-byte access per
// lane (fully coalesced 512-byte rows); the 8 warps split the rows, each
// keeping STEP_UNROLL independent row loads in flight before it updates and
// stores them.  The partial q.S sums of the 8 warps meet in shared memory.
// With GroupNorm the CTAs of one (b, h) form a thread-block cluster and
// exchange their row statistics through distributed shared memory.
// Consecutive steps on a stream use programmatic dependent launch: a step's
// CTAs are scheduled while the previous step drains and wait (griddepcontrol)
// until its writes are visible, which hides the launch gap between steps.
//
// Optionally (theta != null) q and k are turned by the xPos rotation of the
// token's position as they are read ("RetNet - Retentive Network - A
// Successor to Transformer for LLMs", core components, item 3): channel pair
// c becomes (x0 cos a - x1 sin a, x0 sin a + x1 cos a), a = pos theta_c, with
// cos and sin taken in double precision (pos theta reaches 1e6 rad and more).
// The rotated rows stay in float32 in shared memory; the inputs are not
// written.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace ret {

constexpr int STEP_COLS = 128;
constexpr int STEP_THREADS = 256;
constexpr int STEP_RG = STEP_THREADS / (STEP_COLS / 4);  // 8 row groups (= warps)
// Residency.  The grid is d_v/128 x B x H CTAs of equal work (512 for the
// 6.7B-class layer at batch 8), all streaming the state at once; what decides
// the time is how evenly they fill the SMs.  Three CTAs per SM (the
// register count the compiler picks by default) run 444 of 512 in a first
// wave and leave a 68-CTA tail: 28.5 us per step.  Without GroupNorm, two
// per SM with eight row loads in flight per warp take 25.0 us (two waves of
// 296 and 216 CTAs, each with ~9 MB of loads in flight); the residency is
// pinned by the shared-memory request (STEP_SMEM_FLOOR), not left to the
// register count.  With GroupNorm (4-CTA clusters) four per SM with four
// row loads in flight, a single wave, measured best (27.3 against 29.3 us).
template <bool GN> struct StepCfg {
  static constexpr int UNROLL = GN ? 4 : 8;
  static constexpr int MIN_BLOCKS = GN ? 4 : 1;
};
constexpr size_t STEP_SMEM_FLOOR = 80 * 1024;  // > 1/3 of an SM's shared memory

__device__ __forceinline__ float block_sum_256(float x, float* scratch /* >= 8 floats */) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[w] = x;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < STEP_THREADS / 32; ++i) t += scratch[i];
  return t;
}

template <typename T, bool GN, bool ROT>
__global__ void __launch_bounds__(STEP_THREADS, StepCfg<GN>::MIN_BLOCKS)
step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
            const float* __restrict__ gammas, float* __restrict__ state,
            const T* __restrict__ gate, T* __restrict__ o, int H, int dk, int dv, float eps,
            const float* __restrict__ theta, long long pos) {
  extern __shared__ float smem[];
  float* qs = smem;                       // [dk]
  float* ks = smem + dk;                  // [dk]
  float* red = smem + 2 * dk;             // [STEP_RG][STEP_COLS]
  __shared__ float scratch[8];
  __shared__ float stats[2];              // this CTA's partial sum, sum of squares

  // the previous grid on the stream (e.g. the step before) must be complete
  // before anything is read; the next one may be scheduled from now on
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int bh = blockIdx.y;
  const int h = bh % H;
  const int c0 = blockIdx.x * STEP_COLS;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int rg = tid >> 5;

  if constexpr (ROT) {
    // dk is even (a multiple of 8): pair c is channels (2c, 2c + 1)
    for (int c = tid; c < dk / 2; c += STEP_THREADS) {
      double sn, cs;
      sincos(static_cast<double>(pos) * static_cast<double>(theta[c]), &sn, &cs);
      const float fc = static_cast<float>(cs), fs = static_cast<float>(sn);
      const size_t at = (size_t)bh * dk + 2 * c;
      const float q0 = Elem<T>::ld(q + at), q1 = Elem<T>::ld(q + at + 1);
      const float k0 = Elem<T>::ld(k + at), k1 = Elem<T>::ld(k + at + 1);
      qs[2 * c] = q0 * fc - q1 * fs;
      qs[2 * c + 1] = q0 * fs + q1 * fc;
      ks[2 * c] = k0 * fc - k1 * fs;
      ks[2 * c + 1] = k0 * fs + k1 * fc;
    }
  } else {
    for (int i = tid; i < dk; i += STEP_THREADS) {
      qs[i] = Elem<T>::ld(q + (size_t)bh * dk + i);
      ks[i] = Elem<T>::ld(k + (size_t)bh * dk + i);
    }
  }
  const float g = gammas[h];
  const int c = c0 + 4 * lane;
  const bool cval = c < dv;  // dv is a multiple of 4, so c..c+3 are all valid
  float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
  if (cval) vv = Elem<T>::ld4(v + (size_t)bh * dv + c);
  __syncthreads();

  constexpr int STEP_UNROLL = StepCfg<GN>::UNROLL;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float* S = state + (size_t)bh * dk * dv + c;
  for (int r0 = rg; r0 < dk; r0 += STEP_RG * STEP_UNROLL) {
    float4 s[STEP_UNROLL];
#pragma unroll
    for (int u = 0; u < STEP_UNROLL; ++u) {
      const int r = r0 + u * STEP_RG;
      if (cval && r < dk) s[u] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)r * dv));
    }
#pragma unroll
    for (int u = 0; u < STEP_UNROLL; ++u) {
      const int r = r0 + u * STEP_RG;
      if (cval && r < dk) {
        const float kr = ks[r], qr = qs[r];
        float4 t;
        t.x = fmaf(kr, vv.x, g * s[u].x);
        t.y = fmaf(kr, vv.y, g * s[u].y);
        t.z = fmaf(kr, vv.z, g * s[u].z);
        t.w = fmaf(kr, vv.w, g * s[u].w);
        __stcs(reinterpret_cast<float4*>(S + (size_t)r * dv), t);
        acc.x = fmaf(qr, t.x, acc.x);
        acc.y = fmaf(qr, t.y, acc.y);
        acc.z = fmaf(qr, t.z, acc.z);
        acc.w = fmaf(qr, t.w, acc.w);
      }
    }
  }
  red[rg * STEP_COLS + 4 * lane + 0] = acc.x;
  red[rg * STEP_COLS + 4 * lane + 1] = acc.y;
  red[rg * STEP_COLS + 4 * lane + 2] = acc.z;
  red[rg * STEP_COLS + 4 * lane + 3] = acc.w;
  __syncthreads();

  const int oc = c0 + tid;
  const bool oval = tid < STEP_COLS && oc < dv;
  float val = 0.f;
  if (tid < STEP_COLS) {
#pragma unroll
    for (int i = 0; i < STEP_RG; ++i) val += red[i * STEP_COLS + tid];
  }
  if constexpr (GN) {
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned nblk = cluster.num_blocks();
    float part = block_sum_256(oval ? val : 0.f, scratch);
    if (tid == 0) stats[0] = part;
    cluster.sync();
    float tot = 0.f;
    for (unsigned r = 0; r < nblk; ++r) tot += cluster.map_shared_rank(stats, r)[0];
    const float mean = tot / static_cast<float>(dv);
    const float dev = oval ? val - mean : 0.f;
    part = block_sum_256(dev * dev, scratch);
    if (tid == 0) stats[1] = part;
    cluster.sync();
    float sq = 0.f;
    for (unsigned r = 0; r < nblk; ++r) sq += cluster.map_shared_rank(stats, r)[1];
    const float inv = 1.0f / sqrtf(sq / static_cast<float>(dv) + eps);
    if (oval) {
      float y = dev * inv;
      if (gate) y *= swishf(Elem<T>::ld(gate + (size_t)bh * dv + oc));
      Elem<T>::st(o + (size_t)bh * dv + oc, y);
    }
    cluster.sync();  // peers may still be reading this CTA's stats
  } else {
    if (oval) {
      if (gate) val *= swishf(Elem<T>::ld(gate + (size_t)bh * dv + oc));
      Elem<T>::st(o + (size_t)bh * dv + oc, val);
    }
  }
}

template <typename T>
static cudaError_t launch_step_t(const void* q, const void* k, const void* v, const float* gammas,
                                 float* state, const void* gate, void* o, int B, int H, int dk,
                                 int dv, float eps, const float* theta, long long pos,
                                 cudaStream_t st) {
  const int nct = cdiv(dv, STEP_COLS);
  dim3 grid(nct, B * H);
  const size_t need = sizeof(float) * (2 * dk + STEP_RG * STEP_COLS);
  // without GroupNorm at most two CTAs per SM (see StepCfg)
  const size_t smem = eps < 0.f && need < STEP_SMEM_FLOOR ? STEP_SMEM_FLOOR : need;
  const T* qq = static_cast<const T*>(q);
  const T* kk = static_cast<const T*>(k);
  const T* vv = static_cast<const T*>(v);
  T* oo = static_cast<T*>(o);
  const T* gg = static_cast<const T*>(gate);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(STEP_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = nct;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  auto go = [&](auto fn, int nattrs) -> cudaError_t {
    if (smem > 48 * 1024) {
      cudaError_t e =
          cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    cfg.numAttrs = nattrs;
    return cudaLaunchKernelEx(&cfg, fn, qq, kk, vv, gammas, state, gg, oo, H, dk, dv, eps, theta,
                              pos);
  };
  // GroupNorm: the CTAs of one (b, h) form a cluster that exchanges row statistics
  if (eps < 0.f)
    return theta ? go(step_kernel<T, false, true>, 1) : go(step_kernel<T, false, false>, 1);
  return theta ? go(step_kernel<T, true, true>, 2) : go(step_kernel<T, true, false>, 2);
}

cudaError_t launch_step(const void* q, const void* k, const void* v, const float* gammas,
                        float* state, const void* gate, void* o, int B, int H, int dk, int dv,
                        int dtype, float eps, const float* theta, long long pos,
                        cudaStream_t st) {
  if (dtype == RET_BF16)
    return launch_step_t<__nv_bfloat16>(q, k, v, gammas, state, gate, o, B, H, dk, dv, eps,
                                        theta, pos, st);
  return launch_step_t<float>(q, k, v, gammas, state, gate, o, B, H, dk, dv, eps, theta, pos,
                              st);
}

}  // namespace ret
