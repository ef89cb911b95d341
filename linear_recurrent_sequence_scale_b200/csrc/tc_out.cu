// Chunk output on the tensor cores: bf16 operands, float32 accumulation.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations (Parallel Form, Chunkwise Recurrent):
//     O_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + (Q_[i] (.) xi) R_{i-1}
// with D[n][m] = gamma^(n-m) for n >= m (0 above the diagonal) and
// xi_j = gamma^(j+1).  The parallel form is the one-chunk case without R.
//
// One CTA computes a 128-row query tile of one chunk for a slice of up to 256
// output columns; d_v = 512 uses a cluster of two CTAs (one per half) that
// exchange GroupNorm row statistics through distributed shared memory.
//   warp 0     TMA: Q tile once; then, in the order the MMAs consume them,
//              K tiles (QK^T), V tiles (P V) and the state R_{i-1} (inter term)
//              through a 3-stage ring of 32 KB stages
//   warp 1     tcgen05.mma: S_t = Q K_t^T into one of two 128-column TMEM
//              buffers; O += P_t V_t and O += (Q (.) xi) R into 256 columns
//   warps 2-5  (TMEM lanes of the 128 rows) decay mask: S_t -> registers ->
//              P_t = S_t (.) D in bf16 into shared memory; then Q (.) xi in
//              place of Q; then the epilogue: optional GroupNorm, bf16 O
//              staged in shared memory and written with TMA stores.
// The decay mask is never materialised in memory: each thread walks its row
// from the highest column down, multiplying by gamma once per column, with one
// exp2 per 32 columns to start the walk.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace ret {
namespace k3 {

using namespace sm100;

constexpr int BM = 128;                // query rows per CTA
constexpr int BN = 128;                // keys per key tile
constexpr int DVS = 256;               // output columns per CTA
constexpr int RING = 3;
constexpr int STAGE = 32768;
constexpr int QBOX = 128 * 128;        // [128 rows][64] bf16 = 16 KB
constexpr int VBOX = 64 * 128;         // [64 rows][64] bf16 = 8 KB
constexpr int Q_OFF = 0;               // up to 4 boxes
constexpr int P_OFF = 65536;           // two 32 KB P buffers (O staging at the end)
constexpr int RING_OFF = 131072;
constexpr int GN_OFF = RING_OFF + RING * STAGE;  // 2 x 128 floats from the peer CTA
constexpr int BAR_OFF = GN_OFF + 1024;
constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
constexpr int THREADS = 192;

struct Params {
  const float* gammas;
  int H, N, chunk, tpc, nc, dk, dv, dvs, nslices;
  int chunked;     // 1: chunkwise form (R from the workspace), 0: parallel form
  int has_state0;  // workspace slot 0 holds an incoming state
  float eps;       // GroupNorm epsilon (< 0: none)
};

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, uint32_t src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <bool GN>
__global__ void __launch_bounds__(THREADS, 1)
chunk_out_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_r,
             const __grid_constant__ CUtensorMap tm_o, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int slice = blockIdx.x;
  const int bh = blockIdx.z;
  const int h = bh % p.H;
  const int ci = blockIdx.y / p.tpc;
  const int r = p.tpc - 1 - static_cast<int>(blockIdx.y % p.tpc);  // long rows first
  const int cs = ci * p.chunk;
  const int n0 = cs + r * BM;
  if (n0 >= p.N) return;  // the same for every CTA of a cluster
  const int nt = r + 1;   // key tiles of this row tile
  const bool has_r = p.chunked && (ci > 0 || p.has_state0);
  const int c0 = slice * p.dvs;
  const int kq = p.dk / 64;           // 64-wide blocks of d_k
  const int kst = (kq + 1) / 2;       // K-tile stages (two blocks each)
  const int vb = p.dvs / 64;          // 64-wide blocks of the column slice

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full = bars;              // [RING]
  uint64_t* empty = bars + RING;      // [RING]
  uint64_t* s_full = bars + 2 * RING; // [2]
  uint64_t* s_free = s_full + 2;      // [2]
  uint64_t* p_full = s_full + 4;      // [2]
  uint64_t* p_empty = s_full + 6;     // [2]
  uint64_t* q_full = s_full + 8;
  uint64_t* qt_full = s_full + 9;
  uint64_t* o_full = s_full + 10;
  uint64_t* gn_bar = s_full + 11;
  uint64_t* drain = s_full + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 13);
  float* gn_red = reinterpret_cast<float*>(smem + GN_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&p_empty[b], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(qt_full, 4);
    mbar_init(o_full, 1);
    mbar_init(gn_bar, 128);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.nslices > 1) cluster_sync_all();  // peer barriers exist before any remote arrive
  const uint32_t tmem = *tmem_slot;
  const uint32_t q_addr = smem_u32(smem + Q_OFF);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (has_r) tma_prefetch_desc(&tm_r);
      mbar_arrive_expect_tx(q_full, kq * QBOX);
      for (int b = 0; b < kq; ++b)
        tma_load_3d(smem + Q_OFF + b * QBOX, &tm_q, q_full, b * 64, n0, bh);
      int g = 0;
      bool ok = true;
      auto acquire = [&](uint32_t bytes, uint64_t*& bar) -> uint8_t* {
        const int slot = g % RING;
        if (!mbar_wait(&empty[slot], ((g / RING) & 1) ^ 1, 201)) return nullptr;
        bar = &full[slot];
        mbar_arrive_expect_tx(bar, bytes);
        return smem + RING_OFF + slot * STAGE;
      };
      for (int t = 0; t <= nt && ok; ++t) {
        if (t < nt) {
          const int key0 = cs + t * BN;
          for (int s = 0; s < kst && ok; ++s, ++g) {
            const int nb = min(2, kq - 2 * s);
            uint64_t* bar;
            uint8_t* st = acquire(nb * QBOX, bar);
            if (!st) { ok = false; break; }
            for (int b = 0; b < nb; ++b)
              tma_load_3d(st + b * QBOX, &tm_k, bar, (2 * s + b) * 64, key0, bh);
          }
        }
        if (t >= 1 && ok) {
          const int key0 = cs + (t - 1) * BN;
          for (int s = 0; s < 2 && ok; ++s, ++g) {
            uint64_t* bar;
            uint8_t* st = acquire(vb * VBOX, bar);
            if (!st) { ok = false; break; }
            for (int b = 0; b < vb; ++b)
              tma_load_3d(st + b * VBOX, &tm_v, bar, c0 + b * 64, key0 + 64 * s, bh);
          }
        }
      }
      if (has_r && ok) {
        const int zr = bh * p.nc + ci;
        for (int s = 0; s < kq && ok; ++s, ++g) {
          uint64_t* bar;
          uint8_t* st = acquire(vb * VBOX, bar);
          if (!st) { ok = false; break; }
          for (int b = 0; b < vb; ++b) tma_load_3d(st + b * VBOX, &tm_r, bar, c0 + b * 64, 64 * s, zr);
        }
      }
      for (int gg = max(0, g - RING); gg < g; ++gg)
        mbar_wait(&full[gg % RING], (gg / RING) & 1, 208);
      mbar_wait(q_full, 0, 209);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, BN, false, false);
      const uint32_t id_pv = idesc_bf16(128, p.dvs, false, true);
      const uint32_t o_tm = tmem + 256;
      int g = 0;
      bool ok = mbar_wait(q_full, 0, 202);
      tc_fence_after();
      auto take = [&](uint32_t& addr) -> bool {
        const int slot = g % RING;
        if (!mbar_wait(&full[slot], (g / RING) & 1, 203)) return false;
        tc_fence_after();
        addr = smem_u32(smem + RING_OFF + slot * STAGE);
        return true;
      };
      auto give = [&]() {
        umma_commit(&empty[g % RING]);
        ++g;
      };
      for (int t = 0; t <= nt && ok; ++t) {
        if (t < nt) {
          const int b = t & 1, u = t >> 1;
          if (u >= 1 && !mbar_wait(&s_free[b], (u - 1) & 1, 204)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + b * BN;
          for (int s = 0; s < kst && ok; ++s) {
            uint32_t sa;
            if (!take(sa)) { ok = false; break; }
            const int nb = min(2, kq - 2 * s);
            for (int bb = 0; bb < nb; ++bb)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const int kb = 2 * s + bb;
                const uint64_t a = sdesc_sw128(q_addr + kb * QBOX + kk * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(sa + bb * QBOX + kk * 32, 16, 1024);
                umma_bf16_ss(d, a, bd, id_qk, (kb | kk) ? 1u : 0u);
              }
            give();
          }
          if (!ok) break;
          umma_commit(&s_full[b]);
        }
        if (t >= 1) {
          const int tp = t - 1, b = tp & 1;
          if (!mbar_wait(&p_full[b], (tp >> 1) & 1, 205)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pa = smem_u32(smem + P_OFF + b * 32768);
          for (int s = 0; s < 2 && ok; ++s) {
            uint32_t sa;
            if (!take(sa)) { ok = false; break; }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int key = 64 * s + 16 * kk;
              const uint64_t a = sdesc_sw128(pa + (key >> 6) * 16384 + (key & 63) * 2, 16, 1024);
              const uint64_t bd = sdesc_sw128(sa + kk * 2048, VBOX, 1024);
              umma_bf16_ss(o_tm, a, bd, id_pv, (tp | s | kk) ? 1u : 0u);
            }
            give();
          }
          if (!ok) break;
          umma_commit(&p_empty[b]);
        }
      }
      if (has_r && ok) {
        ok = mbar_wait(qt_full, 0, 206);
        tc_fence_after();
        for (int s = 0; s < kq && ok; ++s) {
          uint32_t sa;
          if (!take(sa)) { ok = false; break; }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = sdesc_sw128(q_addr + s * QBOX + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sa + kk * 2048, VBOX, 1024);
            umma_bf16_ss(o_tm, a, bd, id_pv, 1u);
          }
          give();
        }
      }
      if (ok) umma_commit(o_full);
      umma_commit(drain);
      mbar_wait(drain, 0, 207);
    }
  } else {
    // ---------------- decay mask, Q (.) xi, epilogue ----------------
    const int q = warp & 3;
    const int i = 32 * q + lane;                  // row in the tile = TMEM lane
    const int j = r * BM + i;                     // row position inside the chunk
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const float gam = p.gammas[h];
    const float lg = log2f(gam);
    bool ok = true;
    for (int t = 0; t < nt && ok; ++t) {
      const int b = t & 1, u = t >> 1;
      if (!mbar_wait(&s_full[b], u & 1, 210)) { ok = false; break; }
      tc_fence_after();
      if (u >= 1 && !mbar_wait(&p_empty[b], (u - 1) & 1, 211)) { ok = false; break; }
      const uint32_t pbase = smem_u32(smem + P_OFF + b * 32768) + i * 128;
#pragma unroll 1
      for (int gq = 0; gq < 4; ++gq) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_addr + b * BN + 32 * gq, sv);
        tmem_wait_ld();
        const int e0 = j - (t * BN + 32 * gq + 31);  // distance to the group's last column
        uint32_t pk[16];
        if (e0 <= -32) {
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = 0u;
        } else {
          float w = e0 > 0 ? exp2f(static_cast<float>(e0) * lg) : (e0 == 0 ? 1.f : 0.f);
          float pv[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            pv[31 - k] = __uint_as_float(sv[31 - k]) * w;
            w = (e0 + k + 1 == 0) ? 1.f : w * gam;
          }
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = pack_bf16(pv[2 * x], pv[2 * x + 1]);
        }
        const uint32_t rowa = pbase + (gq >> 1) * 16384;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int phys = (((gq & 1) * 4 + c) ^ (i & 7));
          st_shared_v4(rowa + phys * 16, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_free[b]);
        mbar_arrive(&p_full[b]);
      }
    }
    if (has_r && ok) {
      // all Q K^T products are done (the last s_full covers them): Q -> Q (.) xi in place
      const float xi = gpow(lg, j + 1);
      for (int bq = 0; bq < kq; ++bq) {
        const uint32_t rowa = q_addr + bq * QBOX + i * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t a = rowa + ((u + lane) & 7) * 16;
          const uint4 v = ld_shared_v4(a);
          const uint32_t in[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[4];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            o[c] = pack_bf16(bf16lo_to_f32(in[c]) * xi, bf16hi_to_f32(in[c]) * xi);
          st_shared_v4(a, o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(qt_full);
    }
    // ---- epilogue ----
    if (ok) ok = mbar_wait(o_full, 0, 212);
    tc_fence_after();
    const uint32_t o_tm = tmem + lane_addr + 256;
    const int ncg = p.dvs / 32;
    float mean = 0.f, inv = 1.f;
    if (GN) {
      float s1 = 0.f;
      for (int cg = 0; cg < ncg; ++cg) {
        uint32_t v[32];
        tmem_ld32(o_tm + 32 * cg, v);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) s1 += __uint_as_float(v[x]);
      }
      if (p.nslices > 1) {
        const uint32_t peer = static_cast<uint32_t>(slice ^ 1);
        st_cluster_f32(&gn_red[i], peer, s1);
        mbar_arrive_cluster(gn_bar, peer);
        if (mbar_wait_cluster(gn_bar, 0, 213)) s1 += gn_red[i];
      }
      mean = s1 / static_cast<float>(p.dv);
      float s2 = 0.f;
      for (int cg = 0; cg < ncg; ++cg) {
        uint32_t v[32];
        tmem_ld32(o_tm + 32 * cg, v);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float d = __uint_as_float(v[x]) - mean;
          s2 = fmaf(d, d, s2);
        }
      }
      if (p.nslices > 1) {
        const uint32_t peer = static_cast<uint32_t>(slice ^ 1);
        st_cluster_f32(&gn_red[128 + i], peer, s2);
        mbar_arrive_cluster(gn_bar, peer);
        if (mbar_wait_cluster(gn_bar, 1, 214)) s2 += gn_red[128 + i];
      }
      inv = 1.0f / sqrtf(s2 / static_cast<float>(p.dv) + p.eps);
    }
    // stage bf16 O in the (now idle) P buffers: vb boxes of [128 rows][64 cols]
    const uint32_t stage_a = smem_u32(smem + P_OFF) + i * 128;
    for (int cg = 0; cg < ncg; ++cg) {
      uint32_t v[32];
      tmem_ld32(o_tm + 32 * cg, v);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int x = 0; x < 16; ++x)
        pk[x] = pack_bf16((__uint_as_float(v[2 * x]) - mean) * inv,
                          (__uint_as_float(v[2 * x + 1]) - mean) * inv);
      const uint32_t rowa = stage_a + (cg >> 1) * 16384;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int phys = (((cg & 1) * 4 + c) ^ (i & 7));
        st_shared_v4(rowa + phys * 16, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
    }
    fence_proxy_async_smem();
    epi_bar();
    if (warp == 2 && lane == 0) {
      if (ok)
        for (int b = 0; b < vb; ++b)
          tma_store_3d(&tm_o, smem_u32(smem + P_OFF) + b * 16384, c0 + b * 64, n0, bh);
      bulk_commit();
      bulk_wait_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (p.nslices > 1) cluster_sync_all();  // no CTA leaves while its peer may touch its smem
}

}  // namespace k3

int tc_out_device_error() { return read_clear_device_error(); }

cudaError_t launch_tc_out(const void* q, const void* k, const void* v, const float* gammas,
                          int chunk, const void* ws, int has_state0, void* o, int B, int H, int N,
                          int dk, int dv, float eps, int parallel_form, cudaStream_t st) {
  using namespace k3;
  const uint64_t BH = (uint64_t)B * H;
  Params p;
  p.gammas = gammas;
  p.H = H;
  p.N = N;
  p.chunk = parallel_form ? cdiv(N, BM) * BM : chunk;
  p.tpc = p.chunk / BM;
  p.nc = parallel_form ? 1 : cdiv(N, chunk);
  p.dk = dk;
  p.dv = dv;
  p.dvs = dv < DVS ? dv : DVS;
  p.nslices = dv / p.dvs;
  p.chunked = parallel_form ? 0 : 1;
  p.has_state0 = has_state0;
  p.eps = eps;
  if ((int64_t)p.nc * p.tpc > 65535) return cudaErrorInvalidConfiguration;

  CUtensorMap tm_q, tm_k, tm_v, tm_r, tm_o;
  cudaError_t e;
  if ((e = make_tmap_bf16_3d(&tm_q, q, dk, N, BH, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_k, k, dk, N, BH, 64, BN)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_v, v, dv, N, BH, 64, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_o, o, dv, N, BH, 64, BM)) != cudaSuccess) return e;
  if (ws) {
    if ((e = make_tmap_bf16_3d(&tm_r, ws, dv, dk, BH * p.nc, 64, 64)) != cudaSuccess) return e;
  } else {
    tm_r = tm_v;  // never read
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nslices, p.nc * p.tpc, (unsigned)BH);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.nslices;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (eps >= 0.f) {
    auto fn = chunk_out_tc<true>;
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
        cudaSuccess)
      return e;
    return cudaLaunchKernelEx(&cfg, fn, tm_q, tm_k, tm_v, tm_r, tm_o, p);
  }
  auto fn = chunk_out_tc<false>;
  if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  return cudaLaunchKernelEx(&cfg, fn, tm_q, tm_k, tm_v, tm_r, tm_o, p);
}

}  // namespace ret
