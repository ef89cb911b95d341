// Chunk output on CTA pairs (tcgen05 cta_group::2): bf16 operands, float32
// accumulation.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations (Parallel Form, Chunkwise Recurrent):
//     O_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + (Q_[i] (.) xi) R_{i-1}
// with D[n][m] = gamma^(n-m) for n >= m and xi_j = gamma^(j+1).
//
// Same computation as the single-CTA kernel, arranged for the tensor cores of
// two SMs at once.  A work tile is a pair of 128-row query tiles (2j, 2j+1)
// of one chunk: each CTA of a pair owns one of them (its Q rows, its P in
// TMEM, its rows of O), and every product runs as one M = 256 MMA issued by
// the pair's even CTA.  The B operands (K tiles, V tiles, the chunk state R)
// are split between the two CTAs by columns, so each SM loads half of them:
// the load on L2 per output row drops by about 40 %, which is what bounds the
// single-CTA kernel.  Rows of tile 2j also multiply key tile 2j+1, which the
// decay mask zeroes; that costs a few percent of MMA work.
// With d_v = 512 two pairs (one per 256-column slice) form a 4-CTA cluster
// and exchange GroupNorm statistics between CTAs holding the same rows.
//
// Roles per CTA (both CTAs of a pair run all of them except the MMA issue):
//   warp 0     TMA: own Q rows; own half of each K / V / R tile, counted on
//              the leader's barriers
//   warp 1     (leader) tcgen05.mma.cta_group::2, commits multicast to the pair
//   warps 2-5  decay mask of own rows (S -> P in own TMEM), then Q (.) xi
//   warps 6-9  epilogue of own rows: optional GroupNorm, bf16 stores
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace ret {
namespace k3p {

using namespace sm100;

constexpr int BM = 128;                // query rows per CTA
constexpr int BN = 128;                // keys per key tile (64 in each CTA)
constexpr int DVS = 256;               // output columns per slice
constexpr int STAGE = 32768;
constexpr int QBOX = 128 * 128;        // [128 rows][64] bf16 = 16 KB
constexpr int HBOX = 64 * 128;         // [64 rows][64] bf16 = 8 KB
constexpr int QBUF = 4 * QBOX;
constexpr int NQB = 2;                 // Q buffers: the next tile's Q loads early
constexpr int RING = 3;
constexpr int Q_OFF = 0;
constexpr int RING_OFF = NQB * QBUF;
constexpr int GN_OFF = RING_OFF + RING * STAGE;  // [2 slots][2 values][128] floats
constexpr int BAR_OFF = GN_OFF + 2048;
constexpr int ALIGN_SLACK = 512;
constexpr int SMEM_BYTES = BAR_OFF + 256 + ALIGN_SLACK;
constexpr int THREADS = 320;

struct Params {
  const float* gammas;
  __nv_bfloat16* o;
  int H, N, chunk, tpc, nc, dk, dv, dvs, nslices, ntiles;
  int chunked;
  int has_state0;
  float eps;
};

struct Tile {
  int bh, ci, r, cs, n0, nt;
  bool has_r;
};

// Pair tile t -> this CTA's row tile (2j + member) of chunk ci of head bh.
__device__ __forceinline__ Tile decode_tile(const Params& p, int t, int member) {
  Tile x;
  const int pairs = p.tpc / 2;
  const int jj = t % pairs;
  const int rest = t / pairs;
  x.ci = rest % p.nc;
  x.bh = rest / p.nc;
  const int j = pairs - 1 - jj;  // longest rows of a chunk first
  x.r = 2 * j + member;
  x.cs = x.ci * p.chunk;
  x.n0 = x.cs + x.r * BM;
  x.nt = 2 * j + 2;              // key tiles of the pair
  x.has_r = p.chunked && (x.ci > 0 || p.has_state0);
  return x;
}

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

__device__ __forceinline__ void chan_merge(float& n_a, float& mean_a, float& m2_a, float n_b,
                                           float mean_b, float m2_b) {
  const float n = n_a + n_b;
  const float d = mean_b - mean_a;
  mean_a += d * (n_b / n);
  m2_a += m2_b + d * d * (n_a * n_b / n);
  n_a = n;
}

template <bool GN>
__global__ void __launch_bounds__(THREADS, 1)
chunk_out_pair(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_r,
               const __grid_constant__ CUtensorMap tm_o, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uintptr_t aligned = (raw + 1023) & ~static_cast<uintptr_t>(1023);
  if (aligned - raw > ALIGN_SLACK) {  // same for every CTA of the cluster
    if (threadIdx.x == 0) record_error(399);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>(aligned);
  const uint32_t rank = cluster_ctarank();
  const int member = rank & 1;           // 0: leader of the pair
  const uint32_t lead = rank & ~1u;
  const uint16_t pair_mask = static_cast<uint16_t>(3u << lead);
  const int slice = rank >> 1;
  const int c0 = slice * p.dvs;
  const int ch = p.dvs / 2;              // columns of each B half
  const int nvb = ch / 64;               // 64-wide column blocks per half
  const int kq = p.dk / 64;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full = bars;                 // [RING]  (leader)
  uint64_t* empty = bars + RING;         // [RING]  (both)
  uint64_t* q_full = bars + 2 * RING;    // [2]     (leader)
  uint64_t* q_empty = q_full + 2;        // [2]     (both)
  uint64_t* s_full = q_full + 4;         // [2]     (both)
  uint64_t* p_full = q_full + 6;         // [2]     (leader, 8 warps)
  uint64_t* qt_full = q_full + 8;        //         (leader, 8 warps)
  uint64_t* o_full = q_full + 9;         //         (both)
  uint64_t* o_free = q_full + 10;        //         (leader, 8 warps)
  uint64_t* gn_bar = q_full + 11;        // [2]
  uint64_t* drain = q_full + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 14);
  float* gn_red = reinterpret_cast<float*>(smem + GN_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);  // arrived by this CTA's epilogue (the buffer stages O)
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 8);
      mbar_init(&gn_bar[b], 128);
    }
    mbar_init(qt_full, 8);
    mbar_init(o_full, 1);
    mbar_init(o_free, 8);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc2(tmem_slot, 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // every barrier of the cluster exists before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int tile0 = blockIdx.y;
  const int tstep = gridDim.y;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (p.chunked) tma_prefetch_desc(&tm_r);
      int g = 0, k = 0;
      bool ok = true;
      auto load_q = [&](int kk, const Tile& x) -> bool {
        const int qb = kk % NQB;
        if (!mbar_wait_cluster(&q_empty[qb], ((kk / NQB) & 1) ^ 1, 301)) return false;
        const uint32_t bar = cluster_addr(&q_full[qb], lead);
        if (member == 0) mbar_arrive_expect_tx(&q_full[qb], 2 * kq * QBOX);
        for (int b = 0; b < kq; ++b)
          tma_load_3d_pair(smem + Q_OFF + qb * QBUF + b * QBOX, &tm_q, bar, b * 64, x.n0, x.bh);
        return true;
      };
      // one ring stage: wait until the pair's MMAs released it, announce the
      // pair's bytes on the leader's barrier (leader only), return its address
      auto acquire = [&](uint32_t bytes_per_cta, uint32_t& bar) -> uint8_t* {
        const int slot = g % RING;
        if (!mbar_wait_cluster(&empty[slot], ((g / RING) & 1) ^ 1, 302)) return nullptr;
        bar = cluster_addr(&full[slot], lead);
        if (member == 0) mbar_arrive_expect_tx(&full[slot], 2 * bytes_per_cta);
        return smem + RING_OFF + slot * STAGE;
      };
      for (int tile = tile0; tile < p.ntiles && ok; tile += tstep, ++k) {
        const Tile x = decode_tile(p, tile, member);
        if (k == 0) ok = load_q(0, x);
        bool next_q = false;
        for (int t = 0; t <= x.nt && ok; ++t) {
          if (t < x.nt) {
            // own 64 keys of key tile t, all of d_k
            uint32_t bar;
            uint8_t* st = acquire(kq * HBOX, bar);
            if (!st) { ok = false; break; }
            const int key0 = x.cs + t * BN + 64 * member;
            for (int b = 0; b < kq; ++b)
              tma_load_3d_pair(st + b * HBOX, &tm_k, bar, b * 64, key0, x.bh);
            ++g;
          }
          if (!next_q && ok) {
            next_q = true;
            if (tile + tstep < p.ntiles) ok = load_q(k + 1, decode_tile(p, tile + tstep, member));
          }
          if (t >= 1 && ok) {
            // own column half of V for key tile t-1: [key half][column block]
            uint32_t bar;
            uint8_t* st = acquire(2 * nvb * HBOX, bar);
            if (!st) { ok = false; break; }
            const int key0 = x.cs + (t - 1) * BN;
            for (int h2 = 0; h2 < 2; ++h2)
              for (int d = 0; d < nvb; ++d)
                tma_load_3d_pair(st + (h2 * nvb + d) * HBOX, &tm_v, bar,
                                 c0 + member * ch + d * 64, key0 + 64 * h2, x.bh);
            ++g;
          }
        }
        if (x.has_r && ok) {
          // own column half of R_{i-1}, 128 rows of d_k per stage
          const int zr = x.bh * p.nc + x.ci;
          for (int s = 0; s < (kq + 1) / 2 && ok; ++s) {
            const int nb = min(2, kq - 2 * s);
            uint32_t bar;
            uint8_t* st = acquire(nb * nvb * HBOX, bar);
            if (!st) { ok = false; break; }
            for (int b = 0; b < nb; ++b)
              for (int d = 0; d < nvb; ++d)
                tma_load_3d_pair(st + (b * nvb + d) * HBOX, &tm_r, bar, c0 + member * ch + d * 64,
                                 128 * s + 64 * b, zr);
            ++g;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only) ----------------
    if (lane == 0 && member == 0) {
      const uint32_t id_qk = idesc_bf16(256, BN, false, false);
      const uint32_t id_pv = idesc_bf16(256, p.dvs, false, true);
      const uint32_t o_tm = tmem + 256;
      int g = 0, sc = 0, k = 0;
      bool ok = true;
      auto take = [&](uint32_t& addr) -> bool {
        const int slot = g % RING;
        if (!mbar_wait_cluster(&full[slot], (g / RING) & 1, 303)) return false;
        tc_fence_after();
        addr = smem_u32(smem + RING_OFF + slot * STAGE);
        return true;
      };
      auto give = [&]() {
        umma2_commit_mc(&empty[g % RING], pair_mask);
        ++g;
      };
      for (int tile = tile0; tile < p.ntiles && ok; tile += tstep, ++k) {
        const Tile x = decode_tile(p, tile, 0);
        const int qb = k % NQB;
        const uint32_t q_addr = smem_u32(smem + Q_OFF + qb * QBUF);
        if (!mbar_wait_cluster(&q_full[qb], (k / NQB) & 1, 304)) { ok = false; break; }
        tc_fence_after();
        const int s0 = sc;
        for (int t = 0; t <= x.nt && ok; ++t) {
          if (t < x.nt) {
            const int b = sc & 1;
            uint32_t sa;
            if (!take(sa)) { ok = false; break; }
            for (int kk = 0; kk < 4 * kq; ++kk) {
              const uint64_t a = sdesc_sw128(q_addr + (kk >> 2) * QBOX + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(sa + (kk >> 2) * HBOX + (kk & 3) * 32, 16, 1024);
              umma2_bf16_ss(tmem + b * BN, a, bd, id_qk, kk ? 1u : 0u);
            }
            give();
            umma2_commit_mc(&s_full[b], pair_mask);
            ++sc;
          }
          if (t >= 1) {
            const int tp = t - 1;
            const int su = s0 + tp;
            const int b = su & 1;
            if (!mbar_wait_cluster(&p_full[b], (su >> 1) & 1, 305)) { ok = false; break; }
            if (tp == 0 && k >= 1 && !mbar_wait_cluster(o_free, (k - 1) & 1, 306)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint32_t sa;
            if (!take(sa)) { ok = false; break; }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // 16 keys each
              const uint32_t boff = (kk >> 2) * nvb * HBOX + (kk & 3) * 2048;
              const uint64_t bd = sdesc_sw128(sa + boff, HBOX, 1024);
              umma2_bf16_ts(o_tm, tmem + b * BN + 8 * kk, bd, id_pv, (tp | kk) ? 1u : 0u);
            }
            give();
          }
        }
        if (!ok) break;
        if (!mbar_wait_cluster(qt_full, k & 1, 307)) { ok = false; break; }
        tc_fence_after();
        if (x.has_r) {
          for (int s = 0; s < (kq + 1) / 2 && ok; ++s) {
            const int nb = min(2, kq - 2 * s);
            uint32_t sa;
            if (!take(sa)) { ok = false; break; }
            for (int kk = 0; kk < 4 * nb; ++kk) {  // 16 rows of d_k each
              const int kb = 2 * s + (kk >> 2);
              const uint64_t a = sdesc_sw128(q_addr + kb * QBOX + (kk & 3) * 32, 16, 1024);
              const uint32_t boff = (kk >> 2) * nvb * HBOX + (kk & 3) * 2048;
              const uint64_t bd = sdesc_sw128(sa + boff, HBOX, 1024);
              umma2_bf16_ss(o_tm, a, bd, id_pv, 1u);
            }
            give();
          }
        }
        umma2_commit_mc(o_full, pair_mask);
      }
      umma2_commit_mc(drain, static_cast<uint16_t>(1u << rank));
      mbar_wait(drain, 0, 309);
    }
  } else if (warp < 6) {
    // ---------------- decay mask and Q (.) xi (own rows) ----------------
    const int q = warp & 3;
    const int i = 32 * q + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    int sc = 0, k = 0;
    bool ok = true;
    for (int tile = tile0; tile < p.ntiles && ok; tile += tstep, ++k) {
      const Tile x = decode_tile(p, tile, member);
      const float gam = p.gammas[x.bh % p.H];
      const float lg = log2f(gam);
      const int j = x.r * BM + i;
      for (int t = 0; t < x.nt && ok; ++t, ++sc) {
        const int b = sc & 1;
        if (!mbar_wait_cluster(&s_full[b], (sc >> 1) & 1, 310)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sbuf = tmem + lane_addr + b * BN;
#pragma unroll 1
        for (int gq = 0; gq < 4; ++gq) {
          uint32_t sv[32];
          tmem_ld32(sbuf + 32 * gq, sv);
          tmem_wait_ld();
          const int e0 = j - (t * BN + 32 * gq + 31);
          uint32_t pk[16];
          if (e0 <= -32) {
#pragma unroll
            for (int xx = 0; xx < 16; ++xx) pk[xx] = 0u;
          } else {
            float w = e0 > 0 ? exp2f(static_cast<float>(e0) * lg) : (e0 == 0 ? 1.f : 0.f);
            float pv[32];
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) {
              pv[31 - kk] = __uint_as_float(sv[31 - kk]) * w;
              w = (e0 + kk + 1 == 0) ? 1.f : w * gam;
            }
#pragma unroll
            for (int xx = 0; xx < 16; ++xx) pk[xx] = pack_bf16(pv[2 * xx], pv[2 * xx + 1]);
          }
          tmem_st16(sbuf + 16 * gq, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(cluster_addr(&p_full[b], lead));
      }
      if (!ok) break;
      if (x.has_r) {
        const float xi = gpow(lg, j + 1);
        const uint32_t qa = smem_u32(smem + Q_OFF + (k % NQB) * QBUF) + i * 128;
        for (int bq = 0; bq < kq; ++bq) {
          uint4 v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = ld_shared_v4(qa + bq * QBOX + ((u + lane) & 7) * 16);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t in[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t o4[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              o4[c] = pack_bf16(bf16lo_to_f32(in[c]) * xi, bf16hi_to_f32(in[c]) * xi);
            st_shared_v4(qa + bq * QBOX + ((u + lane) & 7) * 16, o4[0], o4[1], o4[2], o4[3]);
          }
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(cluster_addr(qt_full, lead));
    }
  } else {
    // ---------------- epilogue (own rows) ----------------
    const int q = warp & 3;
    const int i = 32 * q + lane;
    const uint32_t o_tm = tmem + (static_cast<uint32_t>(32 * q) << 16) + 256;
    const int ncg = p.dvs / 32;
    int k = 0;
    bool ok = true;
    for (int tile = tile0; tile < p.ntiles && ok; tile += tstep, ++k) {
      const Tile x = decode_tile(p, tile, member);
      if (!mbar_wait_cluster(o_full, k & 1, 312)) { ok = false; break; }
      tc_fence_after();
      float mean = 0.f, inv = 1.f;
      if (GN) {
        float n_a = 0.f, m_a = 0.f, q_a = 0.f;
        for (int cg = 0; cg < ncg; ++cg) {
          uint32_t v[32];
          tmem_ld32(o_tm + 32 * cg, v);
          tmem_wait_ld();
          float s1 = 0.f;
#pragma unroll
          for (int xx = 0; xx < 32; ++xx) s1 += __uint_as_float(v[xx]);
          const float m = s1 * (1.f / 32.f);
          float s2 = 0.f;
#pragma unroll
          for (int xx = 0; xx < 32; ++xx) {
            const float d = __uint_as_float(v[xx]) - m;
            s2 = fmaf(d, d, s2);
          }
          if (cg == 0) {
            n_a = 32.f; m_a = m; q_a = s2;
          } else {
            chan_merge(n_a, m_a, q_a, 32.f, m, s2);
          }
        }
        if (p.nslices > 1) {
          const int slot = k & 1;
          const uint32_t peer = rank ^ 2u;  // same rows, other column slice
          st_cluster_f32(&gn_red[slot * 256 + i], peer, m_a);
          st_cluster_f32(&gn_red[slot * 256 + 128 + i], peer, q_a);
          mbar_arrive_cluster(&gn_bar[slot], peer);
          if (!mbar_wait_cluster(&gn_bar[slot], (k >> 1) & 1, 313)) { ok = false; }
          else chan_merge(n_a, m_a, q_a, static_cast<float>(p.dvs), gn_red[slot * 256 + i],
                          gn_red[slot * 256 + 128 + i]);
        }
        mean = m_a;
        inv = 1.0f / sqrtf(q_a / static_cast<float>(p.dv) + p.eps);
      }
      // stage bf16 O in this tile's Q buffer (swizzled, [block][128 rows][128 B])
      // and write it with coalesced TMA stores
      const uint32_t stage_a = smem_u32(smem + Q_OFF + (k % NQB) * QBUF) + i * 128;
      for (int cg = 0; cg < ncg; ++cg) {
        uint32_t v[32];
        tmem_ld32(o_tm + 32 * cg, v);
        tmem_wait_ld();
        if (cg == ncg - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(cluster_addr(o_free, lead));
        }
        uint32_t pk[16];
#pragma unroll
        for (int xx = 0; xx < 16; ++xx)
          pk[xx] = pack_bf16((__uint_as_float(v[2 * xx]) - mean) * inv,
                             (__uint_as_float(v[2 * xx + 1]) - mean) * inv);
        const uint32_t rowa = stage_a + (cg >> 1) * QBOX;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int phys = (((cg & 1) * 4 + c) ^ (i & 7));
          st_shared_v4(rowa + phys * 16, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      epi_bar();
      if (warp == 6 && lane == 0) {
        const uint32_t sb = smem_u32(smem + Q_OFF + (k % NQB) * QBUF);
        for (int b = 0; b < p.dvs / 64; ++b)
          tma_store_3d(&tm_o, sb + b * QBOX, c0 + b * 64, x.n0, x.bh);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(&q_empty[k % NQB]);  // this CTA's loader may refill the buffer
      }
    }
  }

  // The leader's MMAs have drained (its warp 1 waited on `drain`); no TMA of
  // either CTA is still in flight once its consumers have seen every stage.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
  cluster_sync_all();  // no CTA leaves while a peer may touch its shared memory
}

}  // namespace k3p

int tc_out2_device_error() { return read_clear_device_error(); }

static constexpr int kPairEnabled = 0;

bool tc_out2_supported(int dk, int dv, int chunk, int parallel_form) {
  // Measured on B200 at the shapes of the 1.3B/6.7B layers: not faster than
  // the single-CTA kernel, so not selected; kept for shapes where loads bound.
  if (kPairEnabled == 0) return false;
  if (dv < 128) return false;
  (void)dk;
  if (parallel_form) return true;
  return chunk >= 256;
}

cudaError_t launch_tc_out2(const void* q, const void* k, const void* v, const float* gammas,
                           int chunk, const void* ws, int has_state0, void* o, int B, int H, int N,
                           int dk, int dv, float eps, int parallel_form, cudaStream_t st) {
  using namespace k3p;
  const uint64_t BH = (uint64_t)B * H;
  Params p;
  p.gammas = gammas;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.H = H;
  p.N = N;
  // the parallel form is one chunk, padded to a whole number of row-tile pairs
  p.chunk = parallel_form ? cdiv(N, 2 * BM) * 2 * BM : chunk;
  p.tpc = p.chunk / BM;
  p.nc = parallel_form ? 1 : cdiv(N, chunk);
  p.dk = dk;
  p.dv = dv;
  p.dvs = dv < DVS ? dv : DVS;
  p.nslices = dv / p.dvs;
  p.chunked = parallel_form ? 0 : 1;
  p.has_state0 = has_state0;
  p.eps = eps;
  const int64_t ntiles = (int64_t)BH * p.nc * (p.tpc / 2);
  if (ntiles > (int64_t)1 << 30) return cudaErrorInvalidConfiguration;
  p.ntiles = static_cast<int>(ntiles);

  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int cl = 2 * p.nslices;
  int nclusters = nsm / cl;
  if (nclusters > p.ntiles) nclusters = p.ntiles;
  if (nclusters < 1) nclusters = 1;

  CUtensorMap tm_q, tm_k, tm_v, tm_r, tm_o;
  if ((e = make_tmap_bf16_3d(&tm_q, q, dk, N, BH, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_k, k, dk, N, BH, 64, 64)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_o, o, dv, N, BH, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_v, v, dv, N, BH, 64, 64)) != cudaSuccess) return e;
  if (ws) {
    if ((e = make_tmap_bf16_3d(&tm_r, ws, dv, dk, BH * p.nc, 64, 64)) != cudaSuccess) return e;
  } else {
    tm_r = tm_v;  // never read
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cl, nclusters, 1);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // A persistent grid must not exceed the clusters that can be resident at
  // once: clusters live inside one GPC, and GPCs do not split evenly into
  // clusters of 2 or 4, so SM count / cluster size can overshoot.
  auto launch = [&](auto fn) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          SMEM_BYTES);
    if (e2 != cudaSuccess) return e2;
    if (cfg.gridDim.x > 1) {
      e2 = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
      if (e2 != cudaSuccess) return e2;
      int max_clusters = 0;
      e2 = cudaOccupancyMaxActiveClusters(&max_clusters, fn, &cfg);
      if (e2 != cudaSuccess) return e2;
      if (max_clusters < 1) return cudaErrorInvalidConfiguration;
      if (cfg.gridDim.y > static_cast<unsigned>(max_clusters)) cfg.gridDim.y = max_clusters;
    }
    return cudaLaunchKernelEx(&cfg, fn, tm_q, tm_k, tm_v, tm_r, tm_o, p);
  };
  return eps >= 0.f ? launch(chunk_out_pair<true>) : launch(chunk_out_pair<false>);
}

}  // namespace ret
