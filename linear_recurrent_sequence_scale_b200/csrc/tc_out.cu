// Chunk output on the tensor cores: bf16 operands, float32 accumulation.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations (Parallel Form, Chunkwise Recurrent):
//     O_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + (Q_[i] (.) xi) R_{i-1}
// with D[n][m] = gamma^(n-m) for n >= m (0 above the diagonal) and
// xi_j = gamma^(j+1).  The parallel form is the one-chunk case without R.
//
// Persistent kernel.  A work tile is a 128-row query tile of one chunk and a
// slice of up to 256 output columns; d_v = 512 runs two slices as a 2-CTA
// cluster that exchanges GroupNorm row statistics through distributed shared
// memory.  Each CTA (one per SM) walks its tiles in a fixed order (the row
// tiles of a chunk back to back when there are enough chunks, see tile_at)
// and overlaps consecutive tiles:
//   warp 0     TMA: Q of the next tile into the second of two Q buffers while
//              the current tile runs; K, V and R_{i-1} tiles through a 3-stage
//              ring of 32 KB stages, in the order the MMAs consume them
//   warp 1     tcgen05.mma: S_t = Q K_t^T into one of two 128-column TMEM
//              buffers; O += P_t V_t with P_t read from TMEM; O += (Q (.) xi) R
//   warps 2-5  decay mask: S_t -> registers -> P_t = S_t (.) D as bf16, written
//              back into the first 64 columns of S_t's TMEM buffer; then
//              Q (.) xi in place in the tile's Q buffer
//   warps 6-   epilogue (4 warps, or with GroupNorm 8: two per TMEM lane
//              quadrant, each on half of the columns): one pass over O in
//              TMEM, after which O is free for the next tile's P V; with
//              GroupNorm the per-32-column statistics (Chan's merge, the two
//              halves through shared memory, one exchange with the peer CTA)
//              and the deviations held as scaled f16 in registers; bf16 rows
//              staged in the tile's Q buffer (with the optional output gate
//              loaded there by TMA and applied in place) and written by TMA
// When it follows the state scan of the same call the kernel is launched as
// a programmatic dependent: it may start while the scan drains, and the
// loader waits for the scan (griddepcontrol.wait) before the first R_{i-1}.
// The decay mask is never stored: each thread walks its row from the highest
// column down, multiplying by gamma per column, one exp2 per 32 columns.
// S_t's buffer is rewritten by Q K_{t+2}^T only after the MMA reading P_t was
// issued; tcgen05.mma from one thread executes in issue order.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace ret {
namespace k3 {

using namespace sm100;

constexpr int BM = 128;                // query rows per tile
constexpr int BN = 128;                // keys per key tile
constexpr int DVS = 256;               // output columns per CTA
constexpr int STAGE = 32768;
constexpr int QBOX = 128 * 128;        // [128 rows][64] bf16 = 16 KB
constexpr int VBOX = 64 * 128;         // [64 rows][64] bf16 = 8 KB
constexpr int QBUF = 4 * QBOX;         // one Q tile, d_k <= 256
constexpr int Q_OFF = 0;
constexpr int DATA_BYTES = 7 * 32768;  // Q buffers + ring stages
constexpr int GN_OFF = DATA_BYTES;     // [2 slots][2 values][128] floats
constexpr int BAR_OFF = GN_OFF + 2048;
constexpr int ALIGN_SLACK = 512;
constexpr int SMEM_BYTES = BAR_OFF + 256 + ALIGN_SLACK;
// NQB Q buffers (2: the next tile's Q loads while this tile runs; 1: two more
// ring stages in flight instead) and the ring depth that fills the rest.
template <int NQB> struct Layout {
  static constexpr int RING = (DATA_BYTES - NQB * QBUF) / STAGE;
  static constexpr int RING_OFF = NQB * QBUF;
  static_assert(RING >= 2 && RING_OFF + RING * STAGE <= DATA_BYTES, "ring layout");
  static_assert((2 * RING + 17) * 8 <= SMEM_BYTES - ALIGN_SLACK - BAR_OFF, "barrier area");
};
static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per CTA");
// Epilogue warps: with GroupNorm (two passes over O and an exchange) two per
// TMEM lane quadrant, each on half of the columns; without it one per quadrant
// (more warps measured slower there).
template <bool GN> constexpr int epi_warps() { return GN ? 8 : 4; }
template <bool GN> constexpr int threads() { return (6 + epi_warps<GN>()) * 32; }

struct Params {
  const float* gammas;
  const __nv_bfloat16* gate;  // null: no output gate
  __nv_bfloat16* o;
  int H, N, chunk, tpc, nc, dk, dv, dvs, nslices, ntiles;
  int chunked;     // 1: chunkwise form (R from the workspace), 0: parallel form
  int grouped;     // 1: a CTA runs the row tiles of a chunk back to back
  int has_state0;  // workspace slot 0 holds an incoming state
  float eps;       // GroupNorm epsilon (< 0: none)
};

struct Tile {
  int bh, ci, r, cs, n0, nt;
  bool has_r;
};

__device__ __forceinline__ Tile decode_tile(const Params& p, int t) {
  Tile x;
  const int rr = t % p.tpc;
  const int rest = t / p.tpc;
  x.ci = rest % p.nc;
  x.bh = rest / p.nc;
  x.r = p.tpc - 1 - rr;  // longest rows of a chunk first
  x.cs = x.ci * p.chunk;
  x.n0 = x.cs + x.r * BM;
  x.nt = x.r + 1;
  x.has_r = p.chunked && (x.ci > 0 || p.has_state0);
  return x;
}

// The k-th work tile of this CTA (cluster row blockIdx.y of gridDim.y), or -1
// past the end.  Grouped: whole chunks go round-robin over the cluster rows
// and a CTA runs the row tiles of a chunk back to back (longest first), so
// the K/V tiles and the chunk state its later row tiles re-read are still in
// L2 from the first; otherwise (few chunks, e.g. the parallel form) single
// tiles go round-robin.
__device__ __forceinline__ int tile_at(const Params& p, int k) {
  const int t = p.grouped ? (blockIdx.y + (k / p.tpc) * gridDim.y) * p.tpc + k % p.tpc
                          : blockIdx.y + k * gridDim.y;
  return t < p.ntiles ? t : -1;
}

// Named barriers of the epilogue warps (0 is __syncthreads).
// Barrier 1 also ANDs a flag over the epilogue warps, so that they leave the
// tile loop together when a wait has failed and never strand each other on a
// named barrier.
template <int EPI>
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(EPI * 32)
      : "memory");
  return r != 0;
}
template <int EPI>
__device__ __forceinline__ void epi_bar2() {
  asm volatile("bar.sync 2, %0;" ::"n"(EPI * 32) : "memory");
}

__device__ __forceinline__ void chan_merge(float& n_a, float& mean_a, float& m2_a, float n_b,
                                           float mean_b, float m2_b) {
  const float n = n_a + n_b;
  const float d = mean_b - mean_a;
  mean_a += d * (n_b / n);
  m2_a += m2_b + d * d * (n_a * n_b / n);
  n_a = n;
}

// swish(x) = x sigmoid(x) with sigmoid(x) = (1 + tanh(x / 2)) / 2 and the
// hardware tanh approximation: one special-function op per element instead
// of an exponential and a division.  The epilogue runs it on every output
// element, and the special-function unit is what bounds the gated tile
// (output phase on the 8k workload: 2.21 ms with exp and an IEEE division,
// 1.49 ms with fast exp and reciprocal, 1.34 ms with tanh; 1.29 ms ungated).
// The absolute error of sigmoid stays near 2^-12, far below the bf16
// rounding of the gated output at the scale of the tile.
__device__ __forceinline__ float swish_tanh(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return x * fmaf(0.5f, t, 0.5f);
}

// y <- y swish(g) on eight bf16 values (four packed pairs), g read from the
// staged gate piece at the same place.
__device__ __forceinline__ void gate_in_place(uint32_t& y0, uint32_t& y1, uint32_t& y2,
                                              uint32_t& y3, const uint4 g) {
  uint32_t* y[4] = {&y0, &y1, &y2, &y3};
  const uint32_t gi[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)
    *y[e] = pack_bf16(bf16lo_to_f32(*y[e]) * swish_tanh(bf16lo_to_f32(gi[e])),
                      bf16hi_to_f32(*y[e]) * swish_tanh(bf16hi_to_f32(gi[e])));
}

// Sum of 32 values as a balanced tree: depth 5 instead of a 32-long chain.
__device__ __forceinline__ float tree_sum32(const float (&x)[32]) {
  float t[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) t[j] = x[j] + x[j + 16];
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
    for (int j = 0; j < w; ++j) t[j] += t[j + w];
  }
  return t[0];
}

// Sum of squares of 32 values, the same tree.
__device__ __forceinline__ float tree_sumsq32(const float (&x)[32]) {
  float t[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) t[j] = fmaf(x[j], x[j], x[j + 16] * x[j + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
    for (int j = 0; j < w; ++j) t[j] += t[j + w];
  }
  return t[0];
}

template <bool GN, int NQB, int KQ, bool GATE>
__global__ void __launch_bounds__(threads<GN>(), 1)
chunk_out_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_r,
             const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_g,
             const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uintptr_t aligned = (raw + 1023) & ~static_cast<uintptr_t>(1023);
  if (aligned - raw > ALIGN_SLACK) {  // never seen: the dynamic window is 1 KB aligned
    if (threadIdx.x == 0) record_error(299);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>(aligned);
  constexpr int RING = Layout<NQB>::RING;
  constexpr int RING_OFF = Layout<NQB>::RING_OFF;
  constexpr int EPI = epi_warps<GN>();
  constexpr int NH = EPI / 4;          // epilogue warps per TMEM lane quadrant
  constexpr int GN_G = DVS / (32 * NH);  // most 32-column groups an epilogue warp holds
  const int slice = blockIdx.x;
  const int c0 = slice * p.dvs;
  constexpr int kq = KQ;              // 64-wide blocks of d_k
  constexpr int kst = (KQ + 1) / 2;   // K-tile stages (two blocks each)
  constexpr int KST = kst;
  const int vb = p.dvs / 64;          // 64-wide blocks of the column slice

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full = bars;              // [RING]
  uint64_t* empty = bars + RING;      // [RING]
  uint64_t* q_full = bars + 2 * RING; // [2]
  uint64_t* q_empty = q_full + 2;     // [2]
  uint64_t* s_full = q_full + 4;      // [2]
  uint64_t* p_full = q_full + 6;      // [2]
  uint64_t* qt_full = q_full + 8;
  uint64_t* o_full = q_full + 9;
  uint64_t* o_free = q_full + 10;
  uint64_t* gn_bar = q_full + 11;     // [2]
  uint64_t* drain = q_full + 13;
  uint64_t* g_full = q_full + 14;     // [2] gate tile in the staging buffer (boxes >= 1, box 0)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 16);
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
      mbar_init(&q_empty[b], 1);  // arrived by the epilogue: the buffer also stages O
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 4);
      mbar_init(&gn_bar[b], 128);
    }
    mbar_init(qt_full, 4);
    mbar_init(o_full, 1);
    mbar_init(o_free, EPI);
    mbar_init(drain, 1);
    mbar_init(&g_full[0], 1);
    mbar_init(&g_full[1], 1);
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

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (p.chunked) tma_prefetch_desc(&tm_r);
      int g = 0, k = 0;
      bool ok = true;
      // Q of this CTA's tile sequence number qn goes to buffer qn % NQB once
      // that buffer is free (the epilogue of tile qn - NQB has stored its O
      // from it).  The loader never blocks on that while it still has ring
      // stages to issue: it polls between stages and waits only when the tile
      // that needs the Q starts.
      int qn = 0;  // next Q to load (tile sequence number)
      bool r_ready = false;
      auto issue_q = [&](bool block) -> bool {
        const int tile = tile_at(p, qn);
        if (tile < 0 || qn > k + (NQB - 1)) return true;
        const int qb = qn % NQB;
        const uint32_t par = ((qn / NQB) & 1) ^ 1;
        if (block) {
          if (!mbar_wait(&q_empty[qb], par, 201)) return false;
        } else if (!mbar_try_wait(&q_empty[qb], par)) {
          return true;
        }
        const Tile y = decode_tile(p, tile);
        mbar_arrive_expect_tx(&q_full[qb], kq * QBOX);
        for (int b = 0; b < kq; ++b)
          tma_load_3d(smem + Q_OFF + qb * QBUF + b * QBOX, &tm_q, &q_full[qb], b * 64, y.n0, y.bh);
        ++qn;
        return true;
      };
      auto acquire = [&](uint32_t bytes, uint64_t*& bar) -> uint8_t* {
        const int slot = g % RING;
        if (!issue_q(false)) return nullptr;
        if (!mbar_wait(&empty[slot], ((g / RING) & 1) ^ 1, 202)) return nullptr;
        bar = &full[slot];
        mbar_arrive_expect_tx(bar, bytes);
        return smem + RING_OFF + slot * STAGE;
      };
      for (int tile = tile_at(p, k); tile >= 0 && ok; tile = tile_at(p, ++k)) {
        const Tile x = decode_tile(p, tile);
        while (ok && qn <= k) ok = issue_q(true);  // this tile's own Q

        for (int t = 0; t <= x.nt && ok; ++t) {
          if (t < x.nt) {
            const int key0 = x.cs + t * BN;
            for (int s = 0; s < kst && ok; ++s, ++g) {
              const int nb = min(2, kq - 2 * s);
              uint64_t* bar;
              uint8_t* st = acquire(nb * QBOX, bar);
              if (!st) { ok = false; break; }
              for (int b = 0; b < nb; ++b)
                tma_load_3d(st + b * QBOX, &tm_k, bar, (2 * s + b) * 64, key0, x.bh);
            }
          }
          if (t >= 1 && ok) {
            const int key0 = x.cs + (t - 1) * BN;
            for (int s = 0; s < 2 && ok; ++s, ++g) {
              uint64_t* bar;
              uint8_t* st = acquire(vb * VBOX, bar);
              if (!st) { ok = false; break; }
              for (int b = 0; b < vb; ++b)
                tma_load_3d(st + b * VBOX, &tm_v, bar, c0 + b * 64, key0 + 64 * s, x.bh);
            }
          }
        }
        if (x.has_r && ok) {
          if (!r_ready) {
            // The chunk states come from the state scan launched just before
            // this kernel (programmatic dependent launch): this grid may have
            // started while it drained; wait for it before the first read.
            asm volatile("griddepcontrol.wait;" ::: "memory");
            r_ready = true;
          }
          const int zr = x.bh * p.nc + x.ci;
          for (int s = 0; s < kq && ok; ++s, ++g) {
            uint64_t* bar;
            uint8_t* st = acquire(vb * VBOX, bar);
            if (!st) { ok = false; break; }
            for (int b = 0; b < vb; ++b)
              tma_load_3d(st + b * VBOX, &tm_r, bar, c0 + b * 64, 64 * s, zr);
          }
        }
      }
      // no copy may still be landing when the CTA exits
      for (int gg = max(0, g - RING); gg < g; ++gg)
        mbar_wait(&full[gg % RING], (gg / RING) & 1, 208);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, BN, false, false);
      const uint32_t id_pv = idesc_bf16(128, p.dvs, false, true);
      const uint32_t o_tm = tmem + 256;
      int g = 0, sc = 0, k = 0;
      bool ok = true;
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
      // Descriptors: one full descriptor per operand buffer, then constant
      // offsets (the start address sits in the low bits, in 16-byte units), so
      // the issuing thread spends its time on MMAs, not on address arithmetic.
      for (int tile = tile_at(p, k); tile >= 0 && ok; tile = tile_at(p, ++k)) {
        const Tile x = decode_tile(p, tile);
        const int qb = k % NQB;
        const uint64_t qd = sdesc_sw128(smem_u32(smem + Q_OFF + qb * QBUF), 16, 1024);
        if (!mbar_wait(&q_full[qb], (k / NQB) & 1, 204)) { ok = false; break; }
        tc_fence_after();
        const int s0 = sc;  // S-buffer use index of this tile's key tile 0
        for (int t = 0; t <= x.nt && ok; ++t) {
          if (t < x.nt) {
            const int b = sc & 1;
            const uint32_t d = tmem + b * BN;
#pragma unroll
            for (int s = 0; s < KST; ++s) {
              uint32_t sa;
              if (!ok || !take(sa)) { ok = false; break; }
              const uint64_t kd = sdesc_sw128(sa, 16, 1024);
#pragma unroll
              for (int bb = 0; bb < 2; ++bb) {
                if (2 * s + bb >= KQ) break;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  umma_bf16_ss(d, qd + (((2 * s + bb) * QBOX + kk * 32) >> 4),
                               kd + ((bb * QBOX + kk * 32) >> 4), id_qk,
                               (s | bb | kk) ? 1u : 0u);
              }
              give();
            }
            if (!ok) break;
            umma_commit(&s_full[b]);
            ++sc;
          }
          if (t >= 1) {
            const int tp = t - 1;
            const int su = s0 + tp;
            const int b = su & 1;
            if (!mbar_wait(&p_full[b], (su >> 1) & 1, 205)) { ok = false; break; }
            if (tp == 0 && k >= 1 && !mbar_wait(o_free, (k - 1) & 1, 206)) { ok = false; break; }
            tc_fence_after();
            const uint32_t pa = tmem + b * BN;  // P_t: 64 columns of packed bf16
            const uint32_t acc0 = tp ? 1u : 0u;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
              uint32_t sa;
              if (!ok || !take(sa)) { ok = false; break; }
              const uint64_t vd = sdesc_sw128(sa, VBOX, 1024);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_bf16_ts(o_tm, pa + 32 * s + 8 * kk, vd + ((kk * 2048) >> 4), id_pv,
                             (s | kk) ? 1u : acc0);
              give();
            }
          }
        }
        if (!ok) break;
        if (!mbar_wait(qt_full, k & 1, 207)) { ok = false; break; }
        tc_fence_after();
        if (x.has_r) {
#pragma unroll
          for (int s = 0; s < KQ; ++s) {
            uint32_t sa;
            if (!ok || !take(sa)) { ok = false; break; }
            const uint64_t rd = sdesc_sw128(sa, VBOX, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(o_tm, qd + ((s * QBOX + kk * 32) >> 4), rd + ((kk * 2048) >> 4), id_pv,
                           1u);
            give();
          }
        }
        umma_commit(o_full);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, 209);
    }
  } else if (warp < 6) {
    // ---------------- decay mask and Q (.) xi ----------------
    const int q = warp & 3;
    const int i = 32 * q + lane;  // row in the tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    int sc = 0, k = 0;
    bool ok = true;
    for (int tile = tile_at(p, k); tile >= 0 && ok; tile = tile_at(p, ++k)) {
      const Tile x = decode_tile(p, tile);
      const int h = x.bh % p.H;
      const float gam = p.gammas[h];
      const float lg = log2f(gam);
      const int j = x.r * BM + i;  // row position inside the chunk
      for (int t = 0; t < x.nt && ok; ++t, ++sc) {
        const int b = sc & 1;
        if (!mbar_wait(&s_full[b], (sc >> 1) & 1, 210)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sbuf = tmem + lane_addr + b * BN;
#pragma unroll 1
        for (int gq = 0; gq < 4; ++gq) {
          uint32_t sv[32];
          tmem_ld32(sbuf + 32 * gq, sv);
          tmem_wait_ld();
          const int e0 = j - (t * BN + 32 * gq + 31);  // distance to the group's last column
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
          // columns [16 gq, 16 gq + 16) were read by this or an earlier group
          tmem_st16(sbuf + 16 * gq, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
      }
      if (!ok) break;
      if (x.has_r) {
        // every Q K^T of this tile is done (the last s_full covers them):
        // scale row i of the tile's Q buffer by xi_j = gamma^(j+1), in place
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
      if (lane == 0) mbar_arrive(qt_full);
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;
    const int half = (warp - 6) >> 2;     // which part of the slice's columns
    const int i = 32 * q + lane;
    const int ncg = p.dvs / (32 * NH);    // 32-column groups per warp
    const int cg0 = half * ncg;           // first group of this warp
    const uint32_t o_tm = tmem + (static_cast<uint32_t>(32 * q) << 16) + 256;
    int k = 0;
    bool ok = true;
    for (int tile = tile_at(p, k); tile >= 0 && ok; tile = tile_at(p, ++k)) {
      const Tile x = decode_tile(p, tile);
      const uint32_t stage_a = smem_u32(smem + Q_OFF + (k % NQB) * QBUF);
      if (!epi_bar_and<EPI>(mbar_wait(o_full, k & 1, 212))) break;
      tc_fence_after();
      // Output gate: its tile goes by TMA into this tile's Q buffer (the MMAs
      // that read Q are done), where the epilogue stages the output, and is
      // applied in place as each staged 16-byte piece is written.  Box 0 is
      // loaded only after the two halves' GroupNorm statistics, which pass
      // through the buffer's first 2 KB, have been read.
      const int nblk = p.dvs / 64;
      const bool late0 = GN && NH == 2;
      if (GATE && warp == 6 && lane == 0) {
        const int b0 = late0 ? 1 : 0;
        mbar_arrive_expect_tx(&g_full[0], (nblk - b0) * QBOX);
        for (int b = b0; b < nblk; ++b)
          tma_load_3d(smem + Q_OFF + (k % NQB) * QBUF + b * QBOX, &tm_g, &g_full[0], c0 + b * 64,
                      x.n0, x.bh);
      }
      bool xok = true;
      const uint32_t row_a = stage_a + i * 128;
      if (GN) {
        // One pass over O in TMEM: per 32-column group the mean m_g, the
        // squared deviations (Chan's merge across groups) and the deviations
        // x - m_g themselves, scaled by sc_g = 1 / rms(x - m_g) and kept in
        // registers as f16 (11-bit significands at unit scale, so the error
        // stays below the bf16 rounding of the output).  O is released right
        // after the last load; the exchanges and the normalisation
        //     y = (x - m_g) sc_g (inv / sc_g) + (m_g - mean) inv
        // run from registers while the next tile's P V proceeds.
        uint32_t hv[GN_G][16];
        float gm[GN_G], gs[GN_G];
        float n_a = 0.f, m_a = 0.f, q_a = 0.f;
#pragma unroll
        for (int g = 0; g < GN_G; ++g) {
          if (g < ncg) {
            uint32_t v[32];
            tmem_ld32(o_tm + 32 * (cg0 + g), v);
            tmem_wait_ld();
            if (g == ncg - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(o_free);  // O may be overwritten now
            }
            float d[32];
#pragma unroll
            for (int xx = 0; xx < 32; ++xx) d[xx] = __uint_as_float(v[xx]);
            const float m = tree_sum32(d) * (1.f / 32.f);
#pragma unroll
            for (int xx = 0; xx < 32; ++xx) d[xx] -= m;
            const float s2 = tree_sumsq32(d);
            const float sc = s2 > 0.f ? rsqrtf(s2 * (1.f / 32.f)) : 1.f;
#pragma unroll
            for (int xx = 0; xx < 16; ++xx) hv[g][xx] = pack_f16(d[2 * xx] * sc, d[2 * xx + 1] * sc);
            gm[g] = m;
            gs[g] = sc;
            if (g == 0) {
              n_a = 32.f; m_a = m; q_a = s2;
            } else {
              chan_merge(n_a, m_a, q_a, 32.f, m, s2);
            }
          }
        }
        if (NH == 2) {
          // the two halves of a row meet in shared memory (the tile's Q
          // buffer, whose last reader, the inter-chunk MMA, is done); the
          // second barrier keeps the staging writes below off it until both
          // halves have read
          float* part = reinterpret_cast<float*>(smem + Q_OFF + (k % NQB) * QBUF);
          part[(2 * half) * 128 + i] = m_a;
          part[(2 * half + 1) * 128 + i] = q_a;
          epi_bar2<EPI>();
          const float m_o = part[(2 * (half ^ 1)) * 128 + i];
          const float q_o = part[(2 * (half ^ 1) + 1) * 128 + i];
          if (GATE) fence_proxy_async_smem();  // these accesses before box 0's TMA write
          epi_bar2<EPI>();
          if (GATE && warp == 6 && lane == 0) {
            mbar_arrive_expect_tx(&g_full[1], QBOX);
            tma_load_3d(smem + Q_OFF + (k % NQB) * QBUF, &tm_g, &g_full[1], c0, x.n0, x.bh);
          }
          // merged in the same order by both halves: identical statistics
          const float mb = half ? m_a : m_o, qb = half ? q_a : q_o;
          if (half) { m_a = m_o; q_a = q_o; }
          chan_merge(n_a, m_a, q_a, n_a, mb, qb);
        }
        if (p.nslices > 1) {
          const int slot = k & 1;
          const uint32_t peer = static_cast<uint32_t>(slice ^ 1);
          if (half == 0) {
            st_cluster_f32(&gn_red[slot * 256 + i], peer, m_a);
            st_cluster_f32(&gn_red[slot * 256 + 128 + i], peer, q_a);
            mbar_arrive_cluster(&gn_bar[slot], peer);
          }
          if (!mbar_wait_cluster(&gn_bar[slot], (k >> 1) & 1, 213)) { xok = false; }
          else chan_merge(n_a, m_a, q_a, static_cast<float>(p.dvs), gn_red[slot * 256 + i],
                          gn_red[slot * 256 + 128 + i]);
        }
        const float inv = 1.0f / sqrtf(q_a / static_cast<float>(p.dv) + p.eps);
        if (GATE) {
          if (!mbar_wait(&g_full[0], k & 1, 214)) xok = false;
          if (late0 && !mbar_wait(&g_full[1], k & 1, 215)) xok = false;
        }
#pragma unroll
        for (int g = 0; g < GN_G; ++g) {
          if (g < ncg) {
            const int cg = cg0 + g;
            const float a = inv / gs[g];
            const float b = (gm[g] - m_a) * inv;
            uint32_t pk[16];
#pragma unroll
            for (int xx = 0; xx < 16; ++xx)
              pk[xx] = pack_bf16(fmaf(f16lo_to_f32(hv[g][xx]), a, b),
                                 fmaf(f16hi_to_f32(hv[g][xx]), a, b));
            const uint32_t rowa = row_a + (cg >> 1) * QBOX;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int phys = (((cg & 1) * 4 + c) ^ (i & 7));
              if (GATE) gate_in_place(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3],
                                      ld_shared_v4(rowa + phys * 16));
              st_shared_v4(rowa + phys * 16, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                           pk[4 * c + 3]);
            }
          }
        }
      } else {
        // Stage bf16 O in this tile's Q buffer as [64-column block][128 rows]
        // [128 B] with the 128-byte swizzle, then write it with coalesced TMA
        // stores; rows past N are clipped by the tensor map.
        if (GATE && !mbar_wait(&g_full[0], k & 1, 214)) xok = false;
        for (int g = 0; g < ncg; ++g) {
          const int cg = cg0 + g;
          uint32_t v[32];
          tmem_ld32(o_tm + 32 * cg, v);
          tmem_wait_ld();
          if (g == ncg - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);  // O may be overwritten now
          }
          uint32_t pk[16];
#pragma unroll
          for (int xx = 0; xx < 16; ++xx)
            pk[xx] = pack_bf16(__uint_as_float(v[2 * xx]), __uint_as_float(v[2 * xx + 1]));
          const uint32_t rowa = row_a + (cg >> 1) * QBOX;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int phys = (((cg & 1) * 4 + c) ^ (i & 7));
            if (GATE) gate_in_place(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3],
                                    ld_shared_v4(rowa + phys * 16));
            st_shared_v4(rowa + phys * 16, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
      }
      fence_proxy_async_smem();
      ok = epi_bar_and<EPI>(xok);
      if (warp == 6 && lane == 0) {
        for (int b = 0; b < p.dvs / 64; ++b)
          tma_store_3d(&tm_o, stage_a + b * QBOX, c0 + b * 64, x.n0, x.bh);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(&q_empty[k % NQB]);  // the loader may refill the buffer
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // Launched after the state scan, this grid may start before the scan ends.
  // Every CTA waits for it before leaving, so the call completes only after
  // the scan has written everything, the final state included, even when no
  // tile read a chunk state (one chunk, no incoming state).  Without a
  // programmatic dependency the wait returns at once.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (p.nslices > 1) cluster_sync_all();  // no CTA leaves while its peer may touch its smem
}

}  // namespace k3

int tc_out_device_error() { return read_clear_device_error(); }

cudaError_t launch_tc_out(const void* q, const void* k, const void* v, const float* gammas,
                          int chunk, const void* ws, int has_state0, const void* gate, void* o,
                          int B, int H, int N, int dk, int dv, float eps, int parallel_form,
                          int after_states, cudaStream_t st) {
  using namespace k3;
  const uint64_t BH = (uint64_t)B * H;
  Params p;
  p.gammas = gammas;
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.o = static_cast<__nv_bfloat16*>(o);
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
  const int64_t ntiles = (int64_t)BH * p.nc * p.tpc;
  if (ntiles > (int64_t)1 << 30) return cudaErrorInvalidConfiguration;
  p.ntiles = static_cast<int>(ntiles);
  p.grouped = 0;

  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  int nclusters = nsm / p.nslices;
  if (nclusters > p.ntiles) nclusters = p.ntiles;
  if (nclusters < 1) nclusters = 1;
  p.grouped = p.tpc > 1 && ntiles / p.tpc >= 4 * nclusters;

  CUtensorMap tm_q, tm_k, tm_v, tm_r, tm_o, tm_g;
  if ((e = make_tmap_bf16_3d(&tm_q, q, dk, N, BH, 64, BM)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_k, k, dk, N, BH, 64, BN)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16_3d(&tm_o, o, dv, N, BH, 64, BM)) != cudaSuccess) return e;
  if (gate) {
    if ((e = make_tmap_bf16_3d(&tm_g, const_cast<void*>(gate), dv, N, BH, 64, BM)) != cudaSuccess)
      return e;
  } else {
    tm_g = tm_o;  // never read
  }
  if ((e = make_tmap_bf16_3d(&tm_v, v, dv, N, BH, 64, 64)) != cudaSuccess) return e;
  if (ws) {
    if ((e = make_tmap_bf16_3d(&tm_r, ws, dv, dk, BH * p.nc, 64, 64)) != cudaSuccess) return e;
  } else {
    tm_r = tm_v;  // never read
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nslices, nclusters, 1);
  cfg.blockDim = dim3(eps >= 0.f ? threads<true>() : threads<false>());
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.nslices;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // After the state scan of the same call, the grid may be scheduled while
  // that scan drains (it only waits before reading the chunk states); any
  // other launch keeps full stream order.
  cfg.numAttrs = after_states ? 2 : 1;
  // Short tiles (chunkwise) gain most from loading the next Q early; long
  // tiles (parallel form) from a deeper ring (both measured on B200).
  const int nqb = parallel_form ? 1 : 2;
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
    return cudaLaunchKernelEx(&cfg, fn, tm_q, tm_k, tm_v, tm_r, tm_o, tm_g, p);
  };
  auto by_dk = [&](auto gn, auto q, auto gt) -> cudaError_t {
    constexpr bool G = decltype(gn)::value;
    constexpr int QB = decltype(q)::value;
    constexpr bool GT = decltype(gt)::value;
    if (dk == 64) return launch(chunk_out_tc<G, QB, 1, GT>);
    if (dk == 128) return launch(chunk_out_tc<G, QB, 2, GT>);
    return launch(chunk_out_tc<G, QB, 4, GT>);
  };
  using T1 = std::integral_constant<int, 1>;
  using T2 = std::integral_constant<int, 2>;
  auto by_q = [&](auto gn, auto gt) -> cudaError_t {
    return nqb == 1 ? by_dk(gn, T1{}, gt) : by_dk(gn, T2{}, gt);
  };
  auto by_gn = [&](auto gt) -> cudaError_t {
    return eps >= 0.f ? by_q(std::true_type{}, gt) : by_q(std::false_type{}, gt);
  };
  return gate ? by_gn(std::true_type{}) : by_gn(std::false_type{});
}

}  // namespace ret
