// Chunk-state scan on the tensor cores: bf16 operands, float32 state.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations, Chunkwise Recurrent: the state carried between chunks is
//     R_i = gamma^L R_{i-1} + H_i,   H_i = K_[i]^T (V_[i] (.) zeta),
//     zeta_j = gamma^(L-1-j)
// (the in-chunk decay zeta is the reading that makes the chunk state equal
// the recurrent form summed over the chunk).
//
// One CTA owns one (batch, head), MH (1 or 2) 128-row halves of d_k and NT
// (<= 128) state columns, and walks the chunks in order:
//   warp 0      TMA: V tile [T tokens][NT] and K tile [T][128 MH d_k] per
//               stage, each on its own mbarrier (V first: the transform
//               needs only V, the MMA both)
//   warps 2-9   V (.) zeta; when the final state is requested it is split
//               into bf16 hi + lo parts (16 mantissa bits of the product
//               reach the tensor core instead of 8), hi written in place of V
//   warp 1      tcgen05.mma: H_i = K^T (V hi) [+ K^T (V lo)] into a TMEM
//               accumulator that starts from zero in every chunk (M = 128
//               state rows per half, N = NT, K = 16 tokens, MN-major operands)
//   warps 10-17 the carried state R, float32 in a second TMEM region: at each
//               chunk end they read H_i (then hand the accumulator back to the
//               MMA warp), form gamma^L R + H_i with IEEE float32 FMAs, write
//               R back, and store it as bf16 to the workspace (the state
//               entering the next chunk, read by the output kernel; staged
//               per warp in shared memory and written by TMA, since 16-byte
//               stores of every thread's own row cost the transform its
//               shared-memory bandwidth) or, after the last chunk, as the
//               float32 final state.
// Accumulating each chunk afresh keeps the tensor core's running sums short
// (one chunk), so the float32 state stays accurate over any sequence length.
// MH = 2 halves the number of CTAs reading each K tile; MH = 1 gives twice
// the CTAs for small batches (the launcher picks by rounds of CTAs times
// bytes per stage).
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace ret {
namespace k2 {

using namespace sm100;

constexpr int T = 64;                  // tokens per stage (32 measured slower: more
                                       // per-stage waits and fences per token)
constexpr int NT = 128;                // state columns per CTA (d_v = 64 uses 64)
constexpr int BOX = T * 128;           // one [T][64] bf16 box
constexpr int K_OFF = 0;               // 4 boxes: up to 256 rows of d_k
constexpr int V_OFF = 4 * BOX;         // 2 boxes: NT columns of V, becomes V hi
constexpr int LO_OFF = 6 * BOX;        // 2 boxes (V lo, with the hi/lo split only)
// Ring geometry: with the hi/lo split a stage holds K, V hi and V lo (64 KB,
// 3 stages); without it K and V (48 KB), and the same shared memory holds 4
// stages, so more loads are in flight behind the transform and the MMAs.
template <bool SPLIT> struct Ring {
  static constexpr int STAGES = SPLIT ? 3 : 4;
  static constexpr int STAGE_BYTES = (SPLIT ? 8 : 6) * BOX;
};
// After the ring: one 4 KB staging box per state warp (32 state rows x 64
// columns of bf16, 128-byte swizzle) through which the chunk states leave by
// TMA, then the mbarriers.
constexpr int STG_OFF = 3 * 8 * BOX;
constexpr int STG_BYTES = 32 * 128;
constexpr int BAR_OFF = STG_OFF + 8 * STG_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 512 + 1024;
static_assert(Ring<true>::STAGES * Ring<true>::STAGE_BYTES <= STG_OFF &&
              Ring<false>::STAGES * Ring<false>::STAGE_BYTES <= STG_OFF, "ring fits");
static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per CTA");
constexpr int XF_WARPS = 8;            // V (.) zeta warps
#ifndef RET_K2_XG
#define RET_K2_XG 1
#endif
constexpr int XG = RET_K2_XG;          // groups of transform warps, taking stages in turn
constexpr int XG_THREADS = XF_WARPS * 32 / XG;
// Each ring slot must belong to one group, so that a group waiting on a
// slot's mbarrier is never more than one phase ahead of it (a parity wait
// two phases ahead would pass at once).
static_assert(XF_WARPS % XG == 0 && Ring<true>::STAGES % XG == 0 &&
                  Ring<false>::STAGES % XG == 0,
              "transform groups own whole ring slots");
constexpr int EPI_WARP0 = 2 + XF_WARPS;  // first state warp
constexpr int THREADS = (EPI_WARP0 + 8) * 32;  // 18 warps

struct Params {
  const float* gammas;
  const float* state_in;
  float* state_out;
  __nv_bfloat16* ws;  // [B*H*nc][dk][dv]; slot i = state entering chunk i
  int H, N, chunk, nc, dk, dv, nt, mh;
  int write_ws0;      // store state_in (as bf16) in slot 0
  int tma_ws;         // chunk states stored by TMA (64-column halves of NT)
};

template <bool SPLIT, int MH>
__global__ void __launch_bounds__(THREADS, 1)
state_scan_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_ws, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int STAGES = Ring<SPLIT>::STAGES;
  constexpr int STAGE_BYTES = Ring<SPLIT>::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full = bars;                 // TMA (V) -> transform
  uint64_t* xf = bars + STAGES;          // transform -> MMA
  uint64_t* empty = bars + 2 * STAGES;   // MMA -> TMA
  uint64_t* full_k = bars + 3 * STAGES;  // TMA (K) -> MMA
  uint64_t* h_full = bars + 4 * STAGES;  // MMA -> epilogue
  uint64_t* h_free = h_full + 1;         // epilogue -> MMA
  uint64_t* drain = h_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(h_full + 3);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.z;
  const int h = bh % p.H;
  const int r0 = blockIdx.y * 128 * p.mh;  // first d_k row of this CTA
  const int c0 = blockIdx.x * p.nt;        // first state column
  const int vboxes = p.nt / 64;
  const int kboxes = 2 * p.mh;             // d_k = 64 loads an out-of-range (zero) box
  // TMEM: H (accumulator) in [0, MH NT), R (carried state) in [MH NT, 2 MH NT)
  const uint32_t rcol = static_cast<uint32_t>(p.mh * p.nt);
  const uint32_t tmem_cols = 2 * rcol;     // 128, 256 or 512

  // the chunk-output kernel of the same call may be scheduled once every CTA
  // of this grid runs (it waits for this grid before reading the states)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&full_k[s], 1);
      mbar_init(&xf[s], XF_WARPS / XG);
      mbar_init(&empty[s], 1);
    }
    mbar_init(h_full, 1);
    mbar_init(h_free, 8);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float gam = p.gammas[h];
  const float lg = log2f(gam);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int g = 0;
      bool ok = true;
      for (int ci = 0; ci < p.nc && ok; ++ci) {
        const int cs = ci * p.chunk;
        const int L = min(p.chunk, p.N - cs);
        for (int j0 = 0; j0 < L; j0 += T, ++g) {
          const int slot = g % STAGES;
          if (!mbar_wait(&empty[slot], ((g / STAGES) & 1) ^ 1, 101)) { ok = false; break; }
          uint8_t* st = smem + slot * STAGE_BYTES;
          // V first, on its own barrier: the transform starts on it while K
          // (needed only by the MMA) is still landing
          mbar_arrive_expect_tx(&full[slot], vboxes * BOX);
          mbar_arrive_expect_tx(&full_k[slot], kboxes * BOX);
          for (int b = 0; b < vboxes; ++b)
            tma_load_3d(st + V_OFF + b * BOX, &tm_v, &full[slot], c0 + b * 64, cs + j0, bh);
          for (int b = 0; b < kboxes; ++b)
            tma_load_3d(st + K_OFF + b * BOX, &tm_k, &full_k[slot], r0 + b * 64, cs + j0, bh);
        }
      }
      // no copy may still be landing when the CTA exits
      for (int gg = max(0, g - STAGES); gg < g; ++gg) {
        mbar_wait(&full[gg % STAGES], (gg / STAGES) & 1, 108);
        mbar_wait(&full_k[gg % STAGES], (gg / STAGES) & 1, 108);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.nt, true, true);
      // descriptors of ring slot 0, built once; a slot, a d_k half or a
      // 16-token step is a constant offset of the start address (low bits,
      // 16-byte units), so the issue loop does no descriptor arithmetic
      const uint32_t s0 = smem_u32(smem);
      const uint64_t a0 = sdesc_sw128(s0 + K_OFF, BOX, 1024);
      const uint64_t bh0 = sdesc_sw128(s0 + V_OFF, BOX, 1024);
      const uint64_t bl0 = sdesc_sw128(s0 + LO_OFF, BOX, 1024);
      int g = 0;
      bool ok = true;
      for (int ci = 0; ci < p.nc && ok; ++ci) {
        // the epilogue must have read H_{ci-1} before it is overwritten
        if (ci >= 1 && !mbar_wait(h_free, (ci - 1) & 1, 102)) { ok = false; break; }
        tc_fence_after();
        const int L = min(p.chunk, p.N - ci * p.chunk);
        bool first = true;
        for (int j0 = 0; j0 < L; j0 += T, ++g) {
          const int slot = g % STAGES;
          if (!mbar_wait(&xf[slot], (g / STAGES) & 1, 103) ||
              !mbar_wait(&full_k[slot], (g / STAGES) & 1, 110)) { ok = false; break; }
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>((slot * STAGE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < T / 16; ++kk) {
            const uint64_t ko = so + ((kk * 2048) >> 4);
#pragma unroll
            for (int hh = 0; hh < MH; ++hh) {
              const uint64_t a = a0 + ko + ((2 * hh * BOX) >> 4);
              const uint32_t d = tmem + hh * p.nt;
              umma_bf16_ss(d, a, bh0 + ko, idesc, first ? 0u : 1u);
              if (SPLIT) umma_bf16_ss(d, a, bl0 + ko, idesc, 1u);
            }
            first = false;
          }
          umma_commit(&empty[slot]);
        }
        if (!ok) break;
        umma_commit(h_full);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, 109);
    }
  } else if (warp < EPI_WARP0) {
    // ---------------- V (.) zeta, hi/lo split ----------------
    // A stage holds T token rows of NT columns (16-byte chunks, 8 per 64-column
    // box row).  Each thread owns consecutive chunks of one token row, so it
    // needs one zeta per stage and can issue all its loads before any store.
    const int grp = (threadIdx.x - 64) / XG_THREADS;  // takes stages grp, grp + XG, ...
    const int tt = (threadIdx.x - 64) % XG_THREADS;
    const int cpr = p.nt / 8;                  // 16-byte chunks per token row
    const int per = (T * cpr) / XG_THREADS;    // chunks per thread
    const int row = (tt * per) / cpr;
    const int c_first = (tt * per) % cpr;
    int g = 0;
    bool ok = true;
    for (int ci = 0; ci < p.nc && ok; ++ci) {
      const int L = min(p.chunk, p.N - ci * p.chunk);
      for (int j0 = 0; j0 < L; j0 += T, ++g) {
        if (g % XG != grp) continue;
        const int slot = g % STAGES;
        if (!mbar_wait(&full[slot], (g / STAGES) & 1, 104)) { ok = false; break; }
        const uint32_t sb = smem_u32(smem + slot * STAGE_BYTES);
        const int j = j0 + row;
        const float z = (j < L) ? gpow(lg, L - 1 - j) : 0.f;
        constexpr int MAXP = T * (NT / 8) / XG_THREADS;  // chunks per thread at NT = 128
        uint32_t off[MAXP];
        uint4 v[MAXP];
#pragma unroll
        for (int u = 0; u < MAXP; ++u) {
          if (u < per) {
            // chunk within the row (box c/8, position c%8).  A 16-byte access
            // is served a quarter warp at a time, and its eight threads own
            // 8 * per consecutive chunks, so each 128-byte position occurs
            // `per` times among them; rotating the order by the thread's rank
            // among the threads sharing its positions makes every access of a
            // quarter warp hit eight distinct positions: no bank conflicts
            const int c = c_first + ((u + (((tt & 7) * per) >> 3)) & (per - 1));
            off[u] = (c >> 3) * BOX + row * 128 + (c & 7) * 16;
            v[u] = ld_shared_v4(sb + V_OFF + off[u]);
          }
        }
#pragma unroll
        for (int u = 0; u < MAXP; ++u) {
          if (u < per) {
            const uint32_t in[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float a = bf16lo_to_f32(in[c]) * z;
              const float b = bf16hi_to_f32(in[c]) * z;
              hi[c] = pack_bf16(a, b);
              if (SPLIT) lo[c] = pack_bf16(a - bf16lo_to_f32(hi[c]), b - bf16hi_to_f32(hi[c]));
            }
            st_shared_v4(sb + V_OFF + off[u], hi[0], hi[1], hi[2], hi[3]);
            if (SPLIT) st_shared_v4(sb + LO_OFF + off[u], lo[0], lo[1], lo[2], lo[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xf[slot]);
      }
    }
  } else {
    // ---------------- carried state (float32, TMEM region R) ----------------
    const int q = warp & 3;                   // TMEM lane quadrant
    const int part = (warp - EPI_WARP0) >> 2;  // which half of the NT columns
    const int ncol = p.nt / 2;                // 64 (or 32 when d_v = 64)
    const int row = 32 * q + lane;            // state row within a d_k half
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const int cb = c0 + part * ncol;          // first global column of this thread
    // R <- state_in (or zero); slot 0 of the workspace <- bf16(state_in)
    for (int hh = 0; hh < p.mh; ++hh) {
      const int r = r0 + 128 * hh + row;
      const bool live = r < p.dk;
      for (int x0 = 0; x0 < ncol; x0 += 32) {
        uint32_t v[32];
        if (p.state_in && live) {
          const float4* src =
              reinterpret_cast<const float4*>(p.state_in + ((size_t)bh * p.dk + r) * p.dv + cb + x0);
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float4 f = src[x];
            v[4 * x] = __float_as_uint(f.x);
            v[4 * x + 1] = __float_as_uint(f.y);
            v[4 * x + 2] = __float_as_uint(f.z);
            v[4 * x + 3] = __float_as_uint(f.w);
          }
          if (p.write_ws0) {
            uint4* dst = reinterpret_cast<uint4*>(
                p.ws + (((size_t)bh * p.nc) * p.dk + r) * p.dv + cb + x0);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(
                  pack_bf16(__uint_as_float(v[8 * x]), __uint_as_float(v[8 * x + 1])),
                  pack_bf16(__uint_as_float(v[8 * x + 2]), __uint_as_float(v[8 * x + 3])),
                  pack_bf16(__uint_as_float(v[8 * x + 4]), __uint_as_float(v[8 * x + 5])),
                  pack_bf16(__uint_as_float(v[8 * x + 6]), __uint_as_float(v[8 * x + 7])));
          }
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = 0u;
        }
        tmem_st32(tmem + lane_addr + rcol + hh * p.nt + part * ncol + x0, v);
      }
    }
    tmem_wait_st();
    for (int ci = 0; ci < p.nc; ++ci) {
      if (!mbar_wait(h_full, ci & 1, 105)) break;
      tc_fence_after();
      const float gL = gpow(lg, min(p.chunk, p.N - ci * p.chunk));
      const bool last = ci == p.nc - 1;
      // R <- gamma^L R + H, 32 columns at a time, in TMEM only; H goes back to
      // the MMA warp (h_free) as soon as it has been read, and the stores of
      // the new state to global memory follow from TMEM, off that path.
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (hh >= p.mh) continue;
#pragma unroll
        for (int x0 = 0; x0 < 64; x0 += 32) {
          if (x0 >= ncol) continue;
          const uint32_t hoff = lane_addr + hh * p.nt + part * ncol + x0;
          uint32_t hv[32], v[32];
          tmem_ld32(tmem + hoff, hv);
          tmem_ld32(tmem + rcol + hoff, v);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x)
            v[x] = __float_as_uint(fmaf(gL, __uint_as_float(v[x]), __uint_as_float(hv[x])));
          tmem_st32(tmem + rcol + hoff, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(h_free);
      // the new state from TMEM to memory: bf16 to the workspace (staged per
      // warp in shared memory and stored by TMA as one [32 rows][64 columns]
      // box), or float32 to state_out after the last chunk
      const uint32_t stg = smem_u32(smem + STG_OFF + (warp - EPI_WARP0) * STG_BYTES);
      const bool by_tma = !last && p.tma_ws;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (hh >= p.mh) continue;
        const int r = r0 + 128 * hh + row;
        const bool live = r < p.dk;
#pragma unroll
        for (int x0 = 0; x0 < 64; x0 += 32) {
          if (x0 >= ncol) continue;
          const uint32_t hoff = lane_addr + hh * p.nt + part * ncol + x0;
          uint32_t v[32];
          tmem_ld32(tmem + rcol + hoff, v);  // warp-wide: every lane loads
          tmem_wait_ld();
          if (by_tma) {
            // the previous box's store has read this warp's staging
            if (x0 == 0) {
              if (lane == 0) bulk_wait_read0();
              __syncwarp();
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const int c = (x0 / 8 + x) ^ (lane & 7);  // 128-byte swizzle
              st_shared_v4(stg + lane * 128 + c * 16,
                           pack_bf16(__uint_as_float(v[8 * x]), __uint_as_float(v[8 * x + 1])),
                           pack_bf16(__uint_as_float(v[8 * x + 2]), __uint_as_float(v[8 * x + 3])),
                           pack_bf16(__uint_as_float(v[8 * x + 4]), __uint_as_float(v[8 * x + 5])),
                           pack_bf16(__uint_as_float(v[8 * x + 6]), __uint_as_float(v[8 * x + 7])));
            }
            continue;
          }
          if (!live) continue;
          if (!last) {
            uint4* dst = reinterpret_cast<uint4*>(
                p.ws + (((size_t)bh * p.nc + ci + 1) * p.dk + r) * p.dv + cb + x0);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(
                  pack_bf16(__uint_as_float(v[8 * x]), __uint_as_float(v[8 * x + 1])),
                  pack_bf16(__uint_as_float(v[8 * x + 2]), __uint_as_float(v[8 * x + 3])),
                  pack_bf16(__uint_as_float(v[8 * x + 4]), __uint_as_float(v[8 * x + 5])),
                  pack_bf16(__uint_as_float(v[8 * x + 6]), __uint_as_float(v[8 * x + 7])));
          } else if (p.state_out) {
            float4* dst = reinterpret_cast<float4*>(p.state_out + ((size_t)bh * p.dk + r) * p.dv +
                                                    cb + x0);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              dst[x] = make_float4(__uint_as_float(v[4 * x]), __uint_as_float(v[4 * x + 1]),
                                   __uint_as_float(v[4 * x + 2]), __uint_as_float(v[4 * x + 3]));
          }
        }
        if (by_tma) {
          fence_proxy_async_smem();
          __syncwarp();
          const int rb = r0 + 128 * hh + 32 * q;  // first row of the box
          if (lane == 0 && rb < p.dk) {
            tma_store_3d(&tm_ws, stg, cb, rb, bh * p.nc + ci + 1);
            bulk_commit();
          }
        }
      }
    }
    // the staging must have been read before the CTA's shared memory goes
    if (lane == 0) bulk_wait_read0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

}  // namespace k2

int tc_state_device_error() { return read_clear_device_error(); }

cudaError_t launch_tc_state(const void* k, const void* v, const float* gammas, int chunk,
                            const float* state_in, float* state_out, void* ws, int write_ws0,
                            int B, int H, int N, int dk, int dv, cudaStream_t st) {
  using namespace k2;
  CUtensorMap tm_k, tm_v;
  const uint64_t BH = (uint64_t)B * H;
  cudaError_t e = make_tmap_bf16_3d(&tm_k, k, dk, N, BH, 64, T);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16_3d(&tm_v, v, dv, N, BH, 64, T);
  if (e != cudaSuccess) return e;
  // chunk-state boxes of [32 rows][64 columns] (state columns per warp: 64
  // unless d_v = 64, which keeps plain stores)
  CUtensorMap tm_ws;
  memset(&tm_ws, 0, sizeof(tm_ws));
  const int nc = cdiv(N, chunk);
  const int tma_ws = ws != nullptr && nc > 1 && dv >= NT ? 1 : 0;
  if (tma_ws) {
    e = make_tmap_bf16_3d(&tm_ws, ws, dv, dk, BH * nc, 64, 32);
    if (e != cudaSuccess) return e;
  }
  Params p;
  p.gammas = gammas;
  p.state_in = state_in;
  p.state_out = state_out;
  p.ws = static_cast<__nv_bfloat16*>(ws);
  p.H = H;
  p.N = N;
  p.chunk = chunk;
  p.nc = cdiv(N, chunk);
  p.dk = dk;
  p.dv = dv;
  p.nt = dv < NT ? dv : NT;
  p.write_ws0 = write_ws0;
  p.tma_ws = tma_ws;
  // Both d_k halves in one CTA (K read by half as many CTAs, 1.5x the bytes
  // per stage) or one half per CTA (twice the CTAs): a CTA walks its whole
  // sequence, one CTA per SM, so the time goes as the number of rounds of
  // CTAs over the SMs times the bytes each stage loads; take the smaller.
  // (8k layer at batch 8: 4 rounds x 6 boxes against 7 x 4, both halves;
  // 1.3B layer: 1 x 6 against 2 x 4, both halves; 64k at batch 1: 1 x 4
  // against 1 x 6, one half.)
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int halves = cdiv(dk, 128);
  const uint64_t tiles = BH * (uint64_t)(dv / p.nt);
  auto cost = [&](int mh) {
    const uint64_t ctas = tiles * (uint64_t)(halves / mh);
    return ((ctas + nsm - 1) / nsm) * (uint64_t)(2 * mh + p.nt / 64);
  };
  p.mh = (halves == 2 && cost(2) < cost(1)) ? 2 : 1;
  dim3 grid(dv / p.nt, halves / p.mh, (unsigned)BH);
  auto go = [&](auto fn) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          SMEM_BYTES);
    if (e2 != cudaSuccess) return e2;
    fn<<<grid, THREADS, SMEM_BYTES, st>>>(tm_k, tm_v, tm_ws, p);
    return cudaPeekAtLastError();
  };
  if (state_out) return p.mh == 2 ? go(state_scan_tc<true, 2>) : go(state_scan_tc<true, 1>);
  return p.mh == 2 ? go(state_scan_tc<false, 2>) : go(state_scan_tc<false, 1>);
}

}  // namespace ret
