// Chunk-state scan on the tensor cores: bf16 operands, float32 state in TMEM.
//
// "RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
// Equations, Chunkwise Recurrent: the state carried between chunks is
//     R_i = gamma^L R_{i-1} + K_[i]^T (V_[i] (.) zeta),  zeta_j = gamma^(L-1-j)
// (the in-chunk decay zeta is the reading that makes the chunk state equal
// the recurrent form summed over the chunk).
//
// One CTA owns one (batch, head) and NT (<= 128) state columns, all d_k rows
// (two 128-row halves for d_k = 256), and walks the chunks in order:
//   warp 0      TMA: K tile [T tokens][d_k] and V tile [T][NT] per stage
//   warps 2-5   V (.) zeta, split into bf16 hi and lo parts when the final
//               state is requested (hi + lo carries 16 mantissa bits, so the
//               float32 state stays accurate to ~1e-6 instead of the 2^-9 of
//               one bf16 rounding); hi is written in place of V
//   warp 1      tcgen05.mma: R += K^T (V hi) [+ K^T (V lo)], M = 128 state
//               rows, N = NT, K = 16 tokens, A and B both MN-major
//   warps 6-9   at each chunk boundary: read R from TMEM, store it as bf16 to
//               the workspace (the state entering the next chunk, read by the
//               output kernel), scale it by gamma^L of the next chunk and
//               write it back; after the last chunk store the float32 state.
// Two CTAs fit on an SM (256 TMEM columns, ~97 KB shared memory each), so one
// CTA's MMAs run while the other rescales its state.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace ret {
namespace k2 {

using namespace sm100;

constexpr int T = 32;                  // tokens per stage
constexpr int STAGES = 3;
constexpr int BOX = T * 128;           // one [T][64] bf16 box: 4 KB
constexpr int K_OFF = 0;               // 4 boxes (d_k up to 256)
constexpr int V_OFF = 4 * BOX;         // 2 boxes (NT up to 128), becomes V hi
constexpr int LO_OFF = 6 * BOX;        // 2 boxes
constexpr int STAGE_BYTES = 8 * BOX;   // 32 KB
constexpr int BAR_OFF = STAGES * STAGE_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
constexpr int THREADS = 320;

struct Params {
  const float* gammas;
  const float* state_in;
  float* state_out;
  __nv_bfloat16* ws;  // [B*H*nc][dk][dv]; slot i = state entering chunk i
  int H, N, chunk, nc, dk, dv, nt;
  int write_ws0;      // store state_in (as bf16) in slot 0
};

__device__ __forceinline__ void store_bf16_row32(__nv_bfloat16* dst, const uint32_t (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 w;
    w.x = pack_bf16(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]));
    w.y = pack_bf16(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]));
    w.z = pack_bf16(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]));
    w.w = pack_bf16(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]));
    d[c] = w;
  }
}

template <bool SPLIT>
__global__ void __launch_bounds__(THREADS, 2)
state_scan_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full = bars;                 // TMA -> transform
  uint64_t* xf = bars + STAGES;          // transform -> MMA
  uint64_t* empty = bars + 2 * STAGES;   // MMA -> TMA
  uint64_t* acc_ready = bars + 3 * STAGES;
  uint64_t* acc_full = acc_ready + 1;
  uint64_t* drain = acc_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_ready + 3);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int h = bh % p.H;
  const int c0 = blockIdx.x * p.nt;
  const int halves = (p.dk + 127) / 128;
  const int kboxes = 2 * halves;  // d_k = 64 loads one out-of-range (zero) box as padding
  const int vboxes = p.nt / 64;
  const uint32_t tmem_cols = static_cast<uint32_t>(halves * p.nt);  // 64, 128 or 256

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&xf[s], 4);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_ready, 4);
    mbar_init(acc_full, 1);
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
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&empty[slot], ph ^ 1, 101)) { ok = false; break; }
          uint8_t* st = smem + slot * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[slot], (kboxes + vboxes) * BOX);
          for (int b = 0; b < kboxes; ++b)
            tma_load_3d(st + K_OFF + b * BOX, &tm_k, &full[slot], b * 64, cs + j0, bh);
          for (int b = 0; b < vboxes; ++b)
            tma_load_3d(st + V_OFF + b * BOX, &tm_v, &full[slot], c0 + b * 64, cs + j0, bh);
        }
      }
      // no copy may still be landing when the CTA exits
      for (int gg = max(0, g - STAGES); gg < g; ++gg)
        mbar_wait(&full[gg % STAGES], (gg / STAGES) & 1, 108);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.nt, true, true);
      int g = 0;
      bool ok = true;
      for (int ci = 0; ci < p.nc && ok; ++ci) {
        if (!mbar_wait(acc_ready, ci & 1, 102)) { ok = false; break; }
        tc_fence_after();
        const int L = min(p.chunk, p.N - ci * p.chunk);
        for (int j0 = 0; j0 < L; j0 += T, ++g) {
          const int slot = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&xf[slot], ph, 103)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + slot * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < T / 16; ++kk) {
            const uint64_t bhi = sdesc_sw128(sb + V_OFF + kk * 2048, BOX, 1024);
            const uint64_t blo = sdesc_sw128(sb + LO_OFF + kk * 2048, BOX, 1024);
            for (int hh = 0; hh < halves; ++hh) {
              const uint64_t a = sdesc_sw128(sb + K_OFF + 2 * hh * BOX + kk * 2048, BOX, 1024);
              umma_bf16_ss(tmem + hh * p.nt, a, bhi, idesc, 1u);
              if (SPLIT) umma_bf16_ss(tmem + hh * p.nt, a, blo, idesc, 1u);
            }
          }
          umma_commit(&empty[slot]);
        }
        if (!ok) break;
        umma_commit(acc_full);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, 109);
    }
  } else if (warp < 6) {
    // ---------------- V (.) zeta, hi/lo split ----------------
    const int tt = threadIdx.x - 64;
    const int nchunks = vboxes * (BOX / 16);
    int g = 0;
    bool ok = true;
    for (int ci = 0; ci < p.nc && ok; ++ci) {
      const int L = min(p.chunk, p.N - ci * p.chunk);
      for (int j0 = 0; j0 < L; j0 += T, ++g) {
        const int slot = g % STAGES;
        const uint32_t ph = (g / STAGES) & 1;
        if (!mbar_wait(&full[slot], ph, 104)) { ok = false; break; }
        const uint32_t sb = smem_u32(smem + slot * STAGE_BYTES);
        for (int e = tt; e < nchunks; e += 128) {
          const int box = e >> 8;           // 256 16-byte chunks per box
          const int within = e & 255;
          const int j = j0 + (within >> 3);  // token row of this chunk
          const float z = (j < L) ? gpow(lg, L - 1 - j) : 0.f;
          const uint32_t off = box * BOX + within * 16;
          const uint4 v = ld_shared_v4(sb + V_OFF + off);
          const uint32_t in[4] = {v.x, v.y, v.z, v.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float a = bf16lo_to_f32(in[c]) * z;
            const float b = bf16hi_to_f32(in[c]) * z;
            hi[c] = pack_bf16(a, b);
            if (SPLIT) lo[c] = pack_bf16(a - bf16lo_to_f32(hi[c]), b - bf16hi_to_f32(hi[c]));
          }
          st_shared_v4(sb + V_OFF + off, hi[0], hi[1], hi[2], hi[3]);
          if (SPLIT) st_shared_v4(sb + LO_OFF + off, lo[0], lo[1], lo[2], lo[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xf[slot]);
      }
    }
  } else {
    // ---------------- state epilogue (TMEM lanes 32q..32q+31) ----------------
    const int q = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const int ncg = p.nt / 32;
    // the first chunk's MMAs add onto gamma^L0 * state_in
    const float g0 = gpow(lg, min(p.chunk, p.N));
    for (int hh = 0; hh < halves; ++hh) {
      const int r = 128 * hh + 32 * q + lane;
      for (int cgi = 0; cgi < ncg; ++cgi) {
        uint32_t v[32];
        const int c = c0 + 32 * cgi;
        if (p.state_in && r < p.dk) {
          const float4* src =
              reinterpret_cast<const float4*>(p.state_in + ((size_t)bh * p.dk + r) * p.dv + c);
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float4 f = src[x];
            v[4 * x + 0] = __float_as_uint(f.x);
            v[4 * x + 1] = __float_as_uint(f.y);
            v[4 * x + 2] = __float_as_uint(f.z);
            v[4 * x + 3] = __float_as_uint(f.w);
          }
          if (p.write_ws0)
            store_bf16_row32(p.ws + (((size_t)bh * p.nc) * p.dk + r) * p.dv + c, v);
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(__uint_as_float(v[x]) * g0);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) v[x] = 0u;
        }
        tmem_st32(tmem + lane_addr + hh * p.nt + 32 * cgi, v);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_ready);

    for (int ci = 0; ci < p.nc; ++ci) {
      if (!mbar_wait(acc_full, ci & 1, 105)) break;
      tc_fence_after();
      const bool last = ci == p.nc - 1;
      const float gnext = last ? 0.f : gpow(lg, min(p.chunk, p.N - (ci + 1) * p.chunk));
      for (int hh = 0; hh < halves; ++hh) {
        const int r = 128 * hh + 32 * q + lane;
        for (int cgi = 0; cgi < ncg; ++cgi) {
          const int c = c0 + 32 * cgi;
          const uint32_t ta = tmem + lane_addr + hh * p.nt + 32 * cgi;
          uint32_t v[32];
          tmem_ld32(ta, v);
          tmem_wait_ld();
          if (!last) {
            if (r < p.dk)
              store_bf16_row32(p.ws + (((size_t)bh * p.nc + ci + 1) * p.dk + r) * p.dv + c, v);
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(__uint_as_float(v[x]) * gnext);
            tmem_st32(ta, v);
          } else if (p.state_out && r < p.dk) {
            float4* dst =
                reinterpret_cast<float4*>(p.state_out + ((size_t)bh * p.dk + r) * p.dv + c);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              dst[x] = make_float4(__uint_as_float(v[4 * x]), __uint_as_float(v[4 * x + 1]),
                                   __uint_as_float(v[4 * x + 2]), __uint_as_float(v[4 * x + 3]));
          }
        }
      }
      if (!last) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_ready);
      }
    }
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
  p.nt = dv < 128 ? dv : 128;
  p.write_ws0 = write_ws0;
  dim3 grid(dv / p.nt, (unsigned)BH);
  if (state_out) {
    auto fn = state_scan_tc<true>;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    fn<<<grid, THREADS, SMEM_BYTES, st>>>(tm_k, tm_v, p);
  } else {
    auto fn = state_scan_tc<false>;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    fn<<<grid, THREADS, SMEM_BYTES, st>>>(tm_k, tm_v, p);
  }
  return cudaPeekAtLastError();
}

}  // namespace ret
