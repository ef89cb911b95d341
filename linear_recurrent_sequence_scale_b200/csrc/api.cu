// C ABI of libretention.so: argument checks and kernel dispatch.
//
// Every check runs on the host before anything is launched, so a non-zero
// status means no kernel ran and no memory was touched.
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "retention.h"

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return RET_OK;
  g_last_cuda_error = static_cast<int>(e);
  return RET_ECUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int dt) { return dt == RET_F32 || dt == RET_BF16; }

// Sizes shared by the sequence forms.  dk, dv: multiples of 8 in [8, 512].
int check_seq_dims(int B, int H, int N, int dk, int dv, int dtype) {
  if (B < 1 || H < 1 || N < 0 || dk < 8 || dv < 8) return RET_EINVAL;
  if (dk % 8 || dv % 8) return RET_EINVAL;
  if (!valid_dtype(dtype)) return RET_EINVAL;
  if ((int64_t)B * H > 65535) return RET_EUNSUPPORTED;
  if (dk > 512 || dv > 512) return RET_EUNSUPPORTED;
  if ((int64_t)B * H * N * (dk > dv ? dk : dv) > ((int64_t)1 << 40)) return RET_EUNSUPPORTED;
  return RET_OK;
}

int check_eps(float eps) { return isnan(eps) ? RET_EINVAL : RET_OK; }

bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

// Shapes the tensor-core kernels handle (bf16 only).
bool tc_dims(int dk, int dv) { return pow2_in(dk, 64, 256) && pow2_in(dv, 64, 512); }
bool tc_chunk(int chunk) { return pow2_in(chunk, 64, 512); }
// The chunk length the tensor-core kernels work in.  Their row tiles hold 128
// query rows, so a 64-token chunk runs as 128-token chunks: every chunk
// length gives the same output and final state in exact arithmetic (the
// chunkwise form regroups one sum), and this moves only where the bf16
// copies of the carried state are rounded, every 128 tokens instead of 64.
int tc_tile(int chunk) { return chunk < 128 ? 128 : chunk; }

size_t tc_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk) {
  const size_t nc = (size_t)((N + chunk - 1) / chunk);
  return 2 * (size_t)B * H * nc * dk * dv;
}

}  // namespace

extern "C" {

const char* ret_status_string(int status) {
  switch (status) {
    case RET_OK: return "ok";
    case RET_EINVAL: return "invalid argument";
    case RET_EUNSUPPORTED: return "unsupported configuration";
    case RET_ECUDA: return "CUDA runtime error";
    case RET_EWORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

int ret_last_cuda_error(void) { return g_last_cuda_error; }

const char* ret_version(void) { return "retention-b200 0.1 (sm_100a)"; }

int ret_device_error(void) {
  const int a = ret::tc_state_device_error();
  const int b = ret::tc_out_device_error();
  const int c = ret::selftest_device_error();
  if (a < 0 || b < 0 || c < 0) return -1;
  return a ? a : (b ? b : c);
}

int ret_selftest_bounded_wait(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 10000) return RET_EINVAL;
  return cuda_status(
      ret::launch_bounded_wait_selftest(limit_ms, static_cast<cudaStream_t>(stream)));
}

int ret_parallel_gated(const void* q, const void* k, const void* v, const float* gammas,
                       const void* gate, void* o, int B, int H, int N, int dk, int dv, int dtype,
                       float gn_eps, void* stream) {
  int s = check_seq_dims(B, H, N, dk, dv, dtype);
  if (s) return s;
  if ((s = check_eps(gn_eps))) return s;
  if (N == 0) return RET_OK;
  if (!q || !k || !v || !o || !gammas) return RET_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RET_EINVAL;
  if (gate && !aligned16(gate)) return RET_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == RET_BF16 && tc_dims(dk, dv)) {
    if ((int64_t)((N + 127) / 128) > 65535) return RET_EUNSUPPORTED;
    return cuda_status(ret::launch_tc_out(q, k, v, gammas, 0, nullptr, 0, gate, o, B, H, N, dk,
                                          dv, gn_eps, 1, 0, st));
  }
  return cuda_status(ret::launch_simt_parallel(q, k, v, gammas, gate, o, B, H, N, dk, dv, dtype,
                                               gn_eps, st));
}

int ret_parallel(const void* q, const void* k, const void* v, const float* gammas, void* o,
                 int B, int H, int N, int dk, int dv, int dtype, float gn_eps, void* stream) {
  return ret_parallel_gated(q, k, v, gammas, nullptr, o, B, H, N, dk, dv, dtype, gn_eps, stream);
}

size_t ret_chunkwise_workspace(int B, int H, int N, int dk, int dv, int chunk, int dtype) {
  if (check_seq_dims(B, H, N, dk, dv, dtype) != RET_OK || chunk < 1) return 0;
  if (N == 0) return 0;
  if (dtype == RET_BF16 && tc_dims(dk, dv) && tc_chunk(chunk))
    return tc_workspace_bytes(B, H, N, dk, dv, tc_tile(chunk));
  return ret::simt_workspace_bytes(B, H, N, dk, dv, chunk);
}

}  // extern "C"

namespace {

bool tc_config(int dtype, int dk, int dv, int chunk) {
  return dtype == RET_BF16 && tc_dims(dk, dv) && tc_chunk(chunk);
}

// Checks shared by the chunkwise entry points (everything but the pointers
// that only one phase reads).
int check_chunkwise(int B, int H, int N, int dk, int dv, int dtype, int chunk,
                    const float* gammas, const void* workspace, size_t workspace_bytes) {
  int s = check_seq_dims(B, H, N, dk, dv, dtype);
  if (s) return s;
  if (chunk < 1 || !gammas) return RET_EINVAL;
  if (N == 0) return RET_OK;
  const size_t need = ret_chunkwise_workspace(B, H, N, dk, dv, chunk, dtype);
  if (need > 0 && (!workspace || workspace_bytes < need)) return RET_EWORKSPACE;
  if (workspace && !aligned16(workspace)) return RET_EINVAL;
  if (tc_config(dtype, dk, dv, chunk)) {
    const int c = tc_tile(chunk);
    const int nc = (N + c - 1) / c;
    if ((int64_t)nc * (c / 128) > 65535) return RET_EUNSUPPORTED;
  }
  return RET_OK;
}

}  // namespace

extern "C" {

int ret_chunkwise_states(const void* k, const void* v, const float* gammas, int chunk,
                         const float* state_in, float* state_out, int B, int H, int N, int dk,
                         int dv, int dtype, void* workspace, size_t workspace_bytes,
                         void* stream) {
  int s = check_chunkwise(B, H, N, dk, dv, dtype, chunk, gammas, workspace, workspace_bytes);
  if (s) return s;
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return RET_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    // No tokens: the final state is the initial one.
    if (!state_out || state_in == state_out) return RET_OK;
    const size_t state_bytes = sizeof(float) * (size_t)B * H * dk * dv;
    if (state_in)
      return cuda_status(
          cudaMemcpyAsync(state_out, state_in, state_bytes, cudaMemcpyDeviceToDevice, st));
    return cuda_status(cudaMemsetAsync(state_out, 0, state_bytes, st));
  }
  if (!k || !v || !aligned16(k) || !aligned16(v)) return RET_EINVAL;
  if (tc_config(dtype, dk, dv, chunk)) {
    // Needed whenever a state enters, crosses a chunk boundary or is
    // returned; the incoming state is also stored in workspace slot 0.
    const int c = tc_tile(chunk);
    const int nc = (N + c - 1) / c;
    if (nc == 1 && !state_out && !state_in) return RET_OK;
    return cuda_status(ret::launch_tc_state(k, v, gammas, c, state_in, state_out, workspace,
                                            state_in != nullptr, B, H, N, dk, dv, st));
  }
  return cuda_status(ret::launch_simt_states(k, v, gammas, chunk, state_in, state_out, B, H, N,
                                             dk, dv, dtype, workspace, st));
}

}  // extern "C"

namespace {

// The output phase; after_states: the states phase of the same call was
// launched just before it on the stream (programmatic dependent launch).
int chunkwise_output_impl(const void* q, const void* k, const void* v, const float* gammas,
                          int chunk, int has_state_in, const void* gate, void* o, int B, int H,
                          int N, int dk, int dv, int dtype, float gn_eps, const void* workspace,
                          size_t workspace_bytes, void* stream, bool after_states) {
  int s = check_chunkwise(B, H, N, dk, dv, dtype, chunk, gammas, workspace, workspace_bytes);
  if (s) return s;
  if ((s = check_eps(gn_eps))) return s;
  if (N == 0) return RET_OK;
  if (!q || !k || !v || !o) return RET_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RET_EINVAL;
  if (gate && !aligned16(gate)) return RET_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_config(dtype, dk, dv, chunk))
    return cuda_status(ret::launch_tc_out(q, k, v, gammas, tc_tile(chunk), workspace,
                                          has_state_in != 0, gate, o, B, H, N, dk, dv, gn_eps, 0,
                                          after_states, st));
  return cuda_status(ret::launch_simt_output(q, k, v, gammas, chunk, gate, o, B, H, N, dk, dv,
                                             dtype, gn_eps, workspace, st));
}

}  // namespace

extern "C" {

int ret_chunkwise_output_gated(const void* q, const void* k, const void* v, const float* gammas,
                               int chunk, int has_state_in, const void* gate, void* o, int B,
                               int H, int N, int dk, int dv, int dtype, float gn_eps,
                               const void* workspace, size_t workspace_bytes, void* stream) {
  return chunkwise_output_impl(q, k, v, gammas, chunk, has_state_in, gate, o, B, H, N, dk, dv,
                               dtype, gn_eps, workspace, workspace_bytes, stream, false);
}

int ret_chunkwise_output(const void* q, const void* k, const void* v, const float* gammas,
                         int chunk, int has_state_in, void* o, int B, int H, int N, int dk, int dv,
                         int dtype, float gn_eps, const void* workspace, size_t workspace_bytes,
                         void* stream) {
  return ret_chunkwise_output_gated(q, k, v, gammas, chunk, has_state_in, nullptr, o, B, H, N, dk,
                                    dv, dtype, gn_eps, workspace, workspace_bytes, stream);
}

int ret_chunkwise_gated(const void* q, const void* k, const void* v, const float* gammas,
                        int chunk, const float* state_in, float* state_out, const void* gate,
                        void* o, int B, int H, int N, int dk, int dv, int dtype, float gn_eps,
                        void* workspace, size_t workspace_bytes, void* stream) {
  // Every check of both phases runs before the first launch.
  int s = check_chunkwise(B, H, N, dk, dv, dtype, chunk, gammas, workspace, workspace_bytes);
  if (s) return s;
  if ((s = check_eps(gn_eps))) return s;
  if (N > 0) {
    if (!q || !k || !v || !o) return RET_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RET_EINVAL;
    if (gate && !aligned16(gate)) return RET_EINVAL;
  }
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return RET_EINVAL;
  s = ret_chunkwise_states(k, v, gammas, chunk, state_in, state_out, B, H, N, dk, dv, dtype,
                           workspace, workspace_bytes, stream);
  if (s) return s;
  // the states kernel ran (and may still be draining) unless nothing needed it
  const bool scanned = tc_config(dtype, dk, dv, chunk) &&
                       ((N + tc_tile(chunk) - 1) / tc_tile(chunk) > 1 || state_out || state_in);
  return chunkwise_output_impl(q, k, v, gammas, chunk, state_in != nullptr, gate, o, B, H, N, dk,
                               dv, dtype, gn_eps, workspace, workspace_bytes, stream, scanned);
}

int ret_chunkwise(const void* q, const void* k, const void* v, const float* gammas, int chunk,
                  const float* state_in, float* state_out, void* o, int B, int H, int N, int dk,
                  int dv, int dtype, float gn_eps, void* workspace, size_t workspace_bytes,
                  void* stream) {
  return ret_chunkwise_gated(q, k, v, gammas, chunk, state_in, state_out, nullptr, o, B, H, N, dk,
                             dv, dtype, gn_eps, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

// The bf16 backward as three forward calls (backward_tc.cu): reversed copies
// of q, k, v and dO, the prepared states, then the forward calls' workspace.
struct BwdTcLayout {
  size_t qr, kr, vr, dor, sin_t, dso_t, dso, g0, fws, fws_bytes, total;
};

bool bwd_tc(int dtype, int chunk) { return dtype == RET_BF16 && tc_chunk(chunk); }

BwdTcLayout bwd_tc_layout(int B, int H, int N, int dk, int dv, int chunk) {
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t BH = (size_t)B * H;
  const size_t rk = al(BH * N * dk * 2), rv = al(BH * N * dv * 2), st = al(BH * dk * dv * 4);
  BwdTcLayout L;
  L.qr = 0;
  L.kr = L.qr + rk;
  L.vr = L.kr + rk;
  L.dor = L.vr + rv;
  L.sin_t = L.dor + rv;
  L.dso_t = L.sin_t + st;
  L.dso = L.dso_t + st;
  L.g0 = L.dso + st;
  L.fws = L.g0 + st;
  const size_t a = ret_chunkwise_workspace(B, H, N, dv, dk, chunk, RET_BF16);  // dq, dk calls
  const size_t b = ret_chunkwise_workspace(B, H, N, dk, dv, chunk, RET_BF16);  // the dv call
  L.fws_bytes = al(a > b ? a : b);
  L.total = L.fws + L.fws_bytes;
  return L;
}

}  // namespace

extern "C" {

size_t ret_chunkwise_backward_workspace(int B, int H, int N, int dk, int dv, int chunk,
                                        int dtype) {
  if (check_seq_dims(B, H, N, dk, dv, dtype) != RET_OK || chunk < 1 || N == 0) return 0;
  if (bwd_tc(dtype, chunk)) return bwd_tc_layout(B, H, N, dk, dv, chunk).total;
  return ret::backward_workspace_bytes(B, H, N, dk, dv, chunk);
}

int ret_chunkwise_backward(const void* q, const void* k, const void* v, const float* gammas,
                           int chunk, const float* state_in, const void* d_o,
                           const float* d_state_out, void* dq, void* dk_, void* dv_,
                           float* d_state_in, int B, int H, int N, int dk, int dv, int dtype,
                           void* workspace, size_t workspace_bytes, void* stream) {
  int s = check_seq_dims(B, H, N, dk, dv, dtype);
  if (s) return s;
  if (chunk < 1 || !gammas) return RET_EINVAL;
  if ((state_in && !aligned16(state_in)) || (d_state_out && !aligned16(d_state_out)) ||
      (d_state_in && !aligned16(d_state_in)))
    return RET_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t state_bytes = sizeof(float) * (size_t)B * H * dk * dv;
  if (N == 0) {
    // No tokens: the final state is the initial one, so their gradients are equal.
    if (!d_state_in) return RET_OK;
    if (d_state_out)
      return cuda_status(cudaMemcpyAsync(d_state_in, d_state_out, state_bytes,
                                         cudaMemcpyDeviceToDevice, st));
    return cuda_status(cudaMemsetAsync(d_state_in, 0, state_bytes, st));
  }
  if (!q || !k || !v || !d_o || !dq || !dk_ || !dv_) return RET_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_o) || !aligned16(dq) ||
      !aligned16(dk_) || !aligned16(dv_))
    return RET_EINVAL;
  const size_t need = ret_chunkwise_backward_workspace(B, H, N, dk, dv, chunk, dtype);
  if (!workspace || workspace_bytes < need) return RET_EWORKSPACE;
  if (!aligned16(workspace)) return RET_EINVAL;
  if (!bwd_tc(dtype, chunk))
    return cuda_status(ret::launch_chunkwise_backward(q, k, v, gammas, chunk, state_in, d_o,
                                                      d_state_out, dq, dk_, dv_, d_state_in, B,
                                                      H, N, dk, dv, dtype, workspace, st));
  // bf16: each gradient is the forward chunkwise form of permuted inputs
  // (backward_tc.cu states the identities), run by the forward's kernels.
  const BwdTcLayout L = bwd_tc_layout(B, H, N, dk, dv, chunk);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  void *qr = w + L.qr, *kr = w + L.kr, *vr = w + L.vr, *dor = w + L.dor;
  float* sin_t = reinterpret_cast<float*>(w + L.sin_t);
  float* dso_t = reinterpret_cast<float*>(w + L.dso_t);
  float* dso = reinterpret_cast<float*>(w + L.dso);
  float* g0 = reinterpret_cast<float*>(w + L.g0);
  void* fws = w + L.fws;
  const int BH = B * H;
  cudaError_t e;
#define RET_TRY(call)                            \
  do {                                           \
    if ((e = (call)) != cudaSuccess) return cuda_status(e); \
  } while (0)
#define RET_TRY_STATUS(call)                     \
  do {                                           \
    const int s2 = (call);                       \
    if (s2 != RET_OK) return s2;                 \
  } while (0)
  // the forward calls' own checks (e.g. the chunk-count limit) before any
  // launch, so that a failing status still means nothing ran
  RET_TRY_STATUS(check_chunkwise(B, H, N, dv, dk, RET_BF16, chunk, gammas, fws, L.fws_bytes));
  RET_TRY_STATUS(check_chunkwise(B, H, N, dk, dv, RET_BF16, chunk, gammas, fws, L.fws_bytes));
  RET_TRY(ret::launch_reverse_rows(q, qr, BH, N, dk, st));
  RET_TRY(ret::launch_reverse_rows(k, kr, BH, N, dk, st));
  RET_TRY(ret::launch_reverse_rows(v, vr, BH, N, dv, st));
  RET_TRY(ret::launch_reverse_rows(d_o, dor, BH, N, dv, st));
  if (state_in) RET_TRY(ret::launch_prep_state(state_in, sin_t, gammas, BH, H, dk, dv, 1, 0, 0, st));
  if (d_state_out) {
    RET_TRY(ret::launch_prep_state(d_state_out, dso_t, gammas, BH, H, dk, dv, 1, 1, 0, st));
    RET_TRY(ret::launch_prep_state(d_state_out, dso, gammas, BH, H, dk, dv, 0, 1, 0, st));
  }
  // dq = forward(dO, V, K; S_in^T)
  RET_TRY_STATUS(ret_chunkwise(d_o, v, k, gammas, chunk, state_in ? sin_t : nullptr, nullptr, dq,
                               B, H, N, dv, dk, RET_BF16, -1.f, fws, L.fws_bytes, stream));
  // dk, reversed = forward(V', dO', Q'; dS_out^T / gamma)
  RET_TRY_STATUS(ret_chunkwise(vr, dor, qr, gammas, chunk, d_state_out ? dso_t : nullptr, nullptr,
                               dk_, B, H, N, dv, dk, RET_BF16, -1.f, fws, L.fws_bytes, stream));
  // dv, reversed = forward(K', Q', dO'; dS_out / gamma), final state G_0
  RET_TRY_STATUS(ret_chunkwise(kr, qr, dor, gammas, chunk, d_state_out ? dso : nullptr,
                               d_state_in ? g0 : nullptr, dv_, B, H, N, dk, dv, RET_BF16, -1.f,
                               fws, L.fws_bytes, stream));
  RET_TRY(ret::launch_reverse_rows(dk_, dk_, BH, N, dk, st));
  RET_TRY(ret::launch_reverse_rows(dv_, dv_, BH, N, dv, st));
  if (d_state_in) RET_TRY(ret::launch_prep_state(g0, d_state_in, gammas, BH, H, dk, dv, 0, 0, 1, st));
  if (d_state_out)
    RET_TRY(ret::launch_gamma_zero_last_token(k, v, d_state_out, gammas, dk_, dv_, BH, H, N, dk,
                                              dv, st));
#undef RET_TRY
#undef RET_TRY_STATUS
  return RET_OK;
}

int ret_state_combine(const float* locals, const int* spans, int r, const float* gammas,
                      const float* state0, float* state_in, int B, int H, int dk, int dv,
                      void* stream) {
  if (B < 1 || H < 1 || dk < 8 || dv < 8 || dk % 8 || dv % 8) return RET_EINVAL;
  if (r < 0 || (r > 0 && (!locals || !spans)) || !gammas || !state_in) return RET_EINVAL;
  if (r > ret::kMaxSpans) return RET_EUNSUPPORTED;
  if ((int64_t)B * H * dk * dv > ((int64_t)1 << 40)) return RET_EUNSUPPORTED;
  for (int g = 0; g < r; ++g)
    if (spans[g] < 0) return RET_EINVAL;
  if ((locals && !aligned16(locals)) || (state0 && !aligned16(state0)) || !aligned16(state_in))
    return RET_EINVAL;
  return cuda_status(ret::launch_state_combine(locals, spans, r, gammas, state0, state_in, B, H,
                                               dk, dv, static_cast<cudaStream_t>(stream)));
}

int ret_step_rotated(const void* q, const void* k, const void* v, const float* gammas,
                     const float* theta, long long pos, float* state, const void* gate, void* o,
                     int B, int H, int dk, int dv, int dtype, float gn_eps, void* stream) {
  if (B < 1 || H < 1 || dk < 8 || dv < 8 || dk % 8 || dv % 8) return RET_EINVAL;
  if (!valid_dtype(dtype)) return RET_EINVAL;
  int s = check_eps(gn_eps);
  if (s) return s;
  if (dk > 4096 || dv > 1024 || (int64_t)B * H > 65535) return RET_EUNSUPPORTED;
  if (!q || !k || !v || !gammas || !state || !o) return RET_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(o))
    return RET_EINVAL;
  if (gate && !aligned16(gate)) return RET_EINVAL;
  if (theta && (pos < 0 || pos > ((long long)1 << 53))) return RET_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(ret::launch_step(q, k, v, gammas, state, gate, o, B, H, dk, dv, dtype, gn_eps,
                                      theta, theta ? pos : 0, st));
}

int ret_step_gated(const void* q, const void* k, const void* v, const float* gammas,
                   float* state, const void* gate, void* o, int B, int H, int dk, int dv,
                   int dtype, float gn_eps, void* stream) {
  return ret_step_rotated(q, k, v, gammas, nullptr, 0, state, gate, o, B, H, dk, dv, dtype,
                          gn_eps, stream);
}

int ret_step(const void* q, const void* k, const void* v, const float* gammas, float* state,
             void* o, int B, int H, int dk, int dv, int dtype, float gn_eps, void* stream) {
  return ret_step_gated(q, k, v, gammas, state, nullptr, o, B, H, dk, dv, dtype, gn_eps, stream);
}

int ret_rotate(const void* x, void* y, const float* theta, long long pos0, int B, int H, int N,
               int d, int dtype, void* stream) {
  if (B < 1 || H < 1 || N < 0 || d < 2 || d % 2) return RET_EINVAL;
  if (!valid_dtype(dtype)) return RET_EINVAL;
  if (pos0 < 0 || pos0 > ((long long)1 << 53) - N) return RET_EINVAL;
  if (N == 0) return RET_OK;  // nothing to read or write; x, y, theta may be NULL
  if (!x || !y || !theta) return RET_EINVAL;
  if (!aligned16(x) || !aligned16(y)) return RET_EINVAL;
  if ((int64_t)B * H > INT32_MAX || (int64_t)N * d > ((int64_t)1 << 38) ||
      (int64_t)B * H * N * d > ((int64_t)1 << 40))
    return RET_EUNSUPPORTED;
  const uintptr_t bytes = (uintptr_t)((int64_t)B * H * N * d * (dtype == RET_BF16 ? 2 : 4));
  const uintptr_t xs = reinterpret_cast<uintptr_t>(x), ys = reinterpret_cast<uintptr_t>(y);
  if (xs != ys && xs < ys + bytes && ys < xs + bytes) return RET_EINVAL;  // partial overlap
  return cuda_status(ret::launch_rotate(x, y, theta, pos0, B, H, N, d, dtype,
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
