// Internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ret {

// gate (may be null): o is multiplied by swish(gate), same layout and type as o.
// theta (may be null): q and k are rotated by pos * theta[c] per channel pair.
cudaError_t launch_step(const void* q, const void* k, const void* v, const float* gammas,
                        float* state, const void* gate, void* o, int B, int H, int dk, int dv,
                        int dtype, float eps, const float* theta, long long pos,
                        cudaStream_t st);

size_t simt_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk);

// The chunkwise form on the SIMT cores, in its two phases: the float32 chunk
// states into ws, then the outputs from them.
cudaError_t launch_simt_states(const void* k, const void* v, const float* gammas, int chunk,
                               const float* state_in, float* state_out, int B, int H, int N,
                               int dk, int dv, int dtype, void* ws, cudaStream_t st);
cudaError_t launch_simt_output(const void* q, const void* k, const void* v, const float* gammas,
                               int chunk, const void* gate, void* o, int B, int H, int N, int dk,
                               int dv, int dtype, float eps, const void* ws, cudaStream_t st);

// Chunkwise backward on the CUDA cores (backward.cu); ws holds the forward
// and the gradient chunk states and the in-chunk scores in float32.
size_t backward_workspace_bytes(int B, int H, int N, int dk, int dv, int chunk);
cudaError_t launch_chunkwise_backward(const void* q, const void* k, const void* v,
                                      const float* gammas, int chunk, const float* state_in,
                                      const void* dout, const float* d_state_out, void* dq,
                                      void* dk_, void* dv_, float* d_state_in, int B, int H,
                                      int N, int dk, int dv, int dtype, void* ws,
                                      cudaStream_t st);

// Data movement for the bf16 backward built from forward calls (backward_tc.cu).
cudaError_t launch_reverse_rows(const void* src, void* dst, int BH, int N, int d,
                                cudaStream_t st);
cudaError_t launch_prep_state(const float* in, float* out, const float* gammas, int BH, int H,
                              int R, int C, int transpose, int inv_gamma, int by_gamma,
                              cudaStream_t st);
cudaError_t launch_gamma_zero_last_token(const void* k, const void* v, const float* ds,
                                         const float* gammas, void* dk, void* dv, int BH, int H,
                                         int N, int DK, int DV, cudaStream_t st);

// State entering span r of a sequence split across GPUs (seqpar.cu).
constexpr int kMaxSpans = 64;
cudaError_t launch_state_combine(const float* locals, const int* spans, int r,
                                 const float* gammas, const float* state0, float* out, int B,
                                 int H, int dk, int dv, cudaStream_t st);

// xPos-style rotation of q or k rows by pos * theta per channel pair (rotate.cu).
cudaError_t launch_rotate(const void* x, void* y, const float* theta, long long pos0, int B,
                          int H, int N, int d, int dtype, cudaStream_t st);

cudaError_t launch_simt_parallel(const void* q, const void* k, const void* v, const float* gammas,
                                 const void* gate, void* o, int B, int H, int N, int dk, int dv,
                                 int dtype, float eps, cudaStream_t st);

}  // namespace ret

namespace ret {

// Tensor-core (tcgen05) kernels for bf16 inputs.
cudaError_t launch_tc_state(const void* k, const void* v, const float* gammas, int chunk,
                            const float* state_in, float* state_out, void* ws, int write_ws0,
                            int B, int H, int N, int dk, int dv, cudaStream_t st);
cudaError_t launch_tc_out(const void* q, const void* k, const void* v, const float* gammas,
                          int chunk, const void* ws, int has_state0, const void* gate, void* o,
                          int B, int H, int N, int dk, int dv, float eps, int parallel_form,
                          int after_states, cudaStream_t st);
int tc_state_device_error();
int tc_out_device_error();
// Bounded-wait self-test (selftest.cu): a wait that runs out, site code 901.
cudaError_t launch_bounded_wait_selftest(int limit_ms, cudaStream_t st);
int selftest_device_error();

}  // namespace ret
