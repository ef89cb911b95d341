/*
 * retention.h - C ABI of libretention.so: multi-scale retention on NVIDIA
 * B200 (sm_100a).
 *
 * Retention, as defined on the page "RetNet - Retentive Network - A Successor
 * to Transformer for LLMs" (section Key Equations), has three forms that give
 * the same output in exact arithmetic:
 *
 *   recurrent   S_n = gamma * S_{n-1} + k_n^T v_n,     o_n = q_n S_n
 *   parallel    O = (Q K^T (.) D) V,   D[n][m] = gamma^(n-m) if n >= m, else 0
 *   chunkwise   O_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + (Q_[i] (.) xi) R_{i-1}
 *
 * with one decay gamma_h per head (multi-scale retention, same page, section
 * Methods: gamma_h = 1 - 2^(-5-h); here gammas are an input).  The chunk state
 * is R_i = gamma^L R_{i-1} + K_[i]^T (V_[i] (.) zeta) with xi_j = gamma^(j+1)
 * and zeta_j = gamma^(L-1-j) for in-chunk position j of a chunk of length L
 * (the page prints R_i without the in-chunk decay and leaves xi undefined;
 * these are the readings that make the chunkwise form equal the recurrence).
 * An optional per-head GroupNorm (same page, Methods: MSR -> GroupNorm)
 * normalises each (batch, head, token) row of o over its d_v values:
 * (o - mean) / sqrt(var + eps), biased variance, no affine parameters.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates no memory; scratch space comes from the caller (workspace).
 *  - Layouts are dense row-major:
 *        q, k     [B][H][N][dk]        v, o  [B][H][N][dv]
 *        state    [B][H][dk][dv]  float32 always
 *        gammas   [H]             float32, each in [0, 1]; values outside give
 *                                 unspecified (possibly NaN) results
 *    q, k, v and o share the element type `dtype` (RET_F32 or RET_BF16).
 *  - q, k, v, o, state and workspace must be 16-byte aligned; dk and dv must be
 *    multiples of 8.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    is the legacy default stream).  A return value other than RET_OK means
 *    that nothing was launched and no memory was written.  Errors raised by a
 *    kernel while it runs surface on the stream like any CUDA error.
 *  - Accumulation is float32.  With RET_BF16 inputs the products run on the
 *    tensor cores with bf16 operands where the shapes fit their tiles (the
 *    rules under each call); other bf16 shapes (chunk 100, dk 32, dk 512 ...)
 *    run the float32 CUDA-core kernels on the same inputs, whose only bf16
 *    rounding is that of o.  Either way o is rounded to the input type.
 */
#ifndef RETENTION_H_
#define RETENTION_H_

#include <stddef.h>

#if defined(__GNUC__)
#define RET_API __attribute__((visibility("default")))
#else
#define RET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { RET_F32 = 0, RET_BF16 = 1 } ret_dtype;

typedef enum {
  RET_OK = 0,
  RET_EINVAL = -1,        /* invalid argument: NULL, bad size, misalignment  */
  RET_EUNSUPPORTED = -2,  /* valid, but no kernel in this build handles it    */
  RET_ECUDA = -3,         /* a CUDA runtime call failed (ret_last_cuda_error) */
  RET_EWORKSPACE = -4     /* workspace smaller than the size it must have     */
} ret_status;

/*
 * Parallel form, O = (Q K^T (.) D) V, one decay per head; no state enters or
 * leaves.  ("RetNet - Retentive Network - A Successor to Transformer for
 * LLMs", Key Equations, Parallel Form; jisaku.com glossary "RetNet",
 * parallel mode.)
 *   q, k, v, o : layouts above; N >= 0 (N == 0 writes nothing).
 *   gn_eps     : < 0 disables the fused GroupNorm, otherwise its epsilon.
 * Supported: dk, dv in [8, 512]; RET_BF16 runs on the tensor cores when
 * dk in {64,128,256} and dv in {64,128,256,512}.
 */
RET_API int ret_parallel(const void* q, const void* k, const void* v, const float* gammas, void* o,
                 int B, int H, int N, int dk, int dv, int dtype, float gn_eps, void* stream);

/*
 * Bytes of workspace ret_chunkwise needs for these sizes (0 if none).  Returns
 * 0 as well for arguments ret_chunkwise would reject.
 */
RET_API size_t ret_chunkwise_workspace(int B, int H, int N, int dk, int dv, int chunk, int dtype);

/*
 * Chunkwise-recurrent form ("RetNet - Retentive Network - A Successor to
 * Transformer for LLMs", Key Equations, Chunkwise Recurrent; jisaku.com
 * glossary "RetNet", chunkwise mode): the sequence is cut into chunks of
 * `chunk` tokens (the last one may be shorter), each computed in parallel, and
 * a float32 d_k x d_v state per (batch, head) is carried from chunk to chunk.
 *   state_in   : initial state [B][H][dk][dv]; NULL means zero.
 *   state_out  : final state; NULL means not written.  May equal state_in.
 *   workspace  : device scratch of at least ret_chunkwise_workspace() bytes;
 *                its contents on entry do not matter; it is overwritten.
 * The final state is accurate to float32 accumulation (the bf16 path splits
 * the decayed V operand into two bf16 halves when state_out is requested).
 * Supported: chunk >= 1 with either type.  RET_BF16 runs on the tensor cores
 * for chunk in {64, 128, 256, 512} under the dk/dv rules of ret_parallel, and
 * on the float32 CUDA-core kernels otherwise (chunk 100, for instance).  The
 * tensor-core kernels tile 128 query rows, so chunk 64 runs as 128-token
 * chunks: every chunk length gives the same o and final state in exact
 * arithmetic, and only the places where the bf16 copies of the chunk state
 * are rounded move (every 128 tokens instead of 64).  The workspace size and
 * the chunk states in it follow that 128-token chunking.
 */
RET_API int ret_chunkwise(const void* q, const void* k, const void* v, const float* gammas, int chunk,
                  const float* state_in, float* state_out, void* o,
                  int B, int H, int N, int dk, int dv, int dtype, float gn_eps,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * The chunkwise form in its two phases; ret_chunkwise is exactly
 * ret_chunkwise_states followed by ret_chunkwise_output on one stream.
 * ("RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
 * Equations, Chunkwise Recurrent: the states R_i form one pass, the outputs
 * of all chunks the other.)  Callers use them to time the phases apart or to
 * keep the chunk states of a prefill.
 *
 * ret_chunkwise_states: from k, v and the decays, writes into `workspace` the
 *   state entering every chunk (slot i = R_{i-1}; slot 0 = state_in when
 *   given; on the tensor cores chunks of at least 128 tokens, see above) and,
 *   when state_out is not NULL, the final float32 state.  It
 *   launches nothing when there is a single chunk and no state enters or
 *   leaves.  Arguments as for ret_chunkwise.
 * ret_chunkwise_output: from q, k, v, the decays and the workspace that
 *   ret_chunkwise_states wrote with the same B, H, N, dk, dv, chunk and dtype,
 *   writes o (with the fused GroupNorm when gn_eps >= 0).  has_state_in must
 *   say whether that states call was given a state_in.  The workspace is
 *   only read.
 * The workspace layout is internal to the library and differs between the
 * tensor-core and the other paths; nothing but these two calls may read or
 * write it.  Errors as for ret_chunkwise; N == 0 writes nothing (the states
 * call still copies or zeroes state_out).
 */
RET_API int ret_chunkwise_states(const void* k, const void* v, const float* gammas, int chunk,
                         const float* state_in, float* state_out,
                         int B, int H, int N, int dk, int dv, int dtype,
                         void* workspace, size_t workspace_bytes, void* stream);
RET_API int ret_chunkwise_output(const void* q, const void* k, const void* v, const float* gammas,
                         int chunk, int has_state_in, void* o,
                         int B, int H, int N, int dk, int dv, int dtype, float gn_eps,
                         const void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device scratch compiled into the library for ret_chunkwise_noalloc. */
#define RET_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * ret_chunkwise for callers that cannot allocate device memory: a plugin in
 * a host runtime that owns every byte of device memory and offers it no
 * allocator, or a latency-critical loop that must not call cudaMalloc/cudaFree
 * (they can synchronise the device).  The paper has no counterpart; this is a
 * deployment variant of the chunkwise form above, with the same arguments,
 * results and errors except for the workspace.
 *   - Scratch comes from a fixed device array of RET_NOALLOC_SCRATCH_BYTES
 *     (64 MiB) inside the library, present on every GPU that loads it until the
 *     process exits.  Sizes whose ret_chunkwise_workspace() exceeds it are
 *     rejected with RET_EWORKSPACE before anything runs.
 *   - The first call on each device looks the array's device address up (with
 *     that device current); make that first call before any stream capture.
 *     A failed lookup returns RET_ECUDA and is retried by the next call.
 *   - `stream` must belong to the current device, whose copy of the array
 *     the call uses.
 *   - Every call shares the one array: calls that overlap on the GPU race on
 *     it and must be serialised by the caller.  Nothing in it needs to start
 *     at zero; it keeps the last call's contents.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
RET_API int ret_chunkwise_noalloc(const void* q, const void* k, const void* v, const float* gammas,
                          int chunk, const float* state_in, float* state_out, void* o,
                          int B, int H, int N, int dk, int dv, int dtype, float gn_eps,
                          void* stream);

/*
 * One recurrent decode step for every (batch, head) pair ("RetNet - Retentive
 * Network - A Successor to Transformer for LLMs", Key Equations, Recurrent
 * Form):  state <- gamma * state + k^T v,  o = q state  (the updated state).
 *   q, k  : [B][H][dk]      v, o : [B][H][dv]     (element type dtype)
 *   state : [B][H][dk][dv] float32, read and written in place.
 *   gn_eps: < 0 disables the fused GroupNorm of o.
 * Supported: dk in [8, 4096], dv in [8, 1024].
 */
RET_API int ret_step(const void* q, const void* k, const void* v, const float* gammas, float* state,
             void* o, int B, int H, int dk, int dv, int dtype, float gn_eps, void* stream);

/*
 * Gated variants of the three forms ("RetNet - Retentive Network - A
 * Successor to Transformer for LLMs", core components, item 4: GroupNorm with
 * swish gating; abstract page, section 2.2 Gated Multi-Scale Retention):
 *     o = swish(gate) (.) Y,   swish(x) = x / (1 + exp(-x)),
 * where Y is what the ungated call writes (the retention output, after the
 * per-head GroupNorm when gn_eps >= 0).  The gate is computed by the caller
 * (the layer's gate projection); the output projection after it is not part
 * of this library.
 *   gate : same shape, layout and dtype as o ([B][H][N][dv], or [B][H][dv]
 *          for the step), 16-byte aligned, only read; NULL gives exactly the
 *          ungated call.
 * Other arguments, results and errors as for the ungated call.  The gate is
 * applied in the kernel that writes o (fused; no extra pass over o).
 */
RET_API int ret_parallel_gated(const void* q, const void* k, const void* v, const float* gammas,
                       const void* gate, void* o, int B, int H, int N, int dk, int dv,
                       int dtype, float gn_eps, void* stream);
RET_API int ret_chunkwise_gated(const void* q, const void* k, const void* v, const float* gammas,
                        int chunk, const float* state_in, float* state_out, const void* gate,
                        void* o, int B, int H, int N, int dk, int dv, int dtype, float gn_eps,
                        void* workspace, size_t workspace_bytes, void* stream);
RET_API int ret_chunkwise_output_gated(const void* q, const void* k, const void* v,
                               const float* gammas, int chunk, int has_state_in,
                               const void* gate, void* o, int B, int H, int N, int dk, int dv,
                               int dtype, float gn_eps, const void* workspace,
                               size_t workspace_bytes, void* stream);
RET_API int ret_step_gated(const void* q, const void* k, const void* v, const float* gammas,
                   float* state, const void* gate, void* o, int B, int H, int dk, int dv,
                   int dtype, float gn_eps, void* stream);

/*
 * One recurrent decode step with the xPos rotation of q and k fused into it
 * ("RetNet - Retentive Network - A Successor to Transformer for LLMs", core
 * components, item 3: xPos puts relative position into Q and K as a complex
 * rotation).  The token sits at sequence position `pos`; as q and k are read,
 * channel pair c, (x[2c], x[2c+1]) as the real and imaginary parts of z_c,
 * is multiplied by e^{i pos theta[c]} (the reading ret_rotate documents), so
 * the step equals ret_rotate of q and k at pos0 = pos followed by
 * ret_step_gated, without rounding the rotated q and k to the storage type
 * and without writing them.
 *   theta : device [dk/2] float32 angles (radians per position), or NULL
 *           for no rotation (then exactly ret_step_gated).
 *   pos   : 0 .. 2^53 (used only when theta is given).
 * Other arguments, layouts and errors as for ret_step_gated.
 */
RET_API int ret_step_rotated(const void* q, const void* k, const void* v, const float* gammas,
                     const float* theta, long long pos, float* state, const void* gate,
                     void* o, int B, int H, int dk, int dv, int dtype, float gn_eps,
                     void* stream);

/*
 * State entering span r of a sequence split into spans held by different GPUs
 * (sequence parallelism for the chunkwise form).  The carried state obeys
 * the chunk recurrence ("RetNet - Retentive Network - A Successor to
 * Transformer for LLMs", Key Equations, Chunkwise Recurrent) at span
 * granularity: with S_local(g) the end state of span g computed from a zero
 * state (ret_chunkwise_states with state_in = NULL) and N_g its length,
 *     state_in = gamma^(N_0+...+N_(r-1)) state0
 *              + sum_{g<r} gamma^(N_(g+1)+...+N_(r-1)) S_local(g).
 *   locals   : device, [r][B][H][dk][dv] float32 (the gathered end states of
 *              spans 0 .. r-1; may be NULL when r == 0).
 *   spans    : HOST array of r span lengths (tokens, >= 0).
 *   state0   : device [B][H][dk][dv] float32 entering span 0, or NULL (zero).
 *   state_in : device [B][H][dk][dv] float32, written.  r == number of spans
 *              gives the end state of the whole sequence.
 * Supported: r <= 64.  All device pointers 16-byte aligned.
 */
RET_API int ret_state_combine(const float* locals, const int* spans, int r, const float* gammas,
                      const float* state0, float* state_in, int B, int H, int dk, int dv,
                      void* stream);

/*
 * Backward of the chunkwise form (the training role; "RetNet - Retentive
 * Network - A Successor to Transformer for LLMs", Key Equations: the pages
 * give the forms, this is their chain rule): given dO, the gradient of the
 * outputs o of ret_chunkwise without GroupNorm or gate, and d_state_out, that
 * of its final state, it writes
 *   grad_q, grad_k, grad_v : [B][H][N][dk|dv], dtype of the inputs (written)
 *   d_state_in   : [B][H][dk][dv] float32, the gradient of state_in (or NULL)
 *   state_in     : the forward call's initial state, or NULL (zero)
 *   d_state_out  : [B][H][dk][dv] float32, or NULL (zero)
 *   workspace    : at least ret_chunkwise_backward_workspace() bytes.
 * RET_BF16 with chunk in {64, 128, 256, 512}: each gradient of the
 * recurrence is itself a retention operation, so the call runs three forward
 * chunkwise calls (dq = forward(dO, V, K) with the incoming state S_in^T;
 * in reversed time dk = forward(V, dO, Q) and dv = forward(K, Q, dO), whose
 * final state gives d_state_in), on the tensor cores wherever their mapped
 * shapes fit the tiles of ret_chunkwise; the workspace then holds reversed
 * copies of q, k, v and dO, four float32 states and the forward calls'
 * workspace.  Otherwise (float32, or other chunks) it runs the chain rule on
 * the CUDA cores in float32, its workspace holding the forward and gradient
 * chunk states and the masked in-chunk scores for chunks of min(chunk, 128)
 * tokens (the gradients do not depend on the chunk length).
 * Supported: any chunk >= 1, dk, dv in [8, 512].  Errors as for
 * ret_chunkwise.
 */
RET_API size_t ret_chunkwise_backward_workspace(int B, int H, int N, int dk, int dv, int chunk,
                                        int dtype);
RET_API int ret_chunkwise_backward(const void* q, const void* k, const void* v,
                           const float* gammas, int chunk, const float* state_in,
                           const void* d_o, const float* d_state_out, void* grad_q,
                           void* grad_k, void* grad_v, float* d_state_in, int B, int H, int N,
                           int dk, int dv, int dtype, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * xPos-style rotation of q or k rows ("RetNet - Retentive Network - A
 * Successor to Transformer for LLMs", core components, item 3: a complex
 * rotation that puts relative position into Q and K; "RetNet入門", Spiral.AI
 * Tech Blog, LEX Transformer paragraph).  Channels (2c, 2c+1) of a row are
 * the real and imaginary parts of one complex number, and the row at
 * sequence position n is multiplied by e^{i n theta_c}:
 *     y[2c]   = x[2c] cos(n theta_c) - x[2c+1] sin(n theta_c)
 *     y[2c+1] = x[2c] sin(n theta_c) + x[2c+1] cos(n theta_c)
 * Rotating both q and k makes q'_n . k'_m depend on n - m only.  The pages
 * give neither the angles nor the channel pairing: theta is an input and the
 * pairs are adjacent channels.
 *   x     : [B][H][N][d] device, dtype, only read.
 *   y     : [B][H][N][d] device, dtype, written; may equal x (in place), must
 *           not overlap it otherwise.
 *   theta : [d/2] float32 device array, radians per position for each pair.
 *   pos0  : position of row 0 of every sequence (e.g. tokens already
 *           decoded); 0 <= pos0 and pos0 + N <= 2^53.
 * The angle n theta_c and its cos / sin are taken in double precision; the
 * rotation itself in float32.  Supported: d even, N >= 0 (N == 0 writes
 * nothing, and x, y and theta may then be NULL); x and y 16-byte aligned.
 */
RET_API int ret_rotate(const void* x, void* y, const float* theta, long long pos0, int B, int H,
               int N, int d, int dtype, void* stream);

/* Human-readable name of a ret_status value (static storage). */
RET_API const char* ret_status_string(int status);

/* The cudaError_t of the last call that returned RET_ECUDA in this thread. */
RET_API int ret_last_cuda_error(void);

/*
 * Reads and clears the flag the tensor-core kernels set when one of their
 * bounded waits on an mbarrier ran out (a protocol failure that would
 * otherwise hang the GPU): 0 if none, otherwise the code of the wait site, -1
 * if the flag could not be read.  Synchronous with respect to the device.
 */
RET_API int ret_device_error(void);

/*
 * Self-test of the failure path above: launches one thread that waits on an
 * mbarrier nothing will complete, with a limit of limit_ms (1 .. 10000).  The
 * wait gives up, records site code 901 and the kernel returns, so the
 * context stays usable; after the stream has run, ret_device_error() returns
 * 901 (and clears it).  No GPU fault, trap or hang is involved.
 */
RET_API int ret_selftest_bounded_wait(int limit_ms, void* stream);

/* Library version string (static storage). */
RET_API const char* ret_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RETENTION_H_ */
