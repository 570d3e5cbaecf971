/*
 * ttt.h - C ABI of the Test-Time-Training (TTT) layer forward on NVIDIA B200 (sm_100a).
 *
 * The method (TTT write-up "大模型最强架构TTT问世！斯坦福UCSD等5年磨一剑，一夜推翻
 * Transformer", a summary of arXiv 2407.04620):
 *   - §03.1 "TTT hidden state": the layer's hidden state is the weight W of a
 *     small model f; each token takes one gradient step on a self-supervised
 *     loss, W_t = W_{t-1} - eta_t * grad l, and the output is f evaluated at the
 *     updated weight, z_t = f(q_t; W_t).
 *   - §03.5 "self-supervised task": l(W; t) = || f(k_t; W) - v_t ||^2, where
 *     k, v, q are learned projections of the input computed outside this layer.
 *   - §03.6 "mini-batch TTT": tokens are grouped in mini-batches of b; every
 *     gradient of a mini-batch is taken at the state left by the previous one
 *     (t' = t - mod(t, b), tokens 0-indexed).
 *   - §03.7 "dual form": a whole mini-batch is computed with matrix products,
 *     never materialising the b per-token gradients.
 *   - §03.9 "two variants": TTT-Linear f(x) = x W (W square, d x d); TTT-MLP with
 *     hidden width 4d and GELU; f carries a layer norm and a residual,
 *     f(x) = x + LN(f_res(x)).
 * Readings where the text is silent: the loss has no 1/2 (gradients carry a
 * factor 2); LN uses the population variance and the caller's epsilon; gamma
 * and beta are fixed per head and not updated by the inner loop; GELU is the
 * exact x * Phi(x); f has no bias; the per-token step size eta_t scales the
 * gradient of token t.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Row-vector convention: f(x) = x W with W[i][j] mapping input feature i to
 * output feature j.  All arrays are dense, row-major and contiguous:
 *   Q, K, V   [B][H][T][d]   dtype qkv_dtype (TTT_F32 or TTT_BF16)
 *   eta       [B][H][T]      float32, step size of each token
 *   W0        [H][d][d]      float32, initial state per head, shared by the batch
 *   W1_0      [H][d][hidden], W2_0 [H][hidden][d]   (TTT-MLP initial state)
 *   ln_gamma, ln_beta [H][d] float32
 *   Z         [B][H][T][d]   float32 output
 *   W_out     [B][H][d][d]   float32 final state of each (batch, head)
 *   W1_out    [B][H][d][hidden], W2_out [B][H][hidden][d]
 * Every pointer is a DEVICE pointer of the current CUDA device, 16-byte aligned.
 * The caller owns every buffer; the library allocates nothing and keeps no
 * pointer after the call.  Inputs are read only; outputs must not overlap any
 * input or each other.  The work is enqueued on `stream` (a cudaStream_t; NULL
 * is the legacy default stream) and the call returns without synchronising.
 *
 * Supported sizes: d = 64; 1 <= b <= 64 with T % b == 0 (b <= 16 for TTT-MLP);
 * hidden = 4 d; B, H, T >= 0 with B*H*T*d < 2^40.  B*H == 0 is a no-op; T == 0
 * copies the initial state to the outputs.  b = 16 with bf16 inputs runs the
 * tensor-core path; every other supported case runs the exact-fp32 CUDA-core
 * path.
 *
 * Errors: a call returns TTT_OK or a negative ttt_status.  Argument errors are
 * detected on the host BEFORE anything is enqueued (nothing is launched and no
 * CUDA call is made).  Launch failures return TTT_ERR_CUDA.  A device-side
 * wait that runs past its bound stops that CTA, leaves its outputs undefined
 * and records TTT_ERR_TIMEOUT in a device status word that
 * ttt_last_device_status() reports.
 */
#ifndef TTT_H_
#define TTT_H_

#if defined(__GNUC__)
#define TTT_API __attribute__((visibility("default")))
#else
#define TTT_API
#endif

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_OK = 0,
  TTT_ERR_ARG = -1,         /* null pointer, negative size, bad dtype, T % b != 0, overlap */
  TTT_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
  TTT_ERR_UNSUPPORTED = -3, /* well-formed but outside the supported sizes (d, b, hidden) */
  TTT_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
  TTT_ERR_TIMEOUT = -5      /* a bounded device-side wait expired (device status word) */
} ttt_status;

typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;

/*
 * TTT-Linear forward, f(x) = x W (§03.9; configs without LN).
 * Per (batch, head) and mini-batch n with tiles Q, K, V [b x d], eta [b] and
 * state W at the start of the mini-batch (dual form, §03.7):
 *   G      = 2 (K W - V)                       gradient w.r.t. f's output
 *   Z      = Q W - tril(Q K^T) diag(eta) G     (tril keeps s <= t)
 *   W_next = W - K^T diag(eta) G
 * Writes Z for every token and the final state to W_out.
 */
TTT_API int ttt_linear_fwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                   const float *W0, int B, int H, int T, int d, int b, float *Z, float *W_out,
                   void *stream);

/*
 * TTT-Linear with layer norm and residual, f(x) = x + LN(x W) (§03.9).
 * LN(y) = gamma * (y - mean(y)) / sqrt(var(y) + ln_eps) + beta over the d
 * features of one row, population variance.  Per mini-batch:
 *   G      = d l / d(K W) at the mini-batch base, through LN and the residual
 *   Z      = Q + LN(Q W - tril(Q K^T) diag(eta) G)
 *   W_next = W - K^T diag(eta) G
 * ln_eps must be finite and > 0.
 */
TTT_API int ttt_linear_ln_fwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                      const float *W0, const float *ln_gamma, const float *ln_beta, float ln_eps,
                      int B, int H, int T, int d, int b, float *Z, float *W_out, void *stream);

/*
 * TTT-MLP forward, f(x) = x + LN(GELU(x W1) W2), W1 [d x hidden],
 * W2 [hidden x d], hidden = 4 d (§03.9).  Per mini-batch, with X1 = K W1,
 * X2 = GELU(X1) and G3, G2 the loss gradients w.r.t. X2 W2 and X1 at the base:
 *   Z1 = Q W1 - tril(Q K^T) diag(eta) G2,  Z2 = GELU(Z1)
 *   Z  = Q + LN(Z2 W2 - tril(Z2 X2^T) diag(eta) G3)
 *   W1_next = W1 - K^T diag(eta) G2,  W2_next = W2 - X2^T diag(eta) G3
 */
TTT_API int ttt_mlp_fwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                const float *W1_0, const float *W2_0, const float *ln_gamma, const float *ln_beta,
                float ln_eps, int B, int H, int T, int d, int hidden, int b, float *Z,
                float *W1_out, float *W2_out, void *stream);

/*
 * The three forwards above with Q, K, V, eta, the per-head inputs and the outputs
 * in HOST memory (§03.7 dual form, §03.9 variants: the same operation and results
 * as ttt_linear_fwd / ttt_linear_ln_fwd / ttt_mlp_fwd, which it calls).
 *
 * variant: TTT_VARIANT_LINEAR (W0 = the state; W2_0, gamma, beta, ln_eps and
 * hidden ignored), TTT_VARIANT_LINEAR_LN (W0, gamma, beta, ln_eps), or
 * TTT_VARIANT_MLP (W0 = W1_0 [H][d][hidden], W2_0, gamma, beta, ln_eps, hidden;
 * W2_out receives the final W2).  Layouts and sizes as for the device entry
 * points; every host pointer 16-byte aligned.
 *
 * workspace: DEVICE memory owned by the caller, at least
 * ttt_fwd_host_workspace_bytes(variant, qkv_dtype, B, H, T, d, hidden) bytes,
 * 256-byte aligned; it receives the device copies of every input and output.
 * The batch is split into `chunks` (>= 1; at most B are used) contiguous slices:
 * the copy of slice i + 1 to the device, the forward of slice i and the copy of
 * slice i - 1 back run on three streams and overlap.  Host buffers should be
 * page-locked (cudaHostAlloc, or torch's pin_memory) for the copies to be
 * asynchronous; pageable memory works but serialises them.
 *
 * Ordering and ownership: the call returns once everything is enqueued.  All of
 * its work starts after the work already on `stream`, and `stream` waits for its
 * last copy back, so synchronising `stream` (or an event recorded on it after the
 * call) makes Z, W_out and W2_out valid in host memory.  Until then the caller
 * must neither change the host inputs nor read the host outputs nor reuse the
 * workspace.  Calls ordered on one stream may share a workspace.
 *
 * Errors: the argument rules of the device entry points (on the host pointers),
 * plus TTT_ERR_ARG for an unknown variant, chunks < 1 or a workspace that is null
 * or too small, TTT_ERR_ALIGN for a workspace not 256-byte aligned; TTT_ERR_CUDA
 * if a copy, stream or event call fails.  On an error after the first copy was
 * enqueued the outputs are unspecified.
 */
typedef enum { TTT_VARIANT_LINEAR = 0, TTT_VARIANT_LINEAR_LN = 1, TTT_VARIANT_MLP = 2 } ttt_variant;

/* Bytes of device workspace ttt_fwd_host needs (0 for invalid arguments). */
TTT_API size_t ttt_fwd_host_workspace_bytes(int variant, int qkv_dtype, int B, int H, int T, int d,
                                            int hidden);

TTT_API int ttt_fwd_host(int variant, const void *Q, const void *K, const void *V, int qkv_dtype,
                         const float *eta, const float *W0, const float *W2_0, const float *ln_gamma,
                         const float *ln_beta, float ln_eps, int B, int H, int T, int d, int hidden,
                         int b, float *Z, float *W_out, float *W2_out, void *workspace,
                         size_t workspace_bytes, int chunks, void *stream);

/*
 * Forward of TTT-Linear (and, _ln_, TTT-Linear with LN and residual) over whole
 * sequences with the momentum and decay update of the Titans article (§二.1(2):
 * momentum on past surprise, weight decay that forgets), kept to the TTT
 * mini-batch rule: with S_0 = 0 and G_t the loss gradient at the state the
 * mini-batch of token t started from,
 *   S_t = alpha_t S_{t-1} - eta_t k_t^T G_t,  W_t = (1 - lambda_t) W_{t-1} + S_t,
 *   z_t = q_t W_t  (or q_t + LN(q_t W_t)).
 * Inputs as for the forward, plus alpha, lambda [B][H][T] fp32 (per token, like
 * eta).  Outputs: Z [B][H][T][d], W_out and S_out [B][H][d][d] (the final state
 * and momentum), fp32.  1 <= b <= 16 and d = 64 (else TTT_ERR_UNSUPPORTED),
 * T % b == 0.  alpha = lambda = 0 is the plain TTT forward.  Arithmetic: with
 * bf16 Q, K, V and b = 16, the dual form over 64-token chunks on the tensor
 * cores (the recursion unrolled into per-token decay coefficients; W and S as
 * bf16 hi + lo operands, the coefficient-weighted Gram, eta G and K as fp16, fp32
 * accumulation: about 3e-4 relative to an fp64 evaluation), unless
 * ttt_set_path(TTT_PATH_SIMT); every other case, fp32 on the CUDA cores.  Errors
 * as for the forward entry points.
 */
TTT_API int ttt_linear_momentum_fwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                                    const float *eta, const float *alpha, const float *lambda,
                                    const float *W0, int B, int H, int T, int d, int b, float *Z,
                                    float *W_out, float *S_out, void *stream);
TTT_API int ttt_linear_ln_momentum_fwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                                       const float *eta, const float *alpha, const float *lambda,
                                       const float *W0, const float *ln_gamma,
                                       const float *ln_beta, float ln_eps, int B, int H, int T,
                                       int d, int b, float *Z, float *W_out, float *S_out,
                                       void *stream);

/*
 * The same momentum and decay forward on the TTT-MLP memory, f(x) = x + LN(GELU(x
 * W1) W2) (the Titans article's memory is an MLP, §二.1(3)): both layers follow
 *   S_t = alpha_t S_{t-1} - eta_t g_t,  W_t = (1 - lambda_t) W_{t-1} + S_t,
 * with g_t the loss gradient at the mini-batch base, z_t = f(q_t; W1_t, W2_t).
 * Inputs as for ttt_mlp_fwd plus alpha, lambda [B][H][T] fp32.  Outputs: Z
 * [B][H][T][d]; W1_out, S1_out [B][H][d][hidden]; W2_out, S2_out [B][H][hidden][d]
 * (the final states and momenta), fp32.  1 <= b <= 16, d = 64, hidden = 4 d (else
 * TTT_ERR_UNSUPPORTED), T % b == 0.  fp32 arithmetic on the CUDA cores.  Errors as
 * for the forward entry points.
 */
TTT_API int ttt_mlp_momentum_fwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                                 const float *eta, const float *alpha, const float *lambda,
                                 const float *W1_0, const float *W2_0, const float *ln_gamma,
                                 const float *ln_beta, float ln_eps, int B, int H, int T, int d,
                                 int hidden, int b, float *Z, float *W1_out, float *W2_out,
                                 float *S1_out, float *S2_out, void *stream);

/*
 * Backward pass of TTT-Linear (and, _ln_, TTT-Linear with LN and residual): the
 * gradients of L = <dZ, Z> + <dW_T, W_T> through the forward of ttt_linear_fwd /
 * ttt_linear_ln_fwd (the write-up trains the layer end to end and computes the
 * backward in the dual form too, §04.3).  Inputs as for the forward, plus
 *   dZ     [B][H][T][d] fp32: the cotangent of Z.
 *   dW_T   [B][H][d][d] fp32 or NULL (zero): the cotangent of the final state.
 * Outputs (fp32, caller-owned, fully written):
 *   dQ, dK, dV [B][H][T][d];  deta [B][H][T];
 *   dW0    [B][H][d][d]: per (batch, head) unit; the gradient of a W0 shared by
 *          the batch is the sum over the batch;
 *   dgamma, dbeta [B][H][d] (LN only): per unit likewise;
 *   W_ckpt [B][H][T/b][d][d]: the state at the start of every mini-batch
 *          (W_ckpt[.][.][0] = W0), which the reverse pass reads.
 * Mini-batch size 1 <= b <= 16 and d = 64 (else TTT_ERR_UNSUPPORTED); T % b == 0.
 * No output may overlap an input or another output.  Errors as for the forward.
 */
TTT_API int ttt_linear_bwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                           const float *eta, const float *W0, const float *dZ, const float *dW_T,
                           int B, int H, int T, int d, int b, float *dQ, float *dK, float *dV,
                           float *deta, float *dW0, float *W_ckpt, void *stream);
TTT_API int ttt_linear_ln_bwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                              const float *eta, const float *W0, const float *ln_gamma,
                              const float *ln_beta, float ln_eps, const float *dZ,
                              const float *dW_T, int B, int H, int T, int d, int b, float *dQ,
                              float *dK, float *dV, float *deta, float *dW0, float *dgamma,
                              float *dbeta, float *W_ckpt, void *stream);

/*
 * Backward pass of TTT-MLP (the gradients of L = <dZ, Z> + <dW1_T, W1_T> +
 * <dW2_T, W2_T> through the forward of ttt_mlp_fwd; the write-up trains the layer
 * end to end and computes the backward in the dual form too, §04.3).  Inputs as
 * for ttt_mlp_fwd, plus
 *   dZ      [B][H][T][d] fp32: the cotangent of Z.
 *   dW1_T   [B][H][d][hidden], dW2_T [B][H][hidden][d] fp32, or NULL (zero): the
 *           cotangents of the final states.
 * Outputs (fp32, caller-owned, fully written):
 *   dQ, dK, dV [B][H][T][d];  deta [B][H][T];
 *   dW1_0 [B][H][d][hidden], dW2_0 [B][H][hidden][d]: per (batch, head) unit (the
 *           gradient of a state shared by the batch is the sum over the batch);
 *   dgamma, dbeta [B][H][d]: per unit likewise;
 *   W1_ckpt [B][H][T/b][d][hidden], W2_ckpt [B][H][T/b][hidden][d]: the state at
 *           the start of every mini-batch (index 0 = the initial state), which the
 *           reverse pass reads.
 * 1 <= b <= 16, d = 64, hidden = 4 d (else TTT_ERR_UNSUPPORTED); T % b == 0.  No
 * output may overlap an input or another output.  fp32 arithmetic on the CUDA
 * cores.  Errors as for the forward.
 */
TTT_API int ttt_mlp_bwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                        const float *W1_0, const float *W2_0, const float *ln_gamma,
                        const float *ln_beta, float ln_eps, const float *dZ, const float *dW1_T,
                        const float *dW2_T, int B, int H, int T, int d, int hidden, int b, float *dQ,
                        float *dK, float *dV, float *deta, float *dW1_0, float *dW2_0,
                        float *dgamma, float *dbeta, float *W1_ckpt, float *W2_ckpt, void *stream);

/*
 * The backward of TTT-Linear + LN (ttt_linear_ln_bwd) for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a property of
 * the library's interface, not of the method.
 *
 * Who needs it: code that runs under a device allocator it does not own and may
 * not call cudaMalloc itself -- an operator hosted inside another framework or
 * runtime that hands out only its own buffers, or a serving process that
 * reserves all device memory at start-up, where a later cudaMalloc can fail or
 * stall the device -- and that has no way to pass the extra workspace
 * ttt_linear_ln_bwd asks for.  Here the per-mini-batch states that the reverse
 * pass reads back (W_ckpt of ttt_linear_ln_bwd) live in one fixed array of
 * device memory inside the library instead.
 *
 * Arguments, layouts, outputs and errors are those of ttt_linear_ln_bwd without
 * W_ckpt; the outputs are identical to that entry point's.  Limits and rules:
 *   - B * H * (T / b) <= TTT_NOALLOC_BWD_MAX_STATES (4096 states of d x d fp32,
 *     a 64 MiB array).  A larger call returns TTT_ERR_UNSUPPORTED before
 *     anything is enqueued.  Every GPU that loads the library holds the array
 *     until the process exits.
 *   - The array is shared by every call on a device and keeps the last call's
 *     contents.  A call writes every state before it reads it, so nothing needs
 *     clearing, but calls whose kernels overlap on the GPU (different streams,
 *     or different host threads, without an ordering between them) race on it:
 *     order them on one stream or with events.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address once and keeps it; make that first call before
 *     any stream capture.  The lookup follows the size checks and precedes the
 *     pointer checks; it returns TTT_ERR_CUDA if it fails.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 */
#define TTT_NOALLOC_BWD_MAX_STATES 4096
TTT_API int ttt_linear_ln_bwd_noalloc(const void *Q, const void *K, const void *V, int qkv_dtype,
                                      const float *eta, const float *W0, const float *ln_gamma,
                                      const float *ln_beta, float ln_eps, const float *dZ,
                                      const float *dW_T, int B, int H, int T, int d, int b,
                                      float *dQ, float *dK, float *dV, float *deta, float *dW0,
                                      float *dgamma, float *dbeta, void *stream);

/*
 * Primal-form decode step (generation, §04.3 of the TTT write-up: decoding is
 * sequential and takes the primal form): one token per (batch, head) and call,
 * with the state carried in device memory across calls.
 *   q, k, v  [B][H][d] (qkv_dtype), eta [B][H] fp32: this token's views and rate.
 *   W        [B][H][d][d] fp32, in/out: the state W_t after the previous token.
 *   W_base   [B][H][d][d] fp32, in/out: the state the current mini-batch started
 *            from (every gradient of a mini-batch is taken there, §03.6).
 *   pos      this token's position in its mini-batch of b tokens, 0 <= pos < b.
 *   z        [B][H][d] fp32 out.
 * Per (batch, head):
 *   G = d l / d(k W_base)        2 (k W_base - v), or through LN and the residual
 *   W <- W - eta k^T G,  z = q W  (or q + LN(q W)),  and W_base <- W if pos == b-1.
 * Run over a sequence with pos = t mod b, starting from W = W_base = W0, the calls
 * produce exactly the forward's Z and final state.  The caller owns all buffers;
 * W and W_base must not overlap each other or the inputs.  Errors as for the
 * forward entry points (host checks before any launch).
 */
TTT_API int ttt_linear_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                              const float *eta, float *W, float *W_base, int B, int H, int d,
                              int b, int pos, float *z, void *stream);
TTT_API int ttt_linear_ln_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                                 const float *eta, float *W, float *W_base, const float *ln_gamma,
                                 const float *ln_beta, float ln_eps, int B, int H, int d, int b,
                                 int pos, float *z, void *stream);

/*
 * The decode step with the momentum and decay update of the Titans article
 * (§二.1(2): momentum on past surprise, weight decay that forgets), kept to the
 * TTT mini-batch base above.  Besides the arguments of the plain step:
 *   alpha   [B][H] fp32: this token's momentum factor (0 <= alpha < 1 in use).
 *   lambda  [B][H] fp32: this token's weight decay (0 <= lambda <= 1 in use).
 *   S       [B][H][d][d] fp32, in/out: the momentum, all zero before the first token.
 * Per (batch, head), with G at W_base as above:
 *   S <- alpha S - eta k^T G,   W <- (1 - lambda) W + S,   z = q W (or q + LN(q W)),
 *   and W_base <- W if pos == b-1.
 * alpha = lambda = 0 is the plain step.  The caller owns all buffers; W, W_base,
 * S and z must not overlap each other or the inputs.  Errors as for the plain step.
 */
TTT_API int ttt_linear_momentum_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                                       const float *eta, const float *alpha, const float *lambda,
                                       float *W, float *W_base, float *S, int B, int H, int d,
                                       int b, int pos, float *z, void *stream);
TTT_API int ttt_linear_ln_momentum_decode(const void *q, const void *k, const void *v,
                                          int qkv_dtype, const float *eta, const float *alpha,
                                          const float *lambda, float *W, float *W_base, float *S,
                                          const float *ln_gamma, const float *ln_beta,
                                          float ln_eps, int B, int H, int d, int b, int pos,
                                          float *z, void *stream);

/*
 * The same step for TTT-MLP, f(x) = x + LN(GELU(x W1) W2): the state is W1
 * [B][H][d][hidden] and W2 [B][H][hidden][d] (fp32, in/out) with their
 * mini-batch bases W1_base, W2_base (in/out); hidden = 4 d.  Per (batch, head),
 * with X1 = k W1_base, X2 = GELU(X1) and G3, G2 the loss gradients w.r.t.
 * X2 W2_base and X1:  W1 <- W1 - eta k^T G2,  W2 <- W2 - eta X2^T G3,
 * z = q + LN(GELU(q W1) W2), and both bases follow at pos == b - 1.
 */
TTT_API int ttt_mlp_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                           const float *eta, float *W1, float *W2, float *W1_base, float *W2_base,
                           const float *ln_gamma, const float *ln_beta, float ln_eps, int B, int H,
                           int d, int hidden, int b, int pos, float *z, void *stream);

/*
 * The TTT-MLP decode step with the momentum and decay update (the Titans
 * article's MLP memory, §二.1(2); the same reading as the linear momentum step):
 * S1 [B][H][d][hidden] and S2 [B][H][hidden][d] fp32 (in/out, zero before the
 * first token) are the momenta of W1 and W2; alpha, lambda [B][H] fp32.  Per
 * (batch, head), with G2, G3 at the bases as in ttt_mlp_decode:
 *   S1 <- alpha S1 - eta k^T G2,   W1 <- (1 - lambda) W1 + S1,
 *   S2 <- alpha S2 - eta X2^T G3,  W2 <- (1 - lambda) W2 + S2,
 *   z = q + LN(GELU(q W1) W2), and both bases follow at pos == b - 1.
 * The caller owns all buffers; the seven state and output buffers must not
 * overlap each other or the inputs.  Errors as for ttt_mlp_decode.
 */
TTT_API int ttt_mlp_momentum_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                                    const float *eta, const float *alpha, const float *lambda,
                                    float *W1, float *W2, float *W1_base, float *W2_base, float *S1,
                                    float *S2, const float *ln_gamma, const float *ln_beta,
                                    float ln_eps, int B, int H, int d, int hidden, int b, int pos,
                                    float *z, void *stream);

/* Static English text for a ttt_status value (never NULL). */
TTT_API const char *ttt_status_string(int status);

/*
 * Synchronises `stream`, then returns and clears the device status word of the
 * current device: TTT_OK, or TTT_ERR_TIMEOUT if a bounded wait of an earlier
 * launch expired.  Returns TTT_ERR_CUDA if the synchronisation itself fails.
 */
TTT_API int ttt_last_device_status(void *stream);

/*
 * Kernel path selection for the next calls from any thread: TTT_PATH_AUTO
 * (default: tensor cores where supported), TTT_PATH_SIMT (exact-fp32 CUDA-core
 * kernels for every case) or TTT_PATH_TC (tensor cores; calls outside the
 * tensor-core sizes return TTT_ERR_UNSUPPORTED).  It applies to the entry points
 * that have a tensor-core kernel: ttt_linear_fwd, ttt_linear_ln_fwd, ttt_mlp_fwd
 * (and ttt_fwd_host) and ttt_linear_momentum_fwd / ttt_linear_ln_momentum_fwd;
 * the others run their CUDA-core kernels under every path.  Returns the previous
 * path, or TTT_ERR_ARG for an unknown value.
 */
typedef enum { TTT_PATH_AUTO = 0, TTT_PATH_SIMT = 1, TTT_PATH_TC = 2 } ttt_path;
TTT_API int ttt_set_path(int path);

/* Number of CUDA kernels this library enqueued since load (for launch accounting). */
TTT_API long long ttt_launch_count(void);

/*
 * Test hook for the timeout path (no counterpart in the method).  While on,
 * every CTA of the tensor-core kernels launched by later calls first waits on a
 * barrier that nothing arrives at, bounded at ~2^20 SM cycles: the wait
 * expires, the CTA records TTT_ERR_TIMEOUT in the device status word, skips its
 * remaining work (its outputs are then undefined), waits (bounded) for its own
 * loads and tensor-core products in flight, frees its tensor memory and
 * returns.  No GPU fault is involved.  Returns the previous setting (0 or 1).
 */
TTT_API int ttt_debug_inject_timeout(int on);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H_ */
