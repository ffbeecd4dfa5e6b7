/*
 * deco_moe.h -- C ABI of the B200 (sm_100a) DECO sparse MoE FFN layer.
 *
 * The layer is the DECO mixture-of-experts FFN as described in
 *   [arXiv] "DECO: Sparse Mixture-of-Experts with Dense-Comparable Performance
 *           on End-Side Devices" (arXiv 2605.10933), §1 Introduction and §2
 *           "Router design" / "Expert design";
 *   [press] the qidianchuan.cn summary of the same paper, part 2 (core design:
 *           router paragraph, NormSiLU paragraphs, non-gated experts).
 *
 *   z   = x W_r^T + b_r                    router logits, one per routed expert
 *   e is active for a token iff z_e > 0    (a zero or negative score is ignored)
 *   r   = ReLU(z)                          raw routing weight, not renormalised
 *   u   = x W_bar_up^T                     mean up-projection (precomputed mean)
 *   a_e = SiLU(RMSNorm(x W_up[e]^T - u))   NormSiLU, RMS over the d_e features,
 *                                          eps inside the square root, no gain
 *   y   = W_s_down SiLU(W_s_up x)          always-on shared expert
 *       + sum_{e active, ascending} s_e r_e W_down[e] a_e
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument named as a tensor is a DEVICE pointer to memory the
 *    caller owns; the library never allocates, frees or keeps a pointer after
 *    the call returns.  Matrices are row-major with the nn.Linear convention
 *    [out_features][in_features], so every row is contiguous along the
 *    contracted axis.  Device pointers must be 16-byte aligned.
 *  - x, out and all weight matrices use the layer's storage dtype (fp32 or
 *    bf16); b_r and s are always fp32.  Products accumulate in fp32; router
 *    activation decisions are exact (see below).  Intermediates: fp32 layers
 *    keep them in fp32; bf16 batches of up to 16 tokens keep the hidden
 *    activations as bf16 hi/lo pairs (~16 significant bits); larger bf16
 *    batches (tensor-core path) round the hidden activations to bf16 and each
 *    (token, expert) output W_down[e] a, before its s_e r_e scaling, to fp16
 *    ahead of the fixed-order sum, which costs about 1 % of the output RMS at
 *    the largest element on the test layers.
 *  - All calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream) and never synchronise, except
 *    deco_moe_device_error.  They do not allocate, so a sequence of calls can
 *    be captured in a CUDA graph.
 *  - Arguments are checked on the host before anything is launched; on any
 *    error nothing is launched and a non-zero status is returned.  A status of
 *    DECO_ERR_CUDA means a launch failed (cudaGetLastError was not success).
 *  - `x` must not alias `out`.
 *
 * Exact routing: the activation decision z_e > 0 is made on the exact real
 * value of b_r[e] + sum_k x_k W_r[e,k] over the stored operands.  The kernels
 * compute z in fp32 with a rigorous error bound and re-evaluate the sign
 * exactly (integer accumulation of the exact products) whenever the fp32 value
 * lies inside the bound, so active sets, counts and permutations are
 * reproducible bit for bit on any GPU and match an exact CPU evaluation.
 */
#ifndef DECO_MOE_H_
#define DECO_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DECO_OK = 0,
  DECO_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer   */
  DECO_ERR_UNSUPPORTED = 2,   /* valid but unsupported shape or dtype         */
  DECO_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required   */
  DECO_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed         */
  DECO_ERR_DEVICE = 5         /* a kernel reported an error (see device_error) */
} deco_status_t;

typedef enum { DECO_F32 = 0, DECO_BF16 = 1 } deco_dtype_t;

/* Shape of one layer call.
 *   T        tokens in the batch (>= 0; T == 0 is a no-op)
 *   d_model  model width D: multiple of 64, 64..16384
 *   E        routed experts: 1..256
 *   d_e      routed expert width: multiple of 64, 64..512
 *   d_s      shared expert width: multiple of 64, 64..16384
 *   dtype    storage dtype of x, out and every weight matrix
 *   rms_eps  epsilon added to the mean square inside NormSiLU's square root
 *   residual 0: out = layer(x); 1: out = x + layer(x), rounded once
 *   topk     routing rule.  0: DECO's ReLU routing (active iff z_e > 0).
 *            k in 1..E: the TopK baseline of [arXiv] §5 -- each token keeps
 *            its k largest logits (ranked on their exact values, exact ties
 *            to the lower expert index) with weights ReLU(z_e), not
 *            renormalised; everything after the router is unchanged
 *   gated    0: DECO's non-gated experts.  1: the gated variant of the
 *            ablation ([press] part 2, non-gated paragraph; [arXiv] §2
 *            "Expert design"): a_e = NormSiLU(x W_up[e]^T - u) * (x W_val[e]^T),
 *            element-wise, with the value branch W_val (weights.W_val)
 *   experts_on_host
 *            0: every weight is in device memory.  1: the routed experts'
 *            matrices W_up, W_down (and W_val) stay in host memory, pinned
 *            and mapped into the device's address space (cudaHostAlloc, or
 *            cudaHostRegister with cudaHostRegisterMapped, on a system with
 *            unified addressing, so the host pointer is the device pointer),
 *            and the layer reads only the rows of the experts the batch
 *            activates across the host link: the offloaded-parameter setting
 *            behind the paper's memory-access argument ([arXiv] §1).  The
 *            other weights stay in device memory.  These calls take the
 *            general CUDA-core kernels, which read weights with plain loads;
 *            a pointer that is not mapped host memory is rejected with
 *            DECO_ERR_INVALID_ARG before anything is launched.            */
typedef struct {
  int T;
  int d_model;
  int E;
  int d_e;
  int d_s;
  int dtype;      /* deco_dtype_t */
  float rms_eps;
  int residual;
  int topk;
  int gated;
  int experts_on_host;
} deco_moe_shape_t;

/* The layer's weights (device pointers, storage dtype unless noted; with
 * shape->experts_on_host, W_up, W_down and W_val are mapped host pointers).
 *   W_r      [E][D]        router projection
 *   b_r      [E]     fp32  router bias
 *   W_up     [E][d_e][D]   routed up-projections
 *   W_bar_up [d_e][D]      mean of W_up over the E experts (deco_moe_mean_up)
 *   W_down   [E][D][d_e]   routed down-projections
 *   s        [E]     fp32  learnable expert-wise router scaling
 *   W_s_up   [d_s][D]      shared expert up-projection
 *   W_s_down [D][d_s]      shared expert down-projection
 *   W_val    [E][d_e][D]   gated experts' value branch (shape->gated = 1;
 *                          NULL otherwise)                                  */
typedef struct {
  const void* W_r;
  const float* b_r;
  const void* W_up;
  const void* W_bar_up;
  const void* W_down;
  const float* s;
  const void* W_s_up;
  const void* W_s_down;
  const void* W_val;
} deco_moe_weights_t;

/* Routing outputs of deco_moe_routing (device pointers; any may be NULL to
 * skip that output except where noted).
 *   r        [T][E] fp32   ReLU(z): the logit where active, 0 elsewhere
 *   active   [T][E] u8     1 where z > 0 (exact), else 0
 *   counts   [E]    i32    tokens routed to each expert
 *   offsets  [E+1]  i32    exclusive prefix sum of counts; offsets[E] = P
 *   perm     [T*E]  i32    token of each (token, expert) pair, pairs ordered by
 *                          expert then token, ascending; the first P entries
 *                          are valid (capacity must be T*E)
 *   n_tok    [T]    i32    number of active experts of each token          */
typedef struct {
  float* r;
  uint8_t* active;
  int* counts;
  int* offsets;
  int* perm;
  int* n_tok;
} deco_routing_t;

/* Bytes of device workspace deco_moe_forward / deco_moe_routing need for
 * `shape`.  Returns DECO_ERR_INVALID_ARG / DECO_ERR_UNSUPPORTED for a shape the
 * forward call would reject. */
deco_status_t deco_moe_workspace_size(const deco_moe_shape_t* shape, size_t* bytes);

/* Forward pass of one DECO MoE FFN layer ([arXiv] §1; [press] part 2):
 * out[T][D] = layer(x[T][D]) (plus x when shape->residual).
 * `workspace` is device scratch of at least deco_moe_workspace_size bytes,
 * 256-byte aligned, owned by the caller; its contents need no initialisation
 * and are overwritten.  Two calls that overlap on the GPU must not share one
 * workspace.  The kernels are chosen from the shape: bf16 batches of up to 16
 * tokens take the weight-streaming decode kernel (one cooperative launch with
 * one CTA per SM; d_model a multiple of 256 up to 4096, d_e <= 256), other
 * bf16 batches with d_e <= 256 the tensor-core (tcgen05) kernels, everything
 * else the general CUDA-core kernels; all compute the same layer.  The workspace of a tensor-core batch holds one fp16 row of
 * d_model values per possible (token, expert) pair, T * E * d_model * 2 bytes. */
deco_status_t deco_moe_forward(const deco_moe_shape_t* shape, const void* x,
                               const deco_moe_weights_t* w, void* out,
                               void* workspace, size_t workspace_bytes, void* stream);

/* The router and the token->expert tables alone ([press] part 2 router
 * paragraph: a token activates every expert whose ReLU score is positive, so
 * the count per token varies).  Only w->W_r and w->b_r are read.  counts,
 * offsets and perm follow a stable counting sort by expert. */
deco_status_t deco_moe_routing(const deco_moe_shape_t* shape, const void* x,
                               const deco_moe_weights_t* w, const deco_routing_t* out,
                               void* workspace, size_t workspace_bytes, void* stream);

/* The precomputed mean up-projection of NormSiLU ([press] part 2: the mean of
 * all experts' up-projection weights is fixed at inference and computed once):
 * W_bar_up[j][k] = (1/E) sum_{e ascending} W_up[e][j][k], summed and divided in
 * fp64, rounded once (to nearest, ties to even) to `dtype`. */
deco_status_t deco_moe_mean_up(int E, int d_e, int d_model, int dtype, const void* W_up,
                               void* W_bar_up, void* stream);

/* Equal-parameter dense non-gated FFN, the "Dense" comparison of [arXiv] §5:
 * out[T][D] = W2 SiLU(W1 x), W1 [d_ff][D], W2 [D][d_ff].  d_ff multiple of 64,
 * d_model as for the layer. */
deco_status_t deco_dense_ffn_workspace_size(int T, int d_model, int d_ff, int dtype,
                                            size_t* bytes);
deco_status_t deco_dense_ffn_forward(int T, int d_model, int d_ff, int dtype, const void* x,
                                     const void* W1, const void* W2, void* out,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads the device error word a kernel may have
 * set in `workspace` and clears it.  Bits: 1 = a non-finite router operand;
 * 2 = a kernel gave up waiting for its own data after about a second (a
 * library fault, not an input property, unless deco_set_wait_limit lowered
 * the limit); 4 = on the bf16 prefill path (T > 16), an unscaled routed
 * expert output W_down[e] a left the fp16 range (|v| > 65504) in which it is
 * staged before the combine, so the output is not valid.  Since |a_j| <=
 * sqrt(d_e) after the RMS normalisation, |v| <= sqrt(d_e) times the largest
 * row 1-norm of W_down[e]: this depends on the weights only, never on x.
 * 0 = none.  Returns DECO_ERR_CUDA if the synchronisation fails. */
deco_status_t deco_moe_device_error(void* workspace, int* code, void* stream);

/* Size of the library's built-in device scratch used by
 * deco_moe_forward_static: 64 MiB on every GPU that loads the library. */
#define DECO_STATIC_SCRATCH_BYTES (64u << 20)

/* deco_moe_forward without a caller-provided workspace.  The paper has no
 * counterpart for this; it exists for callers that cannot allocate device
 * memory on their execution path -- for example a host whose memory budget is
 * fixed and fully handed out before it starts running layers, or a plugin
 * called back from another runtime that owns every allocation -- where a
 * cudaMalloc would fail, or would synchronise the device and stall the other
 * work on it.  Instead of a workspace argument, it uses a scratch array of
 * DECO_STATIC_SCRATCH_BYTES compiled into the library (static device memory,
 * held by every GPU that loads the library until the process exits).  It
 * allocates nothing, and runs the same kernels, with the same results, as
 * deco_moe_forward.
 *  - Shapes whose deco_moe_workspace_size exceeds DECO_STATIC_SCRATCH_BYTES
 *    are rejected with DECO_ERR_WORKSPACE before anything is launched.  Decode
 *    batches fit: T = 16 needs about 7 MiB at d_model 2048 / 64 experts,
 *    10 MiB at d_model 4096 / 128 experts (12 MiB gated) and 20 MiB with
 *    256 gated experts at d_model 4096.  Larger batches fit while their
 *    workspace, which on the tensor-core path grows with T * E * d_model,
 *    stays within the array.
 *  - The first call on each device looks up the scratch array's device
 *    address (cudaGetSymbolAddress, a runtime call made with that device
 *    current) and keeps it for the life of the process; make that first call
 *    before any stream capture on the device, and do not use this entry point
 *    on a device after cudaDeviceReset.
 *  - All calls on a device share the one array.  Calls whose executions
 *    overlap on the GPU (different streams, or several threads) race on it and
 *    give wrong results; serialise them, e.g. on one stream.  Each call
 *    clears what must start at zero; the rest is overwritten.
 * Other arguments, results and errors are those of deco_moe_forward; the
 * device error word of the last call is read with
 * deco_moe_static_device_error. */
deco_status_t deco_moe_forward_static(const deco_moe_shape_t* shape, const void* x,
                                      const deco_moe_weights_t* w, void* out, void* stream);

/* deco_moe_device_error for deco_moe_forward_static, whose error word lives
 * in the built-in scratch array of the current device: synchronises `stream`,
 * returns the word in *code (bits as for deco_moe_device_error) and clears it.
 * Allocates nothing. */
deco_status_t deco_moe_static_device_error(int* code, void* stream);

/* Fault-injection hook for tests of the kernels' timeout path: every later
 * call's kernels give up a wait for data (a shared-memory barrier or another
 * CTA's counter) after `cycles` SM clock cycles instead of about a second,
 * set bit 2 of the device error word, stop issuing work and, before exiting,
 * still wait (with the default limit) for every copy and tensor-core
 * operation they issued.  A small limit therefore makes the calls give up
 * without faulting; their outputs are then not valid.  0 restores the
 * default.  Process-wide, not thread-safe; not for production use. */
deco_status_t deco_set_wait_limit(long long cycles);

/* Kernel timing hook for benchmarks.  While set (events != NULL), every later
 * deco_moe_forward call on this process records events[2*i] on its stream just
 * before the kernel of timing slot i and events[2*i+1] just after it, for
 * i < n_events/2.  Slots: 0 router, 1 expert counts, 2 expert scatter,
 * 3 up-projection, 4 down-projection (general and tensor-core paths),
 * 5 projections, 6 shared down-projection, 7 combine (tensor-core path),
 * 8 the whole layer (decode path, one kernel).  `events` are cudaEvent_t
 * handles owned by the caller (passed as void*) and must outlive the calls.
 * Pass NULL to stop.  Not thread-safe; meant for a single benchmarking
 * thread. */
deco_status_t deco_moe_set_profiling(void* const* events, int n_events);

/* ---- training side -------------------------------------------------------
 * The backward pass of the layer and the pieces of the paper's adaptive
 * sparsity regularisation ([arXiv] §2 "Auxiliary training objective": an
 * auto-scaling coefficient on the router entropy; [press] part 3: the
 * coefficient is multiplied by a small factor such as 1.002 after every
 * iteration whose activation ratio is above the target, divided by it when
 * below). */

/* Gradients of the loss with respect to the layer's input and weights (device
 * pointers, fp32, the shapes of the corresponding inputs; all written in
 * full).  dW_up includes the mean up-projection's share: W_bar_up is taken as
 * the function mean_e W_up[e], so its gradient reaches every W_up[e] as
 * dW_bar_up / E.  dW_val only for gated experts (NULL otherwise). */
typedef struct {
  float* dx;         /* [T][D]        */
  float* dW_r;       /* [E][D]        */
  float* db_r;       /* [E]           */
  float* dW_up;      /* [E][d_e][D]   */
  float* dW_down;    /* [E][D][d_e]   */
  float* ds;         /* [E]           */
  float* dW_s_up;    /* [d_s][D]      */
  float* dW_s_down;  /* [D][d_s]      */
  float* dW_val;     /* [E][d_e][D]   */
} deco_moe_grads_t;

/* Bytes of device workspace deco_moe_backward needs for `shape`
 * (DECO_ERR_UNSUPPORTED for TopK routing, whose gradient is not provided). */
deco_status_t deco_moe_backward_workspace_size(const deco_moe_shape_t* shape, size_t* bytes);

/* Backward pass: given dy [T][D] (x's dtype) = dLoss/dout, writes every
 * gradient of `grads`.  The routing is recomputed with the forward pass's
 * exact router, so the active sets are those of deco_moe_forward; the
 * gradient of ReLU routing is 1 on the active set (z > 0) and 0 elsewhere.
 * dz_extra [T][E] fp32 (device, may be NULL) is an extra gradient on the
 * router logits from another term of the loss (the entropy regulariser,
 * deco_moe_router_entropy), added where the expert is active.  With
 * shape->residual, dx includes dy.  CUDA-core kernels in fp32 with every sum
 * in a fixed order: bitwise reproducible.  The workspace is as for
 * deco_moe_forward (caller-owned, 256-byte aligned, no initialisation;
 * deco_moe_device_error reads its error word).  Errors as deco_moe_forward. */
deco_status_t deco_moe_backward(const deco_moe_shape_t* shape, const void* x,
                                const deco_moe_weights_t* w, const void* dy, const float* dz_extra,
                                const deco_moe_grads_t* grads, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Router entropy regulariser (device pointers).  For token t, over the experts
 * it activates (active[t][e] = 1), with r = ReLU(z) the routing weights
 * [T][E] fp32 of deco_moe_routing: R = sum r, p = r / R and
 * H_t = -sum p log p (0 when the token activates nothing); H[t] = H_t and
 * H[T] = the mean over tokens (H holds T + 1 floats).  dz [T][E] gets
 * lambda * d(mean_t H_t)/dz = -lambda (log p_e + H_t) / (R T) where active and
 * 0 elsewhere: pass it to deco_moe_backward as dz_extra.  The entropy form is
 * this library's reading (the pages name the router entropy but give no
 * formula). */
deco_status_t deco_moe_router_entropy(int T, int E, const float* r, const uint8_t* active, float lambda,
                                      float* H, float* dz, void* stream);

/* One step of the adaptive sparsity coefficient (host): *lambda is multiplied
 * by factor (> 1) when the iteration's activation ratio is above the target,
 * divided by it when below, unchanged when equal. */
deco_status_t deco_sparsity_controller(double* lambda, double ratio, double target, double factor);

/* The name and description of the CUDA error behind the last DECO_ERR_CUDA
 * status returned on the calling thread ("" if none).  The string is owned by
 * the library and stays valid until the next call on this thread. */
const char* deco_last_cuda_error(void);

/* A static, human-readable name for a status code. */
const char* deco_status_string(deco_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* DECO_MOE_H_ */
