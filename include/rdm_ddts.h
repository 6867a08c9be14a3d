/*
 * rdm_ddts.h -- C ABI of the B200 (sm_100a) DDTS-gated linear-attention
 * recurrence of Rodimus.
 *
 * The operation (per batch b, head h, token t; i runs over d_k, j over d_v):
 *
 *   alpha_t     = exp(-g_t * tau_t)        alpha_hat_t = g_t ^ tau_t
 *   S_t         = diag(alpha_t) S_{t-1} + (alpha_hat_t * k_t)(beta_hat_t * v_t)^T
 *   o_t         = S_t^T q_t
 *
 * Sources: the gate formulas are those of the DDTS mechanism in "Rodimus*:
 * Breaking the Accuracy-Efficiency Trade-Off with Efficient Attentions"
 * (digest.lyk-ai.com summary, section "Method", first Rodimus bullet: selection
 * gate g_t, temperature gate tau_t).  The selection acts only along the key
 * dimension n = d_k, which is what allows chunkwise-parallel training
 * (paperhub.cn OpenReview rebuttal, "Efficient Parallelization" bullet, Sec.
 * 3.1.3 / App. B3); training runs chunkwise in parallel and inference runs token
 * by token on a fixed-size cached state (same page, answer to Q2; state size
 * n x m, answer to Q5-3 on Table 4).  beta_hat gates the input only, never the
 * transition (atlas.scime.ai summary, ablation rows on hat-beta and on beta in
 * the state transition).  The pages do not print the state update itself; the
 * form above is the plainest reading that agrees with all of these.
 *
 * Conventions shared by every entry point:
 *   - Layouts are dense row-major: sequences [B,H,T,D], states [B,H,d_k,d_v],
 *     decode inputs [B,H,D].  D is d_k for q, k, g, tau and d_v for v, beta_hat,
 *     o and their gradients.
 *   - Element type of every sequence tensor is `dtype` (RDM_F32 or RDM_BF16);
 *     states, saved states and dS_0 are always float32.  Arithmetic is float32
 *     throughout; bf16 operands feed the tensor cores with float32 accumulation.
 *   - All pointers are DEVICE pointers of the current device, 16-byte aligned.
 *     The caller owns every buffer.  The library allocates nothing, never
 *     synchronises (except rdm_ddts_sync_status) and launches only on `stream`.
 *   - Domain: g >= 0, tau >= 0.  Values are not checked on the device;
 *     out-of-domain values give NaN as the formulas do.  0^0 = 1, 0^tau = 0.
 *   - Host-side validation failures return a status and launch nothing.
 *     Kernel-side failures (a bounded wait that ran out, a decode position
 *     out of range) set a device status word that rdm_ddts_sync_status reports.
 *   - Supported sizes: d_k, d_v in {16, 32, 64, 128}; any T >= 0; B*H >= 1.
 *     The tensor-core path covers bf16 with d_k in {64, 128} and d_v in
 *     {64, 128} (d_v a multiple of the per-CTA tile); every other supported
 *     shape, and all float32 calls, run the exact-recurrence CUDA-core path.
 */
#ifndef RDM_DDTS_H
#define RDM_DDTS_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *rdm_stream_t;

typedef enum {
    RDM_OK = 0,
    RDM_ERR_INVALID_ARG = 1,  /* bad size, NULL or misaligned pointer      */
    RDM_ERR_UNSUPPORTED = 2,  /* valid request this build does not handle  */
    RDM_ERR_CUDA = 3,         /* a CUDA runtime call failed                 */
    RDM_ERR_TIMEOUT = 4,      /* a bounded on-device wait ran out           */
    RDM_ERR_WORKSPACE = 5     /* workspace missing or too small             */
} rdm_status;

typedef enum { RDM_F32 = 0, RDM_BF16 = 1 } rdm_dtype;

/* Which kernels to use.  AUTO picks the tensor-core path when the shape and
 * dtype allow it.  SIMT forces the exact token-serial CUDA-core path.  TC
 * forces the tensor-core path and fails with RDM_ERR_UNSUPPORTED where it does
 * not apply. */
typedef enum { RDM_IMPL_AUTO = 0, RDM_IMPL_SIMT = 1, RDM_IMPL_TC = 2 } rdm_impl;

/* What the g, tau and beta pointers of rdm_fwd_args / rdm_bwd_args hold.
 * ACTIVATED: the gates themselves (g >= 0, tau >= 0, beta_hat).  PREACT: the
 * gates before their activations; the kernels apply g = softplus(x) =
 * log(1 + e^x), tau = sigmoid(x), beta_hat = sigmoid(x) on the fly (the page
 * names a selection gate, a temperature gate and a low-rank beta_hat without
 * printing the activations; these are the reading this library takes), and the
 * backward returns the gradients with respect to the pre-activations. */
typedef enum { RDM_GATES_ACTIVATED = 0, RDM_GATES_PREACT = 1 } rdm_gate_inputs;

/* ------------------------------------------------------------------ forward
 * Chunkwise-parallel forward over whole sequences (the training / prefill
 * form named in the rebuttal's answer to Q2).
 *
 *   q, k, g, tau : [B,H,T,d_k] dtype      v, beta : [B,H,T,d_v] dtype
 *   S0           : [B,H,d_k,d_v] float32, or NULL for a zero initial state
 *   o            : [B,H,T,d_v] dtype, written
 *   ST           : [B,H,d_k,d_v] float32 final state, written; NULL = skip
 *   saved_states : [B,H,ceil(T/chunk),d_k,d_v] float32, written with the state
 *                  in force before each chunk (S_0 for chunk 0); NULL = skip.
 *                  rdm_ddts_bwd can reuse it instead of recomputing.
 *   chunk        : tokens per chunk (the block over which the intra-chunk
 *                  quadratic form is evaluated and between whose ends the state
 *                  is passed); 0 selects 64.  Allowed: 16, 32, 64, 128.  The
 *                  tensor-core path evaluates chunks of 16, 32 or 64 tokens
 *                  (narrowing any chunk to 16 tokens, then to single tokens,
 *                  where its log-decay span is too wide for one fp32
 *                  reference); chunk 128 runs the exact token-serial path.
 *                  Results agree across chunk sizes up to rounding.
 *                  saved_states then holds one state per chunk of this size.
 *   gate_inputs  : RDM_GATES_ACTIVATED (default, 0) or RDM_GATES_PREACT.
 *   workspace    : optional device scratch of workspace_bytes.  With at least
 *                  rdm_ddts_fwd_workspace_size() bytes the tensor-core path
 *                  may cut each sequence into segments processed by separate
 *                  CTAs (when B*H alone does not fill the GPU); with less, or
 *                  NULL, it runs each sequence in one CTA.  Results agree up
 *                  to rounding either way.  Contents on entry are ignored; two
 *                  calls whose kernels may overlap must not share it.
 *   feedthrough  : [H,d_v] float32 weights d, or NULL for none.  With d the
 *                  output is o_t = S_t^T q_t + d (.) v_t: the feedthrough d_t
 *                  of the paper's Eq. (11), which the rebuttal's answer to Q6
 *                  (paperhub.cn OpenReview page) names the SSM feedthrough, as
 *                  in Mamba and Mamba2 (a learned per-channel skip from the SSM
 *                  input, here v_t, to the output).  The pages print neither
 *                  its shape nor its input; this library takes one weight per
 *                  head and value channel, constant over time, applied to v_t
 *                  (not to beta_hat * v_t).  Added in the store stage of o.
 *   beta_rank    : 0, or the rank r (8 or 16) of a low-rank beta_hat (Rodimus*
 *                  digest.lyk-ai.com summary, "Method": beta_hat is built from
 *                  low-rank matrices to cut parameters and filter input noise).
 *                  The reading taken: a per-token factor beta_u [B,T,r] dtype,
 *                  shared by the heads (the token's input projected down to
 *                  rank r), times an up-projection beta_w [H,r,d_v] float32
 *                  gives beta_hat's pre-activation,
 *                    beta_hat[b,h,t,j] = sigmoid(sum_rho beta_u[b,t,rho] beta_w[h,rho,j]),
 *                  built on chip by the tensor-core kernel (beta is then
 *                  ignored and may be NULL).  Requires RDM_GATES_PREACT and the
 *                  tensor-core path (bf16, d_k and d_v in {64, 128}, chunk 16,
 *                  32 or 64); RDM_ERR_UNSUPPORTED otherwise.
 */
typedef struct {
    int B, H, T, dk, dv;
    int chunk;
    rdm_dtype dtype;
    rdm_impl impl;
    const void *q, *k, *v, *g, *tau, *beta;
    const float *S0;
    void *o;
    float *ST;
    float *saved_states;
    void *workspace;
    size_t workspace_bytes;
    rdm_gate_inputs gate_inputs;
    const float *feedthrough;
    int beta_rank;
    const void *beta_u;
    const float *beta_w;
} rdm_fwd_args;

rdm_status rdm_ddts_fwd(const rdm_fwd_args *args, rdm_stream_t stream);

/* Scratch bytes that let rdm_ddts_fwd segment sequences for `args` (0 when it
 * would not; depends on sizes, dtype, impl and the device's SM count);
 * (size_t)-1 on invalid sizes. */
size_t rdm_ddts_fwd_workspace_size(const rdm_fwd_args *args);

/* Bytes of `saved_states` that rdm_ddts_fwd writes for these sizes
 * (B*H*ceil(T/chunk)*d_k*d_v*4); 0 on invalid sizes. */
size_t rdm_ddts_saved_states_size(int B, int H, int T, int dk, int dv, int chunk);

/* ----------------------------------------------------------------- backward
 * Reverse mode of the forward for the loss L with dL/do = grad_o and
 * dL/dS_T = grad_ST.  The pages print no backward; this is the exact gradient
 * of the recurrence above.
 *
 *   inputs as in rdm_fwd_args (q..beta, S0)
 *   grad_o       : [B,H,T,d_v] dtype
 *   grad_ST      : [B,H,d_k,d_v] float32, or NULL for zero
 *   saved_states : states written by rdm_ddts_fwd with the same inputs and
 *                  chunk, or NULL to recompute them (into the workspace)
 *   grad_q, grad_k, grad_g, grad_tau : [B,H,T,d_k] dtype, written
 *   grad_v, grad_beta                : [B,H,T,d_v] dtype, written
 *   grad_S0      : [B,H,d_k,d_v] float32, written; NULL = skip
 *   gate_inputs  : as for rdm_ddts_fwd; with RDM_GATES_PREACT, grad_g, grad_tau
 *                  and grad_beta are with respect to the pre-activations.
 *   workspace    : device scratch of at least rdm_ddts_bwd_workspace_size()
 *                  bytes (may be NULL when that size is 0); contents on entry
 *                  are ignored and on exit are unspecified.
 *   feedthrough  : the forward's feedthrough weights [H,d_v] float32, or NULL
 *                  (then grad_v has no feedthrough term and grad_feedthrough
 *                  is not written).  grad_v then includes d (.) grad_o.
 *   grad_feedthrough : [H,d_v] float32, written with sum over b and t of
 *                  grad_o (.) v when non-NULL (requires feedthrough non-NULL;
 *                  accumulated with float32 atomics, so the summation order
 *                  may differ between calls).
 *   beta_rank, beta_u, beta_w : the forward's low-rank beta_hat (beta_rank 0 =
 *                  none).  With it grad_beta is not written (may be NULL) and
 *                  grad_beta_u [B,T,r] dtype and grad_beta_w [H,r,d_v] float32
 *                  receive the gradients of the factors (grad_beta_w summed with
 *                  float32 atomics).  The backward expands the pre-activation
 *                  into the workspace and contracts its gradient afterwards, so
 *                  rdm_ddts_bwd_workspace_size grows by two [B,H,T,d_v] dtype
 *                  buffers; both the tensor-core and the exact path take it.
 * Gradients with respect to g are undefined where g = 0 (g^(tau-1) is
 * unbounded there); d/dtau uses alpha_hat * ln g = 0 where alpha_hat = 0.
 */
typedef struct {
    int B, H, T, dk, dv;
    int chunk;
    rdm_dtype dtype;
    rdm_impl impl;
    const void *q, *k, *v, *g, *tau, *beta;
    const float *S0;
    const void *grad_o;
    const float *grad_ST;
    const float *saved_states;
    void *grad_q, *grad_k, *grad_v, *grad_g, *grad_tau, *grad_beta;
    float *grad_S0;
    void *workspace;
    size_t workspace_bytes;
    rdm_gate_inputs gate_inputs;
    const float *feedthrough;
    float *grad_feedthrough;
    int beta_rank;
    const void *beta_u;
    const float *beta_w;
    void *grad_beta_u;
    float *grad_beta_w;
} rdm_bwd_args;

rdm_status rdm_ddts_bwd(const rdm_bwd_args *args, rdm_stream_t stream);

/* Scratch bytes rdm_ddts_bwd needs for `args` (depends on sizes, dtype, impl
 * and whether saved_states is given); (size_t)-1 on invalid sizes. */
size_t rdm_ddts_bwd_workspace_size(const rdm_bwd_args *args);

/* Backward without a caller-provided workspace.  The pages have no
 * counterpart of this: it exists for callers that cannot allocate device
 * memory when they need the gradient (a process that reserved its device
 * memory once at start-up and may not grow it, or a callback that must not
 * call cudaMalloc / cudaFree because those can synchronise the device).
 *
 * Same arguments and results as rdm_ddts_bwd computed by the exact CUDA-core
 * path (args->impl, args->workspace and args->workspace_bytes are ignored).
 * The scratch comes from one 16 MiB array inside the library, allocated on
 * every device that loads it and held until the process exits.
 *   - The first call on a device, with that device current, loads the
 *     library's module there if that has not happened yet (CUDA loads modules
 *     lazily), which allocates the 16 MiB and may synchronise the device, and
 *     looks up the array's device address.  Make one call at start-up, before
 *     relying on the no-allocation guarantee and before any stream capture.
 *     The address is looked up again on every call (it is cheap once the
 *     module is loaded), so it stays right across cudaDeviceReset.
 *   - Problems needing more scratch than 16 MiB return RDM_ERR_WORKSPACE
 *     and launch nothing.  The figure is rdm_ddts_bwd_workspace_size with
 *     impl = RDM_IMPL_SIMT: B*H*T*d_k*4 + B*H*d_k*4 + 4*(B*H+1) bytes (each
 *     part rounded up to 256), plus, when T >= 1024 (the sweeps then run in
 *     P = min(8, T/512) sequence segments), B*H*P*d_k*(d_v+2)*4 bytes.
 *   - All calls share the one array and it keeps whatever the last call left;
 *     nothing in it has to start at zero (each call writes every scratch
 *     element before reading it).  Calls whose kernels overlap on the GPU
 *     (several streams, or several host threads on one device) race on it:
 *     serialise them.
 */
rdm_status rdm_ddts_bwd_noalloc(const rdm_bwd_args *args, rdm_stream_t stream);

/* ------------------------------------------------------------ decode step
 * One token of sequential inference on a cached fixed-size state, O(1) per
 * token (rebuttal answers to Q1 and Q2).  For every (b,h):
 *   S <- diag(alpha) S + (alpha_hat * k)(beta_hat * v)^T ;  o = S^T q
 *
 *   q, k, g, tau : [B,H,d_k] dtype     v, beta : [B,H,d_v] dtype
 *   S            : [B,H,d_k,d_v] float32, read and updated in place
 *   o            : [B,H,d_v] dtype, written
 */
rdm_status rdm_ddts_decode_step(int B, int H, int dk, int dv, rdm_dtype dtype,
                                const void *q, const void *k, const void *v,
                                const void *g, const void *tau, const void *beta,
                                float *S, void *o, rdm_stream_t stream);

/* The same decode step with the arguments in a struct and the feedthrough:
 * o = S^T q + d (.) v when feedthrough ([H,d_v] float32) is non-NULL.
 * rdm_ddts_decode_step is this call with feedthrough = NULL. */
typedef struct {
    int B, H, dk, dv;
    rdm_dtype dtype;
    const void *q, *k, *v, *g, *tau, *beta;
    float *S;
    void *o;
    const float *feedthrough;
} rdm_decode_args;

rdm_status rdm_ddts_decode(const rdm_decode_args *args, rdm_stream_t stream);

/* -------------------------------------------------------------- ShortConv
 * The short convolution of the Rodimus block (Rodimus* digest.lyk-ai.com
 * summary, "Method", third Rodimus bullet: ShortConv next to the GLU for local
 * context aggregation).  The pages print neither its width, its activation nor
 * where it sits; this library takes a causal depthwise convolution along the
 * tokens with one filter of width W <= 4 per (head, channel), an optional bias
 * and an optional SiLU, on sequences in the layout of the recurrence's inputs:
 *
 *   z[b,h,t,c] = bias[h,c] + sum_{i=0}^{W-1} w[h,c,i] * x[b,h,t-i,c]
 *   y = z   or   y = z * sigmoid(z)  (silu = 1)
 *
 * x at t - i < 0 comes from the carried-in state (the W-1 inputs before the
 * sequence, oldest first), or is zero without one; the state after the
 * sequence (its last W-1 inputs) can be written out, so sequences can be cut
 * into pieces and decoded token by token with T = 1.
 *
 *   x, y        : [B,H,T,D] dtype        D in {16, 32, 64, 128}; W in {1,2,3,4}
 *   weight      : [H,D,W] float32        bias : [H,D] float32 or NULL
 *   state_in    : [B,H,W-1,D] dtype or NULL (zeros)
 *   state_out   : [B,H,W-1,D] dtype or NULL (not written)
 * Outputs must not alias inputs (y, state_out vs x, state_in; in the backward
 * grad_x, grad_state_in vs x, state_in, grad_y, grad_state_out): the kernels
 * read their inputs through the read-only path.
 * All pointers are device pointers, 16-byte aligned; nothing is allocated.
 */
typedef struct {
    int B, H, T, D, W;
    rdm_dtype dtype;
    int silu;
    const void *x;
    const float *weight;
    const float *bias;
    const void *state_in;
    void *y;
    void *state_out;
} rdm_shortconv_args;

rdm_status rdm_shortconv_fwd(const rdm_shortconv_args *args, rdm_stream_t stream);

/* Reverse mode of rdm_shortconv_fwd for dL/dy = grad_y and dL/d(state_out) =
 * grad_state_out (NULL = zero).  Writes grad_x [B,H,T,D] dtype, grad_weight
 * [H,D,W] float32, grad_bias [H,D] float32 (when bias and grad_bias are
 * non-NULL) and grad_state_in [B,H,W-1,D] dtype (when state_in and
 * grad_state_in are non-NULL).  The weight and bias gradients are sums over
 * batch and tokens accumulated with float32 atomics (summation order may vary
 * between calls). */
typedef struct {
    rdm_shortconv_args fwd;      /* the forward's arguments (y, state_out unused) */
    const void *grad_y;
    const void *grad_state_out;
    void *grad_x;
    float *grad_weight;
    float *grad_bias;
    void *grad_state_in;
} rdm_shortconv_bwd_args;

rdm_status rdm_shortconv_bwd(const rdm_shortconv_bwd_args *args, rdm_stream_t stream);

/* Several independent ShortConv problems in one launch (the q, k and v
 * convolutions of a layer, say): args[0 .. n-1], 1 <= n <= 4, each exactly as
 * for rdm_shortconv_fwd / rdm_shortconv_bwd (own B, H, T, D, pointers), all with
 * the same dtype, W and silu (else RDM_ERR_INVALID_ARG; nothing is launched
 * when any problem fails its checks).  Their tiles share the persistent
 * blocks of one kernel, so the launch pays one ramp and one tail for all of
 * them.  The single-problem calls above are these with n = 1. */
rdm_status rdm_shortconv_fwd_many(const rdm_shortconv_args *args, int n, rdm_stream_t stream);
rdm_status rdm_shortconv_bwd_many(const rdm_shortconv_bwd_args *args, int n, rdm_stream_t stream);

/* ------------------------------------------------------------------ SW-SKA
 * Sliding-window shared-key attention, the attention half of the Rodimus+
 * block (Rodimus* digest.lyk-ai.com summary, "Method", Rodimus+ bullets: a
 * sliding window for local context and one key shared by all heads to shrink
 * the KV cache; paperhub.cn OpenReview rebuttal, answer to Q1: multi-head query
 * and value projections, a multi-query key projection).  The pages print
 * neither the window nor the score scale; this library takes, per batch b,
 * head h and token t,
 *
 *   s_u = scale * q[b,h,t] . k[b,u]      for u = max(0, t-window+1) .. t
 *   o[b,h,t] = sum_u softmax(s)_u v[b,h,u]
 *
 * with one key row per token shared by every head, scale = 1/sqrt(d_k) when
 * 0 is passed.
 *
 *   q : [B,H,T,d_k] bf16     k : [B,T,d_k] bf16     v, o : [B,H,T,d_v] bf16
 *   d_k, d_v in {64, 128}; window >= 1; T >= 0; dtype must be RDM_BF16.
 * Arithmetic: bf16 tensor-core products with float32 accumulation; the
 * softmax weights enter the second product rounded to bf16.
 *
 * Decode keeps a ring KV cache of `window` slots: the token at position p
 * (counted from 0 at the start of the sequence) lives in slot p mod window.
 *   k_cache : [B,window,d_k] bf16     v_cache : [B,H,window,d_v] bf16
 *   pos     : [B] int32, tokens of each sequence seen before this step
 * The forward fills the caches from a prompt when k_cache / v_cache are given
 * (the last min(T, window) keys and values at their slots) and sets pos[b] = T
 * when pos is given.  A decode step writes the new key and value into slot
 * pos[b] mod window, attends to positions max(0, pos-window+1) .. pos, and adds
 * one to pos[b] when advance_pos != 0.  Sequences of one batch may be at
 * different positions.  Decode takes window <= 32768.  A negative pos[b]
 * leaves that sequence untouched and makes rdm_ddts_sync_status return
 * RDM_ERR_INVALID_ARG.
 * All pointers are device pointers, 16-byte aligned (pos: 4-byte aligned);
 * outputs must not alias inputs; nothing is allocated.
 */
typedef struct {
    int B, H, T, dk, dv, window;
    float scale;                 /* > 0, or 0 for 1/sqrt(d_k) */
    rdm_dtype dtype;
    const void *q, *k, *v;
    void *o;
    void *k_cache;               /* NULL = not filled */
    void *v_cache;               /* NULL = not filled */
    int *pos;                    /* NULL = not written */
} rdm_ska_fwd_args;

rdm_status rdm_ska_fwd(const rdm_ska_fwd_args *args, rdm_stream_t stream);

typedef struct {
    int B, H, dk, dv, window;
    float scale;                 /* > 0, or 0 for 1/sqrt(d_k) */
    rdm_dtype dtype;
    const void *q;               /* [B,H,d_k] */
    const void *k;               /* [B,d_k] */
    const void *v;               /* [B,H,d_v] */
    void *k_cache, *v_cache;     /* updated in place */
    int *pos;                    /* [B] int32 */
    int advance_pos;             /* != 0: pos[b] += 1 after the step */
    void *o;                     /* [B,H,d_v] */
} rdm_ska_decode_args;

rdm_status rdm_ska_decode(const rdm_ska_decode_args *args, rdm_stream_t stream);

/* ------------------------------------------------------------------ status */

/* Synchronises `stream`, then reports (and clears) the device status word of
 * the current device: RDM_ERR_TIMEOUT if a bounded wait in a kernel ran out,
 * RDM_ERR_CUDA if the stream holds a CUDA error, RDM_OK otherwise. */
rdm_status rdm_ddts_sync_status(rdm_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char *rdm_status_string(rdm_status status);

/* ----------------------------------------------------------------- testing
 * Test hooks for the failure path of the bounded on-device waits; not for
 * production use.  They apply to every later call in the process (all host
 * threads) until reset with (0, 0).
 *   wait_limit_cycles      : SM clock cycles after which a bounded wait gives
 *                            up (0 = the default, about one second).
 *   withhold_segment_flags : 1 = CTAs of a sequence-segmented tensor-core
 *                            launch never publish the flag that tells later
 *                            segments their input is ready, the SW-SKA forward
 *                            never loads its value tiles and the ShortConv
 *                            kernels never issue their staging copies, so the
 *                            waits on them run out: the kernel then stops, sets
 *                            the device status word and returns, and
 *                            rdm_ddts_sync_status reports RDM_ERR_TIMEOUT.
 *                            Outputs of such a call are unspecified.
 * Returns RDM_ERR_INVALID_ARG for a negative limit or a flag other than 0/1. */
rdm_status rdm_ddts_set_test_hooks(long long wait_limit_cycles, int withhold_segment_flags);

/* Library ABI version (major*10000 + minor*100 + patch). */
int rdm_ddts_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RDM_DDTS_H */
