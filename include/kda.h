/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) library.
 *
 * The library computes the forward hot path of KDA for one GPU:
 *
 *   decay   St  = Diag(alpha_t) S_{t-1}               alpha_t per key channel
 *   erase + write  S_t = St + beta_t k_t (v_t - St^T k_t)^T
 *   read    o_t = scale * S_t^T q_t                   (post-write state)
 *
 * Page "Kimi K3 の KDA(1): KDA が Gated MLA と AttnRes とどのように連携するか",
 * section 1.2.1 (decay -> erase -> write; the read sees S_t; q and k are L2
 * normalised per head inside the kernel); page "GDN, KDA の整理", section
 * "Kimi Delta Attention" (S_t in R^{dk x dv}, o_t = S_t^T q_t, per-channel
 * decay D_t = Diag(alpha_t)).  Complex-KDA (signed gate in [-1, 1], beta in
 * [0, 2]): page "Complex KDA: 理解并增强 Kimi Delta Attention 的表达能力".
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - Memory: every tensor pointer is DEVICE memory owned by the caller.  The
 *    library never allocates or frees memory and keeps no state between calls.
 *  - Asynchrony: work is enqueued on `stream`; the return value reports
 *    argument and launch errors only.  Kernel faults surface at the caller's
 *    next synchronisation.  The tensor-core chunk kernels wait on each other
 *    only through bounded loops (mbarriers of their own CTA; in the one-launch
 *    form, the scan CTAs on flags the prep CTAs publish); a wait that runs out
 *    sets a device error word and the kernel returns with its outputs
 *    unwritten.  kda_device_status() reads and clears that word.
 *  - Errors: a negative status (see kda_status); no exception and no device
 *    trap ever crosses the ABI.  Arguments are checked on the host before any
 *    CUDA call is made.
 *  - Alignment: every pointer must be 16-byte aligned (KDA_ERR_ALIGN).
 *  - Layouts (contiguous, row-major, "BTHD"):
 *        q, k, g      [B, T, H, dk]
 *        v, out       [B, T, H, dv]
 *        beta         [B, T, H]
 *        S0, S_T, S   [B, H, dk, dv]  FP32, rows = key channels
 *  - Element types: opts->dtype selects the type of q, k, v, g, beta and out
 *    (bf16 or fp32).  The recurrent state is always FP32 and all arithmetic
 *    is FP32 (or BF16 tensor-core operands with FP32 accumulation).
 *  - Shapes: dk and dv must each be 64 or 128 (KDA_ERR_UNSUPPORTED otherwise).
 *    T need not be a multiple of the 64-token chunk.  T == 0 is the identity:
 *    S_T = S0 (zero when S0 is NULL).  B == 0 or H == 0 is a no-op.
 */
#ifndef KDA_B200_KDA_H
#define KDA_B200_KDA_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of the activation tensors. */
typedef enum { KDA_BF16 = 0, KDA_F32 = 1 } kda_dtype;

/* Status codes returned by every entry point. */
typedef enum {
    KDA_OK = 0,
    KDA_ERR_ARG = -1,          /* NULL pointer, negative size, unknown flag bit */
    KDA_ERR_SHAPE = -2,        /* inconsistent sizes, size overflow            */
    KDA_ERR_ALIGN = -3,        /* a pointer is not 16-byte aligned             */
    KDA_ERR_UNSUPPORTED = -4,  /* valid but not implemented (dk/dv, flags)     */
    KDA_ERR_CUDA = -5,         /* a CUDA launch or copy reported an error      */
    KDA_ERR_TIMEOUT = -6,      /* a bounded device wait gave up               */
    KDA_ERR_WORKSPACE = -7     /* workspace missing or smaller than required   */
} kda_status;

/* Flag bits of kda_opts.flags. */
enum {
    KDA_QK_L2NORM = 1u,  /* q, k <- x / sqrt(sum x^2 + 1e-6) per head, in-kernel
                            (use_qk_l2norm_in_kernel, "Kimi K3 の KDA(1)" 1.2.1) */
    KDA_COMPLEX = 2u,    /* Complex-KDA: `g` holds the signed gate alpha itself,
                            |alpha| in [e^-5, 1], alpha != 0; beta in [0, 2]   */
    KDA_FUSED = 4u,      /* bf16 dk = dv = 128 only: run the chunk forward as one
                            fused kernel per sequence (no workspace)          */
    KDA_SPLIT = 8u,      /* bf16 dk = dv = 128 only: run it as the parallel
                            per-chunk prep kernel + per-sequence scan pair
                            (workspace: one record per chunk and head).
                            With neither flag the library picks the one its
                            cost model, from B*H and the device's SM count,
                            says is faster; KDA_FUSED | KDA_SPLIT is an error */
    KDA_UNBOUNDED_DECAY = 16u, /* g may lie anywhere in (-inf, 0]: no -5 floor.
                            The bounded tensor-core forms reference decay
                            factors to 16-token band starts, which needs the
                            floor (page "Kimi K3 模型结构（2）", Q&A on the -5
                            bound).  With this flag the bf16 dk = dv = 128
                            chunk forward takes the split form with the
                            off-diagonal band pairs on the tensor cores (every
                            factor one exponential of an exponent <= 0) and the
                            diagonal 16 x 16 blocks as FP32 position pairs;
                            with KDA_COMPLEX, fp32 data or d = 64 it takes the
                            exact-FP32 chunk path.  Cannot be combined with
                            KDA_FUSED or KDA_SPLIT (KDA_ERR_ARG).  The decode
                            step is exact for any g and ignores the flag.   */
    KDA_GATE_SOFTPLUS = 32u /* prologue entry points: the Kimi Linear gate
                            g = -exp(A_h) * softplus(z), range (-inf, 0), in
                            place of the bounded -5 * sigmoid(exp(A_h) z)
                            (same Q&A item, "与 Kimi Linear 的负 softplus 有何
                            不同").  Implies KDA_UNBOUNDED_DECAY everywhere. */
};

/* Options.  Passing NULL means {KDA_BF16, KDA_QK_L2NORM, 1.0f, NULL, 0, NULL, 0}. */
typedef struct {
    kda_dtype dtype;        /* type of q, k, v, g, beta, out                  */
    unsigned flags;         /* KDA_QK_L2NORM | KDA_COMPLEX | KDA_FUSED | KDA_SPLIT |
                               KDA_UNBOUNDED_DECAY | KDA_GATE_SOFTPLUS */
    float scale;            /* read-out scale; the pages use 1                 */
    void *workspace;        /* device scratch, >= kda_*_workspace_bytes()     */
    size_t workspace_bytes;
    /* Optional instrumentation: when non-NULL, events[i] is recorded on
       `stream` just before the i-th kernel launch of the call and
       events[launches] right after the last one, for i < n_events. */
    cudaEvent_t *events;
    int n_events;
} kda_opts;

/*
 * kda_chunk_fwd -- chunkwise-parallel forward (chunk_kda; training/prefill).
 *
 * Page "Kimi K3 模型结构（2）：序列维度（下），chunkwise 并行与下界衰减",
 * Q&A items: the sequence is cut into chunks of C = 64 tokens, one state
 * update per chunk, matmuls inside a chunk through the WY representation and
 * one C x C triangular (UT) inverse; A = Tril[(Q*Gamma)(K/Gamma)^T] with its
 * diagonal and O = (Gamma*Q) S + A V~.  The result equals the token
 * recurrence above up to rounding.
 *
 *   q, k     [B,T,H,dk]  queries/keys (normalised in-kernel if KDA_QK_L2NORM)
 *   v        [B,T,H,dv]  values
 *   g        [B,T,H,dk]  log-decay g = log(alpha), expected in [-5, 0] for
 *                        unsigned KDA (bounded decay) unless
 *                        KDA_UNBOUNDED_DECAY is set; with KDA_COMPLEX, the
 *                        signed gate alpha itself
 *   beta     [B,T,H]     write strength (already through the sigmoid)
 *   S0       [B,H,dk,dv] FP32 initial state, NULL means zero
 *   out      [B,T,H,dv]  outputs o_t
 *   S_T      [B,H,dk,dv] FP32 final state, NULL to skip
 *   opts->workspace must hold kda_chunk_workspace_bytes(...) bytes (may be
 *   NULL when that is 0).
 */
int kda_chunk_fwd(const void *q, const void *k, const void *v, const void *g,
                  const void *beta, const float *S0, void *out, float *S_T,
                  int B, int T, int H, int dk, int dv, const kda_opts *opts,
                  cudaStream_t stream);

/*
 * kda_chunk_fwd_gated -- kda_chunk_fwd with the branch's output epilogue fused in.
 *
 * Page "Kimi K3 の KDA(1)", section 1.2.1, the full-rank output gate:
 * o = FusedRMSNormGated(o, g_out) = RMSNorm(o) * sigmoid(g_out), the RMS taken per
 * (token, head) over the dv values, the norm before the gate.  Computed as
 *     out = o / sqrt(mean(o^2) + norm_eps) * norm_weight * sigmoid(out_gate)
 * in FP32 (the pages give neither the weight nor eps; norm_weight is one dv-vector
 * shared by the heads, NULL = ones).  On the split tensor-core form with B*H >= 64 it
 * is applied inside the scan, before the outputs leave the chip; otherwise as one
 * bandwidth-bound pass over out (cheaper when few sequences make the scan the chain).
 *
 *   out_gate    [B,T,H,dv] gate logits (dtype of out), required
 *   norm_weight [dv] FP32 or NULL;  norm_eps >= 0 (1e-5 is the usual choice)
 * Everything else, the workspace included, as kda_chunk_fwd.
 */
int kda_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *g,
                        const void *beta, const float *S0, void *out, float *S_T,
                        const void *out_gate, const float *norm_weight, float norm_eps,
                        int B, int T, int H, int dk, int dv, const kda_opts *opts,
                        cudaStream_t stream);

/* Workspace bytes kda_chunk_fwd needs for these sizes and options. */
size_t kda_chunk_workspace_bytes(int B, int T, int H, int dk, int dv,
                                 const kda_opts *opts);

/*
 * kda_recurrent_step -- one-token recurrent step (fused_recurrent_kda; decode).
 *
 * Page "Kimi K3 模型结构（2）", Q&A item on train/prefill vs decode: decode
 * generates one token at a time with the recurrent form.  One call advances
 * N independent sequences by one token, updating S in place.
 *
 *   q, k, g  [N,H,dk]   v, out [N,H,dv]   beta [N,H]
 *   S        [N,H,dk,dv] FP32, read and overwritten with S_t
 * Needs no workspace.
 */
int kda_recurrent_step(const void *q, const void *k, const void *v, const void *g,
                       const void *beta, float *S, void *out, int N, int H, int dk,
                       int dv, const kda_opts *opts, cudaStream_t stream);

/*
 * kda_chunk_fwd_prologue -- the branch prologue fused ahead of kda_chunk_fwd.
 *
 * Page "Kimi K3 の KDA(1)", section 1.2.1: q, k and v each pass a causal
 * depthwise ShortConvolution (kernel 4, SiLU): every channel independent,
 * the current token and the three before it (zero history before t = 0, no
 * bias); the tap order is that of a causal Conv1d weight [channels, 4], tap 3
 * multiplying the current token.  The decay is the bounded map
 * g = -5 * sigmoid(exp(A_h) * z) (page "Kimi K3 模型结构（2）", Q&A on the
 * decay function) and beta = sigmoid(beta_logit) in FP32 (section 1.2.1,
 * `.float()` of b_proj).  q and k are then L2 normalised in the chunk kernel
 * (KDA_QK_L2NORM is implied).
 *
 *   q_pre, k_pre [B,T,H,dk], v_pre [B,T,H,dv]   pre-conv activations (dtype)
 *   conv_w       [3, H*dk, 4]  taps for q, k, v (dtype); needs dk == dv
 *   z            [B,T,H,dk]   decay logits (dtype)
 *   A            [H]          per-head log-scale A_h (FP32)
 *   beta_logit   [B,T,H]      FP32
 *   S0, out, S_T as in kda_chunk_fwd.
 * KDA_COMPLEX is not supported here (the pages define no signed-gate map).
 * KDA_GATE_SOFTPLUS selects the Kimi Linear gate g = -exp(A_h) * softplus(z)
 * (unbounded below) and the unbounded chunk forward with it (KDA_UNBOUNDED_DECAY):
 * for bf16 d = 128 the gate is computed inside the split form's prep, otherwise
 * by the FP32 prologue ahead of the exact-FP32 chunk path.
 */
int kda_chunk_fwd_prologue(const void *q_pre, const void *k_pre, const void *v_pre,
                           const void *conv_w, const void *z, const float *A,
                           const float *beta_logit, const float *S0, void *out,
                           float *S_T, int B, int T, int H, int dk, int dv,
                           const kda_opts *opts, cudaStream_t stream);

/* Workspace bytes kda_chunk_fwd_prologue needs. */
size_t kda_prologue_workspace_bytes(int B, int T, int H, int dk, int dv,
                                    const kda_opts *opts);

/*
 * kda_recurrent_step_prologue -- the decode step with its branch prologue fused in.
 *
 * Page "Kimi K3 の KDA(1)", section 1.2.1 (short convolution k = 4 + SiLU on q, k,
 * v; beta = sigmoid(b) in FP32) and page "Kimi K3 模型结构（2）", Q&A on the decay
 * function (g = -5 * sigmoid(exp(A_h) * z)), applied to one new token per sequence.
 * The convolution's three earlier inputs per channel come from conv_state, which
 * is shifted by the new token in place; then q, k are L2 normalised (implied) and
 * the recurrent step of kda_recurrent_step runs.  All of it in FP32, in one kernel.
 *
 *   q_pre, k_pre, v_pre [N,H,d]   the new token's raw branch inputs (dtype)
 *   conv_w       [3, H*d, 4]      taps of q, k, v, tap 3 on the current token (dtype)
 *   conv_state   [N, 3, 3, H*d]   per sequence, branch (q, k, v) and tap
 *                                 (t-3, t-2, t-1): the previous raw inputs (dtype),
 *                                 read and overwritten.  Zeros = no history.
 *   z            [N,H,d]          gate logits (dtype);  A [H] FP32;  beta_logit [N,H] FP32
 *   S, out       as in kda_recurrent_step
 * Needs dk == dv; KDA_COMPLEX is not supported (no signed-gate map on the pages).
 * KDA_GATE_SOFTPLUS selects the Kimi Linear gate g = -exp(A_h) * softplus(z).
 */
int kda_recurrent_step_prologue(const void *q_pre, const void *k_pre, const void *v_pre,
                                const void *conv_w, void *conv_state, const void *z,
                                const float *A, const float *beta_logit, float *S, void *out,
                                int N, int H, int dk, int dv, const kda_opts *opts,
                                cudaStream_t stream);

/*
 * kda_conv_state_from_prefill -- the handoff from a prefill to decode: writes the
 * conv state [B, 3, 3, H*d] that kda_recurrent_step_prologue continues from, i.e.
 * the raw q, k, v inputs [B,T,H,d] of tokens T-3, T-2, T-1 (zeros where t < 0).
 * With the final state S_T of kda_chunk_fwd_prologue, decode then continues the
 * same sequence exactly.  opts->dtype gives the element type; d is 64 or 128.
 */
int kda_conv_state_from_prefill(const void *q_pre, const void *k_pre, const void *v_pre,
                                void *conv_state, int B, int T, int H, int d,
                                const kda_opts *opts, cudaStream_t stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate.
 *
 * The pages have no counterpart: this is a deployment variant, not part of
 * the method.  Some callers cannot call cudaMalloc -- code that must not
 * synchronise the device, loops that forbid allocation once running, host
 * applications that own the device pool and give a component no allocator.
 * This entry point takes the same arguments as kda_chunk_fwd, checked by the
 * same rules (opts->workspace is ignored), and runs the exact-FP32 two-phase
 * chunk path with its scratch in a fixed device array of
 * KDA_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
 * until the process exits.  It calls no allocator.  The flags that only pick
 * one of kda_chunk_fwd's paths (KDA_FUSED, KDA_SPLIT, KDA_UNBOUNDED_DECAY,
 * KDA_GATE_SOFTPLUS) are accepted and change nothing: the exact-FP32 path
 * takes any g <= 0.
 *
 *  - Sizes whose scratch (kda_chunk_workspace_bytes of the FP32 path: about
 *    148 KB per 64-token chunk and head at dk = dv = 128) exceeds the array
 *    are rejected with KDA_ERR_WORKSPACE before any CUDA call.
 *  - The first call on a device (with that device current) looks up the
 *    array's device address once; make that first call before any stream
 *    capture.  The address belongs to the device's primary context: after
 *    cudaDeviceReset, do not call this entry point again in that process.
 *  - All calls share the array.  Calls whose work overlaps on the GPU race;
 *    serialise them (one stream per device).  No scratch content carries over:
 *    each call writes every element it reads.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (32u << 20)
int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *g,
                          const void *beta, const float *S0, void *out, float *S_T,
                          int B, int T, int H, int dk, int dv, const kda_opts *opts,
                          cudaStream_t stream);

/*
 * kda_chunk_bwd -- backward of the chunk forward (chunk_kda training).
 *
 * Page "Kimi K3 模型结构（2）", Q&A on the train / prefill / decode forms: training
 * runs chunk_kda, so it needs the gradient of the forward.  Given the upstream
 * gradients dout = dL/dO and dS_T = dL/dS_T of a call of kda_chunk_fwd with the
 * same q, k, v, g, beta, S0 and opts, this writes the gradients of
 * L = <dout, O> + <dS_T, S_T> with respect to every input:
 *
 *   grad_q, grad_k, grad_g [B,T,H,dk] FP32   (q, k before the in-kernel L2 norm
 *                                             when KDA_QK_L2NORM is set; g as
 *                                             passed: log-decay, or with
 *                                             KDA_COMPLEX the signed gate alpha)
 *   grad_v [B,T,H,dv] FP32,  grad_beta [B,T,H] FP32
 *   grad_S0 [B,H,dk,dv] FP32, NULL to skip
 *
 * dout has the activation dtype (bf16 or fp32) with the layout of out; dS_T is
 * FP32 [B,H,dk,dv], NULL meaning zero; S0 NULL means zero.  All arithmetic is
 * FP32 and exact for any g <= 0 (no -5 floor needed).  The gradient outputs
 * are written, not accumulated.  opts->workspace must hold
 * kda_chunk_bwd_workspace_bytes(...) bytes: the FP32 state at every 8-token
 * window start and its gradient at every window end, 2*B*H*ceil(T/8)*dk*dv*4
 * bytes.  T == 0 writes grad_S0 = dS_T only.
 */
int kda_chunk_bwd(const void *q, const void *k, const void *v, const void *g,
                  const void *beta, const float *S0, const void *dout,
                  const float *dS_T, float *grad_q, float *grad_k, float *grad_v,
                  float *grad_g, float *grad_beta, float *grad_S0, int B, int T,
                  int H, int dk, int dv, const kda_opts *opts, cudaStream_t stream);

/* Workspace bytes kda_chunk_bwd needs. */
size_t kda_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv,
                                     const kda_opts *opts);

/*
 * kda_segment_pair -- the affine pair of a segment of tokens (for splitting one long
 * sequence over several GPUs: context parallelism over T).
 *
 * Page "Kimi K3 の KDA(1)", section 2.3 (the algebraic view): each token maps the
 * state by S -> T_t S + beta_t k_t v_t^T, T_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
 * so a segment maps it by one affine pair S -> M S + B, and pairs compose in order.
 * For the segment held in q, k, v, g, beta ([B,T,H,*], as kda_chunk_fwd) this writes
 *
 *   M_out [B,H,dk,dk] FP32   M = T_T ... T_1   (the final state from S0 = I, v = 0)
 *   B_out [B,H,dk,dv] FP32   B = the final state from S0 = 0
 *
 * For bf16 dk = dv = 128 (the split tensor-core form, any gate it takes) one prep pass
 * writes the segment's chunk records into opts->workspace and two scans over them run
 * side by side: B from S0 = 0, M from S0 = I with the chunks' U taken as zero (the state's
 * columns evolve independently, so column i is M e_i).  The records stay in the workspace
 * for kda_segment_forward.  Otherwise (fp32, d = 64, Complex-KDA with an unbounded gate)
 * it runs the chunk forward twice, the second time from S0 = I with v = 0.  Same flags
 * and tolerances as kda_chunk_fwd.  opts->workspace must hold
 * kda_segment_pair_workspace_bytes(...).  T == 0 gives the identity pair (I, 0).
 */
int kda_segment_pair(const void *q, const void *k, const void *v, const void *g,
                     const void *beta, float *M_out, float *B_out, int B, int T, int H,
                     int dk, int dv, const kda_opts *opts, cudaStream_t stream);

/* Workspace bytes kda_segment_pair (and kda_segment_forward after it) needs. */
size_t kda_segment_pair_workspace_bytes(int B, int T, int H, int dk, int dv,
                                        const kda_opts *opts);

/*
 * kda_segment_forward -- the segment's chunk forward from a start state S0 (the fold of the
 * earlier segments' pairs, kda_affine_combine), after kda_segment_pair on the SAME inputs with
 * the SAME opts (flags and workspace, untouched in between).  Same page and section.
 *
 * Arguments as kda_chunk_fwd.  On the split tensor-core form (bf16, dk = dv = 128) only the
 * scan runs, over the records kda_segment_pair left in opts->workspace (the inputs are not
 * read); otherwise this is kda_chunk_fwd (opts->workspace large enough for it: a
 * kda_segment_pair workspace is).  The result equals kda_chunk_fwd from S0 up to rounding.
 */
int kda_segment_forward(const void *q, const void *k, const void *v, const void *g,
                        const void *beta, const float *S0, void *out, float *S_T, int B, int T,
                        int H, int dk, int dv, const kda_opts *opts, cudaStream_t stream);

/*
 * kda_affine_combine -- fold the first n segment pairs onto a start state, in order:
 * S <- M_r S + B_r for r = 0, ..., n-1 (same page and section as kda_segment_pair).
 * With the pairs of segments 0..r-1 of a sequence this gives the state at the start of
 * segment r; with all of them, the sequence's final state.
 *
 *   M  [n, BH, dk, dk] FP32,  Bp [n, BH, dk, dv] FP32  (BH independent sequences)
 *   S0 [BH, dk, dv] FP32 start state, NULL means zero;  S_out [BH, dk, dv] FP32
 *      (may be S0 itself).
 * n == 0 copies S0 (or zeros) to S_out.  FP32 arithmetic on CUDA cores.
 */
int kda_affine_combine(const float *M, const float *Bp, int n, const float *S0,
                       float *S_out, int BH, int dk, int dv, cudaStream_t stream);

/*
 * kda_selftest_bounded_wait -- exercises the give-up path of the library's bounded waits.
 *
 * The pages have no counterpart: this is a check of the library's failure handling.  The
 * tensor-core kernels wait only in bounded loops (on mbarriers of their own CTA, and on
 * flags between CTAs of one launch); a wait that runs out sets an error word and the kernel
 * returns.  This launches one tiny kernel that waits, with at most `limit` polls each, on an
 * mbarrier no one arrives at and on a flag no one writes, then reads its status back and
 * synchronises `stream`.  It returns KDA_ERR_TIMEOUT when both waits gave up (the expected
 * outcome, for any limit, 0 included) and KDA_ERR_CUDA if the launch or the copy failed.
 * Nothing faults and nothing can hang; the CUDA context stays usable afterwards.
 */
int kda_selftest_bounded_wait(unsigned limit, cudaStream_t stream);

/*
 * kda_device_status -- the outcome of the kernels already enqueued on `stream`.
 *
 * The pages have no counterpart: this is the library's failure reporting.  Synchronises
 * `stream`, then reads and clears the device error words the tensor-core chunk kernels set
 * when one of their bounded waits gives up.  Returns KDA_OK when none did, KDA_ERR_TIMEOUT
 * when one did since the last call (that call's out and S_T are not valid), KDA_ERR_CUDA if
 * the synchronisation or the copies failed.  The words are per device and shared by all
 * streams: call it with no other chunk work in flight on the device.
 */
int kda_device_status(cudaStream_t stream);

/*
 * kda_set_wait_limit -- polls a bounded wait of the split tensor-core form makes before it
 * gives up (the prep kernel's waits and the one-launch form's wait for published records).
 *
 * The pages have no counterpart: this exists so failure handling can be tested on a GPU
 * without a fault.  0 makes those waits give up at once: the call then ends early with
 * KDA_ERR_TIMEOUT reported by kda_device_status(), copies and products already in flight
 * are drained first, and nothing faults.  KDA_WAIT_LIMIT_DEFAULT restores normal operation.
 * Returns the previous limit.  Host-global; not thread-safe against concurrent calls.
 */
#define KDA_WAIT_LIMIT_DEFAULT (1u << 22)
unsigned kda_set_wait_limit(unsigned polls);

/* Static description of a status code (never NULL). */
const char *kda_status_string(int status);

/* Library ABI version: 100 * major + minor (1.3: kda_chunk_fwd_gated;
   1.4: KDA_UNBOUNDED_DECAY, KDA_GATE_SOFTPLUS; 1.5: kda_chunk_bwd;
   1.6: kda_segment_pair, kda_affine_combine; 1.7: kda_selftest_bounded_wait;
   1.8: kda_device_status, kda_set_wait_limit; 1.9: kda_segment_forward;
   1.10: the kda_chunk_bwd workspace holds the state gradients too). */
int kda_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KDA_B200_KDA_H */
