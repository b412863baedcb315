// kda_internal.h -- launch descriptors passed from the C ABI layer to kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include "kda_common.cuh"

namespace kda {

struct DecodeArgs {
    const void *q, *k, *v, *g, *beta;
    float *S;
    void *out;
    long long units;   // N * H
    int dk, dv;
    bool bf16;
    KernelFlags fl;
    // decode prologue (conv_w != nullptr): q, k, v are the raw new token, g is the gate
    // logit z, beta is unused; the short convolution reads and shifts conv_state
    const void *conv_w;     // [3, H * d, 4]
    void *conv_state;       // [N, 3 branches, 3 taps (t-3, t-2, t-1), H * d], dtype of q
    const float *A;         // [H]
    const float *b_logit;   // [N, H]
    int H;
    int gate_softplus;      // gate g = -exp(A_h) softplus(z) instead of -5 sigmoid(exp(A_h) z)
};

// Last three raw rows of each branch of a prefill, as the decode prologue's conv state.
cudaError_t launch_conv_state_from_prefill(const void *q_pre, const void *k_pre, const void *v_pre,
                                           void *conv_state, int B, int T, int H, int d, bool bf16,
                                           cudaStream_t st);

// Element types of the chunk path's inputs.
enum class Elt : int { BF16 = 0, F32 = 1 };

struct ChunkArgs {
    const void *q, *k, *v, *g, *beta;   // inputs ([B,T,H,*])
    Elt t_qkv, t_g, t_beta, t_out;
    const float *S0;                     // nullable
    void *out;
    float *S_T;                          // nullable
    int B, T, H, dk, dv;
    KernelFlags fl;
    void *workspace;
    size_t workspace_bytes;
    cudaEvent_t *events;
    int n_events;
    int *launch_idx;                     // running launch counter for events
    // output epilogue (FusedRMSNormGated): out = o / sqrt(mean(o^2) + eps) * w * sigmoid(gate)
    // per (token, head) row of dv values; out_gate == nullptr: no epilogue
    const void *out_gate;                // [B,T,H,dv], dtype of out
    const float *norm_w;                 // [dv], nullable = ones
    float norm_eps;
    // g may fall below -5 per token: only the exact-FP32 path takes such inputs
    bool exact_decay;
};

// The output epilogue as its own pass over out (in place), for the paths that do not fuse it.
cudaError_t launch_out_epilogue(const ChunkArgs &a, cudaStream_t st);

struct PrologueArgs {
    const void *q_pre, *k_pre, *v_pre, *conv_w, *z;
    const float *A, *beta_logit;
    bool bf16;                           // element type of the raw inputs
    bool out_bf16;                       // outputs in bf16 (tensor-core path) or FP32
    int B, T, H, dk, dv;
    void *qc, *kc, *vc, *g, *beta;       // outputs in the workspace
    int gate_softplus;                   // g = -exp(A_h) softplus(z) (unbounded; FP32 outputs)
};

// Workspace of the FP32 two-phase chunk path.
size_t chunk_ref_workspace_bytes(int B, int T, int H, int dk, int dv);

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);
// Fused tensor-core chunk path (bf16, dk = dv = 128); needs no workspace.
bool chunk_tc_supported(const ChunkArgs &a);
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t st);
// Read and clear the fused form's device error word (1 = a bounded wait gave up); synchronises st.
cudaError_t chunk_tc_take_error(int *flag, cudaStream_t st);
// Two-kernel tensor-core chunk path (parallel prep + per-head scan); needs a workspace.
size_t chunk_tc2_workspace_bytes(int B, int T, int H);
cudaError_t launch_chunk_tc2(const ChunkArgs &a, cudaStream_t st);
// Read and clear the split form's device error word; synchronises st.
cudaError_t chunk_tc2_take_error(int *flag, cudaStream_t st);
// Polls before a bounded wait of the split form gives up (the prep's waits, the one-launch
// scan's wait for published records); returns the previous value.
uint32_t set_wait_limit(uint32_t polls);
// The split form with the prologue fused into its prep kernel: the prep stages the raw
// q, k, v, z tiles with a 3-row halo and applies the short convolution, SiLU, the gate and
// beta = sigmoid(logit) on chip.  Uses a.out, a.S0, a.S_T, sizes, flags, workspace, events.
cudaError_t launch_chunk_tc2_prologue(const PrologueArgs &p, const ChunkArgs &a, cudaStream_t st);
// The segment pair on the split form (kda_segment_pair): prep records into a.workspace, then the
// scans from S0 = 0 (B_out) and from S0 = eye with U taken as zero (M_out) in one launch.
cudaError_t launch_segment_pair_tc2(const ChunkArgs &a, const float *eye, float *M_out, float *B_out,
                                    cudaStream_t st);
// The scan alone from a.S0 over the records a preceding launch_segment_pair_tc2 left in
// a.workspace (kda_segment_forward).
cudaError_t launch_segment_scan_tc2(const ChunkArgs &a, cudaStream_t st);
cudaError_t launch_chunk_ref(const ChunkArgs &a, cudaStream_t st);
cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t st);

// Backward of the chunk forward (kda_chunk_bwd): gradients in FP32.
struct BwdArgs {
    const void *q, *k, *v, *g, *beta;    // forward inputs ([B,T,H,*], dtype)
    const float *S0;                     // nullable
    const void *dout;                    // [B,T,H,dv], dtype
    const float *dS_T;                   // nullable
    float *dq, *dk, *dv, *dg, *dbeta;    // [B,T,H,dk] x3 / [B,T,H,dv] / [B,T,H]
    float *dS0;                          // nullable
    void *workspace;                     // chunk_bwd_workspace_bytes
    int B, T, H, dk_, dv_;
    bool bf16;
    KernelFlags fl;
    cudaEvent_t *events;                 // kda_opts.events: one before each launch, one after
    int n_events;
};
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t st);

// Affine pairs of segments (context parallelism over T): the identity start state and the
// ordered fold S <- M_r S + B_r of n pairs ([n, BH, dk, dk] and [n, BH, dk, dv], FP32).
cudaError_t launch_identity(float *S, long long count, int d, cudaStream_t st);
cudaError_t launch_affine_combine(const float *M, const float *Bp, int n, const float *S0, float *S_out,
                                  int BH, int dk, int dv, cudaStream_t st);

// Self-test of the bounded waits: one kernel whose mbarrier wait and flag poll both run out
// (nothing arrives); *status gets bit 0 / bit 1 for each that gave up.  Synchronises `st`.
cudaError_t run_bounded_wait_selftest(unsigned limit, int *status, cudaStream_t st);

// Record a.events[*a.launch_idx] (if requested) and advance the counter.
inline void mark_launch(const ChunkArgs &a, cudaStream_t st) {
    if (a.events && a.launch_idx && *a.launch_idx < a.n_events)
        cudaEventRecord(a.events[*a.launch_idx], st);
    if (a.launch_idx) ++*a.launch_idx;
}

}  // namespace kda
