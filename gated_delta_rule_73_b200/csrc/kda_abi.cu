// kda_abi.cu -- the C ABI: argument checks, workspace sizing and dispatch.
//
// Every check runs on the host before the first CUDA call, so a rejected call
// touches no device state.  See include/kda.h for the contract.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/kda.h"
#include "kda_internal.h"
#include "kda_checks.h"

using namespace kda;

namespace {

constexpr size_t kAlignWs = 256;
constexpr long long kMaxElems = 1LL << 40;   // refuse sizes whose byte offsets could overflow

kda_opts resolve(const kda_opts *o) {
    kda_opts r;
    memset(&r, 0, sizeof(r));
    r.dtype = KDA_BF16;
    r.flags = KDA_QK_L2NORM;
    r.scale = 1.0f;
    if (o) r = *o;
    return r;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
// g without the -5 floor (Kimi Linear's softplus gate, or the caller says so): the split
// tensor-core form takes it with FP32 diagonal blocks (its fused form and its signed-gate steps
// rely on the floor); with Complex-KDA it runs on the FP32 path
bool unbounded(const kda_opts &o) { return (o.flags & (KDA_UNBOUNDED_DECAY | KDA_GATE_SOFTPLUS)) != 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

KernelFlags kflags(const kda_opts &o) {
    KernelFlags f;
    f.l2norm = (o.flags & KDA_QK_L2NORM) ? 1 : 0;
    f.complex_gate = (o.flags & KDA_COMPLEX) ? 1 : 0;
    f.scale = o.scale;
    return f;
}

// The bf16 dk = dv = 128 chunk forward runs on tensor cores, in one of two forms:
//  * split: a parallel per-chunk prep kernel and a per-sequence scan (workspace: one
//    record per chunk and head).  Cost ~ B*H*nch*t_prep / SMs + waves * nch * t_scan.
//  * fused: one kernel per sequence, prep and scan step serially in one CTA (no
//    workspace).  Cost ~ waves * nch * t_fused, waves = ceil(B*H / SMs).
// Measured on B200 at d = 128: t_fused = 14.0 us per chunk of a wave of sequences, t_prep =
// 6.8 us of one SM per (chunk, head) item (the two-group prep), t_scan = 2.4 us per chunk (one
// CTA per head); the model uses their ratios.  With the two-group prep the split form wins at
// every B*H; the fused form stays available through KDA_FUSED.  KDA_SPLIT forces the split.
// An unbounded gate always takes the split form.
bool use_tc(const kda_opts &o, int dk, int dv) {
    return o.dtype == KDA_BF16 && dk == 128 && dv == 128 && !(unbounded(o) && (o.flags & KDA_COMPLEX));
}
int device_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}
bool use_fused(const kda_opts &o, int B, int H) {
    if (unbounded(o)) return false;
    if (o.flags & KDA_FUSED) return true;
    if (o.flags & KDA_SPLIT) return false;
    const double x = (double)B * H / device_sms();
    const double waves = ceil(x);
    const double t_fused = 1.0, t_prep = 6.8 / 14.0, t_scan = 2.4 / 14.0;
    return waves * t_fused < x * t_prep + waves * t_scan;
}
size_t tc_ws(const kda_opts &o, int B, int T, int H) {
    if (B <= 0 || T <= 0 || H <= 0 || use_fused(o, B, H)) return 0;
    return round_up(chunk_tc2_workspace_bytes(B, T, H), kAlignWs);
}

size_t chunk_ws(int B, int T, int H, int dk, int dv) {
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    return round_up(chunk_ref_workspace_bytes(B, T, H, dk, dv), kAlignWs);
}

// The prologue's outputs are bf16 when the tensor-core chunk kernel follows
// (bf16 activations, dk = dv = 128; it needs no further workspace), FP32 otherwise.
size_t prologue_ws_parts(int B, int T, int H, int dk, int dv, bool tc, size_t tc_extra, size_t *off,
                         bool fused_pro = false) {
    // off[0..5]: qc, kc, vc, g, beta, chunk workspace.  With the prologue fused into the
    // split form's prep kernel there are no intermediates: only the chunk workspace.
    if (fused_pro) {
        for (int i = 0; i < 6; ++i) off[i] = 0;
        return tc_extra;
    }
    const size_t rows = (size_t)B * T * H;
    const size_t e = tc ? 2 : 4;
    size_t o = 0;
    off[0] = o; o = round_up(o + rows * dk * e, kAlignWs);
    off[1] = o; o = round_up(o + rows * dk * e, kAlignWs);
    off[2] = o; o = round_up(o + rows * dv * e, kAlignWs);
    off[3] = o; o = round_up(o + rows * dk * e, kAlignWs);
    off[4] = o; o = round_up(o + rows * e, kAlignWs);
    off[5] = o; o += tc ? tc_extra : chunk_ws(B, T, H, dk, dv);
    return o;
}

int finish_identity(const float *S0, float *S_T, int B, int H, int dk, int dv, cudaStream_t st) {
    if (!S_T || B == 0 || H == 0) return KDA_OK;
    const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
    cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st)
                       : cudaMemsetAsync(S_T, 0, bytes, st);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int run_chunk(ChunkArgs &a, bool fused, cudaStream_t st) {
    int launches = 0;
    a.launch_idx = &launches;
    // Output epilogue: the split form can apply it inside its scan, on the per-chunk chain of
    // every sequence (about 1 us per chunk); a separate pass costs the bytes of out and the
    // gate instead.  Measured on B200 the chain wins from about 64 sequences on (T=8192:
    // 96 heads 0.14 vs 0.22 ms; T=4096, 16 heads: 0.048 vs 0.020 ms).
    const bool tc = chunk_tc_supported(a) && !(a.exact_decay && a.fl.complex_gate);
    if (a.exact_decay) fused = false;
    const bool split = tc && !fused;
    const bool fuse_epi = split && a.out_gate && (long long)a.B * a.H >= 64;
    const void *gate = a.out_gate;
    if (split && !fuse_epi) a.out_gate = nullptr;
    cudaError_t e = !tc                     ? launch_chunk_ref(a, st)
                    : fused                 ? launch_chunk_tc(a, st)
                                            : launch_chunk_tc2(a, st);
    a.out_gate = gate;
    if (e == cudaSuccess && a.out_gate && !fuse_epi) e = launch_out_epilogue(a, st);
    if (e == cudaSuccess && a.events && launches < a.n_events) cudaEventRecord(a.events[launches], st);
    if (e == cudaErrorInvalidValue) return KDA_ERR_UNSUPPORTED;
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

namespace kda {
// Shared by every entry point (kda_noalloc.cu included), so the argument rules cannot drift.
int check_opts(const kda_opts &o) {
    if (o.dtype != KDA_BF16 && o.dtype != KDA_F32) return KDA_ERR_ARG;
    if (o.flags & ~(unsigned)(KDA_QK_L2NORM | KDA_COMPLEX | KDA_FUSED | KDA_SPLIT |
                              KDA_UNBOUNDED_DECAY | KDA_GATE_SOFTPLUS))
        return KDA_ERR_ARG;
    if ((o.flags & KDA_FUSED) && (o.flags & KDA_SPLIT)) return KDA_ERR_ARG;
    if (unbounded(o) && (o.flags & (KDA_FUSED | KDA_SPLIT))) return KDA_ERR_ARG;
    if ((o.flags & KDA_GATE_SOFTPLUS) && (o.flags & KDA_COMPLEX)) return KDA_ERR_ARG;
    if (!isfinite(o.scale)) return KDA_ERR_ARG;
    if (o.n_events < 0 || (o.n_events > 0 && !o.events)) return KDA_ERR_ARG;
    return KDA_OK;
}

int check_dims(long long B, long long T, long long H, int dk, int dv) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    const long long d = dk > dv ? dk : dv;
    if (B > 0 && T > 0 && H > 0) {
        if (B > kMaxElems / T) return KDA_ERR_SHAPE;
        const long long bt = B * T;
        if (bt > kMaxElems / H) return KDA_ERR_SHAPE;
        if (bt * H > kMaxElems / d) return KDA_ERR_SHAPE;
    }
    if (B * H > 65535) return KDA_ERR_UNSUPPORTED;   // grid y of the chunk kernels
    return KDA_OK;
}
}  // namespace kda

extern "C" {

int kda_abi_version(void) { return 110; }

const char *kda_status_string(int s) {
    switch (s) {
        case KDA_OK: return "ok";
        case KDA_ERR_ARG: return "invalid argument (NULL pointer, negative size or unknown flag)";
        case KDA_ERR_SHAPE: return "inconsistent or overflowing sizes";
        case KDA_ERR_ALIGN: return "pointer not 16-byte aligned";
        case KDA_ERR_UNSUPPORTED: return "unsupported configuration (dk, dv other than 64 or 128, or an option the entry point does not take)";
        case KDA_ERR_CUDA: return "CUDA launch or copy failed";
        case KDA_ERR_TIMEOUT: return "a bounded device wait gave up";
        case KDA_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

size_t kda_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, const kda_opts *opts) {
    const kda_opts o = resolve(opts);
    if (check_opts(o) != KDA_OK || check_dims(B, T, H, dk, dv) != KDA_OK) return 0;
    if (use_tc(o, dk, dv)) return tc_ws(o, B, T, H);
    return chunk_ws(B, T, H, dk, dv);
}

size_t kda_prologue_workspace_bytes(int B, int T, int H, int dk, int dv, const kda_opts *opts) {
    const kda_opts o = resolve(opts);
    if (check_opts(o) != KDA_OK || check_dims(B, T, H, dk, dv) != KDA_OK) return 0;
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    size_t off[6];
    const bool tc = use_tc(o, dk, dv);
    return prologue_ws_parts(B, T, H, dk, dv, tc, tc_ws(o, B, T, H), off, tc && !use_fused(o, B, H));
}

static int chunk_fwd_impl(const void *q, const void *k, const void *v, const void *g, const void *beta,
                   const float *S0, void *out, float *S_T, const void *out_gate, const float *norm_w,
                   float norm_eps, int B, int T, int H, int dk, int dv, const kda_opts *opts,
                   cudaStream_t stream) {
    const kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if ((s = check_dims(B, T, H, dk, dv)) != KDA_OK) return s;
    if (B == 0 || H == 0) return KDA_OK;
    if (T == 0) {
        if (!aligned16(S0) || !aligned16(S_T)) return KDA_ERR_ALIGN;
        return finish_identity(S0, S_T, B, H, dk, dv, stream);
    }
    if (!q || !k || !v || !g || !beta || !out) return KDA_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, out, S_T, o.workspace, out_gate, norm_w};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    const size_t need = use_tc(o, dk, dv) ? tc_ws(o, B, T, H) : chunk_ws(B, T, H, dk, dv);
    if (need > 0 && (!o.workspace || o.workspace_bytes < need)) return KDA_ERR_WORKSPACE;

    ChunkArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
    const Elt t = o.dtype == KDA_BF16 ? Elt::BF16 : Elt::F32;
    a.t_qkv = a.t_g = a.t_beta = a.t_out = t;
    a.S0 = S0; a.out = out; a.S_T = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
    a.fl = kflags(o);
    a.workspace = o.workspace; a.workspace_bytes = o.workspace_bytes;
    a.events = o.events; a.n_events = o.n_events;
    a.out_gate = out_gate; a.norm_w = norm_w; a.norm_eps = norm_eps;
    a.exact_decay = unbounded(o);
    return run_chunk(a, use_fused(o, B, H), stream);
}

// Workspace of kda_segment_pair: a zero v [B,T,H,dk] and an identity S0 [B,H,dk,dk] for the
// run that yields M, a scratch out [B,T,H,max(dk,dv)] both runs write, and the chunk
// forward's own workspace (the larger of the two runs').
// Split tensor-core form (bf16, d = 128): the chunk records (kept for kda_segment_forward),
// then the identity start state of the M scan.
static size_t segment_ws_tc(int B, int T, int H, int dk, size_t *eye_off) {
    *eye_off = round_up(chunk_tc2_workspace_bytes(B, T, H), kAlignWs);
    return *eye_off + (size_t)B * H * dk * dk * 4;
}

static size_t segment_ws_parts(const kda_opts &o, int B, int T, int H, int dk, int dv, size_t *off) {
    const size_t e = o.dtype == KDA_BF16 ? 2 : 4;
    const size_t rows = (size_t)B * T * H;
    const int dmax = dk > dv ? dk : dv;
    auto cws = [&](int dvv) { return use_tc(o, dk, dvv) ? tc_ws(o, B, T, H) : chunk_ws(B, T, H, dk, dvv); };
    const size_t c1 = cws(dv), c2 = cws(dk);
    size_t x = 0;
    off[0] = x; x = round_up(x + rows * dk * e, kAlignWs);
    off[1] = x; x = round_up(x + (size_t)B * H * dk * dk * 4, kAlignWs);
    off[2] = x; x = round_up(x + rows * dmax * e, kAlignWs);
    off[3] = x; x += c1 > c2 ? c1 : c2;
    return x;
}

size_t kda_segment_pair_workspace_bytes(int B, int T, int H, int dk, int dv, const kda_opts *opts) {
    const kda_opts o = resolve(opts);
    if (check_opts(o) != KDA_OK || check_dims(B, T, H, dk, dv) != KDA_OK) return 0;
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    size_t off[4];
    if (use_tc(o, dk, dv)) return segment_ws_tc(B, T, H, dk, off);
    return segment_ws_parts(o, B, T, H, dk, dv, off);
}

int kda_chunk_fwd(const void *q, const void *k, const void *v, const void *g, const void *beta,
                  const float *S0, void *out, float *S_T, int B, int T, int H, int dk, int dv,
                  const kda_opts *opts, cudaStream_t stream) {
    return chunk_fwd_impl(q, k, v, g, beta, S0, out, S_T, nullptr, nullptr, 0.f, B, T, H, dk, dv,
                          opts, stream);
}

int kda_segment_pair(const void *q, const void *k, const void *v, const void *g, const void *beta,
                     float *M_out, float *B_out, int B, int T, int H, int dk, int dv,
                     const kda_opts *opts, cudaStream_t stream) {
    const kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if ((s = check_dims(B, T, H, dk, dv)) != KDA_OK) return s;
    if (B == 0 || H == 0) return KDA_OK;
    if (!M_out || !B_out) return KDA_ERR_ARG;
    if (!aligned16(M_out) || !aligned16(B_out)) return KDA_ERR_ALIGN;
    if (T == 0) {   // the empty segment is the identity pair (I, 0)
        if (launch_identity(M_out, (long long)B * H, dk, stream) != cudaSuccess) return KDA_ERR_CUDA;
        return cudaMemsetAsync(B_out, 0, (size_t)B * H * dk * dv * 4, stream) == cudaSuccess ? KDA_OK
                                                                                         : KDA_ERR_CUDA;
    }
    if (!q || !k || !v || !g || !beta) return KDA_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, o.workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    size_t off[4];
    if (use_tc(o, dk, dv)) {
        // one prep pass (its records stay in the workspace for kda_segment_forward), then the
        // scans from S0 = 0 (B) and from S0 = I with U taken as zero (M) side by side
        const size_t need = segment_ws_tc(B, T, H, dk, off);
        if (!o.workspace || o.workspace_bytes < need) return KDA_ERR_WORKSPACE;
        float *eye = (float *)((char *)o.workspace + off[0]);
        if (launch_identity(eye, (long long)B * H, dk, stream) != cudaSuccess) return KDA_ERR_CUDA;
        ChunkArgs a;
        memset(&a, 0, sizeof(a));
        a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
        a.t_qkv = a.t_g = a.t_beta = a.t_out = Elt::BF16;
        a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
        a.fl = kflags(o);
        a.workspace = o.workspace; a.workspace_bytes = need;
        a.exact_decay = unbounded(o);
        int launches = 0;
        a.launch_idx = &launches;
        cudaError_t e = launch_segment_pair_tc2(a, eye, M_out, B_out, stream);
        if (e == cudaErrorInvalidValue) return KDA_ERR_UNSUPPORTED;
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    const size_t need = segment_ws_parts(o, B, T, H, dk, dv, off);
    if (!o.workspace || o.workspace_bytes < need) return KDA_ERR_WORKSPACE;
    char *ws = (char *)o.workspace;
    void *zv = ws + off[0];
    float *eye = (float *)(ws + off[1]);
    void *scratch_out = ws + off[2];
    kda_opts oc = o;
    oc.workspace = ws + off[3];
    oc.workspace_bytes = need - off[3];
    oc.events = nullptr;
    oc.n_events = 0;
    const size_t e = o.dtype == KDA_BF16 ? 2 : 4;
    if (cudaMemsetAsync(zv, 0, (size_t)B * T * H * dk * e, stream) != cudaSuccess) return KDA_ERR_CUDA;
    if (launch_identity(eye, (long long)B * H, dk, stream) != cudaSuccess) return KDA_ERR_CUDA;
    // B: the segment's final state from S0 = 0
    s = chunk_fwd_impl(q, k, v, g, beta, nullptr, scratch_out, B_out, nullptr, nullptr, 0.f, B, T, H,
                       dk, dv, &oc, stream);
    if (s != KDA_OK) return s;
    // M: from S0 = I with v = 0 (column i of the final state is M e_i)
    return chunk_fwd_impl(q, k, zv, g, beta, eye, scratch_out, M_out, nullptr, nullptr, 0.f, B, T, H,
                          dk, dk, &oc, stream);
}

int kda_segment_forward(const void *q, const void *k, const void *v, const void *g, const void *beta,
                        const float *S0, void *out, float *S_T, int B, int T, int H, int dk, int dv,
                        const kda_opts *opts, cudaStream_t stream) {
    const kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if ((s = check_dims(B, T, H, dk, dv)) != KDA_OK) return s;
    if (!use_tc(o, dk, dv))   // no records on this path: the whole chunk forward
        return chunk_fwd_impl(q, k, v, g, beta, S0, out, S_T, nullptr, nullptr, 0.f, B, T, H, dk, dv, opts,
                              stream);
    if (B == 0 || H == 0) return KDA_OK;
    if (T == 0) {
        if (!aligned16(S0) || !aligned16(S_T)) return KDA_ERR_ALIGN;
        return finish_identity(S0, S_T, B, H, dk, dv, stream);
    }
    if (!out) return KDA_ERR_ARG;
    const void *ptrs[] = {S0, out, S_T, o.workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    size_t eye_off;
    const size_t need = segment_ws_tc(B, T, H, dk, &eye_off);
    if (!o.workspace || o.workspace_bytes < need) return KDA_ERR_WORKSPACE;
    ChunkArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
    a.t_qkv = a.t_g = a.t_beta = a.t_out = Elt::BF16;
    a.S0 = S0; a.out = out; a.S_T = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
    a.fl = kflags(o);
    a.workspace = o.workspace; a.workspace_bytes = need;
    a.events = o.events; a.n_events = o.n_events;
    int launches = 0;
    a.launch_idx = &launches;
    cudaError_t e = launch_segment_scan_tc2(a, stream);
    if (e == cudaSuccess && o.events && launches < o.n_events) cudaEventRecord(o.events[launches], stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_affine_combine(const float *M, const float *Bp, int n, const float *S0, float *S_out, int BH,
                       int dk, int dv, cudaStream_t stream) {
    if (n < 0 || BH < 0 || dk <= 0 || dv <= 0) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    if (BH == 0) return KDA_OK;
    if (!S_out || (n > 0 && (!M || !Bp))) return KDA_ERR_ARG;
    const void *ptrs[] = {M, Bp, S0, S_out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    return launch_affine_combine(M, Bp, n, S0, S_out, BH, dk, dv, stream) == cudaSuccess ? KDA_OK
                                                                                      : KDA_ERR_CUDA;
}

int kda_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *g, const void *beta,
                        const float *S0, void *out, float *S_T, const void *out_gate,
                        const float *norm_weight, float norm_eps, int B, int T, int H, int dk,
                        int dv, const kda_opts *opts, cudaStream_t stream) {
    if (!isfinite(norm_eps) || norm_eps < 0.f) return KDA_ERR_ARG;
    if (!out_gate && B > 0 && T > 0 && H > 0) return KDA_ERR_ARG;
    return chunk_fwd_impl(q, k, v, g, beta, S0, out, S_T, out_gate, norm_weight, norm_eps, B, T, H,
                          dk, dv, opts, stream);
}

size_t kda_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, const kda_opts *opts) {
    const kda_opts o = resolve(opts);
    if (check_opts(o) != KDA_OK || check_dims(B, T, H, dk, dv) != KDA_OK) return 0;
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    return round_up(chunk_bwd_workspace_bytes(B, T, H, dk, dv), kAlignWs);
}

int kda_chunk_bwd(const void *q, const void *k, const void *v, const void *g, const void *beta,
                  const float *S0, const void *dout, const float *dS_T, float *grad_q,
                  float *grad_k, float *grad_v, float *grad_g, float *grad_beta, float *grad_S0,
                  int B, int T, int H, int dk, int dv, const kda_opts *opts, cudaStream_t stream) {
    const kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if ((s = check_dims(B, T, H, dk, dv)) != KDA_OK) return s;
    if (B == 0 || H == 0) return KDA_OK;
    if (T == 0) {   // the identity: dS0 = dS_T, nothing else to write
        if (!aligned16(dS_T) || !aligned16(grad_S0)) return KDA_ERR_ALIGN;
        if (!grad_S0) return KDA_OK;
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        cudaError_t e = dS_T ? cudaMemcpyAsync(grad_S0, dS_T, bytes, cudaMemcpyDeviceToDevice, stream)
                             : cudaMemsetAsync(grad_S0, 0, bytes, stream);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    if (!q || !k || !v || !g || !beta || !dout || !grad_q || !grad_k || !grad_v || !grad_g || !grad_beta)
        return KDA_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, dout, dS_T, grad_q, grad_k, grad_v, grad_g,
                          grad_beta, grad_S0, o.workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    const size_t need = round_up(chunk_bwd_workspace_bytes(B, T, H, dk, dv), kAlignWs);
    if (!o.workspace || o.workspace_bytes < need) return KDA_ERR_WORKSPACE;
    BwdArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.dout = dout; a.dS_T = dS_T;
    a.dq = grad_q; a.dk = grad_k; a.dv = grad_v; a.dg = grad_g; a.dbeta = grad_beta; a.dS0 = grad_S0;
    a.workspace = o.workspace;
    a.B = B; a.T = T; a.H = H; a.dk_ = dk; a.dv_ = dv;
    a.bf16 = o.dtype == KDA_BF16;
    a.fl = kflags(o);
    a.events = o.events; a.n_events = o.n_events;
    cudaError_t e = launch_chunk_bwd(a, stream);   // two launches: the sweeps, the blocks
    if (e == cudaSuccess && o.events && o.n_events > 2) cudaEventRecord(o.events[2], stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_device_status(cudaStream_t stream) {
    int f1 = 0, f2 = 0;
    if (chunk_tc_take_error(&f1, stream) != cudaSuccess) return KDA_ERR_CUDA;
    if (chunk_tc2_take_error(&f2, stream) != cudaSuccess) return KDA_ERR_CUDA;
    return (f1 || f2) ? KDA_ERR_TIMEOUT : KDA_OK;
}

unsigned kda_set_wait_limit(unsigned polls) { return set_wait_limit(polls); }

int kda_selftest_bounded_wait(unsigned limit, cudaStream_t stream) {
    int status = 0;
    if (run_bounded_wait_selftest(limit, &status, stream) != cudaSuccess) return KDA_ERR_CUDA;
    return status == 3 ? KDA_ERR_TIMEOUT : KDA_ERR_CUDA;
}

int kda_recurrent_step(const void *q, const void *k, const void *v, const void *g, const void *beta,
                       float *S, void *out, int N, int H, int dk, int dv, const kda_opts *opts,
                       cudaStream_t stream) {
    const kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if (N < 0 || H < 0 || dk <= 0 || dv <= 0) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    const long long units = (long long)N * H;
    if (units == 0) return KDA_OK;
    if (units > 0x7fffffffLL) return KDA_ERR_SHAPE;
    if (!q || !k || !v || !g || !beta || !S || !out) return KDA_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.out = out;
    a.units = units; a.dk = dk; a.dv = dv;
    a.bf16 = o.dtype == KDA_BF16;
    a.fl = kflags(o);
    if (o.events && o.n_events > 0) cudaEventRecord(o.events[0], stream);
    cudaError_t e = launch_decode(a, stream);
    if (e == cudaSuccess && o.events && o.n_events > 1) cudaEventRecord(o.events[1], stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_recurrent_step_prologue(const void *q_pre, const void *k_pre, const void *v_pre,
                                const void *conv_w, void *conv_state, const void *z, const float *A,
                                const float *beta_logit, float *S, void *out, int N, int H, int dk,
                                int dv, const kda_opts *opts, cudaStream_t stream) {
    kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if (N < 0 || H < 0 || dk <= 0 || dv <= 0) return KDA_ERR_ARG;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
    if (dk != dv || (o.flags & KDA_COMPLEX)) return KDA_ERR_UNSUPPORTED;
    const long long units = (long long)N * H;
    if (units == 0) return KDA_OK;
    if (units > 0x7fffffffLL) return KDA_ERR_SHAPE;
    if (!q_pre || !k_pre || !v_pre || !conv_w || !conv_state || !z || !A || !beta_logit || !S || !out)
        return KDA_ERR_ARG;
    const void *ptrs[] = {q_pre, k_pre, v_pre, conv_w, conv_state, z, A, beta_logit, S, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q_pre; a.k = k_pre; a.v = v_pre; a.g = z; a.S = S; a.out = out;
    a.units = units; a.dk = dk; a.dv = dv;
    a.bf16 = o.dtype == KDA_BF16;
    o.flags |= KDA_QK_L2NORM;
    a.fl = kflags(o);
    a.conv_w = conv_w; a.conv_state = conv_state; a.A = A; a.b_logit = beta_logit; a.H = H;
    a.gate_softplus = (o.flags & KDA_GATE_SOFTPLUS) ? 1 : 0;
    if (o.events && o.n_events > 0) cudaEventRecord(o.events[0], stream);
    cudaError_t e = launch_decode(a, stream);
    if (e == cudaSuccess && o.events && o.n_events > 1) cudaEventRecord(o.events[1], stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_conv_state_from_prefill(const void *q_pre, const void *k_pre, const void *v_pre,
                                void *conv_state, int B, int T, int H, int d,
                                const kda_opts *opts, cudaStream_t stream) {
    const kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_ARG;
    if (d != 64 && d != 128) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return KDA_OK;
    if ((long long)B * T * H * d > kMaxElems) return KDA_ERR_SHAPE;
    if (!conv_state || (T > 0 && (!q_pre || !k_pre || !v_pre))) return KDA_ERR_ARG;
    const void *ptrs[] = {q_pre, k_pre, v_pre, conv_state};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    cudaError_t e = launch_conv_state_from_prefill(q_pre, k_pre, v_pre, conv_state, B, T, H, d,
                                                   o.dtype == KDA_BF16, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_chunk_fwd_prologue(const void *q_pre, const void *k_pre, const void *v_pre,
                           const void *conv_w, const void *z, const float *A,
                           const float *beta_logit, const float *S0, void *out, float *S_T, int B,
                           int T, int H, int dk, int dv, const kda_opts *opts, cudaStream_t stream) {
    kda_opts o = resolve(opts);
    int s = check_opts(o);
    if (s != KDA_OK) return s;
    if ((s = check_dims(B, T, H, dk, dv)) != KDA_OK) return s;
    if (o.flags & KDA_COMPLEX) return KDA_ERR_UNSUPPORTED;
    if (dk != dv) return KDA_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return KDA_OK;
    if (T == 0) {
        if (!aligned16(S0) || !aligned16(S_T)) return KDA_ERR_ALIGN;
        return finish_identity(S0, S_T, B, H, dk, dv, stream);
    }
    if (!q_pre || !k_pre || !v_pre || !conv_w || !z || !A || !beta_logit || !out) return KDA_ERR_ARG;
    const void *ptrs[] = {q_pre, k_pre, v_pre, conv_w, z, A, beta_logit, S0, out, S_T, o.workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    size_t off[6];
    const bool tc = use_tc(o, dk, dv);
    const bool fused_pro = tc && !use_fused(o, B, H);   // split form: prologue inside its prep
    const size_t need = prologue_ws_parts(B, T, H, dk, dv, tc, tc ? tc_ws(o, B, T, H) : 0, off, fused_pro);
    if (!o.workspace || o.workspace_bytes < need) return KDA_ERR_WORKSPACE;
    char *ws = (char *)o.workspace;

    PrologueArgs p;
    p.q_pre = q_pre; p.k_pre = k_pre; p.v_pre = v_pre; p.conv_w = conv_w; p.z = z;
    p.A = A; p.beta_logit = beta_logit;
    p.bf16 = o.dtype == KDA_BF16;
    p.out_bf16 = tc;
    p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv;
    p.qc = ws + off[0]; p.kc = ws + off[1]; p.vc = ws + off[2];
    p.g = ws + off[3]; p.beta = ws + off[4];
    p.gate_softplus = (o.flags & KDA_GATE_SOFTPLUS) ? 1 : 0;

    int launches = 0;
    if (fused_pro) {
        ChunkArgs a;
        memset(&a, 0, sizeof(a));
        a.t_qkv = a.t_g = a.t_beta = a.t_out = Elt::BF16;
        a.S0 = S0; a.out = out; a.S_T = S_T;
        a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
        o.flags |= KDA_QK_L2NORM;
        a.fl = kflags(o);
        a.workspace = ws;
        a.workspace_bytes = need;
        a.exact_decay = unbounded(o);
        a.events = o.events; a.n_events = o.n_events;
        a.launch_idx = &launches;
        cudaError_t e = launch_chunk_tc2_prologue(p, a, stream);
        if (e == cudaSuccess && o.events && launches < o.n_events) cudaEventRecord(o.events[launches], stream);
        if (e == cudaErrorInvalidValue) return KDA_ERR_UNSUPPORTED;
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    if (o.events && launches < o.n_events) cudaEventRecord(o.events[launches], stream);
    ++launches;
    cudaError_t e = launch_prologue(p, stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;

    ChunkArgs a;
    memset(&a, 0, sizeof(a));
    a.q = p.qc; a.k = p.kc; a.v = p.vc; a.g = p.g; a.beta = p.beta;
    a.t_qkv = a.t_g = a.t_beta = tc ? Elt::BF16 : Elt::F32;
    a.t_out = p.bf16 ? Elt::BF16 : Elt::F32;
    a.S0 = S0; a.out = out; a.S_T = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
    o.flags |= KDA_QK_L2NORM;
    a.fl = kflags(o);
    a.workspace = ws + off[5];
    a.workspace_bytes = need - off[5];
    a.exact_decay = unbounded(o);
    a.events = o.events; a.n_events = o.n_events;
    a.launch_idx = &launches;
    e = !tc ? launch_chunk_ref(a, stream) : use_fused(o, B, H) ? launch_chunk_tc(a, stream) : launch_chunk_tc2(a, stream);
    if (e == cudaSuccess && o.events && launches < o.n_events) cudaEventRecord(o.events[launches], stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
