// kda_prologue.cu -- branch prologue of a KDA layer, ahead of the chunk kernel.
//
// Page "Kimi K3 の KDA(1): KDA が Gated MLA と AttnRes とどのように連携するか",
// section 1.2.1:
//   * q, k, v: ShortConvolution(kernel_size=4, activation='silu') -- causal,
//     depthwise (every channel independent), the current token and the three
//     before it, then SiLU.  Tap order of a causal Conv1d weight [channels, 4]:
//     y_t = sum_j w[c, j] x_{t-3+j} (tap 3 multiplies the current token), zero
//     history before t = 0, no bias.
//   * beta = sigmoid(b) per head, in FP32 (b_proj(...).float()).
// Page "Kimi K3 模型结构（2）", Q&A on the decay function: the bounded log-decay
// g = -5 * sigmoid(exp(A_h) * z), g in (-5, 0); with gate_softplus the Kimi Linear map the
// same Q&A item contrasts it with, g = -exp(A_h) * softplus(z), g in (-inf, 0).
//
// Outputs are bf16 when the tensor-core chunk kernel follows (its operands are
// bf16 anyway) and FP32 for the FP32 chunk path; the L2 norm of q and k is
// applied by the chunk kernel.  The bf16 -> bf16 case has a vectorised kernel
// (8 channels x a run of tokens per thread); the others use the one-element kernel.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {
__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + expf(-x)); }
// softplus(x) = log(1 + e^x) = max(x, 0) + log1p(e^-|x|): no overflow for large x, and
// log1p keeps the tail e^x accurate for very negative x
__device__ __forceinline__ float softplus(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

template <typename T, typename TO>
__global__ void __launch_bounds__(256)
prologue_kernel(const T *__restrict__ q_pre, const T *__restrict__ k_pre,
                const T *__restrict__ v_pre, const T *__restrict__ conv_w,
                const T *__restrict__ z, const float *__restrict__ A,
                const float *__restrict__ b_logit, int T_, int H, int D, long long total,
                TO *__restrict__ qc, TO *__restrict__ kc, TO *__restrict__ vc,
                TO *__restrict__ g, TO *__restrict__ beta, int gate_softplus) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int d = (int)(idx % D);
    const long long bth = idx / D;               // (b * T + t) * H + h
    const int h = (int)(bth % H);
    const int t = (int)((bth / H) % T_);
    const long long HD = (long long)H * D;
    const long long nch = HD;                    // channels per branch
    const long long ch = (long long)h * D + d;
    const T *src[3] = {q_pre, k_pre, v_pre};
    TO *dst[3] = {qc, kc, vc};
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        const T *w = conv_w + ((long long)s * nch + ch) * 4;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int tt = t - 3 + j;
            if (tt >= 0) acc += to_f32(w[j]) * to_f32(src[s][idx - (long long)(3 - j) * HD]);
        }
        dst[s][idx] = from_f32<TO>(acc * sigm(acc));
    }
    const float zv = to_f32(z[idx]);
    g[idx] = from_f32<TO>(gate_softplus ? -expf(A[h]) * softplus(zv) : -5.f * sigm(expf(A[h]) * zv));
    if (d == 0) beta[bth] = from_f32<TO>(sigm(b_logit[bth]));
}

// bf16 in, bf16 out (the tensor-core path): thread = 8 consecutive channels of one head
// over a run of RUN tokens.  The three previous input rows of each branch stay in
// registers as the window slides, so every input row is read once per run (plus a
// three-row halo); loads and stores are 16 bytes.
constexpr int RUN = 16;

__device__ __forceinline__ void ld8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h2[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void st8(__nv_bfloat16 *p, const float (&x)[8]) {
    uint4 raw;
    __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h2[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    *reinterpret_cast<uint4 *>(p) = raw;
}

__global__ void __launch_bounds__(256)
prologue_bf16_kernel(const __nv_bfloat16 *__restrict__ q_pre, const __nv_bfloat16 *__restrict__ k_pre,
                     const __nv_bfloat16 *__restrict__ v_pre, const __nv_bfloat16 *__restrict__ conv_w,
                     const __nv_bfloat16 *__restrict__ z, const float *__restrict__ A,
                     const float *__restrict__ b_logit, int T_, int H, int D, int nruns,
                     long long total, __nv_bfloat16 *__restrict__ qc, __nv_bfloat16 *__restrict__ kc,
                     __nv_bfloat16 *__restrict__ vc, __nv_bfloat16 *__restrict__ g,
                     __nv_bfloat16 *__restrict__ beta) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int HD = H * D, ngroups = HD / 8;
    const int cgrp = (int)(idx % ngroups);
    const long long rest = idx / ngroups;
    const int run = (int)(rest % nruns), b = (int)(rest / nruns);
    const int ch0 = cgrp * 8, h = ch0 / D;
    const int t0 = run * RUN, t1 = min(T_, t0 + RUN);
    const long long rowstride = HD;
    const long long base = ((long long)b * T_) * HD + ch0;
    // one branch at a time keeps only its taps and window live
#pragma unroll 1
    for (int s = 0; s < 3; ++s) {
        const __nv_bfloat16 *src = s == 0 ? q_pre : s == 1 ? k_pre : v_pre;
        __nv_bfloat16 *dst = s == 0 ? qc : s == 1 ? kc : vc;
        float w[4][8];   // [tap][channel]
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float x8[8];   // channels 2m, 2m+1, taps 0-3 each
            ld8(conv_w + ((long long)s * HD + ch0) * 4 + 8 * m, x8);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                w[j][2 * m] = x8[j];
                w[j][2 * m + 1] = x8[4 + j];
            }
        }
        float win[3][8];   // x_{t-3}, x_{t-2}, x_{t-1}
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int tt = t0 - 3 + j;
            if (tt >= 0) {
                ld8(src + base + tt * rowstride, win[j]);
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c) win[j][c] = 0.f;
            }
        }
        // four rows are loaded before any is used, so each thread keeps four loads in flight
        for (int tb = t0; tb < t1; tb += 4) {
            float x[4][8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (tb + i < t1) {
                    ld8(src + base + (tb + i) * rowstride, x[i]);
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) x[i][c] = 0.f;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float y[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float acc = w[0][c] * win[0][c] + w[1][c] * win[1][c] + w[2][c] * win[2][c] +
                                      w[3][c] * x[i][c];
                    y[c] = silu_fast(acc);
                    win[0][c] = win[1][c];
                    win[1][c] = win[2][c];
                    win[2][c] = x[i][c];
                }
                if (tb + i < t1) st8(dst + base + (tb + i) * rowstride, y);
            }
        }
    }
    const float ea = expf(A[h]);
    for (int tb = t0; tb < t1; tb += 4) {
        float zz[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (tb + i < t1) ld8(z + base + (tb + i) * rowstride, zz[i]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (tb + i >= t1) break;
            float gg[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) gg[c] = -5.f * sigmoid_fast(ea * zz[i][c]);
            st8(g + base + (tb + i) * rowstride, gg);
            if (ch0 % D == 0) {
                const long long bth = ((long long)b * T_ + tb + i) * H + h;
                beta[bth] = __float2bfloat16_rn(sigmoid_fast(b_logit[bth]));
            }
        }
    }
}
}  // namespace

// conv_state[b][branch][j][c] = raw input of that branch at token T - 3 + j (zero before t = 0):
// the three inputs the next token's short convolution reads.
template <typename T>
__global__ void __launch_bounds__(256)
conv_state_kernel(const T *__restrict__ q_pre, const T *__restrict__ k_pre, const T *__restrict__ v_pre,
                  T *__restrict__ cs, int T_, long long HD, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long c = idx % HD, r = idx / HD;   // r = (b * 3 + branch) * 3 + j
    const int j = (int)(r % 3), br = (int)((r / 3) % 3);
    const long long b = r / 9;
    const int t = T_ - 3 + j;
    const T *src = br == 0 ? q_pre : br == 1 ? k_pre : v_pre;
    cs[idx] = t >= 0 ? src[(b * T_ + t) * HD + c] : from_f32<T>(0.f);
}

template <typename T, typename TO>
static void launch_t(const PrologueArgs &a, long long total, unsigned blocks, cudaStream_t st) {
    prologue_kernel<T, TO><<<blocks, 256, 0, st>>>(
        (const T *)a.q_pre, (const T *)a.k_pre, (const T *)a.v_pre, (const T *)a.conv_w,
        (const T *)a.z, a.A, a.beta_logit, a.T, a.H, a.dk, total, (TO *)a.qc, (TO *)a.kc,
        (TO *)a.vc, (TO *)a.g, (TO *)a.beta, a.gate_softplus);
}

cudaError_t launch_conv_state_from_prefill(const void *q_pre, const void *k_pre, const void *v_pre,
                                           void *conv_state, int B, int T, int H, int d, bool bf16,
                                           cudaStream_t st) {
    const long long HD = (long long)H * d, total = (long long)B * 9 * HD;
    const unsigned blocks = (unsigned)((total + 255) / 256);
    if (bf16)
        conv_state_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)q_pre, (const __nv_bfloat16 *)k_pre, (const __nv_bfloat16 *)v_pre,
            (__nv_bfloat16 *)conv_state, T, HD, total);
    else
        conv_state_kernel<float><<<blocks, 256, 0, st>>>((const float *)q_pre, (const float *)k_pre,
                                                         (const float *)v_pre, (float *)conv_state, T,
                                                         HD, total);
    return cudaGetLastError();
}

cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t st) {
    if (a.bf16 && a.out_bf16 && a.dk % 8 == 0 && !a.gate_softplus) {
        const int nruns = (a.T + RUN - 1) / RUN;
        const long long total = (long long)a.B * nruns * (a.H * a.dk / 8);
        prologue_bf16_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
            (const __nv_bfloat16 *)a.q_pre, (const __nv_bfloat16 *)a.k_pre, (const __nv_bfloat16 *)a.v_pre,
            (const __nv_bfloat16 *)a.conv_w, (const __nv_bfloat16 *)a.z, a.A, a.beta_logit, a.T, a.H,
            a.dk, nruns, total, (__nv_bfloat16 *)a.qc, (__nv_bfloat16 *)a.kc, (__nv_bfloat16 *)a.vc,
            (__nv_bfloat16 *)a.g, (__nv_bfloat16 *)a.beta);
        return cudaGetLastError();
    }
    const long long total = (long long)a.B * a.T * a.H * a.dk;
    const unsigned blocks = (unsigned)((total + 255) / 256);
    if (a.bf16 && a.out_bf16) launch_t<__nv_bfloat16, __nv_bfloat16>(a, total, blocks, st);
    else if (a.bf16) launch_t<__nv_bfloat16, float>(a, total, blocks, st);
    else if (a.out_bf16) launch_t<float, __nv_bfloat16>(a, total, blocks, st);
    else launch_t<float, float>(a, total, blocks, st);
    return cudaGetLastError();
}

}  // namespace kda
