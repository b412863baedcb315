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
// g = -5 * sigmoid(exp(A_h) * z), g in (-5, 0).
//
// Outputs are bf16 when the tensor-core chunk kernel follows (its operands are
// bf16 anyway) and FP32 for the FP32 chunk path; the L2 norm of q and k is
// applied by the chunk kernel.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {
__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + expf(-x)); }

template <typename T, typename TO>
__global__ void __launch_bounds__(256)
prologue_kernel(const T *__restrict__ q_pre, const T *__restrict__ k_pre,
                const T *__restrict__ v_pre, const T *__restrict__ conv_w,
                const T *__restrict__ z, const float *__restrict__ A,
                const float *__restrict__ b_logit, int T_, int H, int D, long long total,
                TO *__restrict__ qc, TO *__restrict__ kc, TO *__restrict__ vc,
                TO *__restrict__ g, TO *__restrict__ beta) {
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
    g[idx] = from_f32<TO>(-5.f * sigm(expf(A[h]) * to_f32(z[idx])));
    if (d == 0) beta[bth] = from_f32<TO>(sigm(b_logit[bth]));
}
}  // namespace

template <typename T, typename TO>
static void launch_t(const PrologueArgs &a, long long total, unsigned blocks, cudaStream_t st) {
    prologue_kernel<T, TO><<<blocks, 256, 0, st>>>(
        (const T *)a.q_pre, (const T *)a.k_pre, (const T *)a.v_pre, (const T *)a.conv_w,
        (const T *)a.z, a.A, a.beta_logit, a.T, a.H, a.dk, total, (TO *)a.qc, (TO *)a.kc,
        (TO *)a.vc, (TO *)a.g, (TO *)a.beta);
}

cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t st) {
    const long long total = (long long)a.B * a.T * a.H * a.dk;
    const unsigned blocks = (unsigned)((total + 255) / 256);
    if (a.bf16 && a.out_bf16) launch_t<__nv_bfloat16, __nv_bfloat16>(a, total, blocks, st);
    else if (a.bf16) launch_t<__nv_bfloat16, float>(a, total, blocks, st);
    else if (a.out_bf16) launch_t<float, __nv_bfloat16>(a, total, blocks, st);
    else launch_t<float, float>(a, total, blocks, st);
    return cudaGetLastError();
}

}  // namespace kda
