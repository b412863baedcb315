// kda_segment.cu -- affine pairs of sequence segments, for splitting one long sequence
// over several GPUs (context parallelism over T).
//
// Page "Kimi K3 の KDA(1)", section 2.3 (the algebraic view of the recurrence): a token
// acts on the state by the affine map S -> T_t S + beta_t k_t v_t^T with
// T_t = (I - beta_t k_t k_t^T) Diag(alpha_t); a segment of tokens composes to one pair
// (M, B), S -> M S + B, and pairs compose in order (a monoid), so the state at the start
// of any segment follows from the pairs of the segments before it.
//
//  * identity_kernel fills the identity start state used to obtain M: M is the segment's
//    final state from S0 = I with v = 0 (the state's columns evolve independently, so
//    column i of the result is M e_i).  B is the final state from S0 = 0 with the real v.
//    Both runs are the chunk forward itself (kda_abi.cu).
//  * affine_combine_kernel folds pairs onto a start state: S <- M_r S + B_r, r = 0..n-1.
//    One CTA per (sequence, 32 value columns): its slice of S stays in shared memory
//    (double-buffered); thread = (value column, 16 key rows); rows of M_r are read by the
//    whole warp at once (a broadcast).  n is small (the number of segments), so this is a
//    few 128^3 products per sequence.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

__global__ void __launch_bounds__(256)
identity_kernel(float *__restrict__ S, long long total, int d) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const long long e = idx % ((long long)d * d);
    S[idx] = (e / d == e % d) ? 1.f : 0.f;
}

constexpr int CW = 32;    // value columns per CTA

template <int DK>
__global__ void __launch_bounds__(256)
affine_combine_kernel(const float *__restrict__ M, const float *__restrict__ Bp, int n,
                      const float *__restrict__ S0, float *__restrict__ S_out, int BH, int dv) {
    constexpr int RPT = DK / 8;              // key rows per thread (8 warps)
    __shared__ float sb[2][DK][CW];
    const int bh = blockIdx.x, j0 = blockIdx.y * CW;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const size_t sbase = (size_t)bh * DK * dv;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = w + 8 * m;
        sb[0][i][lane] = S0 ? S0[sbase + (size_t)i * dv + j0 + lane] : 0.f;
    }
    __syncthreads();
    int cur = 0;
    for (int r = 0; r < n; ++r) {
        const float *Mr = M + ((size_t)r * BH + bh) * DK * DK;
        const float *Br = Bp + ((size_t)r * BH + bh) * DK * dv;
        float acc[RPT];
#pragma unroll
        for (int m = 0; m < RPT; ++m) acc[m] = Br[(size_t)(w + 8 * m) * dv + j0 + lane];
        for (int c = 0; c < DK; ++c) {
            const float s = sb[cur][c][lane];
#pragma unroll
            for (int m = 0; m < RPT; ++m) acc[m] = fmaf(__ldg(&Mr[(size_t)(w + 8 * m) * DK + c]), s, acc[m]);
        }
#pragma unroll
        for (int m = 0; m < RPT; ++m) sb[cur ^ 1][w + 8 * m][lane] = acc[m];
        cur ^= 1;
        __syncthreads();
    }
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = w + 8 * m;
        S_out[sbase + (size_t)i * dv + j0 + lane] = sb[cur][i][lane];
    }
}

}  // namespace

cudaError_t launch_identity(float *S, long long count, int d, cudaStream_t st) {
    const long long total = count * d * d;
    if (total == 0) return cudaSuccess;
    identity_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(S, total, d);
    return cudaGetLastError();
}

cudaError_t launch_affine_combine(const float *M, const float *Bp, int n, const float *S0, float *S_out,
                                  int BH, int dk, int dv, cudaStream_t st) {
    const dim3 grid((unsigned)BH, (unsigned)(dv / CW));
    if (dk == 128)
        affine_combine_kernel<128><<<grid, 256, 0, st>>>(M, Bp, n, S0, S_out, BH, dv);
    else
        affine_combine_kernel<64><<<grid, 256, 0, st>>>(M, Bp, n, S0, S_out, BH, dv);
    return cudaGetLastError();
}

}  // namespace kda
