// kda_epilogue.cu -- the output epilogue of a KDA branch as its own pass.
//
// Page "Kimi K3 の KDA(1): KDA が Gated MLA と AttnRes とどのように連携するか", section
// 1.2.1, the full-rank output gate: o = FusedRMSNormGated(o, g) = RMSNorm(o) * sigmoid(g),
// the RMS taken per head over its head_dim values, the norm applied before the gate.
// Readings (the page gives neither): out = o / sqrt(mean(o^2) + eps) * w * sigmoid(g) with a
// weight w of head_dim values shared by the heads (NULL = ones) and eps passed by the caller.
//
// The split tensor-core form applies the same epilogue inside its scan kernel, before the
// outputs leave the chip; this pass serves the other calls.  In place on out, DV / 8 lanes per
// (token, head) row, 8 values each.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {
// 8 consecutive values of one row per thread (16-byte bf16 / 32-byte FP32 accesses)
template <typename T>
__device__ __forceinline__ void load8(const T *p, float *x) {
    if constexpr (sizeof(T) == 2) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    } else {
        const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
}
template <typename T>
__device__ __forceinline__ void store8(T *p, const float *x) {
    if constexpr (sizeof(T) == 2) {
        uint4 u;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        *reinterpret_cast<uint4 *>(p) = u;
    } else {
        reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
}

// DV / 8 lanes per (token, head) row; the row's sum of squares is reduced over those lanes
template <typename T, int DV>
__global__ void __launch_bounds__(256)
out_epilogue_kernel(T *__restrict__ out, const T *__restrict__ gate, const float *__restrict__ w,
                    float eps, long long rows) {
    constexpr int LPR = DV / 8;
    const long long gt = (long long)blockIdx.x * 256 + threadIdx.x;
    const long long row = gt / LPR;
    const int j0 = (int)(gt % LPR) * 8;
    const bool live = row < rows;   // whole row groups of lanes share this, so the shuffles below are safe
    float x[8], g[8], ss = 0.f;
    if (live) {
        load8(out + row * DV + j0, x);
        load8(gate + row * DV + j0, g);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss += x[i] * x[i];
    }
#pragma unroll
    for (int m = LPR / 2; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    if (!live) return;
    const float r = rsqrtf(ss / DV + eps);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float wj = w ? w[j0 + i] : 1.f;
        x[i] = x[i] * r * wj / (1.f + expf(-g[i]));
    }
    store8(out + row * DV + j0, x);
}

template <typename T>
cudaError_t launch_t(const ChunkArgs &a, cudaStream_t st) {
    const long long rows = (long long)a.B * a.T * a.H;
    const unsigned blocks = (unsigned)((rows * (a.dv / 8) + 255) / 256);
    if (a.dv == 128)
        out_epilogue_kernel<T, 128><<<blocks, 256, 0, st>>>((T *)a.out, (const T *)a.out_gate, a.norm_w,
                                                            a.norm_eps, rows);
    else
        out_epilogue_kernel<T, 64><<<blocks, 256, 0, st>>>((T *)a.out, (const T *)a.out_gate, a.norm_w,
                                                           a.norm_eps, rows);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_out_epilogue(const ChunkArgs &a, cudaStream_t st) {
    mark_launch(a, st);
    return a.t_out == Elt::BF16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<float>(a, st);
}

}  // namespace kda
