// kda_epilogue.cu -- the output epilogue of a KDA branch as its own pass.
//
// Page "Kimi K3 の KDA(1): KDA が Gated MLA と AttnRes とどのように連携するか", section
// 1.2.1, the full-rank output gate: o = FusedRMSNormGated(o, g) = RMSNorm(o) * sigmoid(g),
// the RMS taken per head over its head_dim values, the norm applied before the gate.
// Readings (the page gives neither): out = o / sqrt(mean(o^2) + eps) * w * sigmoid(g) with a
// weight w of head_dim values shared by the heads (NULL = ones) and eps passed by the caller.
//
// The split tensor-core form applies the same epilogue inside its scan kernel, before the
// outputs leave the chip; this pass serves the fused form and the FP32 path.  One warp per
// (token, head) row, in place on out.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {
template <typename T, int DV>
__global__ void __launch_bounds__(256)
out_epilogue_kernel(T *__restrict__ out, const T *__restrict__ gate, const float *__restrict__ w,
                    float eps, long long rows) {
    constexpr int PER = DV / 32;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    T *o = out + row * DV;
    const T *g = gate + row * DV;
    float x[PER], ss = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        x[i] = to_f32(o[lane + 32 * i]);
        ss += x[i] * x[i];
    }
    const float r = rsqrtf(warp_sum(ss) / DV + eps);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int j = lane + 32 * i;
        const float wj = w ? w[j] : 1.f;
        o[j] = from_f32<T>(x[i] * r * wj / (1.f + expf(-to_f32(g[j]))));
    }
}

template <typename T>
cudaError_t launch_t(const ChunkArgs &a, cudaStream_t st) {
    const long long rows = (long long)a.B * a.T * a.H;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
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
