// kda_common.cuh -- small device helpers shared by the KDA kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr float kL2Eps = 1e-6f;   // epsilon inside the square root of the L2 norm
constexpr int kChunk = 64;        // chunk length C

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Activations of the bf16 prologue (standalone and fused into the split form's prep):
// __expf and a hardware reciprocal (x * rcp(1 + e^-x)).  Both errors are a few ulp, far below
// the bf16 rounding of the outputs; for x -> -inf the reciprocal of inf is 0, so the limits
// stay exact (sigmoid -> 0, SiLU -> -0).
// sigmoid(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh: one special-function operation
// (the exp + reciprocal form takes two), absolute error about 2^-12, below the bf16 rounding
// of the prologue's outputs; SiLU(x) = x sigmoid(x)
__device__ __forceinline__ float sigmoid_fast(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}
__device__ __forceinline__ float silu_fast(float x) { return x * sigmoid_fast(x); }

// Options the kernels see (a device-side copy of the host flags).
struct KernelFlags {
    int l2norm;
    int complex_gate;
    float scale;
};

}  // namespace kda
