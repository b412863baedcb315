// kda_selftest.cu -- the bounded waits' give-up path, exercised on the GPU.
//
// The tensor-core kernels wait only through bounded loops: mbar_wait_bounded on mbarriers
// of their own CTA, and polls of release/acquire flags between CTAs of one launch.  When a
// wait runs out it sets an error word and the kernel returns, leaving the context usable.
// This self-test drives both forms into giving up on purpose, with nothing that can arrive:
// an mbarrier that expects one arrival nobody makes, and a device flag nobody writes.  It
// faults nothing and cannot hang: each loop runs at most `limit` polls.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

namespace {
using namespace sm100;

__device__ int g_selftest_flag;      // never written: the flag no producer publishes
__device__ int g_selftest_status;    // bit 0: the mbarrier wait gave up; bit 1: the flag poll

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(uint32_t limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        mbar_fence_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        int status = 0;
        if (!mbar_wait_bounded(smem_u32(&bar), 0u, limit)) status |= 1;
        bool seen = false;
        for (uint32_t i = 0; i < limit && !seen; ++i) seen = flag_acquire(&g_selftest_flag) != 0;
        if (!seen) status |= 2;
        g_selftest_status = status;
    }
}
}  // namespace

cudaError_t run_bounded_wait_selftest(unsigned limit, int *status, cudaStream_t st) {
    const int zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_selftest_status, &zero, sizeof(int), 0,
                                            cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return e;
    bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(limit);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaMemcpyFromSymbolAsync(status, g_selftest_status, sizeof(int), 0,
                                       cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return e;
    return cudaStreamSynchronize(st);
}

}  // namespace kda
