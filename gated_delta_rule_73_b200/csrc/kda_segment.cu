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
//    One CTA per (sequence, 16 value columns): its slice of S stays in shared memory
//    (double-buffered); each M_r is staged transposed in shared memory by coalesced reads,
//    the next one loaded into registers while the current products run; thread = 4 (or 2)
//    key rows x 2 value columns.
//    n is small (the number of segments), so this is a few 128^3 products per sequence.
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

constexpr int CW = 16;    // value columns per CTA
constexpr int CPT = 2;    // value columns per thread

// Shared memory of one fold CTA: M_r transposed ([c][i], rows padded to keep float4 reads
// aligned and the transposing writes at most 4-way conflicted) and the state slice, twice.
template <int DK>
struct FoldSmem {
    static constexpr int MP = DK + 4;
    float mt[DK][MP];
    float sb[2][DK][CW];
};

template <int DK>
__global__ void __launch_bounds__(256)
affine_combine_kernel(const float *__restrict__ M, const float *__restrict__ Bp, int n,
                      const float *__restrict__ S0, float *__restrict__ S_out, int BH, int dv) {
    // thread = RPT x 2 tile: key rows RPT rg .. RPT rg + RPT - 1, value columns 2 cg, 2 cg + 1
    constexpr int MP = FoldSmem<DK>::MP;
    constexpr int RPT = DK / 32;             // rows per thread: 4 (DK = 128) or 2 (DK = 64)
    constexpr int NM = DK * DK / 256;        // elements of M_r per thread
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FoldSmem<DK> &sm = *reinterpret_cast<FoldSmem<DK> *>(smem_raw);
    const int bh = blockIdx.x, j0 = blockIdx.y * CW;
    const int tid = threadIdx.x, rg = tid >> 3, cg = tid & 7;
    const int i0 = RPT * rg, c2 = CPT * cg;
    const size_t sbase = (size_t)bh * DK * dv;
    // every load of a staging loop is issued before its first shared store (unrolled), and the
    // next pair's M is loaded while this pair's products run: the load latency is paid once
#pragma unroll
    for (int idx = tid; idx < DK * CW; idx += 256) {
        const int i = idx / CW, j = idx % CW;
        sm.sb[0][i][j] = S0 ? S0[sbase + (size_t)i * dv + j0 + j] : 0.f;
    }
    float mreg[NM];
    if (n > 0) {
        const float *M0 = M + (size_t)bh * DK * DK;
#pragma unroll
        for (int u = 0; u < NM; ++u) mreg[u] = M0[tid + 256 * u];   // coalesced rows
    }
    int cur = 0;
    for (int r = 0; r < n; ++r) {
        const float *Br = Bp + ((size_t)r * BH + bh) * DK * dv;
        __syncthreads();   // the previous step's reads of mt are done
#pragma unroll
        for (int u = 0; u < NM; ++u) {
            const int idx = tid + 256 * u, i = idx / DK, c = idx % DK;
            sm.mt[c][i] = mreg[u];
        }
        __syncthreads();
        if (r + 1 < n) {   // the next pair's M, in flight during this pair's products
            const float *Mn = M + ((size_t)(r + 1) * BH + bh) * DK * DK;
#pragma unroll
            for (int u = 0; u < NM; ++u) mreg[u] = Mn[tid + 256 * u];
        }
        float acc[RPT][CPT];
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float2 b2 = *reinterpret_cast<const float2 *>(&Br[(size_t)(i0 + m) * dv + j0 + c2]);
            acc[m][0] = b2.x; acc[m][1] = b2.y;
        }
#pragma unroll 8
        for (int c = 0; c < DK; ++c) {
            const float2 s2 = *reinterpret_cast<const float2 *>(&sm.sb[cur][c][c2]);
            float mv[RPT];
            if constexpr (RPT == 4) {
                const float4 m4 = *reinterpret_cast<const float4 *>(&sm.mt[c][i0]);
                mv[0] = m4.x; mv[1] = m4.y; mv[2] = m4.z; mv[3] = m4.w;
            } else {
                const float2 m2 = *reinterpret_cast<const float2 *>(&sm.mt[c][i0]);
                mv[0] = m2.x; mv[1] = m2.y;
            }
#pragma unroll
            for (int m = 0; m < RPT; ++m) {
                acc[m][0] = fmaf(mv[m], s2.x, acc[m][0]);
                acc[m][1] = fmaf(mv[m], s2.y, acc[m][1]);
            }
        }
#pragma unroll
        for (int m = 0; m < RPT; ++m)
            *reinterpret_cast<float2 *>(&sm.sb[cur ^ 1][i0 + m][c2]) = make_float2(acc[m][0], acc[m][1]);
        cur ^= 1;
    }
    __syncthreads();
#pragma unroll
    for (int idx = tid; idx < DK * CW; idx += 256) {
        const int i = idx / CW, j = idx % CW;
        S_out[sbase + (size_t)i * dv + j0 + j] = sm.sb[cur][i][j];
    }
}

}  // namespace

cudaError_t launch_identity(float *S, long long count, int d, cudaStream_t st) {
    const long long total = count * d * d;
    if (total == 0) return cudaSuccess;
    identity_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(S, total, d);
    return cudaGetLastError();
}

template <int DK>
static cudaError_t launch_fold(const float *M, const float *Bp, int n, const float *S0, float *S_out,
                               int BH, int dv, cudaStream_t st) {
    const size_t smem = sizeof(FoldSmem<DK>);
    cudaError_t e = cudaFuncSetAttribute(affine_combine_kernel<DK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)BH, (unsigned)(dv / CW));
    affine_combine_kernel<DK><<<grid, 256, smem, st>>>(M, Bp, n, S0, S_out, BH, dv);
    return cudaGetLastError();
}

cudaError_t launch_affine_combine(const float *M, const float *Bp, int n, const float *S0, float *S_out,
                                  int BH, int dk, int dv, cudaStream_t st) {
    return dk == 128 ? launch_fold<128>(M, Bp, n, S0, S_out, BH, dv, st)
                     : launch_fold<64>(M, Bp, n, S0, S_out, BH, dv, st);
}

}  // namespace kda
