// kda_chunk_tc2.cu -- the split tensor-core chunkwise KDA forward for sm_100a.
//
// The chunkwise form (page "Kimi K3 模型结构（2）：序列维度（下），chunkwise 并行与
// 下界衰减", Q&A items on the chunkwise algorithm, the -5 decay floor and the
// intra-chunk matrix A) splits into work that does not depend on the state --
// everything up to the WY vectors -- and a short state-dependent scan.
//
//   prep (kda_chunk_prep.cuh): every (chunk, head) item in parallel, two items in flight per SM;
//        writes one 74,240-byte record per item: W and Q e^gamma (one [128][128] K-major tile),
//        K e^{gamma_C - gamma}, U, A_qk (K-major [r][i]) and sigma_C e^{gamma_C} (FP32 [128]),
//        bf16 tiles already in the layouts the scan's tensor-core products read
//   scan, TMEM form (kda_chunk_scan.cuh): one CTA per sequence, the state and the chunk's
//        products in TMEM; the second launch when the sequences fill the SMs
//   scan, sliced form (below): one CTA per (sequence, value-column slice), the state in
//        registers and shared memory; beside the prep in one cooperative launch when the
//        sequences are few, and with whole-row slices when the output epilogue is fused:
//          [P ; O] = [W ; Q e^gamma] S;  V~ = U - P;  dS = Kd^T V~;  O += A_qk V~
//          S <- diag(sigma_C e^{gamma_C}) S + dS in FP32 registers
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

namespace {
using namespace sm100;

constexpr int D = 128;
constexpr int C = 64;
constexpr uint32_t kWaitLimit = 1u << 22;

// the per-(chunk, head) record written by kernel 1 and read by kernel 2
constexpr uint32_t IMG_W = 0;           // bf16 W, K-major [64 r][128 c] (with Q e^gamma: one [128][128] tile)
constexpr uint32_t IMG_QG = 16384;      // bf16 Q e^gamma, K-major [64 r][128 c]
constexpr uint32_t IMG_KD = 32768;      // bf16 K e^{gamma_C - gamma}, [64 r][128 c]
constexpr uint32_t IMG_U = 49152;       // bf16 U as eight 16-column slabs of [64 r][16 j] (2 KB each)
constexpr uint32_t IMG_AQK = 65536;     // bf16 A_qk, K-major [64 r][64 i]
constexpr uint32_t IMG_GC = 73728;      // fp32 sigma_C e^{gamma_C} [128]
constexpr uint32_t IMG_BYTES = 74240;

__device__ __forceinline__ uint32_t off_r128(int r, int c) {
    return (uint32_t)((r & 7) * 16 + (r >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 2);
}
__device__ __forceinline__ uint32_t off_r64(int r, int c) {
    return (uint32_t)((r & 7) * 16 + (r >> 3) * 1024 + (c >> 3) * 128 + (c & 7) * 2);
}
// [rows][n] bf16 tile of n columns in the no-swizzle core-matrix layout (8 rows x 16 bytes per
// core matrix, row groups n * 16 bytes apart)
__device__ __forceinline__ uint32_t off_rn(int r, int c, int n) {
    return (uint32_t)((r & 7) * 16 + (r >> 3) * (n * 16) + (c >> 3) * 128 + (c & 7) * 2);
}
// U in the record: value column j lives in slab j / 16, a [64 r][16 j] tile of its own, so any
// run of 16-column slabs (one value-column slice of the scan) is one contiguous copy
__device__ __forceinline__ uint32_t off_u(int r, int j) {
    return (uint32_t)((j >> 4) * 2048) + off_rn(r, j & 15, 16);
}
__device__ __forceinline__ int pair_of(int b, int j) { return (j == 0 ? 0 : j == 1 ? 4 : j == 2 ? 7 : 9) + b - j; }

__device__ __forceinline__ void unpack8(uint4 raw, float (&x)[8]) {
    const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
    uint4 u;
    u.x = pack_bf16(x[0], x[1]);
    u.y = pack_bf16(x[2], x[3]);
    u.z = pack_bf16(x[4], x[5]);
    u.w = pack_bf16(x[6], x[7]);
    return u;
}

__device__ int g_kda_tc2_error;   // set when a bounded wait gives up


// Inputs of the prologue fused into the prep kernel (kda_chunk_fwd_prologue on the split
// form).  conv_w == nullptr: the tiles are q, k, v, g and beta is given.
struct PrepPrologue {
    const __nv_bfloat16 *conv_w;   // [3, H * D, 4]: taps of q, k, v
    const float *A;                // [H] per-head log-scale of the gate
    const float *b_logit;          // [B, T, H] beta logits (FP32)
    // the raw branch inputs (the rows before a chunk, for its first convolution outputs)
    const __nv_bfloat16 *raw_q, *raw_k, *raw_v;
    // U in the record as 16-column slabs (the sliced scan) rather than rows like W (the TMEM scan)
    int u_slabs;
    // the gate map: Kimi Linear's g = -e^A softplus(z) instead of -5 sigmoid(e^A z)
    int softplus;
};

#include "kda_chunk_prep.cuh"

// The prep with two item groups per CTA (kda_chunk_prep.cuh): one 512-thread CTA per SM, its
// TMEM split between the groups.  MEGA: CTA `cta` of `ncta` prep CTAs of the one-launch form.
// UNB: g without the -5 floor.
template <bool PRO, bool MEGA, bool UNB>
__device__ __forceinline__ void
prep2_cta(const CUtensorMap *ptm_q, const CUtensorMap *ptm_k, const CUtensorMap *ptm_v, const CUtensorMap *ptm_g,
          const __nv_bfloat16 *beta, uint8_t *ws, int T, int H, int BH, KernelFlags fl, PrepPrologue pro,
          int cta, int ncta, int *flags, uint32_t wait_limit) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t prep_tmem_base;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        tmem_alloc(smem_u32(&prep_tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = prep_tmem_base;
    // the scan kernel, launched with a programmatic dependency on this one, may be scheduled now
    if (!MEGA) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int gi = threadIdx.x / prep2::GT;
    prep2_group<PRO, MEGA, UNB>(ptm_q, ptm_k, ptm_v, ptm_g, beta, ws, T, H, BH, fl, pro, gi,
                           smem + gi * prep2::GROUP_STRIDE, tbase + 256u * gi, prep2::NG * cta + gi,
                           prep2::NG * ncta, flags, wait_limit);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

template <bool PRO, bool UNB>
__global__ void __launch_bounds__(prep2::NT, 1)
chunk_prep2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                   const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ ws, int T, int H, int BH,
                   KernelFlags fl, PrepPrologue pro, uint32_t wait_limit) {
    prep2_cta<PRO, false, UNB>(&tm_q, &tm_k, &tm_v, &tm_g, beta, ws, T, H, BH, fl, pro, (int)blockIdx.x,
                          (int)gridDim.x, nullptr, wait_limit);
}

// ============================================================== kernel 2: the scan
// The value columns of the state evolve independently (column j of S sees only v_{t,j}), so
// the scan splits a head's dv = 128 columns into slices of NS columns, one CTA each: a slice
// runs the same dependent chain with N = NS products and 1/(128/NS) of the per-thread work,
// and few heads still fill the SMs.  One CTA per (b, h, slice).
//
// Warp roles.  4 * NS / CPT state warps: TMEM lane = key channel c for the state and = token
// row for the chunk products; thread (lane, cq) owns the FP32 state row slice
// S[c][j0 + CPT cq .. + CPT - 1] (j0 = the slice's first column).  One MMA warp issues every
// tensor-core product and keeps the record ring full, so no state thread ever waits for an
// issuing lane and the chain's hand-offs are mbarrier arrivals, not block-wide barriers.
// Per chunk ch (record in stage ch % NSTG of a ring refilled NSTG - 1 chunks ahead):
//   MMA warp:      [P ; O] = [W ; Q e^gamma] S         one M = 128, N = NS product into D[ch & 1]
//   lanes 0-63:    V~ = U - P -> bf16 shared memory, then arrive on "V~ ready"
//   lanes 64-127:  the outputs of chunk ch - 1 leave D[(ch - 1) & 1] (16-byte stores)
//   MMA warp:      dS = Kd^T V~;  O += A_qk V~           (A_qk padded with 64 zero rows to M = 128)
//   state warps:   S <- diag(sigma_C e^{gamma_C}) S + dS in FP32, its bf16 copy, then arrive
//                  on "S ready", which releases the next chunk's first product.
namespace scan {
// stage: [W;Qg] and Kd (the record's first 48 KB), the slice's U slabs, 8 KB of zeros, then
// A_qk and sigma_C e^{gamma_C}
template <int NS>
struct Layout {
    static constexpr int CPT = NS < 32 ? NS : 32;       // state columns per thread
    static constexpr int NSW = 4 * (NS / CPT);          // state warps
    static constexpr int NPW = NSW / 2;                 // of which hold rows 0-63 (P, V~)
    static constexpr int NT = 32 * NSW + 32;            // + the MMA warp
    static constexpr uint32_t HEAD = IMG_U;             // [W;Qg], Kd
    static constexpr uint32_t U = IMG_U;
    static constexpr uint32_t U_BYTES = (uint32_t)NS * 128;
    static constexpr uint32_t ZERO = U + U_BYTES;
    static constexpr uint32_t AQK = ZERO + 8192;
    static constexpr uint32_t GC = AQK + (IMG_GC - IMG_AQK);
    static constexpr uint32_t TAIL_BYTES = IMG_BYTES - IMG_AQK;   // A_qk and sigma_C e^{gamma_C}
    static constexpr uint32_t STAGE = (GC + 512 + 1023) / 1024 * 1024;
    static constexpr int NSTG = NS <= 32 ? 3 : 2;                   // record stages in the ring
    static constexpr uint32_t OFF_S = NSTG * STAGE;                 // bf16 S [128 c][NS j]
    static constexpr uint32_t OFF_VT = OFF_S + 128u * NS * 2;       // bf16 V~ [64 r][NS j]
    static constexpr uint32_t SMEM_BYTES = OFF_VT + 64u * NS * 2 + 1024;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    // TMEM columns: D0 = [P ; O] [0,NS), D1 [NS,2NS), dS [2NS,3NS)
    static constexpr uint32_t TC_D0 = 0, TC_D1 = NS, TC_S = 2 * NS;
    static constexpr uint32_t TMEM_COLS = NS == 16 ? 64 : NS == 32 ? 128 : NS == 64 ? 256 : 512;
};
}  // namespace scan

// sigmoid(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh (relative error about 2^-11, below
// the bf16 rounding of the epilogue's output)
__device__ __forceinline__ float sigmoid_tanh(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}

// barrier over `count` threads (a multiple of 32) of the CTA, id != 0 (0 is __syncthreads)
__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, float (&v)[N]) {
    if constexpr (N == 32) tmem_ld32(taddr, v);
    else tmem_ld16(taddr, v);
}

// wait until the grids this one depends on (the prep kernel) have completed and their
// memory is visible; a no-op when the launch has no programmatic dependency
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

struct alignas(8) ScanBars {
    uint64_t stage[3];
    uint64_t mV, mS, mO[2];    // tensor-core commits: [P;O], dS, O of D[0] / D[1]
    uint64_t bV, bS;           // thread arrivals: V~ ready (one per P warp), S ready (one per state warp)
    uint32_t tmem_base;
    int abort;                 // a bounded wait gave up: every other wait returns at once
    int s_done;                // MEGA: state-warp updates done (NSW per chunk)
    int o_done;                // MEGA: O products seen complete by the output warps (NSW / 2 per chunk)
    // completions issued to each barrier (stage[0..2], mV, mS, mO[0], mO[1]): each is written by
    // the one lane that issues to it, and read at exit to drain what is still in flight
    int issued[7];
};

// The scan's work for slice CTA `cta`.  MEGA (run beside the prep in one launch): each record is
// fetched only after the prep has published it (flags, chunk-major).  There the warp after the
// MMA warp issues every stage refill: it watches the flags in chunk order and two shared
// counters that tell when a stage's last readers are done, which keeps the bulk copies (and
// the stall of the warp that issues them) off the MMA warp and the chain; any further warps
// only join the block-wide barriers.
template <int NS, bool GATED, bool MEGA>
__device__ __forceinline__ void
scan_body(const uint8_t *__restrict__ ws, const float *__restrict__ S0, __nv_bfloat16 *__restrict__ out,
          float *__restrict__ S_T, int T, int H, float scale, const __nv_bfloat16 *__restrict__ gate,
          const float *__restrict__ norm_w, float norm_eps, int cta, const int *__restrict__ flags,
          int nseq, uint32_t poll_limit = kWaitLimit) {
    using L = scan::Layout<NS>;
    constexpr int CPT = L::CPT, NSL = D / NS;
    static_assert(!GATED || NS == D, "the output epilogue normalises whole rows: one slice per head");
    extern __shared__ uint8_t smem_raw[];
    __shared__ ScanBars sh;
    __shared__ float rms_part[GATED ? C * 4 : 1];   // output epilogue: per-row partial sums of squares
    __shared__ float w_s[GATED ? D : 1];            // output epilogue: the RMSNorm weight (ones if absent)
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool mma_warp = warp == L::NSW;
    const bool state_warp = warp < L::NSW;
    const bool load_warp = MEGA && warp == L::NSW + 1;   // (later warps: MEGA only, idle)
    const int quad = warp & 3, cq = warp >> 2;   // lane quadrant, column group of the slice
    const int row = quad * 32 + lane;            // TMEM lane
    const bool p_lane = row < 64;                // warp-uniform: rows of P (else of O)
    const int bh = cta / NSL, sl = cta % NSL, b = bh / H, h = bh % H;
    const int j0 = sl * NS;                      // first value column of this slice
    const int nch = (T + C - 1) / C;
    const uint8_t *recs = ws + (size_t)bh * nch * IMG_BYTES;
    const uint32_t b_mV = smem_u32(&sh.mV), b_mS = smem_u32(&sh.mS);
    const uint32_t b_bV = smem_u32(&sh.bV), b_bS = smem_u32(&sh.bS);

    if (tid == 0) {
        for (int i = 0; i < L::NSTG; ++i) mbar_init(smem_u32(&sh.stage[i]), 1);
        mbar_init(b_mV, 1);
        mbar_init(b_mS, 1);
        mbar_init(smem_u32(&sh.mO[0]), 1);
        mbar_init(smem_u32(&sh.mO[1]), 1);
        mbar_init(b_bV, L::NPW);
        mbar_init(b_bS, L::NSW);
        mbar_fence_init();
        sh.abort = 0;
        sh.s_done = 0;
        sh.o_done = 0;
        for (int i = 0; i < 7; ++i) sh.issued[i] = 0;
    }
    // the zero rows under each stage's A_qk
    for (int i = tid; i < L::NSTG * 512; i += (int)blockDim.x)
        *reinterpret_cast<uint4 *>(smem + (i >> 9) * L::STAGE + L::ZERO + (i & 511) * 16) = make_uint4(0, 0, 0, 0);
    if (warp == 0) {
        tmem_alloc(smem_u32(&sh.tmem_base), L::TMEM_COLS);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sh.tmem_base;
    const uint32_t tl = tbase + ((uint32_t)(quad * 32) << 16);
    const uint64_t dK64 = sdesc(sbase, 128, 2048, kSwizzleNone);
    const uint64_t dMN64 = sdesc(sbase, 2048, 128, kSwizzleNone);
    const uint64_t dK32 = sdesc(sbase, 128, 1024, kSwizzleNone);
    const uint64_t dMNs = sdesc(sbase, NS * 16, 128, kSwizzleNone);   // S copy and V~: [K rows][NS]
    auto at = [](uint64_t base, uint32_t off) -> uint64_t { return base + (uint64_t)(off >> 4); };
    const uint32_t a_sdone = smem_u32(&sh.s_done), a_odone = smem_u32(&sh.o_done);
    auto fetch = [&](int ch) {
        const int s = ch % L::NSTG;
        const uint32_t bar = smem_u32(&sh.stage[s]);
        ++sh.issued[s];
        const uint8_t *src = recs + (size_t)ch * IMG_BYTES;
        mbar_arrive_expect_tx(bar, L::HEAD + L::U_BYTES + L::TAIL_BYTES);
        bulk_load(sbase + s * L::STAGE, src, L::HEAD, bar);
        bulk_load(sbase + s * L::STAGE + L::U, src + IMG_U + (uint32_t)sl * L::U_BYTES, L::U_BYTES, bar);
        bulk_load(sbase + s * L::STAGE + L::AQK, src + IMG_AQK, L::TAIL_BYTES, bar);
    };
    // Bounded wait by every calling thread.  A wait that gives up raises the CTA's abort flag;
    // every wait returns false as soon as it sees the flag, so no warp is left waiting on an
    // arrival that will not come, and all warps leave their loops.
    auto wait = [&](uint32_t bar, uint32_t phase) -> bool {
        for (uint32_t i = 0; i < kWaitLimit; ++i) {
            if (mbar_try_wait(bar, phase)) return true;
            if (*reinterpret_cast<volatile int *>(&sh.abort)) return false;
            if (i > 64) __nanosleep(32);
        }
        *reinterpret_cast<volatile int *>(&sh.abort) = 1;
        g_kda_tc2_error = 1;
        return false;
    };
    // outputs of chunk c (O rows are TMEM lanes 64-127): this thread's token r, CPT values.
    // With the output epilogue (FusedRMSNormGated) the row's RMS is summed over the four warps
    // that hold its quarters (named barrier of the eight output warps), then
    // out = o / sqrt(mean(o^2) + eps) * w * sigmoid(gate) leaves the chip directly.
    if (GATED && tid < D) w_s[tid] = norm_w ? norm_w[tid] : 1.f;   // read after the next barrier
    // gate rows of the chunk the next emit stores, loaded one chunk ahead (registers)
    uint4 gpre[GATED ? CPT / 8 : 1];
    auto prefetch_gate = [&](int c) {
        const int r = row - 64, t0 = c * C;
        if (GATED && c < nch && t0 + r < T) {
            const uint4 *gsrc = reinterpret_cast<const uint4 *>(gate + (((size_t)b * T + t0 + r) * H + h) * D + 32 * cq);
#pragma unroll
            for (int m = 0; m < CPT / 8; ++m) gpre[m] = gsrc[m];
        }
    };
    auto emit = [&](int c) {
        const uint32_t dcol = ((c & 1) ? L::TC_D1 : L::TC_D0) + CPT * cq;
        const int r = row - 64, t0 = c * C;
        float o[CPT];
        __syncwarp();
        tmem_ldn<CPT>(tl + dcol, o);
#pragma unroll
        for (int e = 0; e < CPT; ++e) o[e] *= scale;
        const size_t orow = (((size_t)b * T + t0 + r) * H + h) * D + j0 + CPT * cq;
        if constexpr (GATED) {
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < CPT; ++e) ss += o[e] * o[e];
            rms_part[r * 4 + cq] = ss;
            named_bar(1, 256);
            const float rr = rsqrtf((rms_part[r * 4] + rms_part[r * 4 + 1] + rms_part[r * 4 + 2] +
                                     rms_part[r * 4 + 3]) / D + norm_eps);
            if (t0 + r < T) {
#pragma unroll
                for (int m = 0; m < CPT / 8; ++m) {
                    float gv[8];
                    unpack8(gpre[m], gv);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        o[8 * m + e] *= rr * w_s[32 * cq + 8 * m + e] * sigmoid_tanh(gv[e]);
                }
            }
            named_bar(1, 256);   // rms_part is rewritten by the next emit
        }
        if (t0 + r < T) {
            uint4 *dst = reinterpret_cast<uint4 *>(out + orow);
#pragma unroll
            for (int m = 0; m < CPT / 8; ++m) {
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = o[8 * m + e];
                dst[m] = pack8(y);
            }
        }
    };
    // FP32 state row slice S[c = row][j0 + CPT cq + e] and its bf16 copy (B operand, [c][j]
    // core layout of NS columns)
    float S[CPT];
    auto store_state_operand = [&]() {
#pragma unroll
        for (int m = 0; m < CPT / 8; ++m) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = S[8 * m + e];
            *reinterpret_cast<uint4 *>(smem + L::OFF_S + off_rn(row, CPT * cq + 8 * m, NS)) = pack8(y);
        }
        fence_proxy_async();
    };

    if (state_warp) {
        if (S0) {
            const float4 *src = reinterpret_cast<const float4 *>(S0 + ((size_t)bh * D + row) * D + j0 + CPT * cq);
#pragma unroll
            for (int m = 0; m < CPT / 4; ++m) *reinterpret_cast<float4 *>(S + 4 * m) = src[m];
        } else {
#pragma unroll
            for (int e = 0; e < CPT; ++e) S[e] = 0.f;
        }
        store_state_operand();
    }
    // everything above overlaps the end of the prep kernel; the records are read from here on
    if (!MEGA) grid_dependency_wait();
    if (!MEGA && tid == 0)
        for (int c = 0; c < L::NSTG && c < nch; ++c) fetch(c);
    tc_fence_before();
    __syncthreads();

    if (load_warp) {
        // MEGA: chunk c's record goes into stage c % NSTG once the prep has published it (item =
        // chunk * nseq + sequence) and, from c = NSTG on, once every reader of chunk c - NSTG
        // is done: the state warps' updates (sigma_C, U) and its O product (A_qk; the output
        // warps count it when they see it complete).  Counters, not barrier phases: this warp
        // may fall any number of chunks behind without mistaking a phase.
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const int *f = flags + (size_t)c * (size_t)nseq + bh;
                const int need = c - L::NSTG + 1;   // chunks whose stage must be free
                bool go = false;
                for (uint32_t i = 0; i < poll_limit; ++i) {
                    if ((need <= 0 || (smem_acquire_load(a_sdone) >= need * L::NSW &&
                                       smem_acquire_load(a_odone) >= need * L::NPW)) &&
                        flag_acquire(f)) {
                        go = true;
                        break;
                    }
                    if (*reinterpret_cast<volatile int *>(&sh.abort)) break;
                    __nanosleep(32);
                }
                if (!go) {
                    *reinterpret_cast<volatile int *>(&sh.abort) = 1;
                    g_kda_tc2_error = 1;
                    break;
                }
                fence_proxy_async_global();   // the bulk copies read what the prep wrote
                fetch(c);
            }
        }
        __syncwarp();
    } else if (mma_warp) {
        // ---- the MMA warp: every lane waits, lane 0 issues, the warp reconverges
        for (int ch = 0; ch < nch; ++ch) {
            const int s = ch & 1, sg = ch % L::NSTG;
            const uint32_t st = sg * L::STAGE;
            const uint32_t dbuf = s ? L::TC_D1 : L::TC_D0;
            if (ch > 0 && !wait(b_bS, (uint32_t)(ch - 1) & 1u)) break;            // S(ch) is in place
            if (!wait(smem_u32(&sh.stage[sg]), (uint32_t)(ch / L::NSTG) & 1u)) break;
            tc_fence_after();
            if (lane == 0) {
                constexpr uint32_t id = idesc_bf16(128, NS, 0, 1, 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ss(tbase + dbuf, at(dK64, st + 256 * k), at(dMNs, L::OFF_S + NS * 32 * k), id, k > 0);
                mma_commit(b_mV);
                ++sh.issued[3];
            }
            __syncwarp();
            // the stage of chunk ch - 1 is free once its last products are done and every state
            // thread has passed its update (S(ch) ready): refill it (MEGA: the loader warp does)
            if (!MEGA && ch >= 1 && ch - 1 + L::NSTG < nch) {
                if (!wait(smem_u32(&sh.mO[(ch - 1) & 1]), (uint32_t)((ch - 1) >> 1) & 1u)) break;
                if (lane == 0) fetch(ch - 1 + L::NSTG);
                __syncwarp();
            }
            if (!wait(b_bV, (uint32_t)ch & 1u)) break;                              // V~(ch) is in place
            tc_fence_after();
            if (lane == 0) {
                // dS = Kd^T V~ (the state's path), then O += [0 ; A_qk] V~
                constexpr uint32_t id_s = idesc_bf16(128, NS, 1, 1, 0);
                constexpr uint32_t id_o = idesc_bf16(128, NS, 0, 1, 0);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ss(tbase + L::TC_S, at(dMN64, st + IMG_KD + 4096 * k), at(dMNs, L::OFF_VT + NS * 32 * k), id_s, k > 0);
                mma_commit(b_mS);
                ++sh.issued[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ss(tbase + dbuf, at(dK32, st + L::ZERO + 256 * k), at(dMNs, L::OFF_VT + NS * 32 * k), id_o, 1);
                mma_commit(smem_u32(&sh.mO[s]));
                ++sh.issued[5 + s];
            }
            __syncwarp();
        }
    } else if (state_warp) {
        if (!p_lane) prefetch_gate(0);
        for (int ch = 0; ch < nch; ++ch) {
            const int s = ch & 1, sg = ch % L::NSTG;
            const uint32_t st = sg * L::STAGE;
            const uint32_t sbar = smem_u32(&sh.stage[sg]);
            const uint32_t sph = (uint32_t)(ch / L::NSTG) & 1u;
            const uint32_t dbuf = s ? L::TC_D1 : L::TC_D0;
            if (p_lane) {
                // V~ = U - P (this thread: token row, CPT columns of the slice)
                if (!wait(sbar, sph) || !wait(b_mV, (uint32_t)ch & 1u)) break;
                tc_fence_after();
                float p[CPT];
                __syncwarp();
                tmem_ldn<CPT>(tl + dbuf + CPT * cq, p);
#pragma unroll
                for (int m = 0; m < CPT / 8; ++m) {
                    const int jj = CPT * cq + 8 * m;   // column within the slice
                    float u[8], y[8];
                    unpack8(*reinterpret_cast<const uint4 *>(smem + st + L::U + off_u(row, jj)), u);
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = u[e] - p[8 * m + e];
                    *reinterpret_cast<uint4 *>(smem + L::OFF_VT + off_rn(row, jj, NS)) = pack8(y);
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_bV);
            } else if (ch > 0) {
                // the outputs of chunk ch - 1, while this chunk's first product runs
                const int c = ch - 1;
                if (!wait(smem_u32(&sh.mO[c & 1]), (uint32_t)(c >> 1) & 1u)) break;
                if (MEGA && lane == 0) smem_release_add(a_odone, 1);   // the O product has read A_qk
                tc_fence_after();
                emit(c);
                prefetch_gate(ch);   // consumed by the next emit (chunk ch)
            }
            // S <- diag(gC) S + dS (FP32) and its bf16 copy
            if (!wait(sbar, sph) || !wait(b_mS, (uint32_t)ch & 1u)) break;
            tc_fence_after();
            {
                const float gc = reinterpret_cast<const float *>(smem + st + L::GC)[row];
                float v[CPT];
                __syncwarp();
                tmem_ldn<CPT>(tl + L::TC_S + CPT * cq, v);
#pragma unroll
                for (int e = 0; e < CPT; ++e) S[e] = fmaf(gc, S[e], v[e]);
                store_state_operand();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(b_bS);
                if (MEGA) smem_release_add(a_sdone, 1);   // this warp is done with the stage's sigma_C
            }
        }
        if (!p_lane && nch > 0 && !*reinterpret_cast<volatile int *>(&sh.abort)) {
            const int c = nch - 1;
            if (wait(smem_u32(&sh.mO[c & 1]), (uint32_t)(c >> 1) & 1u)) {
                tc_fence_after();
                emit(c);
            }
        }
        if (S_T && !*reinterpret_cast<volatile int *>(&sh.abort)) {
            float4 *dst = reinterpret_cast<float4 *>(S_T + ((size_t)bh * D + row) * D + j0 + CPT * cq);
#pragma unroll
            for (int m = 0; m < CPT / 4; ++m) dst[m] = *reinterpret_cast<const float4 *>(S + 4 * m);
        }
    }
    tc_fence_before();
    __syncthreads();
    // drain: after a give-up, copies and products may still be in flight; let each barrier
    // reach its last issued completion (built-in limit) before TMEM and shared memory go
    if (tid == 0 && *reinterpret_cast<volatile int *>(&sh.abort)) {
        const uint32_t bars[7] = {smem_u32(&sh.stage[0]), smem_u32(&sh.stage[1]), smem_u32(&sh.stage[2]),
                                  b_mV, b_mS, smem_u32(&sh.mO[0]), smem_u32(&sh.mO[1])};
        for (int i = 0; i < 7; ++i) {
            const int k = *reinterpret_cast<volatile int *>(&sh.issued[i]);
            if (k > 0) (void)mbar_wait_bounded(bars[i], (uint32_t)(k - 1) & 1u, kWaitLimit);
        }
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, L::TMEM_COLS);
}

#include "kda_chunk_scan.cuh"

__global__ void __launch_bounds__(scan3::NT, 1)
chunk_scan3_kernel(const uint8_t *__restrict__ ws, const float *__restrict__ S0, __nv_bfloat16 *__restrict__ out,
                   float *__restrict__ S_T, int T, int H, float scale) {
    scan3_body<false>(ws, S0, out, S_T, T, H, scale, (int)blockIdx.x, nullptr, 0, kWaitLimit);
}

// The affine pair of a segment from its records (kda_segment_pair): CTAs [0, BH) run the scan
// from S0 = 0 (the final state is B), CTAs [BH, 2 BH) from S0 = I with U taken as zero (the
// final state is M); no outputs.
__global__ void __launch_bounds__(scan3::NT, 1)
chunk_scan3_pair_kernel(const uint8_t *__restrict__ ws, const float *__restrict__ eye, float *__restrict__ B_out,
                        float *__restrict__ M_out, int T, int H, int BH) {
    const int cta = (int)blockIdx.x, bh = cta % BH;
    if (cta < BH)
        scan3_body<false>(ws, nullptr, nullptr, B_out, T, H, 1.f, bh, nullptr, 0, kWaitLimit, false);
    else
        scan3_body<false>(ws, eye, nullptr, M_out, T, H, 1.f, bh, nullptr, 0, kWaitLimit, true);
}

template <int NS, bool GATED>
__global__ void __launch_bounds__(scan::Layout<NS>::NT, 1)
chunk_scan_tc_kernel(const uint8_t *__restrict__ ws, const float *__restrict__ S0,
                     __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, int T, int H,
                     float scale, const __nv_bfloat16 *__restrict__ gate,
                     const float *__restrict__ norm_w, float norm_eps) {
    scan_body<NS, GATED, false>(ws, S0, out, S_T, T, H, scale, gate, norm_w, norm_eps, (int)blockIdx.x,
                                nullptr, 0);
}

// The scan's role is kept out of line: inlined beside the prep, its code interleaves with the
// prep's, and the prep's first item, which runs from a cold instruction cache whenever the
// call's working set has left L2, takes about twice as long.
template <int NS>
__device__ __noinline__ void mega_scan(const uint8_t *ws, const float *S0, __nv_bfloat16 *out, float *S_T, int T,
                                       int H, float scale, int cta, const int *flags, int BH,
                                       uint32_t poll_limit = kWaitLimit) {
    scan_body<NS, false, true>(ws, S0, out, S_T, T, H, scale, nullptr, nullptr, 0.f, cta, flags, BH, poll_limit);
}

// The one-launch form with the two-group prep: prep CTAs are 512 threads of two item groups.
template <int NS>
constexpr uint32_t mega2_smem_bytes() {
    return prep2::SMEM_BYTES > scan::Layout<NS>::SMEM_BYTES ? prep2::SMEM_BYTES : scan::Layout<NS>::SMEM_BYTES;
}

template <bool PRO, int NS, bool UNB>
__global__ void __launch_bounds__(prep2::NT, 1)
chunk_mega2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                   const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ ws, int T, int H,
                   int BH, KernelFlags fl, PrepPrologue pro, const float *__restrict__ S0,
                   __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, int n_scan,
                   int *__restrict__ flags, uint32_t wait_limit) {
    if ((int)blockIdx.x < n_scan)
        mega_scan<NS>(ws, S0, out, S_T, T, H, fl.scale, (int)blockIdx.x, flags, BH, wait_limit);
    else
        prep2_cta<PRO, true, UNB>(&tm_q, &tm_k, &tm_v, &tm_g, beta, ws, T, H, BH, fl, pro, (int)blockIdx.x - n_scan,
                             (int)gridDim.x - n_scan, flags, wait_limit);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn2() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

bool make_map2(CUtensorMap *m, const void *ptr, int B, int T, int H, int rows = C) {
    auto enc = encode_fn2();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
}  // namespace

static int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    return n;
}

size_t chunk_tc2_workspace_bytes(int B, int T, int H) {
    const size_t nch = ((size_t)T + C - 1) / C, items = nch * (size_t)B * (size_t)H;
    return items * IMG_BYTES + (items * sizeof(int) + 255) / 256 * 256;   // records, then one flag per record
}

static cudaError_t launch_split(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                                const CUtensorMap &mv, const CUtensorMap &mg, PrepPrologue pro,
                                cudaStream_t st);

cudaError_t launch_chunk_tc2(const ChunkArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mg;
    if (!make_map2(&mq, a.q, a.B, a.T, a.H) || !make_map2(&mk, a.k, a.B, a.T, a.H) ||
        !make_map2(&mv, a.v, a.B, a.T, a.H) || !make_map2(&mg, a.g, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    return launch_split(a, mq, mk, mv, mg, PrepPrologue{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0}, st);
}

cudaError_t launch_chunk_tc2_prologue(const PrologueArgs &p, const ChunkArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mz;
    // 64-row tiles: the prep reads the three rows before a chunk from global memory
    const int rows = C;
    if (!make_map2(&mq, p.q_pre, a.B, a.T, a.H, rows) || !make_map2(&mk, p.k_pre, a.B, a.T, a.H, rows) ||
        !make_map2(&mv, p.v_pre, a.B, a.T, a.H, rows) || !make_map2(&mz, p.z, a.B, a.T, a.H, rows))
        return cudaErrorInvalidValue;
    return launch_split(a, mq, mk, mv, mz,
                        PrepPrologue{(const __nv_bfloat16 *)p.conv_w, p.A, p.beta_logit, (const __nv_bfloat16 *)p.q_pre,
                                     (const __nv_bfloat16 *)p.k_pre, (const __nv_bfloat16 *)p.v_pre, 0, p.gate_softplus},
                        st);
}

// Value-column slice width of the scan: the widest slice (fewest redundant record reads)
// whose B*H*(128/NS) CTAs still fit one wave on the SMs; the output epilogue normalises whole
// rows and keeps one slice per head.
int scan_slice_width(int BH, bool gated) {
    if (gated) return D;
    const int sms = num_sms();
    int ns = D;
    while (ns > 16 && (long long)BH * (D / (ns / 2)) <= sms) ns /= 2;
    return ns;
}

template <int NS, bool GATED>
static cudaError_t launch_scan(const ChunkArgs &a, const uint8_t *ws, cudaStream_t st) {
    using L = scan::Layout<NS>;
    auto k = chunk_scan_tc_kernel<NS, GATED>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // programmatic dependency on the prep kernel: the scan's CTAs may start (barriers, TMEM,
    // S0) on SMs the prep has left and wait in the kernel for its records
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.H * (D / NS)));
    cfg.blockDim = dim3(L::NT);
    cfg.dynamicSmemBytes = L::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, ws, a.S0, (__nv_bfloat16 *)a.out, a.S_T, a.T, a.H, a.fl.scale,
                              (const __nv_bfloat16 *)a.out_gate, a.norm_w, a.norm_eps);
}

// Per-(chunk, head) prep cost of one SM (cycles; two items in flight per SM; with the FP32
// diagonal blocks of an unbounded gate) and the per-chunk chain of the sliced scan at d = 128 on
// a B200 SM (measured).
constexpr double kPrepItemCycles = 13300.0, kPrepItemCyclesUnb = 24800.0;
static double scan_chunk_cycles(int ns) { return ns == 16 ? 2900.0 : ns == 32 ? 3000.0 : ns == 64 ? 3100.0 : 4900.0; }

// Polls of a bounded wait before it gives up (kda_set_wait_limit; failure-handling tests only).
static uint32_t g_wait_limit = kWaitLimit;

// Slice width of the one-launch form (prep and sliced-scan CTAs side by side), or 0 when the two
// launches are faster: prep on all SMs, then the TMEM scan, against the prep on the SMs the scan's
// CTAs leave, overlapped with the sliced scan, plus one item of ramp.
constexpr double kScan3ChunkCycles = 4100.0;   // the TMEM scan's chain, one CTA per sequence
int mega_slice_width(int BH, int nch, int sms, bool unb) {
    const double t_item = unb ? kPrepItemCyclesUnb : kPrepItemCycles;
    const double items = (double)BH * nch;
    const double waves = ceil((double)BH / sms);
    const double two = ceil(items / sms) * t_item + waves * nch * kScan3ChunkCycles;
    int best = 0;
    double best_t = 0.9 * two;
    for (int ns : {32, 64}) {
        const int n_scan = BH * (D / ns);
        if (n_scan > sms / 2) continue;
        const double t = fmax(ceil(items / (sms - n_scan)) * t_item, nch * scan_chunk_cycles(ns)) + t_item;
        if (t < best_t) {
            best = ns;
            best_t = t;
        }
    }
    return best;
}

cudaError_t chunk_tc2_take_error(int *flag, cudaStream_t st) {
    const int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(flag, g_kda_tc2_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_kda_tc2_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}

uint32_t set_wait_limit(uint32_t polls) {
    const uint32_t prev = g_wait_limit;
    g_wait_limit = polls;
    return prev;
}

// The one-launch form: CTAs [0, n_scan) are sliced-scan CTAs, the rest prep CTAs of two item
// groups, all resident at once (a cooperative launch; the scan CTAs wait for the records the
// prep CTAs publish).
template <bool PRO, int NS, bool UNB>
static cudaError_t launch_mega(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                               const CUtensorMap &mv, const CUtensorMap &mg, PrepPrologue pro, cudaStream_t st) {
    auto k = chunk_mega2_kernel<PRO, NS, UNB>;
    constexpr uint32_t smem = mega2_smem_bytes<NS>();
    static_assert(smem <= 232448, "shared memory budget");
    static_assert(scan::Layout<NS>::NT + 32 <= prep2::NT, "the scan's warps and the loader warp fit the prep's block");
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nch = (a.T + C - 1) / C, BH = a.B * a.H, n_scan = BH * (D / NS);
    uint8_t *ws = (uint8_t *)a.workspace;
    int *flags = reinterpret_cast<int *>(ws + (size_t)nch * BH * IMG_BYTES);
    e = cudaMemsetAsync(flags, 0, (size_t)nch * BH * sizeof(int), st);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms());
    cfg.blockDim = dim3(prep2::NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    mark_launch(a, st);
    return cudaLaunchKernelEx(&cfg, k, mq, mk, mv, mg, (const __nv_bfloat16 *)a.beta, ws, a.T, a.H, BH, a.fl, pro,
                              a.S0, (__nv_bfloat16 *)a.out, a.S_T, n_scan, flags, g_wait_limit);
}

static cudaError_t launch_scan3(const ChunkArgs &a, const uint8_t *ws, cudaStream_t st) {
    auto k = chunk_scan3_kernel;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan3::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // programmatic dependency on the prep kernel: the scan's CTAs may start (barriers, TMEM,
    // S0) on SMs the prep has left and wait in the kernel for its records
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.H));
    cfg.blockDim = dim3(scan3::NT);
    cfg.dynamicSmemBytes = scan3::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, ws, a.S0, (__nv_bfloat16 *)a.out, a.S_T, a.T, a.H, a.fl.scale);
}

// The split form: few sequences take the one-launch form with value-column slices (its chain is
// the shorter one there); otherwise the prep kernel, then the TMEM scan (one CTA per sequence),
// or with the output epilogue the sliced scan with whole-row slices (it normalises rows in its
// registers).  U's layout in the record follows the scan that reads it.  An unbounded gate
// (a.exact_decay) takes the prep with FP32 diagonal blocks; the scans are the same.
// The prep kernel over every (chunk, head) item: records into a.workspace (U as rows unless
// pro.u_slabs), unbounded prep when a.exact_decay.
static cudaError_t launch_prep2(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                                const CUtensorMap &mv, const CUtensorMap &mg, PrepPrologue pro, cudaStream_t st) {
    const bool p = pro.conv_w != nullptr, unb = a.exact_decay;
    const int nitems = ((a.T + C - 1) / C) * a.B * a.H;
    auto prep_k = p ? (unb ? chunk_prep2_kernel<true, true> : chunk_prep2_kernel<true, false>)
                    : (unb ? chunk_prep2_kernel<false, true> : chunk_prep2_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(prep_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep2::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    mark_launch(a, st);
    const int ctas = std::min((nitems + prep2::NG - 1) / prep2::NG, num_sms());
    prep_k<<<(unsigned)ctas, prep2::NT, prep2::SMEM_BYTES, st>>>(mq, mk, mv, mg, (const __nv_bfloat16 *)a.beta,
                                                                (uint8_t *)a.workspace, a.T, a.H, a.B * a.H, a.fl,
                                                                pro, g_wait_limit);
    return cudaGetLastError();
}

template <bool UNB>
static cudaError_t launch_mega_any(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                                   const CUtensorMap &mv, const CUtensorMap &mg, PrepPrologue pro, int ns,
                                   cudaStream_t st) {
    const bool p = pro.conv_w != nullptr;
    return ns == 32 ? (p ? launch_mega<true, 32, UNB>(a, mq, mk, mv, mg, pro, st)
                         : launch_mega<false, 32, UNB>(a, mq, mk, mv, mg, pro, st))
                    : (p ? launch_mega<true, 64, UNB>(a, mq, mk, mv, mg, pro, st)
                         : launch_mega<false, 64, UNB>(a, mq, mk, mv, mg, pro, st));
}

static cudaError_t launch_split(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                                const CUtensorMap &mv, const CUtensorMap &mg, PrepPrologue pro,
                                cudaStream_t st) {
    const bool p = pro.conv_w != nullptr, unb = a.exact_decay;
    const int nch = (a.T + C - 1) / C;
    if (!a.out_gate) {
        const int ns = mega_slice_width(a.B * a.H, nch, num_sms(), unb);
        if (ns) {
            pro.u_slabs = 1;
            cudaError_t e = unb ? launch_mega_any<true>(a, mq, mk, mv, mg, pro, ns, st)
                                : launch_mega_any<false>(a, mq, mk, mv, mg, pro, ns, st);
            if (e != cudaErrorCooperativeLaunchTooLarge) return e;
            (void)cudaGetLastError();   // not enough room to co-schedule: the two launches below
        }
    }
    pro.u_slabs = a.out_gate ? 1 : 0;
    cudaError_t e = launch_prep2(a, mq, mk, mv, mg, pro, st);
    if (e != cudaSuccess) return e;
    mark_launch(a, st);
    uint8_t *ws = (uint8_t *)a.workspace;
    if (a.out_gate) return launch_scan<D, true>(a, ws, st);
    return launch_scan3(a, ws, st);
}

// kda_segment_pair on the split form: the segment's records, then its two scans (B from S0 = 0,
// M from S0 = I with U taken as zero) side by side in one launch.  The records stay in the
// workspace for kda_segment_forward.
cudaError_t launch_segment_pair_tc2(const ChunkArgs &a, const float *eye, float *M_out, float *B_out,
                                    cudaStream_t st) {
    CUtensorMap mq, mk, mv, mg;
    if (!make_map2(&mq, a.q, a.B, a.T, a.H) || !make_map2(&mk, a.k, a.B, a.T, a.H) ||
        !make_map2(&mv, a.v, a.B, a.T, a.H) || !make_map2(&mg, a.g, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_prep2(a, mq, mk, mv, mg, PrepPrologue{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0}, st);
    if (e != cudaSuccess) return e;
    auto k = chunk_scan3_pair_kernel;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scan3::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * a.B * a.H));
    cfg.blockDim = dim3(scan3::NT);
    cfg.dynamicSmemBytes = scan3::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    mark_launch(a, st);
    return cudaLaunchKernelEx(&cfg, k, (const uint8_t *)a.workspace, eye, B_out, M_out, a.T, a.H, a.B * a.H);
}

// kda_segment_forward on the split form: the scan alone, from S0 over the records
// kda_segment_pair left in the workspace.
cudaError_t launch_segment_scan_tc2(const ChunkArgs &a, cudaStream_t st) {
    mark_launch(a, st);
    return launch_scan3(a, (const uint8_t *)a.workspace, st);
}

}  // namespace kda
