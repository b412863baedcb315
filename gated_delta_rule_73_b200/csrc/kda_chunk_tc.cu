// kda_chunk_tc.cu -- fused tensor-core chunkwise KDA forward for sm_100a.
//
// One CTA owns one (b, h) sequence and walks its 64-token chunks in order,
// keeping the FP32 state on chip for the whole scan: nothing but the inputs,
// the outputs, S0 and S_T touches HBM.  Per chunk (page "Kimi K3 模型结构（2）：
// 序列维度（下），chunkwise 并行与下界衰减", Q&A items on the chunkwise algorithm,
// on the -5 decay floor and on the intra-chunk matrix A):
//
//   TMA      q, k, v, g tiles [64 tokens x 128] (bf16, 128-byte swizzle), the
//            next chunk's tiles in flight while this chunk's scan runs
//   CUDA     gamma = chunk-local cumsum of log|alpha| per key channel; band
//   cores    references p_j = gamma just before 16-token band j; per row the
//            factor E = e^{gamma_r - p_band(r)} in [e^-80, 1] (bounded decay)
//   tcgen05  A_qk / A_kk sub-tiles: for column band j, D[:, 16j..] =
//            [Q e^{gamma - p_j}; beta K e^{gamma - p_j}] (A in TMEM) x
//            (K e^{p_j - gamma})^T -- every factor stays inside the bf16 range
//            because a band spans 16 tokens and g > -5 (cumulative >= -80)
//   CUDA     Tm = (I + A_kk)^{-1} (UT transform) in FP32, 16x16 blocks
//   tcgen05  W^T = (K e^gamma)^T Tm'^T,  U^T = V^T Tm'^T   (Tm' = Tm diag(beta))
//   tcgen05  V~^T = U^T - S^T W^T,  O^T = S^T (Q e^gamma)^T
//   tcgen05  O^T += V~^T A_qk^T,  dS = (K e^{gamma_C - gamma})^T V~
//   CUDA     O -> bf16 -> HBM;  S <- diag(sigma_C e^{gamma_C}) S + dS (FP32, registers)
//
// Every matrix product runs with M = 128 (the 128 lanes of TMEM) by putting
// the 128-wide head dimension on M and the 64 tokens on N or K.  Complex-KDA
// (signed gate) folds the sign parity sigma_r = prod_{s<=r} sign(alpha_s) into
// q and k, and sigma_C into the state update.
//
// Requirements checked by the host: bf16 activations, dk = dv = 128, 16-byte
// aligned pointers.  The bounded decay g >= -5 (|alpha| >= e^-5 for
// Complex-KDA) is what keeps every band factor finite; larger decays lose
// accuracy on this path (the FP32 path has no such limit).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {

namespace {
using namespace sm100;

constexpr int D = 128;          // dk = dv
constexpr int C = 64;           // chunk
constexpr int NT = 256;         // threads
constexpr uint32_t kTmaBytes = 4u * C * D * 2u;   // q, k, v, g tiles per chunk

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_STG_Q = 0;
constexpr uint32_t OFF_STG_K = 16384;
constexpr uint32_t OFF_STG_V = 32768;
constexpr uint32_t OFF_STG_G = 49152;
constexpr uint32_t OFF_GAM = 65536;           // fp32 gamma [64][132]; later AKK/TMF/RS; later VT
constexpr uint32_t GAM_STRIDE = 132;          // floats per row (conflict-free 16-byte row reads)
constexpr uint32_t OFF_AKK = OFF_GAM;         // fp32 [64][65]
constexpr uint32_t OFF_TMF = OFF_GAM + 16640; // fp32 [64][65]
constexpr uint32_t OFF_RS = OFF_GAM + 33280;  // fp32 [3][16][17]
constexpr uint32_t OFF_VT = OFF_GAM;          // bf16 V~^T, K-major [128 j][64 r]
constexpr uint32_t OFF_QG = OFF_GAM + 36864;  // bf16 Q e^gamma, [64 r][128 c]
constexpr uint32_t OFF_XR = OFF_QG + 16384;   // bf16 K e^{p-gamma} [64][128]; later A_qk + Tm'
constexpr uint32_t OFF_AQK = OFF_XR;          // bf16 [64 r][64 i]
constexpr uint32_t OFF_TMB = OFF_XR + 8192;   // bf16 [64 r][64 i]
constexpr uint32_t OFF_YR = OFF_XR + 16384;   // bf16 K e^gamma [64][128]; later W^T [128][64]
constexpr uint32_t OFF_KD = OFF_YR + 16384;   // bf16 K e^{gamma_C-gamma} [64][128]
constexpr uint32_t OFF_SB = OFF_KD + 16384;   // bf16 S [128 c][128 j]
constexpr uint32_t OFF_TAB = OFF_SB + 32768;  // fp32 tables
constexpr uint32_t TAB_P = 0;                 // [4][128]
constexpr uint32_t TAB_F = TAB_P + 2048;      // [4][4][128]
constexpr uint32_t TAB_G = TAB_F + 8192;      // [4][128]
constexpr uint32_t TAB_H = TAB_G + 2048;      // [4][128]
constexpr uint32_t TAB_GC = TAB_H + 2048;     // [128]
constexpr uint32_t TAB_NRM = TAB_GC + 512;    // [128]
constexpr uint32_t TAB_BET = TAB_NRM + 512;   // [64]
constexpr uint32_t TAB_SGN = TAB_BET + 256;   // uint32 [64][4]
constexpr uint32_t TAB_SGNC = TAB_SGN + 1024; // uint32 [4]
constexpr uint32_t TAB_BYTES = TAB_SGNC + 256;
constexpr uint32_t SMEM_USED = OFF_TAB + TAB_BYTES;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // slack for the 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (512 allocated)
constexpr uint32_t TC_AOP = 0;     // A operands of the A_qk/A_kk products: band j at 64 j
constexpr uint32_t TC_S = 0;       // dS accumulator (after the band products)
constexpr uint32_t TC_O = 128;     // O^T
constexpr uint32_t TC_A = 256;     // A_qk (lanes 0-63) / A_kk (lanes 64-127)
constexpr uint32_t TC_W = 320;     // W^T
constexpr uint32_t TC_U = 384;     // U^T, then V~^T

constexpr uint32_t kWaitLimit = 1u << 22;

// byte offset of (row, col) in a [rows][128] bf16 tile written as 8x8 core
// matrices (8 rows x 16 bytes): row groups at 2048 B, column groups at 128 B.
__device__ __forceinline__ uint32_t off_r128(int r, int c) {
    return (uint32_t)((r & 7) * 16 + (r >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 2);
}
// same for [rows][64] tiles: row groups at 1024 B
__device__ __forceinline__ uint32_t off_r64(int r, int c) {
    return (uint32_t)((r & 7) * 16 + (r >> 3) * 1024 + (c >> 3) * 128 + (c & 7) * 2);
}
// bf16 element (r, c) of a TMA tile [64][128] stored as two 128-byte-swizzled halves
__device__ __forceinline__ uint32_t off_sw128(int r, int c) {
    const int hf = c >> 6, cc = c & 63;
    return (uint32_t)(hf * 8192 + r * 128 + ((((cc >> 3) ^ (r & 7))) << 4) + (cc & 7) * 2);
}

struct alignas(8) TcShared {
    uint64_t bar_tma;
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort;
};

__device__ int g_kda_tc_error;   // set when a bounded wait gives up

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

__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                const __nv_bfloat16 *__restrict__ beta, const float *__restrict__ S0,
                __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, int T, int H,
                KernelFlags fl) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ TcShared sh;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    float *GAM = reinterpret_cast<float *>(smem + OFF_GAM);
    float *AKK = reinterpret_cast<float *>(smem + OFF_AKK);
    float *TMF = reinterpret_cast<float *>(smem + OFF_TMF);
    float *RS = reinterpret_cast<float *>(smem + OFF_RS);
    float *TP = reinterpret_cast<float *>(smem + OFF_TAB + TAB_P);
    float *TF = reinterpret_cast<float *>(smem + OFF_TAB + TAB_F);
    float *TG = reinterpret_cast<float *>(smem + OFF_TAB + TAB_G);
    float *TH = reinterpret_cast<float *>(smem + OFF_TAB + TAB_H);
    float *TGC = reinterpret_cast<float *>(smem + OFF_TAB + TAB_GC);
    float *NRM = reinterpret_cast<float *>(smem + OFF_TAB + TAB_NRM);
    float *BET = reinterpret_cast<float *>(smem + OFF_TAB + TAB_BET);
    uint32_t *SGN = reinterpret_cast<uint32_t *>(smem + OFF_TAB + TAB_SGN);
    uint32_t *SGNC = reinterpret_cast<uint32_t *>(smem + OFF_TAB + TAB_SGNC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;                 // TMEM lane owned by this thread
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int nch = (T + C - 1) / C;
    const uint32_t bar_tma = smem_u32(&sh.bar_tma), bar_mma = smem_u32(&sh.bar_mma);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        sh.abort = 0;
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sh.tmem_base), 512);
        tmem_relinquish();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sh.tmem_base;

    auto issue_tma = [&](int ch) {
        mbar_arrive_expect_tx(bar_tma, kTmaBytes);
        const int t0 = ch * C;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(sbase + OFF_STG_Q + hf * 8192, &tm_q, bar_tma, hf * 64, h, t0, b);
            tma_load_4d(sbase + OFF_STG_K + hf * 8192, &tm_k, bar_tma, hf * 64, h, t0, b);
            tma_load_4d(sbase + OFF_STG_V + hf * 8192, &tm_v, bar_tma, hf * 64, h, t0, b);
            tma_load_4d(sbase + OFF_STG_G + hf * 8192, &tm_g, bar_tma, hf * 64, h, t0, b);
        }
    };
    // every thread waits; a give-up anywhere makes the whole CTA stop together
    auto wait_all = [&](uint32_t bar, uint32_t phase) -> bool {
        if (!mbar_wait_bounded(bar, phase, kWaitLimit)) {
            sh.abort = 1;
            g_kda_tc_error = 1;
        }
        __syncthreads();
        return sh.abort == 0;
    };
    if (tid == 0 && nch > 0) issue_tma(0);

    // the FP32 state: thread (row = key channel c, half) owns S[c][64 half .. 64 half + 63]
    float S[64];
    {
        const int c = row;
        const float *src = S0 ? S0 + ((size_t)bh * D + c) * D + 64 * half : nullptr;
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
            float4 v4 = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0, 0, 0, 0);
            S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
        }
#pragma unroll
        for (int jg = 0; jg < 8; ++jg) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = S[jg * 8 + e];
            *reinterpret_cast<uint4 *>(smem + OFF_SB + off_r128(c, 64 * half + 8 * jg)) = pack8(x);
        }
    }

    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;
    for (int ch = 0; ch < nch && ok; ++ch) {
        const int t0 = ch * C;
        const int n = min(C, T - t0);
        if (!(ok = wait_all(bar_tma, ph_tma))) break;
        ph_tma ^= 1;

        // ---- step 1: cumulative log-decay per key channel | row norms and beta
        if (tid < D) {
            const int c = tid;
            float gam = 0.f;
            uint32_t par = 0;
            for (int r = 0; r < C; ++r) {
                float lg = 0.f;
                if (r < n) {
                    const float a = __bfloat162float(
                        *reinterpret_cast<const __nv_bfloat16 *>(smem + OFF_STG_G + off_sw128(r, c)));
                    if (fl.complex_gate) {
                        lg = __logf(fabsf(a));
                        par ^= (a < 0.f) ? 1u : 0u;
                    } else {
                        lg = a;
                    }
                }
                gam += lg;
                GAM[r * GAM_STRIDE + c] = gam;
                if (fl.complex_gate) {
                    const uint32_t bits = __ballot_sync(0xffffffffu, par != 0);
                    if (lane == 0) SGN[r * 4 + warp] = bits;
                }
                if ((r & 15) == 15 && r < 63) TP[((r + 1) >> 4) * D + c] = gam;
            }
            TP[c] = 0.f;
            const uint32_t bits = __ballot_sync(0xffffffffu, par != 0);
            if (lane == 0) SGNC[warp] = fl.complex_gate ? bits : 0u;
        } else {
            const int rr = tid - D;      // 0..63 q rows, 64..127 k rows
            const int r = rr & 63;
            const uint32_t tile = rr < 64 ? OFF_STG_Q : OFF_STG_K;
            float ss = 0.f;
#pragma unroll
            for (int cg = 0; cg < 16; ++cg) {
                float x[8];
                unpack8(*reinterpret_cast<const uint4 *>(smem + tile + off_sw128(r, cg * 8)), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss += x[e] * x[e];
            }
            NRM[rr] = fl.l2norm ? rsqrtf(ss + kL2Eps) : 1.f;
            if (rr < 64)
                BET[r] = r < n ? __bfloat162float(beta[((size_t)b * T + t0 + r) * H + h]) : 0.f;
        }
        __syncthreads();

        // ---- step 2: per-band factor tables
        for (int idx = tid; idx < 11 * D; idx += NT) {
            const int e = idx / D, c = idx % D;
            const float gC = GAM[63 * GAM_STRIDE + c];
            if (e < 6) {
                const int bb = e < 1 ? 1 : (e < 3 ? 2 : 3);
                const int jj = e < 1 ? 0 : (e < 3 ? e - 1 : e - 3);
                TF[(bb * 4 + jj) * D + c] = __expf(TP[bb * D + c] - TP[jj * D + c]);
            } else if (e < 10) {
                const int bb = e - 6;
                TG[bb * D + c] = __expf(gC - TP[bb * D + c]);
                TH[bb * D + c] = __expf(TP[bb * D + c]);
                TF[(bb * 4 + bb) * D + c] = 1.f;
            } else {
                const float sg = ((SGNC[c >> 5] >> (c & 31)) & 1u) ? -1.f : 1.f;
                TGC[c] = sg * __expf(gC);
            }
        }
        __syncthreads();

        // ---- step 3: band-scaled operands (thread = row, half = 64 channels)
        {
            const bool isq = row < 64;
            const int r = row & 63;
            const int band = r >> 4;
            const float nrm = NRM[row];
            const float bet = BET[r];
            const uint32_t tile = isq ? OFF_STG_Q : OFF_STG_K;
#pragma unroll 1
            for (int cg = 0; cg < 8; ++cg) {
                const int c0 = 64 * half + 8 * cg;
                float x[8], gm[8], pb[8];
                unpack8(*reinterpret_cast<const uint4 *>(smem + tile + off_sw128(r, c0)), x);
                *reinterpret_cast<float4 *>(gm) = *reinterpret_cast<const float4 *>(GAM + r * GAM_STRIDE + c0);
                *reinterpret_cast<float4 *>(gm + 4) = *reinterpret_cast<const float4 *>(GAM + r * GAM_STRIDE + c0 + 4);
                *reinterpret_cast<float4 *>(pb) = *reinterpret_cast<const float4 *>(TP + band * D + c0);
                *reinterpret_cast<float4 *>(pb + 4) = *reinterpret_cast<const float4 *>(TP + band * D + c0 + 4);
                const uint32_t sb = fl.complex_gate ? (SGN[r * 4 + (c0 >> 5)] >> (c0 & 31)) : 0u;
                const uint32_t sbc = SGNC[c0 >> 5] >> (c0 & 31);
                float xe[8], inv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xv = x[e] * nrm * (((sb >> e) & 1u) ? -1.f : 1.f);
                    const float E = __expf(fmaxf(gm[e] - pb[e], -85.f));
                    xe[e] = xv * E;
                    inv[e] = isq ? 0.f : __fdividef(xv, E);
                }
                // A operands of the band products, bands j <= band(r), in TMEM
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float f = (j <= band) ? TF[(band * 4 + j) * D + c0 + e] : 0.f;
                        y[e] = (isq ? xe[e] : bet * xe[e]) * f;
                    }
                    tmem_st4(tbase + lane_off + TC_AOP + 64 * j + 32 * half + 4 * cg,
                             pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                             pack_bf16(y[6], y[7]));
                }
                float hb[8];
                *reinterpret_cast<float4 *>(hb) = *reinterpret_cast<const float4 *>(TH + band * D + c0);
                *reinterpret_cast<float4 *>(hb + 4) = *reinterpret_cast<const float4 *>(TH + band * D + c0 + 4);
                if (isq) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = xe[e] * hb[e];
                    *reinterpret_cast<uint4 *>(smem + OFF_QG + off_r128(r, c0)) = pack8(y);
                } else {
                    float gb[8], y1[8], y2[8];
                    *reinterpret_cast<float4 *>(gb) = *reinterpret_cast<const float4 *>(TG + band * D + c0);
                    *reinterpret_cast<float4 *>(gb + 4) = *reinterpret_cast<const float4 *>(TG + band * D + c0 + 4);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        y1[e] = xe[e] * hb[e];
                        y2[e] = (((sbc >> e) & 1u) ? -1.f : 1.f) * inv[e] * gb[e];
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_XR + off_r128(r, c0)) = pack8(inv);
                    *reinterpret_cast<uint4 *>(smem + OFF_YR + off_r128(r, c0)) = pack8(y1);
                    *reinterpret_cast<uint4 *>(smem + OFF_KD + off_r128(r, c0)) = pack8(y2);
                }
            }
        }
        tmem_wait_st();
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- step 4: A_qk / A_kk band products
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 16, 0, 0, 0);
#pragma unroll 1
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ts(tbase + TC_A + 16 * j, tbase + TC_AOP + 64 * j + 8 * s,
                           sdesc(sbase + OFF_XR + 4096 * j + 256 * s, 128, 2048, kSwizzleNone), id,
                           s > 0);
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();

        // ---- step 5: A_qk -> bf16 (lower with diagonal); A_kk -> FP32 (strictly lower)
        {
            float v[32];
            tmem_ld32(tbase + lane_off + TC_A + 32 * half, v);
            const int r = row & 63;
            if (row < 64) {
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 32 * half + 8 * g8 + e;
                        y[e] = (i <= r) ? v[8 * g8 + e] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_AQK + off_r64(r, 32 * half + 8 * g8)) = pack8(y);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * half + e;
                    AKK[r * 65 + i] = (i < r) ? v[e] : 0.f;
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- step 6: Tm = (I + A_kk)^{-1}, 16x16 blocks, FP32; Tm' = Tm diag(beta) -> bf16
        if (tid < 64) {
            const int bb = tid >> 4, jj = tid & 15;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < rr; ++i)
                    if (i >= jj) acc += AKK[(16 * bb + rr) * 65 + 16 * bb + i] * x[i];
                x[rr] = rr < jj ? 0.f : (rr == jj ? 1.f : -acc);
            }
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) TMF[(16 * bb + rr) * 65 + 16 * bb + jj] = x[rr];
        }
        __syncthreads();
#pragma unroll 1
        for (int bb = 1; bb < 4; ++bb) {
            for (int o = tid; o < bb * 256; o += NT) {
                const int j = o >> 8, rr = (o >> 4) & 15, cc = o & 15;
                float acc = 0.f;
                for (int m = j; m < bb; ++m)
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        acc += AKK[(16 * bb + rr) * 65 + 16 * m + k] * TMF[(16 * m + k) * 65 + 16 * j + cc];
                RS[(j * 16 + rr) * 17 + cc] = acc;
            }
            __syncthreads();
            for (int o = tid; o < bb * 256; o += NT) {
                const int j = o >> 8, rr = (o >> 4) & 15, cc = o & 15;
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (k <= rr) acc += TMF[(16 * bb + rr) * 65 + 16 * bb + k] * RS[(j * 16 + k) * 17 + cc];
                TMF[(16 * bb + rr) * 65 + 16 * j + cc] = -acc;
            }
            __syncthreads();
        }
        for (int o = tid; o < 64 * 8; o += NT) {
            const int r = o >> 3, ig = o & 7;
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * ig + e;
                y[e] = (i <= r) ? TMF[r * 65 + i] * BET[i] : 0.f;
            }
            *reinterpret_cast<uint4 *>(smem + OFF_TMB + off_r64(r, 8 * ig)) = pack8(y);
        }
        fence_proxy_async();
        __syncthreads();

        // ---- step 7: W^T = KG^T Tm'^T,  U^T = V^T Tm'^T
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 64, 1, 0, 0);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t bdesc = sdesc(sbase + OFF_TMB + 256 * s, 128, 1024, kSwizzleNone);
                mma_ss(tbase + TC_W, sdesc(sbase + OFF_YR + 4096 * s, 2048, 128, kSwizzleNone), bdesc, id, s > 0);
                mma_ss(tbase + TC_U, sdesc(sbase + OFF_STG_V + 2048 * s, 8192, 1024, kSwizzle128B), bdesc, id, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();

        // ---- step 8: prefetch the next chunk; W^T -> bf16 (MN-major [c][r])
        if (tid == 0 && ch + 1 < nch) issue_tma(ch + 1);
        {
            float v[32];
            tmem_ld32(tbase + lane_off + TC_W + 32 * half, v);
            const int c = row;
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = v[8 * g8 + e];
                *reinterpret_cast<uint4 *>(smem + OFF_YR + off_r64(c, 32 * half + 8 * g8)) = pack8(y);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- step 9: V~^T = U^T - S^T W^T;  O^T = S^T Qg^T
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id_v = idesc_bf16(128, 64, 1, 1, 1);
            constexpr uint32_t id_o = idesc_bf16(128, 64, 1, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t adesc = sdesc(sbase + OFF_SB + 4096 * s, 2048, 128, kSwizzleNone);
                mma_ss(tbase + TC_U, adesc, sdesc(sbase + OFF_YR + 2048 * s, 1024, 128, kSwizzleNone), id_v, 1);
                mma_ss(tbase + TC_O, adesc, sdesc(sbase + OFF_QG + 256 * s, 128, 2048, kSwizzleNone), id_o, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();

        // ---- step 10: V~^T -> bf16 (K-major [j][r])
        {
            float v[32];
            tmem_ld32(tbase + lane_off + TC_U + 32 * half, v);
            const int j = row;
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = v[8 * g8 + e];
                *reinterpret_cast<uint4 *>(smem + OFF_VT + off_r64(j, 32 * half + 8 * g8)) = pack8(y);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- step 11: O^T += V~^T A_qk^T;  dS = Kd^T V~
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id_o = idesc_bf16(128, 64, 0, 0, 0);
            constexpr uint32_t id_s = idesc_bf16(128, 128, 1, 0, 0);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t vt = sdesc(sbase + OFF_VT + 256 * s, 128, 1024, kSwizzleNone);
                mma_ss(tbase + TC_O, vt, sdesc(sbase + OFF_AQK + 256 * s, 128, 1024, kSwizzleNone), id_o, 1);
                mma_ss(tbase + TC_S, sdesc(sbase + OFF_KD + 4096 * s, 2048, 128, kSwizzleNone), vt, id_s, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();

        // ---- step 12: outputs; S <- gC * S + dS (FP32) and its bf16 copy
        {
            float v[32];
            tmem_ld32(tbase + lane_off + TC_O + 32 * half, v);
            const int j = row;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int r = 32 * half + e;
                if (r < n)
                    out[(((size_t)b * T + t0 + r) * H + h) * D + j] = __float2bfloat16_rn(fl.scale * v[e]);
            }
            const int c = row;
            const float gc = TGC[c];
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                tmem_ld32(tbase + lane_off + TC_S + 64 * half + 32 * part, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) S[32 * part + e] = fmaf(gc, S[32 * part + e], v[e]);
            }
#pragma unroll
            for (int jg = 0; jg < 8; ++jg) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = S[jg * 8 + e];
                *reinterpret_cast<uint4 *>(smem + OFF_SB + off_r128(c, 64 * half + 8 * jg)) = pack8(x);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (ok && S_T) {
        float *dst = S_T + ((size_t)bh * D + row) * D + 64 * half;
#pragma unroll
        for (int j = 0; j < 64; j += 4)
            *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    if (!ok) {
        // drain what may still be in flight (bounded), then release TMEM
        mbar_wait_bounded(bar_tma, ph_tma, kWaitLimit);
        mbar_wait_bounded(bar_mma, ph_mma, kWaitLimit);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool make_map(CUtensorMap *m, const void *ptr, int B, int T, int H) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
}  // namespace

bool chunk_tc_supported(const ChunkArgs &a) {
    return a.dk == D && a.dv == D && a.t_qkv == Elt::BF16 && a.t_g == Elt::BF16 &&
           a.t_beta == Elt::BF16 && a.t_out == Elt::BF16;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mg;
    if (!make_map(&mq, a.q, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, a.B, a.T, a.H) || !make_map(&mg, a.g, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    mark_launch(a, st);
    chunk_tc_kernel<<<a.B * a.H, NT, SMEM_BYTES, st>>>(mq, mk, mv, mg, (const __nv_bfloat16 *)a.beta,
                                                      a.S0, (__nv_bfloat16 *)a.out, a.S_T, a.T, a.H,
                                                      a.fl);
    return cudaGetLastError();
}

int chunk_tc_read_error() {
    int v = 0;
    cudaMemcpyFromSymbol(&v, g_kda_tc_error, sizeof(int));
    return v;
}

}  // namespace kda
