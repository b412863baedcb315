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
//   tcgen05  A_qk / A_kk: all ten (row band b, column band j <= b) pairs as one
//            N = 160 product.  A = [Q E; beta K E] (rows scaled by their own band
//            reference, in TMEM); the B rows of pair (b, j) are k_i e^{p_b - gamma_i}
//            for the 16 tokens i of band j.  Every factor stays inside the bf16
//            range because a band spans 16 tokens and g > -5 (cumulative >= -80)
//   CUDA     Tm = (I + A_kk)^{-1} (UT transform) in FP32, 32x32 blocks
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
constexpr int NT = 512;         // threads: 16 warps, 4 per TMEM lane quarter
constexpr uint32_t kTmaBytes = 4u * C * D * 2u;   // q, k, v, g tiles per chunk

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_STG_Q = 0;
constexpr uint32_t OFF_STG_K = 16384;
constexpr uint32_t OFF_STG_V = 32768;
constexpr uint32_t OFF_STG_G = 49152;
constexpr uint32_t OFF_GAM = 65536;           // fp32 E = e^{band-local cumsum} [64][132]; later AKK/TMF; later V~^T
constexpr uint32_t E_STRIDE = 132;            // floats per row (conflict-free 16-byte row reads)
constexpr uint32_t AS = 68;                   // row stride (floats) of AKK / TMF
constexpr uint32_t OFF_AKK = OFF_GAM;         // fp32 [64][68]
constexpr uint32_t OFF_TMF = OFF_GAM + 17408; // fp32 [64][68]
constexpr uint32_t OFF_VT = OFF_GAM;          // bf16 V~^T, K-major [128 j][64 r]
constexpr uint32_t OFF_QG = OFF_GAM + 36864;  // bf16 Q e^gamma [64 r][128 c]; later O staging [64][128]
constexpr uint32_t OFF_BOP = OFF_QG + 16384;  // bf16 band-pair B operand [160][128]; later A_qk, Tm'
constexpr uint32_t OFF_AQK = OFF_BOP;         // bf16 [64 r][64 i]
constexpr uint32_t OFF_TMB = OFF_BOP + 8192;  // bf16 [64 r][64 i]
constexpr uint32_t OFF_YR = OFF_BOP + 40960;  // bf16 K e^gamma [64][128]; later W^T [128][64]
constexpr uint32_t OFF_KD = OFF_YR + 16384;   // bf16 K e^{gamma_C-gamma} [64][128]
constexpr uint32_t OFF_TAB = OFF_KD + 16384;  // tables
constexpr uint32_t TAB_TOT = 0;               // fp32 [4][128] band sums of log-decay
constexpr uint32_t TAB_F = TAB_TOT + 2048;    // fp32 [4][4][128] e^{p_b - p_j}
constexpr uint32_t TAB_G = TAB_F + 8192;      // fp32 [4][128] e^{gamma_C - p_b}
constexpr uint32_t TAB_H = TAB_G + 2048;      // fp32 [4][128] e^{p_b}
constexpr uint32_t TAB_GC = TAB_H + 2048;     // fp32 [128] sigma_C e^{gamma_C}
constexpr uint32_t TAB_NRM = TAB_GC + 512;    // fp32 [128] inverse norms (q rows, k rows)
constexpr uint32_t TAB_BET = TAB_NRM + 512;   // fp32 [64]
constexpr uint32_t TAB_SGNL = TAB_BET + 256;  // u32 [64][4] band-local sign parity bits
constexpr uint32_t TAB_BPAR = TAB_SGNL + 1024;// u32 [4][4] parity of each band
constexpr uint32_t TAB_PP = TAB_BPAR + 256;   // u32 [4][4] parity of the bands before
constexpr uint32_t TAB_SGNC = TAB_PP + 256;   // u32 [4] parity of the whole chunk
constexpr uint32_t TAB_BYTES = TAB_SGNC + 256;
constexpr uint32_t SMEM_USED = OFF_TAB + TAB_BYTES;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // slack for the 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_TMF + 64 * AS * 4 <= OFF_QG, "inverse scratch fits");

// The ten (row band b, column band j <= b) pairs of the 64 x 64 intra-chunk
// matrices, as 16-column groups of one N = 160 product: pair(b, j) = P0[j] + b - j.
__device__ __forceinline__ int pair_of(int b, int j) { return (j == 0 ? 0 : j == 1 ? 4 : j == 2 ? 7 : 9) + b - j; }

// TMEM columns (512 allocated)
//   [0,64)    X: rows scaled by their own band reference (A of the band product), steps 3-4
//   [64,224)  D: the ten band-pair products, steps 4-5
//   [224,288) W^T (7-8)   [288,352) U^T, then V~^T (7-10)
//   [128,192) O^T (9-12)  [0,128) dS^T (11-12)
//   [448,512) S^T in bf16: the A operand of the state products (persistent)
constexpr uint32_t TC_X = 0, TC_D = 64, TC_W = 224, TC_U = 288, TC_O = 128, TC_S = 0, TC_SOP = 448;

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
__device__ __forceinline__ void ld8f(const float *p, float (&x)[8]) {
    *reinterpret_cast<float4 *>(x) = *reinterpret_cast<const float4 *>(p);
    *reinterpret_cast<float4 *>(x + 4) = *reinterpret_cast<const float4 *>(p + 4);
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
    float *EX = reinterpret_cast<float *>(smem + OFF_GAM);
    float *AKK = reinterpret_cast<float *>(smem + OFF_AKK);
    float *TMF = reinterpret_cast<float *>(smem + OFF_TMF);
    float *TOT = reinterpret_cast<float *>(smem + OFF_TAB + TAB_TOT);
    float *TF = reinterpret_cast<float *>(smem + OFF_TAB + TAB_F);
    float *TG = reinterpret_cast<float *>(smem + OFF_TAB + TAB_G);
    float *TH = reinterpret_cast<float *>(smem + OFF_TAB + TAB_H);
    float *TGC = reinterpret_cast<float *>(smem + OFF_TAB + TAB_GC);
    float *NRM = reinterpret_cast<float *>(smem + OFF_TAB + TAB_NRM);
    float *BET = reinterpret_cast<float *>(smem + OFF_TAB + TAB_BET);
    uint32_t *SGNL = reinterpret_cast<uint32_t *>(smem + OFF_TAB + TAB_SGNL);
    uint32_t *BPAR = reinterpret_cast<uint32_t *>(smem + OFF_TAB + TAB_BPAR);
    uint32_t *PP = reinterpret_cast<uint32_t *>(smem + OFF_TAB + TAB_PP);
    uint32_t *SGNC = reinterpret_cast<uint32_t *>(smem + OFF_TAB + TAB_SGNC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, qq = warp >> 2;       // lane quarter; column quarter
    const int row = quad * 32 + lane;                // TMEM lane owned by this thread
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
    const uint32_t tl = tbase + lane_off;             // this warp's lane quarter
    // descriptor bases (start address = the smem base); a tile at byte offset `off`
    // is base + (off >> 4) since every address stays below 256 KB
    const uint64_t dK64 = sdesc(sbase, 128, 2048, kSwizzleNone);    // K-major [rows][128]
    const uint64_t dMN64 = sdesc(sbase, 2048, 128, kSwizzleNone);   // MN-major [K rows][128]
    const uint64_t dK32 = sdesc(sbase, 128, 1024, kSwizzleNone);    // K-major [rows][64]
    const uint64_t dMN32 = sdesc(sbase, 1024, 128, kSwizzleNone);   // MN-major [K rows][64]
    const uint64_t dV = sdesc(sbase, 8192, 1024, kSwizzle128B);     // MN-major TMA v tile
    auto at = [](uint64_t base, uint32_t off) -> uint64_t { return base + (uint64_t)(off >> 4); };

    // the next chunk's q, k, g tiles are requested as soon as this chunk's operands are
    // built (they are free then), its v tile once the U product has read it
    auto issue_tma_qkg = [&](int ch) {
        fence_proxy_async();   // order the threads' earlier reads of the tiles before the overwrite
        mbar_arrive_expect_tx(bar_tma, kTmaBytes);
        const int t0 = ch * C;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(sbase + OFF_STG_Q + hf * 8192, &tm_q, bar_tma, hf * 64, h, t0, b);
            tma_load_4d(sbase + OFF_STG_K + hf * 8192, &tm_k, bar_tma, hf * 64, h, t0, b);
            tma_load_4d(sbase + OFF_STG_G + hf * 8192, &tm_g, bar_tma, hf * 64, h, t0, b);
        }
    };
    auto issue_tma_v = [&](int ch) {
        fence_proxy_async();
        const int t0 = ch * C;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
            tma_load_4d(sbase + OFF_STG_V + hf * 8192, &tm_v, bar_tma, hf * 64, h, t0, b);
    };
    // one thread polls the mbarrier (512 pollers would compete with the tensor core for
    // shared memory); the rest wait at the CTA barrier.  A give-up stops the whole CTA.
    auto wait_all = [&](uint32_t bar, uint32_t phase) -> bool {
        if (tid == 0 && !mbar_wait_bounded(bar, phase, kWaitLimit)) {
            sh.abort = 1;
            g_kda_tc_error = 1;
        }
        __syncthreads();
        return sh.abort == 0;
    };
    if (tid == 32 && nch > 0) {
        issue_tma_qkg(0);
        issue_tma_v(0);
    }
    // beta of the first chunk; later chunks' beta is fetched a chunk ahead
    if (tid < C) BET[tid] = tid < T ? __bfloat162float(beta[((size_t)b * T + tid) * H + h]) : 0.f;

    // The FP32 state, transposed: thread (lane j, qq) owns S^T[j][32 qq .. 32 qq + 31],
    // i.e. S[c][j] for its 32 key channels c; its bf16 copy lives in TMEM.
    float S[32];
    auto store_state_operand = [&]() {
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4)
            tmem_st4(tl + TC_SOP + 16 * qq + 4 * e4, pack_bf16(S[8 * e4], S[8 * e4 + 1]),
                     pack_bf16(S[8 * e4 + 2], S[8 * e4 + 3]), pack_bf16(S[8 * e4 + 4], S[8 * e4 + 5]),
                     pack_bf16(S[8 * e4 + 6], S[8 * e4 + 7]));
    };
    {
        const int j = row;
#pragma unroll
        for (int e = 0; e < 32; ++e)
            S[e] = S0 ? S0[((size_t)bh * D + 32 * qq + e) * D + j] : 0.f;
        store_state_operand();
        tmem_wait_st();
    }

    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;
    for (int ch = 0; ch < nch && ok; ++ch) {
        const int t0 = ch * C;
        const int n = min(C, T - t0);
        if (!(ok = wait_all(bar_tma, ph_tma))) break;
        ph_tma ^= 1;

        // ---- step 1: band-local cumulative log-decay (4 bands x 128 channels) | row norms
        {
            const int c = tid & 127, p = tid >> 7;
            float gv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                gv[i] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(
                    smem + OFF_STG_G + off_sw128(16 * p + i, c)));
            float loc = 0.f;
            uint32_t par = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * p + i;
                float lg = 0.f;
                if (r < n) {
                    if (fl.complex_gate) {
                        lg = __logf(fabsf(gv[i]));
                        par ^= (gv[i] < 0.f) ? 1u : 0u;
                    } else {
                        lg = gv[i];
                    }
                }
                loc += lg;
                EX[r * E_STRIDE + c] = __expf(fmaxf(loc, -85.f));
                if (fl.complex_gate) {
                    const uint32_t bits = __ballot_sync(0xffffffffu, par != 0);
                    if (lane == 0) SGNL[r * 4 + quad] = bits;
                }
            }
            TOT[p * D + c] = loc;
            const uint32_t bp = __ballot_sync(0xffffffffu, par != 0);
            if (lane == 0) BPAR[p * 4 + quad] = bp;
        }
        {
            const int rr = tid >> 2, part = tid & 3;     // 4 lanes per row, 32 channels each
            const int r = rr & 63;
            const uint32_t tile = rr < 64 ? OFF_STG_Q : OFF_STG_K;
            float ss = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float x[8];
                unpack8(*reinterpret_cast<const uint4 *>(smem + tile + off_sw128(r, 32 * part + 8 * m)), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss += x[e] * x[e];
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            if (part == 0) NRM[rr] = fl.l2norm ? rsqrtf(ss + kL2Eps) : 1.f;
        }
        __syncthreads();

        // ---- step 2: per-channel band factors from the four band sums
        if (tid < D) {
            const int c = tid;
            float et[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) et[p] = __expf(TOT[p * D + c]);
            // H[b] = e^{p_b}, F[b][j] = e^{p_b - p_j}, G[b] = e^{gamma_C - p_b}
            TH[0 * D + c] = 1.f;
            TH[1 * D + c] = et[0];
            TH[2 * D + c] = et[0] * et[1];
            TH[3 * D + c] = et[0] * et[1] * et[2];
            const float eC = et[0] * et[1] * et[2] * et[3];
            TG[0 * D + c] = eC;
            TG[1 * D + c] = et[1] * et[2] * et[3];
            TG[2 * D + c] = et[2] * et[3];
            TG[3 * D + c] = et[3];
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) TF[(bb * 4 + bb) * D + c] = 1.f;
            TF[(1 * 4 + 0) * D + c] = et[0];
            TF[(2 * 4 + 1) * D + c] = et[1];
            TF[(2 * 4 + 0) * D + c] = et[0] * et[1];
            TF[(3 * 4 + 2) * D + c] = et[2];
            TF[(3 * 4 + 1) * D + c] = et[1] * et[2];
            TF[(3 * 4 + 0) * D + c] = et[0] * et[1] * et[2];
            const int w = c >> 5, bit = c & 31;
            const uint32_t pc = BPAR[0 * 4 + w] ^ BPAR[1 * 4 + w] ^ BPAR[2 * 4 + w] ^ BPAR[3 * 4 + w];
            TGC[c] = ((pc >> bit) & 1u) ? -eC : eC;
            if (c < 4) {
                PP[0 * 4 + c] = 0u;
                PP[1 * 4 + c] = BPAR[0 * 4 + c];
                PP[2 * 4 + c] = BPAR[0 * 4 + c] ^ BPAR[1 * 4 + c];
                PP[3 * 4 + c] = BPAR[0 * 4 + c] ^ BPAR[1 * 4 + c] ^ BPAR[2 * 4 + c];
                SGNC[c] = BPAR[0 * 4 + c] ^ BPAR[1 * 4 + c] ^ BPAR[2 * 4 + c] ^ BPAR[3 * 4 + c];
            }
        }
        __syncthreads();

        // ---- step 3: operands (thread = row, 32 channels).  Rows are scaled by their own
        //      band reference; the band-pair factor e^{p_b - p_j} goes onto the B operand.
        {
            const bool isq = row < 64;
            const int r = row & 63;
            const int band = r >> 4;
            const float nrm = NRM[row];
            const float bet = BET[r];
            const uint32_t tile = isq ? OFF_STG_Q : OFF_STG_K;
            const uint32_t sw = fl.complex_gate ? (SGNL[r * 4 + qq] ^ PP[band * 4 + qq]) : 0u;
            const uint32_t swc = SGNC[qq];
#pragma unroll
            for (int cg = 0; cg < 4; ++cg) {
                const int c0 = 32 * qq + 8 * cg;
                float x[8], E[8], hb[8];
                unpack8(*reinterpret_cast<const uint4 *>(smem + tile + off_sw128(r, c0)), x);
                ld8f(EX + r * E_STRIDE + c0, E);
                ld8f(TH + band * D + c0, hb);
                float xe[8], y1[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[e] *= ((sw >> (8 * cg + e)) & 1u) ? -nrm : nrm;
                    xe[e] = x[e] * E[e];
                    y1[e] = xe[e] * hb[e];
                }
                const float rs = isq ? 1.f : bet;
                tmem_st4(tl + TC_X + 16 * qq + 4 * cg, pack_bf16(rs * xe[0], rs * xe[1]),
                         pack_bf16(rs * xe[2], rs * xe[3]), pack_bf16(rs * xe[4], rs * xe[5]),
                         pack_bf16(rs * xe[6], rs * xe[7]));
                if (isq) {
                    *reinterpret_cast<uint4 *>(smem + OFF_QG + off_r128(r, c0)) = pack8(y1);
                } else {
                    float gb[8], inv[8], y2[8];
                    ld8f(TG + band * D + c0, gb);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        inv[e] = __fdividef(x[e], E[e]);
                        y2[e] = (((swc >> (8 * cg + e)) & 1u) ? -inv[e] : inv[e]) * gb[e];
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_YR + off_r128(r, c0)) = pack8(y1);
                    *reinterpret_cast<uint4 *>(smem + OFF_KD + off_r128(r, c0)) = pack8(y2);
                }
            }
        }
        // B rows of the pairs (b, band(i)) for b = band(i)..3, spread evenly: warp = 8-channel
        // group, lane = key row i in bands 0-1 plus the mirrored row 63 - i in bands 3-2
        // (five copies per lane)
        {
            const int c0 = 8 * warp;
            const int w32 = c0 >> 5, sh8 = c0 & 31;
#pragma unroll
            for (int side = 0; side < 2; ++side) {
                const int i = side ? 63 - lane : lane;
                const int bi = i >> 4;
                const float nk = NRM[64 + i];
                const uint32_t swi = fl.complex_gate ? (SGNL[i * 4 + w32] ^ PP[bi * 4 + w32]) >> sh8 : 0u;
                float x[8], E[8], inv[8];
                unpack8(*reinterpret_cast<const uint4 *>(smem + OFF_STG_K + off_sw128(i, c0)), x);
                ld8f(EX + i * E_STRIDE + c0, E);
#pragma unroll
                for (int e = 0; e < 8; ++e) inv[e] = __fdividef(((swi >> e) & 1u) ? -nk * x[e] : nk * x[e], E[e]);
                for (int bb = bi; bb < 4; ++bb) {
                    float f[8], y3[8];
                    ld8f(TF + (bb * 4 + bi) * D + c0, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) y3[e] = inv[e] * f[e];
                    const int brow = 16 * pair_of(bb, bi) + (i & 15);
                    *reinterpret_cast<uint4 *>(smem + OFF_BOP + off_r128(brow, c0)) = pack8(y3);
                }
            }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();

        // ---- step 4: all ten band-pair products in one N = 160 product
        //      (one thread issues the next chunk's q, k, g loads, another the MMAs)
        if (tid == 0) {
            fence_proxy_async();   // the threads' smem writes (ordered by the barrier) -> async proxy
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 160, 0, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_ts(tbase + TC_D, tbase + TC_X + 8 * s, at(dK64, OFF_BOP + 256 * s), id, s > 0);
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();
        if (tid == 32 && ch + 1 < nch) issue_tma_qkg(ch + 1);

        // ---- step 5: A_qk -> bf16 (lower with diagonal); A_kk -> FP32 (strictly lower), transposed
        //      (AKK[i][r] = A_kk[r][i]).
        //      A warp's 32 rows span two row bands; it reads both bands' columns for
        //      column band j = qq and each thread keeps its own.
        {
            const int r = row & 63, band = r >> 4;
            const int b_lo = (quad & 1) * 2;
            float v[16], v2[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0.f;
            if (qq <= b_lo) tmem_ld16(tl + TC_D + 16 * pair_of(b_lo, qq), v);
            if (qq <= b_lo + 1) {
                tmem_ld16(tl + TC_D + 16 * pair_of(b_lo + 1, qq), v2);
                if (band == b_lo + 1) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = v2[e];
                }
            }
            if (row < 64) {
#pragma unroll
                for (int g8 = 0; g8 < 2; ++g8) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 16 * qq + 8 * g8 + e;
                        y[e] = (i <= r) ? v[8 * g8 + e] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_AQK + off_r64(r, 16 * qq + 8 * g8)) = pack8(y);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int i = 16 * qq + e;
                    AKK[i * AS + r] = (i < r) ? v[e] : 0.f;   // a warp writes 32 consecutive r
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- step 6: Tm = (I + A_kk)^{-1} in FP32 by 32 x 32 blocks, [T1 0; T21 T2]:
        //   T1 = (I + A11)^{-1}, T2 = (I + A22)^{-1}: one warp each, lane = column; column sweep in
        //   registers (x_i is final once the rows above it are done, then x_r -= A[r][i] x_i for
        //   every r > i); Y = A21 T1;  T21 = -T2 Y;  Tm' = Tm diag(beta) -> bf16, K-major [r][i].
        // TMF holds T1 (rows 0-31, columns 0-31), Y (rows 0-31, columns 32-63) and T2 (rows
        // 32-63, columns 32-63).
        if (warp < 2) {
            const int base = 32 * warp;
            float x[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) x[r] = (r == lane) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < 31; ++i) {
                const float xi = x[i];
                const float *col = AKK + (base + i) * AS + base;   // A[base + r][base + i] over r
#pragma unroll
                for (int r4 = ((i + 1) >> 2) << 2; r4 < 32; r4 += 4) {   // rows r <= i hold 0
                    const float4 av = *reinterpret_cast<const float4 *>(col + r4);
                    x[r4] = fmaf(-av.x, xi, x[r4]);
                    x[r4 + 1] = fmaf(-av.y, xi, x[r4 + 1]);
                    x[r4 + 2] = fmaf(-av.z, xi, x[r4 + 2]);
                    x[r4 + 3] = fmaf(-av.w, xi, x[r4 + 3]);
                }
            }
#pragma unroll
            for (int r = 0; r < 32; ++r) TMF[(base + r) * AS + base + lane] = x[r];
        }
        __syncthreads();
        // Y = A21 T1 and T21 = -T2 Y as 2 x 4 register tiles (threads 0-127: row pair rg, column
        // group cg); meanwhile threads 128-511 pack [T1 b | 0 ; . | T2 b'] (b = beta_j) to bf16
        {
            const int rg = tid >> 3, cg = tid & 7;
            if (tid < 128) {
                float acc[2][4] = {};
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float2 av = *reinterpret_cast<const float2 *>(AKK + i * AS + 32 + 2 * rg);   // A21[2rg..][i]
                    const float4 tv = *reinterpret_cast<const float4 *>(TMF + i * AS + 4 * cg);       // T1[i][4cg..]
                    acc[0][0] = fmaf(av.x, tv.x, acc[0][0]);
                    acc[0][1] = fmaf(av.x, tv.y, acc[0][1]);
                    acc[0][2] = fmaf(av.x, tv.z, acc[0][2]);
                    acc[0][3] = fmaf(av.x, tv.w, acc[0][3]);
                    acc[1][0] = fmaf(av.y, tv.x, acc[1][0]);
                    acc[1][1] = fmaf(av.y, tv.y, acc[1][1]);
                    acc[1][2] = fmaf(av.y, tv.z, acc[1][2]);
                    acc[1][3] = fmaf(av.y, tv.w, acc[1][3]);
                }
#pragma unroll
                for (int k = 0; k < 2; ++k)
                    *reinterpret_cast<float4 *>(TMF + (2 * rg + k) * AS + 32 + 4 * cg) =
                        make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
            } else {
                const int u = tid - 128;
                const int r = u < 256 ? (u >> 3) : 32 + ((u - 256) >> 2);
                const int g = u < 256 ? (u & 7) : 4 + ((u - 256) & 3);
                float y[8];
                if (r < 32 && g >= 4) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = 0.f;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = TMF[r * AS + 8 * g + e] * BET[8 * g + e];
                }
                *reinterpret_cast<uint4 *>(smem + OFF_TMB + off_r64(r, 8 * g)) = pack8(y);
            }
        }
        __syncthreads();
        if (tid < 128) {
            const int rg = tid >> 3, cg = tid & 7;
            float acc[2][4] = {};
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 ta = *reinterpret_cast<const float4 *>(TMF + (32 + 2 * rg) * AS + 32 + i);   // T2[2rg][i..]
                const float4 tb = *reinterpret_cast<const float4 *>(TMF + (33 + 2 * rg) * AS + 32 + i);   // T2[2rg+1][i..]
                const float a0[4] = {ta.x, ta.y, ta.z, ta.w}, a1[4] = {tb.x, tb.y, tb.z, tb.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 yv = *reinterpret_cast<const float4 *>(TMF + (i + k) * AS + 32 + 4 * cg);   // Y[i+k][4cg..]
                    acc[0][0] = fmaf(a0[k], yv.x, acc[0][0]);
                    acc[0][1] = fmaf(a0[k], yv.y, acc[0][1]);
                    acc[0][2] = fmaf(a0[k], yv.z, acc[0][2]);
                    acc[0][3] = fmaf(a0[k], yv.w, acc[0][3]);
                    acc[1][0] = fmaf(a1[k], yv.x, acc[1][0]);
                    acc[1][1] = fmaf(a1[k], yv.y, acc[1][1]);
                    acc[1][2] = fmaf(a1[k], yv.z, acc[1][2]);
                    acc[1][3] = fmaf(a1[k], yv.w, acc[1][3]);
                }
            }
            // T21 b -> Tm' rows 32 + 2rg + k, columns 4cg .. 4cg + 3 (8 bytes)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint32_t lo = pack_bf16(-acc[k][0] * BET[4 * cg], -acc[k][1] * BET[4 * cg + 1]);
                const uint32_t hi = pack_bf16(-acc[k][2] * BET[4 * cg + 2], -acc[k][3] * BET[4 * cg + 3]);
                *reinterpret_cast<uint2 *>(smem + OFF_TMB + off_r64(32 + 2 * rg + k, 4 * cg)) = make_uint2(lo, hi);
            }
        }
        __syncthreads();

        // ---- step 7: W^T = KG^T Tm'^T,  U^T = V^T Tm'^T
        if (tid == 0) {
            fence_proxy_async();   // the threads' smem writes (ordered by the barrier) -> async proxy
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, 64, 1, 0, 0);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t bdesc = at(dK32, OFF_TMB + 256 * s);
                mma_ss(tbase + TC_W, at(dMN64, OFF_YR + 4096 * s), bdesc, id, s > 0);
                mma_ss(tbase + TC_U, at(dV, OFF_STG_V + 2048 * s), bdesc, id, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();

        // ---- step 8: prefetch the next chunk's v and beta; W^T -> bf16 (MN-major [c][r])
        if (tid == 32 && ch + 1 < nch) issue_tma_v(ch + 1);
        float beta_next = 0.f;
        if (tid < C && ch + 1 < nch && t0 + C + tid < T)
            beta_next = __bfloat162float(beta[((size_t)b * T + t0 + C + tid) * H + h]);
        {
            float v[16];
            tmem_ld16(tl + TC_W + 16 * qq, v);
            const int c = row;
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = v[8 * g8 + e];
                *reinterpret_cast<uint4 *>(smem + OFF_YR + off_r64(c, 16 * qq + 8 * g8)) = pack8(y);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- step 9: V~^T = U^T - S^T W^T;  O^T = S^T Qg^T  (S^T from TMEM)
        if (tid == 0) {
            fence_proxy_async();   // the threads' smem writes (ordered by the barrier) -> async proxy
            tc_fence_after();
            constexpr uint32_t id_v = idesc_bf16(128, 64, 0, 1, 1);
            constexpr uint32_t id_o = idesc_bf16(128, 64, 0, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                mma_ts(tbase + TC_U, tbase + TC_SOP + 8 * s, at(dMN32, OFF_YR + 2048 * s), id_v, 1);
                mma_ts(tbase + TC_O, tbase + TC_SOP + 8 * s, at(dK64, OFF_QG + 256 * s), id_o, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();

        // ---- step 10: V~^T -> bf16 (K-major [j][r])
        {
            float v[16];
            tmem_ld16(tl + TC_U + 16 * qq, v);
            const int j = row;
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = v[8 * g8 + e];
                *reinterpret_cast<uint4 *>(smem + OFF_VT + off_r64(j, 16 * qq + 8 * g8)) = pack8(y);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- step 11: O^T += V~^T A_qk^T;  dS^T = V~^T Kd
        if (tid == 0) {
            fence_proxy_async();   // the threads' smem writes (ordered by the barrier) -> async proxy
            tc_fence_after();
            constexpr uint32_t id_o = idesc_bf16(128, 64, 0, 0, 0);
            constexpr uint32_t id_s = idesc_bf16(128, 128, 0, 1, 0);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t vt = at(dK32, OFF_VT + 256 * s);
                mma_ss(tbase + TC_O, vt, at(dK32, OFF_AQK + 256 * s), id_o, 1);
                mma_ss(tbase + TC_S, vt, at(dMN64, OFF_KD + 4096 * s), id_s, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;
        ph_mma ^= 1;
        tc_fence_after();

        // ---- step 12: outputs through a smem staging tile; S <- diag(gC) S + dS in FP32
        //      and its bf16 copy back into TMEM
        {
            __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(smem + OFF_QG);   // [64 r][128 j]
            {
                float o[16];
                tmem_ld16(tl + TC_O + 16 * qq, o);
                const int j = row;
#pragma unroll
                for (int e = 0; e < 16; ++e) ost[(16 * qq + e) * D + j] = __float2bfloat16_rn(fl.scale * o[e]);
            }
            float v[32], gcv[32];
            tmem_ld32(tl + TC_S + 32 * qq, v);
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4 *>(gcv + e) = *reinterpret_cast<const float4 *>(TGC + 32 * qq + e);
#pragma unroll
            for (int e = 0; e < 32; ++e) S[e] = fmaf(gcv[e], S[e], v[e]);
            store_state_operand();
            tmem_wait_st();
        }
        if (tid < C) BET[tid] = beta_next;
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int q16 = tid + NT * m, r = q16 >> 4, cj = q16 & 15;
            if (r < n) {
                const uint4 val = *reinterpret_cast<const uint4 *>(smem + OFF_QG + r * 256 + cj * 16);
                *reinterpret_cast<uint4 *>(out + (((size_t)b * T + t0 + r) * H + h) * D + 8 * cj) = val;
            }
        }
        __syncthreads();
    }

    if (ok && S_T) {
        const int j = row;
#pragma unroll
        for (int e = 0; e < 32; ++e) S_T[((size_t)bh * D + 32 * qq + e) * D + j] = S[e];
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

cudaError_t chunk_tc_take_error(int *flag, cudaStream_t st) {
    const int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(flag, g_kda_tc_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_kda_tc_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace kda
