// kda_chunk_tc2.cu -- two-kernel tensor-core chunkwise KDA forward for sm_100a.
//
// The chunkwise form (page "Kimi K3 模型结构（2）：序列维度（下），chunkwise 并行与
// 下界衰减", Q&A items on the chunkwise algorithm, the -5 decay floor and the
// intra-chunk matrix A) splits into work that does not depend on the state --
// everything up to the WY vectors -- and a short state-dependent scan.  The
// first kernel runs the former for every (chunk, head) in parallel, so it fills
// the GPU however few heads there are; the second walks each head's chunks in
// order with nothing but the scan on its critical path.
//
// Kernel 1 (one CTA per chunk and head), with the same arithmetic as the fused
// kernel of kda_chunk_tc.cu:
//   gamma = band-local cumsum of log|alpha|, E = e^{gamma - p_band}, band factors
//   A_qk / A_kk: all ten (row band, column band) pairs as one N = 160 tcgen05 product
//   Tm = (I + A_kk)^{-1} in FP32;  W = Tm' (K e^gamma),  U = Tm' V
//   writes, per chunk and head, a 74,240-byte record of bf16 tiles already in the
//   shared-memory layouts the scan's tensor-core products read:
//     W and Q e^gamma (K-major [r][c], stacked into one [128][128] tile),
//     K e^{gamma_C-gamma} ([r][c]), U (16-column slabs of [r][j]), A_qk (K-major [r][i])
//     and sigma_C e^{gamma_C} (FP32 [128]).
// Kernel 2 (one CTA per head): per chunk, the record is bulk-copied into one of two
// stages, then
//   [P ; O] = [W ; Q e^gamma] S                          (S in shared memory as bf16)
//   V~ = U - P;  dS = Kd^T V~;  O += A_qk V~             (V~ in shared memory as bf16)
//   S <- diag(sigma_C e^{gamma_C}) S + dS in FP32 registers;  O -> HBM while the
//   next chunk's first product runs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <stdlib.h>

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
// staging tile of 64 (or, with the halo of the fused prologue, 67) token rows x 128 channels
// as two 64-channel halves of 128-byte-swizzled rows, the halves 9 KB apart
constexpr uint32_t kHalf = 9216;
__device__ __forceinline__ uint32_t off_sw128(int r, int c) {
    const int hf = c >> 6, cc = c & 63;
    return (uint32_t)(hf * kHalf + r * 128 + ((((cc >> 3) ^ (r & 7))) << 4) + (cc & 7) * 2);
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
__device__ __forceinline__ uint2 pack4(const float (&x)[4]) {
    return make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
}
__device__ __forceinline__ void ld8f(const float *p, float (&x)[8]) {
    *reinterpret_cast<float4 *>(x) = *reinterpret_cast<const float4 *>(p);
    *reinterpret_cast<float4 *>(x + 4) = *reinterpret_cast<const float4 *>(p + 4);
}

__device__ int g_kda_tc2_error;   // set when a bounded wait gives up

struct alignas(8) Bars {
    uint64_t bar0;
    uint64_t bar1;
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort;
};

// ============================================================== kernel 1: per-chunk prep
namespace prep {
constexpr int NT = 512;
constexpr uint32_t kTile = 2 * kHalf;         // one staged tensor
constexpr uint32_t OFF_STG_Q = 0, OFF_STG_K = kTile, OFF_STG_V = 2 * kTile, OFF_STG_G = 3 * kTile;
constexpr int kHalo = 3;                       // rows before the chunk the short convolution reads
constexpr uint32_t OFF_GAM = 4 * kTile;        // fp32 E [64][132]; later AKK / TMF
constexpr uint32_t E_STRIDE = 132;
constexpr uint32_t AS = 68;
constexpr uint32_t OFF_AKK = OFF_GAM;
constexpr uint32_t OFF_TMF = OFF_GAM + 17408;
constexpr uint32_t OFF_BOP = OFF_GAM + 36864;  // bf16 band-pair B operand [160][128]; later Tm'
constexpr uint32_t OFF_TMB = OFF_BOP;          // bf16 [128][64 i]: Tm' rows r, then the same rows again
constexpr uint32_t OFF_YR = OFF_BOP + 40960;   // bf16 K e^gamma [64][128]
constexpr uint32_t OFF_TAB = OFF_YR + 16384;
constexpr uint32_t TAB_TOT = 0, TAB_F = 2048, TAB_G = 10240, TAB_H = 12288, TAB_GC = 14336,
                   TAB_NRM = 14848, TAB_BET = 15360, TAB_SGNL = 15616, TAB_BPAR = 16640,
                   TAB_PP = 16896, TAB_SGNC = 17152, TAB_BYTES = 17408;
// the record leaves through shared memory by bulk stores: Q e^gamma and Kd here, then W and U in
// the same 32 KB at the item's end (first rewritten by the next item's operands), A_qk in the
// band-pair operand's region, sigma_C e^{gamma_C} in the tables
constexpr uint32_t OFF_RQG = OFF_TAB + TAB_BYTES;    // bf16 Q e^gamma, the record's layout
constexpr uint32_t OFF_RKD = OFF_RQG + 16384;        // bf16 Kd
constexpr uint32_t OFF_RAQ = OFF_BOP + 16384;        // bf16 A_qk (after Tm')
constexpr uint32_t OFF_RWU = OFF_RQG;                // bf16 W, then U (16-column slabs)
constexpr uint32_t OFF_CW = OFF_RKD + 16384;        // bf16 conv taps of q, k, v [3][128 c][4] (prologue)
constexpr uint32_t SMEM_BYTES = OFF_CW + 3072 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
// TMEM: X [0,64), D [64,224), then W and U, each in lanes 0-63 with lanes 64-127 repeating
// them: U [224,352), W [352,480)
constexpr uint32_t TC_X = 0, TC_D = 64, TC_U = 224, TC_W = 352;
}  // namespace prep

// Inputs of the prologue fused into the prep kernel (kda_chunk_fwd_prologue on the split
// form).  conv_w == nullptr: the tiles are q, k, v, g and beta is given.
struct PrepPrologue {
    const __nv_bfloat16 *conv_w;   // [3, H * D, 4]: taps of q, k, v
    const float *A;                // [H] per-head log-scale of the gate
    const float *b_logit;          // [B, T, H] beta logits (FP32)
    // the raw branch inputs (the rows before a chunk, for its first convolution outputs)
    const __nv_bfloat16 *raw_q, *raw_k, *raw_v;
};

#include "kda_chunk_prep.cuh"

// The prep's work, run by CTA `cta` of `ncta` prep CTAs.  MEGA (the fused prep + scan launch of
// few-head calls): items are taken chunk-major, so every head's early chunks come first, and
// each finished record is published by a release of flags[item] once its bulk stores are
// complete.  Otherwise items are taken chunk-fastest and the scan runs as the next kernel.
template <bool PRO, bool MEGA>
__device__ __forceinline__ void
prep_body(const CUtensorMap *ptm_q, const CUtensorMap *ptm_k, const CUtensorMap *ptm_v,
          const CUtensorMap *ptm_g, const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ ws, int T,
          int H, int BH, KernelFlags fl, PrepPrologue pro, int cta, int ncta, int *__restrict__ flags) {
    using namespace prep;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Bars sh;
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
    const int quad = warp & 3, qq = warp >> 2;
    const int row = quad * 32 + lane;
    const int nch = (T + C - 1) / C;
    const int nitems = nch * BH;
    const uint32_t bar_tma = smem_u32(&sh.bar0), bar_v = smem_u32(&sh.bar1), bar_mma = smem_u32(&sh.bar_mma);

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        sh.abort = 0;
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sh.tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sh.tmem_base;
    const uint32_t tl = tbase + ((uint32_t)(quad * 32) << 16);
    // the scan kernel, launched with a programmatic dependency on this one, may be scheduled
    // now: its CTAs take SMs as this grid's CTAs leave and wait in-kernel for its completion
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint64_t dK64 = sdesc(sbase, 128, 2048, kSwizzleNone);
    const uint64_t dMN64 = sdesc(sbase, 2048, 128, kSwizzleNone);
    const uint64_t dK32 = sdesc(sbase, 128, 1024, kSwizzleNone);
    const uint64_t dV = sdesc(sbase, kHalf, 1024, kSwizzle128B);
    auto at = [](uint64_t base, uint32_t off) -> uint64_t { return base + (uint64_t)(off >> 4); };
    auto wait_all = [&](uint32_t bar, uint32_t phase) -> bool {
        if (tid == 0 && !mbar_wait_bounded(bar, phase, kWaitLimit)) {
            sh.abort = 1;
            g_kda_tc2_error = 1;
        }
        __syncthreads();
        return sh.abort == 0;
    };

    // work item = (chunk, b * H + h), chunk fastest; each CTA walks items with a stride of the
    // grid and fetches the next item's tiles as soon as their staging buffers are free
    // with the fused prologue the maps cover the raw inputs and their boxes are 67 rows high,
    // starting 3 rows before the chunk (rows before t = 0 read as zeros: no history)
    constexpr bool fused_pro = PRO;
    const int rows = fused_pro ? C + kHalo : C, row0 = fused_pro ? -kHalo : 0;
    const uint32_t tile_bytes = (uint32_t)rows * D * 2u;
    // item -> (chunk, b * H + h)
    auto item_ch = [&](int item) { return MEGA ? item / BH : item % nch; };
    auto item_bh = [&](int item) { return MEGA ? item % BH : item / nch; };
    auto issue_qkg = [&](int item) {
        const int ich = item_ch(item), ibh = item_bh(item);
        const int ib = ibh / H, ih = ibh % H, it0 = ich * C + row0;
        mbar_arrive_expect_tx(bar_tma, 3u * tile_bytes + (fused_pro ? 3072u : 0u));
        if (fused_pro) {
            // the item's conv taps: 1 KB per branch, [c][tap] for the head's 128 channels
#pragma unroll
            for (int br = 0; br < 3; ++br)
                bulk_load(sbase + OFF_CW + 1024 * br, pro.conv_w + ((size_t)br * H * D + (size_t)ih * D) * 4, 1024, bar_tma);
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(sbase + OFF_STG_Q + hf * kHalf, ptm_q, bar_tma, hf * 64, ih, it0, ib);
            tma_load_4d(sbase + OFF_STG_K + hf * kHalf, ptm_k, bar_tma, hf * 64, ih, it0, ib);
            tma_load_4d(sbase + OFF_STG_G + hf * kHalf, ptm_g, bar_tma, hf * 64, ih, it0, ib);
        }
    };
    auto issue_v = [&](int item) {
        const int ich = item_ch(item), ibh = item_bh(item);
        const int ib = ibh / H, ih = ibh % H, it0 = ich * C + row0;
        mbar_arrive_expect_tx(bar_v, tile_bytes);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
            tma_load_4d(sbase + OFF_STG_V + hf * kHalf, ptm_v, bar_v, hf * 64, ih, it0, ib);
    };
    if (tid == 0 && cta < nitems) {
        issue_qkg(cta);
        issue_v(cta);
    }
    // beta (with the fused prologue: its logit) of token row tid < C of an item, loaded one
    // item ahead so its global-memory latency overlaps the current item
    auto load_beta = [&](int it) -> float {
        if (tid >= C || it >= nitems) return 0.f;
        const int ich = item_ch(it), ibh = item_bh(it);
        const int t = ich * C + tid;
        if (t >= T) return 0.f;
        const size_t bth = ((size_t)(ibh / H) * T + t) * H + ibh % H;
        return fused_pro ? pro.b_logit[bth] : __bfloat162float(beta[bth]);
    };
    float bpre = load_beta(cta);
    bool ok = true;
    uint32_t li = 0;   // items done by this CTA: parity of the TMA barriers
    int done = -1;     // the item whose record is published next (MEGA)
    // MEGA: the previous record's bulk stores are complete; publish it
    auto publish = [&]() {
        bulk_wait_all();
        if (done >= 0) {
            fence_proxy_async_global();
            flag_release(flags + done, 1);
            done = -1;
        }
    };
    for (int item = cta; item < nitems && ok; item += ncta, ++li) {
        const int ch = item_ch(item), bh = item_bh(item), h = bh % H;
        const int t0 = ch * C, n = min(C, T - t0);
        const int next = item + ncta;
        uint8_t *img = ws + ((size_t)bh * nch + ch) * IMG_BYTES;
        if (tid < C) {
            // the fused prologue rounds beta to bf16 like the standalone prologue kernel
            BET[tid] = tid >= n ? 0.f
                       : fused_pro ? __bfloat162float(__float2bfloat16_rn(sigmoid_fast(bpre)))
                                   : bpre;
        }
        bpre = load_beta(next);
        // MEGA: the first record of each CTA is published at once (the scan starts on the first
        // wave); later ones once the next item reaches its operands, by when the stores are done
        if (MEGA && tid == 0 && li == 1) publish();
        ok = wait_all(bar_tma, li & 1u);
        if (ok && fused_pro) ok = wait_all(bar_v, li & 1u);
        if (ok && fused_pro) {
            // ---- fused prologue: short convolution k = 4 + SiLU of q, k, v and the bounded
            // gate, in place on the staged tiles (halo row i = token t0 - 3 + i; output row r
            // = token t0 + r).  Thread = (branch, 8-channel group, 8-row segment); every input
            // row it needs is read before the barrier, so in-place writes cannot race.
            const int br = tid >> 7, cg = tid & 15, seg = (tid >> 4) & 7;
            const int c0 = 8 * cg, r0 = 8 * seg;
            const uint32_t tile = br == 0 ? OFF_STG_Q : br == 1 ? OFF_STG_K : br == 2 ? OFF_STG_V : OFF_STG_G;
            uint4 raw[C / 8 + kHalo];
#pragma unroll
            for (int i = 0; i < C / 8 + kHalo; ++i)
                raw[i] = *reinterpret_cast<const uint4 *>(smem + tile + off_sw128(r0 + i, c0));
            __syncthreads();
            float w[4][8];   // [tap][channel]; the gate branch needs none
            if (br < 3) {
                const uint8_t *wsrc = smem + OFF_CW + 1024 * br + c0 * 8;   // staged with the tiles
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    float x8[8];
                    unpack8(*reinterpret_cast<const uint4 *>(wsrc + 16 * m), x8);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        w[j][2 * m] = x8[j];
                        w[j][2 * m + 1] = x8[4 + j];
                    }
                }
            }
            const float ea = br == 3 ? expf(pro.A[h]) : 0.f;
            if (br < 3) {
                float x0[8], x1[8], x2[8];   // sliding window: each staged row is unpacked once
                unpack8(raw[0], x0);
                unpack8(raw[1], x1);
                unpack8(raw[2], x2);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float x3[8], y[8];
                    unpack8(raw[i + kHalo], x3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float acc = w[0][e] * x0[e] + w[1][e] * x1[e] + w[2][e] * x2[e] + w[3][e] * x3[e];
                        y[e] = silu_fast(acc);
                        x0[e] = x1[e];
                        x1[e] = x2[e];
                        x2[e] = x3[e];
                    }
                    *reinterpret_cast<uint4 *>(smem + tile + off_sw128(r0 + i, c0)) = pack8(y);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float x3[8], y[8];
                    unpack8(raw[i + kHalo], x3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = -5.f * sigmoid_fast(ea * x3[e]);
                    *reinterpret_cast<uint4 *>(smem + tile + off_sw128(r0 + i, c0)) = pack8(y);
                }
            }
            __syncthreads();
        }

        if (ok) {
            // ---- band-local cumulative log-decay | row norms
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
                const int rr = tid >> 2, part = tid & 3;
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

            // ---- per-channel band factors
            if (tid < D) {
                const int c = tid;
                float et[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) et[p] = __expf(TOT[p * D + c]);
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
                const float gc = ((pc >> bit) & 1u) ? -eC : eC;
                TGC[c] = gc;
                if (c < 4) {
                    PP[0 * 4 + c] = 0u;
                    PP[1 * 4 + c] = BPAR[0 * 4 + c];
                    PP[2 * 4 + c] = BPAR[0 * 4 + c] ^ BPAR[1 * 4 + c];
                    PP[3 * 4 + c] = BPAR[0 * 4 + c] ^ BPAR[1 * 4 + c] ^ BPAR[2 * 4 + c];
                    SGNC[c] = BPAR[0 * 4 + c] ^ BPAR[1 * 4 + c] ^ BPAR[2 * 4 + c] ^ BPAR[3 * 4 + c];
                }
            }
            // the operands overwrite the previous record's sources (W, U, A_qk)
            if (tid == 0) {
                if (MEGA) publish();
                else bulk_wait_read_all();
            }
            __syncthreads();

            // ---- operands (thread = row, 32 channels); Q e^gamma and Kd go straight to the record
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
                        *reinterpret_cast<uint4 *>(smem + OFF_RQG + off_r128(r, c0)) = pack8(y1);
                    } else {
                        float gb[8], inv[8], y2[8];
                        ld8f(TG + band * D + c0, gb);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            inv[e] = __fdividef(x[e], E[e]);
                            y2[e] = (((swc >> (8 * cg + e)) & 1u) ? -inv[e] : inv[e]) * gb[e];
                        }
                        *reinterpret_cast<uint4 *>(smem + OFF_YR + off_r128(r, c0)) = pack8(y1);
                        *reinterpret_cast<uint4 *>(smem + OFF_RKD + off_r128(r, c0)) = pack8(y2);
                    }
                }
                // The band-pair B rows k_i e^{p_b - gamma_i} (one copy per row band b >= band(i)),
                // spread evenly: warp = 8-channel group, lane = key row i in bands 0-1 plus the
                // mirrored row 63 - i in bands 3-2, five copies per lane.
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
                // each writer orders its shared-memory operands (and record parts) before the
                // tensor-core and bulk-copy reads
                fence_proxy_async();
            }
            tmem_wait_st();
            tc_fence_before();
            __syncthreads();

            // ---- all ten band-pair products as one N = 160 product
            if (tid == 0) {
                if (next < nitems) issue_qkg(next);   // q, k, g staging is free from here on
                tc_fence_after();
                constexpr uint32_t id = idesc_bf16(128, 160, 0, 0, 0);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ts(tbase + TC_D, tbase + TC_X + 8 * s, at(dK64, OFF_BOP + 256 * s), id, s > 0);
                mma_commit(bar_mma);
                bulk_store(img + IMG_QG, sbase + OFF_RQG, 16384);
                bulk_store(img + IMG_KD, sbase + OFF_RKD, 16384);
                bulk_store(img + IMG_GC, sbase + OFF_TAB + TAB_GC, 512);
                bulk_commit();
            }
            ok = wait_all(bar_mma, 0);
        }
        if (ok) {
            tc_fence_after();
            // ---- A_kk -> FP32, transposed (AKK[i][r] = A_kk[r][i] for i < r, else 0); A_qk goes to
            // the record while W/U are on the tensor cores
            auto band_rows = [&](float (&v)[16]) {
                const int r = row & 63, band = r >> 4;
                const int b_lo = (quad & 1) * 2;
                float v2[16];
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
            };
            if (row >= 64) {
                const int r = row & 63;
                float v[16];
                band_rows(v);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int i = 16 * qq + e;
                    AKK[i * AS + r] = (i < r) ? v[e] : 0.f;   // a warp writes 32 consecutive r
                }
            }
            tc_fence_before();
            __syncthreads();

            // ---- Tm = (I + A_kk)^{-1} in FP32 by 32 x 32 blocks, [T1 0; T21 T2]:
            //   T1 = (I + A11)^{-1}, T2 = (I + A22)^{-1} from their 16 x 16 diagonal blocks (column
            //   sweeps in registers: x_i is final once the rows above it are done, then
            //   x_r -= A[r][i] x_i for every r > i) and X = -D1 (A10 D0) below them;
            //   Y = A21 T1;  T21 = -T2 Y;  Tm' = Tm diag(beta) in bf16, stacked twice.
            // TMF holds T1 (rows 0-31, columns 0-31), Y (rows 0-31, columns 32-63) and T2 (rows
            // 32-63, columns 32-63).  AKK holds A_kk transposed, zero on and above the diagonal.
            // T1 and T2 from their 16 x 16 diagonal blocks: D_b = (I + A_bb)^{-1} by a column sweep
            // (lane = column, two blocks per warp); then, for each 32-block, Z = A10 D0 and
            // X = -D1 Z (its lower-left quarter), one output per thread, Z in the columns Y takes
            // later.  The upper-right quarters are zero.
            if (warp < 2) {
                const int blk = 2 * warp + (lane >> 4), base = 16 * blk, j = lane & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < 15; ++i) {
                    const float xi = x[i];
                    const float *col = AKK + (base + i) * AS + base;   // A[base + r][base + i] over r
#pragma unroll
                    for (int r4 = ((i + 1) >> 2) << 2; r4 < 16; r4 += 4) {   // rows r <= i hold 0
                        const float4 av = *reinterpret_cast<const float4 *>(col + r4);
                        x[r4] = fmaf(-av.x, xi, x[r4]);
                        x[r4 + 1] = fmaf(-av.y, xi, x[r4 + 1]);
                        x[r4 + 2] = fmaf(-av.z, xi, x[r4 + 2]);
                        x[r4 + 3] = fmaf(-av.w, xi, x[r4 + 3]);
                    }
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) TMF[(base + r) * AS + base + j] = x[r];
                if ((blk & 1) == 0) {
#pragma unroll
                    for (int r = 0; r < 16; ++r) TMF[(base + r) * AS + base + 16 + j] = 0.f;
                }
            }
            __syncthreads();
            {
                // Z = A10 D0 (per 32-block h = tid / 256): row r, column j of the 16 x 16 product
                const int hb = tid >> 8, r = (tid >> 4) & 15, j = tid & 15, base = 32 * hb;
                float z0 = 0.f, z1 = 0.f;
#pragma unroll
                for (int k = 0; k < 16; k += 2) {
                    z0 = fmaf(AKK[(base + k) * AS + base + 16 + r], TMF[(base + k) * AS + base + j], z0);
                    z1 = fmaf(AKK[(base + k + 1) * AS + base + 16 + r], TMF[(base + k + 1) * AS + base + j], z1);
                }
                TMF[r * AS + 32 + 16 * hb + j] = z0 + z1;
            }
            __syncthreads();
            {
                // X = -D1 Z -> rows 16-31 of the 32-block, columns 0-15
                const int hb = tid >> 8, r = (tid >> 4) & 15, j = tid & 15, base = 32 * hb;
                const float *d1 = TMF + (base + 16 + r) * AS + base + 16;
                float x0 = 0.f, x1 = 0.f;
#pragma unroll
                for (int k = 0; k < 16; k += 2) {
                    x0 = fmaf(d1[k], TMF[k * AS + 32 + 16 * hb + j], x0);
                    x1 = fmaf(d1[k + 1], TMF[(k + 1) * AS + 32 + 16 * hb + j], x1);
                }
                TMF[(base + 16 + r) * AS + base + j] = -(x0 + x1);
            }
            __syncthreads();
            // Y = A21 T1 and T21 = -T2 Y as 2 x 4 register tiles (threads 0-127: row pair rg,
            // column group cg), so a warp's loads of a row of one factor and a column group of
            // the other are one shared-memory wavefront each.  Meanwhile threads 128-511 pack the
            // finished blocks of Tm' = [T1 b | 0 ; . | T2 b'] (b = beta_j) to bf16, 16 bytes each.
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
                    // unit u: rows 0-31 x eight 8-column groups (T1 b, then zeros), then rows
                    // 32-63 x the four groups of columns 32-63 (T2 b')
                    const int u = tid - 128;
                    const int r = u < 256 ? (u >> 3) : 32 + ((u - 256) >> 2);
                    const int g = u < 256 ? (u & 7) : 4 + ((u - 256) & 3);
                    float y[8];
                    if (r < 32 && g >= 4) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = 0.f;
                    } else {
                        float t[8], bb[8];
                        ld8f(TMF + r * AS + 8 * g, t);
                        ld8f(BET + 8 * g, bb);
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = t[e] * bb[e];
                    }
                    const uint4 pk = pack8(y);
                    *reinterpret_cast<uint4 *>(smem + OFF_TMB + off_r64(r, 8 * g)) = pk;
                    *reinterpret_cast<uint4 *>(smem + OFF_TMB + off_r64(r + 64, 8 * g)) = pk;
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
                // T21 b -> Tm' rows 32 + 2rg + k, columns 4cg .. 4cg + 3 (8 bytes, both copies)
                const float4 bv = *reinterpret_cast<const float4 *>(BET + 4 * cg);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float y4[4] = {-acc[k][0] * bv.x, -acc[k][1] * bv.y, -acc[k][2] * bv.z, -acc[k][3] * bv.w};
                    const uint2 pk = pack4(y4);
                    *reinterpret_cast<uint2 *>(smem + OFF_TMB + off_r64(32 + 2 * rg + k, 4 * cg)) = pk;
                    *reinterpret_cast<uint2 *>(smem + OFF_TMB + off_r64(96 + 2 * rg + k, 4 * cg)) = pk;
                }
            }
            fence_proxy_async();   // Tm' is read by the tensor cores next
            __syncthreads();

            // ---- W = Tm' (K e^gamma),  U = Tm' V  (M = 128: Tm' stacked twice)
            if (tid == 0) {
                if (!mbar_wait_bounded(bar_v, li & 1u, kWaitLimit)) {
                    sh.abort = 1;
                    g_kda_tc2_error = 1;
                }
                tc_fence_after();
                constexpr uint32_t id = idesc_bf16(128, 128, 0, 1, 0);
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint64_t tdesc = at(dK32, OFF_TMB + 256 * s);
                    mma_ss(tbase + TC_W, tdesc, at(dMN64, OFF_YR + 4096 * s), id, s > 0);
                    mma_ss(tbase + TC_U, tdesc, at(dV, OFF_STG_V + 2048 * s), id, s > 0);
                }
                mma_commit(bar_mma);
            }
            __syncwarp();
            if (row < 64) {
                // A_qk (lower with diagonal) -> bf16 in shared memory, then the record
                const int r = row;
                float v[16];
                band_rows(v);
#pragma unroll
                for (int g8 = 0; g8 < 2; ++g8) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 16 * qq + 8 * g8 + e;
                        y[e] = (i <= r) ? v[8 * g8 + e] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(smem + OFF_RAQ + off_r64(r, 16 * qq + 8 * g8)) = pack8(y);
                }
                fence_proxy_async();
            }
            if (tid == 0) bulk_wait_read_all();   // W and U are staged where Q e^gamma and Kd left from
            ok = wait_all(bar_mma, 1);
            if (ok && tid == 0) {
                if (next < nitems) issue_v(next);   // the v staging is free again
                bulk_store(img + IMG_AQK, sbase + OFF_RAQ, 8192);
                bulk_commit();
            }
        }
        if (ok) {
            tc_fence_after();
            // ---- W ([r][c], K-major core layout) and U (16-column slabs) -> the record; lanes
            // 0-63 write W, lanes 64-127 (the repeated rows) write U
            {
                const int r = row & 63;
                float w[32];
                tmem_ld32(tl + (row < 64 ? TC_W : TC_U) + 32 * qq, w);
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = w[8 * g8 + e];
                    const int c0 = 32 * qq + 8 * g8;
                    *reinterpret_cast<uint4 *>(smem + OFF_RWU + (row < 64 ? off_r128(r, c0) : 16384 + off_u(r, c0))) =
                        pack8(y);
                }
                fence_proxy_async();
            }
        }
        // the next item rewrites TMEM and shared memory: everyone is done with this one
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (ok && tid == 0) {
            bulk_store(img + IMG_W, sbase + OFF_RWU, 16384);
            bulk_store(img + IMG_U, sbase + OFF_RWU + 16384, 16384);
            bulk_commit();
            done = item;
        }
    }
    if (tid == 0) {
        if (MEGA) publish();
        else bulk_wait_all();   // the records are complete before the scan reads them
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

template <bool PRO>
__global__ void __launch_bounds__(prep::NT, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ ws, int T, int H,
                  int BH, KernelFlags fl, PrepPrologue pro) {
    prep_body<PRO, false>(&tm_q, &tm_k, &tm_v, &tm_g, beta, ws, T, H, BH, fl, pro, (int)blockIdx.x,
                          (int)gridDim.x, nullptr);
}

// The prep with two item groups per CTA (kda_chunk_prep.cuh): one 512-thread CTA per SM, its
// TMEM split between the groups.  MEGA: CTA `cta` of `ncta` prep CTAs of the one-launch form.
template <bool PRO, bool MEGA>
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
    prep2_group<PRO, MEGA>(ptm_q, ptm_k, ptm_v, ptm_g, beta, ws, T, H, BH, fl, pro, gi,
                           smem + gi * prep2::GROUP_STRIDE, tbase + 256u * gi, prep2::NG * cta + gi,
                           prep2::NG * ncta, flags, wait_limit);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

template <bool PRO>
__global__ void __launch_bounds__(prep2::NT, 1)
chunk_prep2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                   const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ ws, int T, int H, int BH,
                   KernelFlags fl, PrepPrologue pro, uint32_t wait_limit) {
    prep2_cta<PRO, false>(&tm_q, &tm_k, &tm_v, &tm_g, beta, ws, T, H, BH, fl, pro, (int)blockIdx.x,
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

template <int NS, bool GATED>
__global__ void __launch_bounds__(scan::Layout<NS>::NT, 1)
chunk_scan_tc_kernel(const uint8_t *__restrict__ ws, const float *__restrict__ S0,
                     __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, int T, int H,
                     float scale, const __nv_bfloat16 *__restrict__ gate,
                     const float *__restrict__ norm_w, float norm_eps) {
    scan_body<NS, GATED, false>(ws, S0, out, S_T, T, H, scale, gate, norm_w, norm_eps, (int)blockIdx.x,
                                nullptr, 0);
}

// One launch for few-head calls: CTAs [0, n_scan) run the scan's slice CTAs, the rest the prep,
// all resident at once (a cooperative launch), the scan reading each record as soon as the
// prep has published it.  The block has the prep's 512 threads; a scan CTA uses its first
// 32 * (NSW + 2) (state warps, the MMA warp, the loader warp).
// dynamic shared memory of the one-launch form: the larger of the two roles' layouts
template <int NS>
constexpr uint32_t mega_smem_bytes() {
    return prep::SMEM_BYTES > scan::Layout<NS>::SMEM_BYTES ? prep::SMEM_BYTES : scan::Layout<NS>::SMEM_BYTES;
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

template <bool PRO, int NS>
__global__ void __launch_bounds__(prep::NT, 1)
chunk_mega_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ ws, int T, int H,
                  int BH, KernelFlags fl, PrepPrologue pro, const float *__restrict__ S0,
                  __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, int n_scan,
                  int *__restrict__ flags) {
    if ((int)blockIdx.x < n_scan)
        mega_scan<NS>(ws, S0, out, S_T, T, H, fl.scale, (int)blockIdx.x, flags, BH);
    else
        prep_body<PRO, true>(&tm_q, &tm_k, &tm_v, &tm_g, beta, ws, T, H, BH, fl, pro,
                             (int)blockIdx.x - n_scan, (int)gridDim.x - n_scan, flags);
}

// The one-launch form with the two-group prep: prep CTAs are 512 threads of two item groups.
template <int NS>
constexpr uint32_t mega2_smem_bytes() {
    return prep2::SMEM_BYTES > scan::Layout<NS>::SMEM_BYTES ? prep2::SMEM_BYTES : scan::Layout<NS>::SMEM_BYTES;
}

template <bool PRO, int NS>
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
        prep2_cta<PRO, true>(&tm_q, &tm_k, &tm_v, &tm_g, beta, ws, T, H, BH, fl, pro, (int)blockIdx.x - n_scan,
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
static bool use_prep2(const ChunkArgs &a);

cudaError_t launch_chunk_tc2(const ChunkArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mg;
    if (!make_map2(&mq, a.q, a.B, a.T, a.H) || !make_map2(&mk, a.k, a.B, a.T, a.H) ||
        !make_map2(&mv, a.v, a.B, a.T, a.H) || !make_map2(&mg, a.g, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    return launch_split(a, mq, mk, mv, mg, PrepPrologue{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr}, st);
}

cudaError_t launch_chunk_tc2_prologue(const PrologueArgs &p, const ChunkArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mz;
    // the one-group prep stages a 3-row halo with each tile; the two-group prep reads those rows
    // from global memory and stages 64-row tiles
    const int rows = use_prep2(a) ? C : C + prep::kHalo;
    if (!make_map2(&mq, p.q_pre, a.B, a.T, a.H, rows) || !make_map2(&mk, p.k_pre, a.B, a.T, a.H, rows) ||
        !make_map2(&mv, p.v_pre, a.B, a.T, a.H, rows) || !make_map2(&mz, p.z, a.B, a.T, a.H, rows))
        return cudaErrorInvalidValue;
    return launch_split(a, mq, mk, mv, mz,
                        PrepPrologue{(const __nv_bfloat16 *)p.conv_w, p.A, p.beta_logit, (const __nv_bfloat16 *)p.q_pre,
                                     (const __nv_bfloat16 *)p.k_pre, (const __nv_bfloat16 *)p.v_pre},
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

// Per-(chunk, head) prep cost per SM (cycles; the two-group prep overlaps two items per SM) and
// per-chunk scan chain at d = 128 on a B200 SM (measured).
constexpr double kPrepItemCycles = 21000.0;
constexpr double kPrep2ItemCycles = 7000.0;
static double scan_chunk_cycles(int ns) { return ns == 16 ? 2900.0 : ns == 32 ? 3000.0 : ns == 64 ? 3100.0 : 4900.0; }

// Polls of a bounded wait before it gives up (kda_set_wait_limit; failure-handling tests only).
static uint32_t g_wait_limit = kWaitLimit;

// Slice width of the one-launch form (prep and scan CTAs side by side), or 0 when the two
// launches are faster: prep on all SMs, then the scan, against the prep on the SMs the scan's
// CTAs leave, overlapped with the scan, plus one item of ramp.
int mega_slice_width(int BH, int nch, int sms, double t_item) {
    const double items = (double)BH * nch;
    const double two = ceil(items / sms) * t_item + nch * scan_chunk_cycles(scan_slice_width(BH, false));
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

// Whether the two-group prep runs (all unsigned-gate calls; Complex-KDA keeps the one-group prep).
static bool use_prep2(const ChunkArgs &a) { return !a.fl.complex_gate && getenv("KDA_PREP_FORM") == nullptr; }

template <bool PRO, int NS>
static cudaError_t launch_mega(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                               const CUtensorMap &mv, const CUtensorMap &mg, PrepPrologue pro, cudaStream_t st) {
    const bool v2 = use_prep2(a);
    auto k = chunk_mega_kernel<PRO, NS>;
    auto k2 = chunk_mega2_kernel<PRO, NS>;
    constexpr uint32_t smem1 = mega_smem_bytes<NS>(), smem2 = mega2_smem_bytes<NS>();
    static_assert(smem1 <= 232448 && smem2 <= 232448, "shared memory budget");
    static_assert(scan::Layout<NS>::NT + 32 <= prep::NT, "the scan's warps and the loader warp fit the prep's block");
    static_assert(prep::NT == prep2::NT, "one block size for both prep forms");
    const uint32_t smem = v2 ? smem2 : smem1;
    cudaError_t e = v2 ? cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
                       : cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nch = (a.T + C - 1) / C, BH = a.B * a.H, n_scan = BH * (D / NS);
    uint8_t *ws = (uint8_t *)a.workspace;
    int *flags = reinterpret_cast<int *>(ws + (size_t)nch * BH * IMG_BYTES);
    e = cudaMemsetAsync(flags, 0, (size_t)nch * BH * sizeof(int), st);
    if (e != cudaSuccess) return e;
    // every CTA resident at once (the scan CTAs wait for records the prep CTAs publish)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms());
    cfg.blockDim = dim3(prep::NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    mark_launch(a, st);
    if (v2)
        return cudaLaunchKernelEx(&cfg, k2, mq, mk, mv, mg, (const __nv_bfloat16 *)a.beta, ws, a.T, a.H, BH, a.fl,
                                  pro, a.S0, (__nv_bfloat16 *)a.out, a.S_T, n_scan, flags, g_wait_limit);
    return cudaLaunchKernelEx(&cfg, k, mq, mk, mv, mg, (const __nv_bfloat16 *)a.beta, ws, a.T, a.H, BH, a.fl, pro,
                              a.S0, (__nv_bfloat16 *)a.out, a.S_T, n_scan, flags);
}

static cudaError_t launch_split(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                                const CUtensorMap &mv, const CUtensorMap &mg, PrepPrologue pro,
                                cudaStream_t st) {
    const bool v2 = use_prep2(a);
    if (!a.out_gate) {
        const int ns = mega_slice_width(a.B * a.H, (a.T + C - 1) / C, num_sms(), v2 ? kPrep2ItemCycles : kPrepItemCycles);
        if (ns) {
            const bool p = pro.conv_w != nullptr;
            cudaError_t e = ns == 32 ? (p ? launch_mega<true, 32>(a, mq, mk, mv, mg, pro, st)
                                          : launch_mega<false, 32>(a, mq, mk, mv, mg, pro, st))
                                     : (p ? launch_mega<true, 64>(a, mq, mk, mv, mg, pro, st)
                                          : launch_mega<false, 64>(a, mq, mk, mv, mg, pro, st));
            if (e != cudaErrorCooperativeLaunchTooLarge) return e;
            (void)cudaGetLastError();   // not enough room to co-schedule: the two launches below
        }
    }
    // the plain instantiations carry none of the prologue or epilogue code
    const int nch = (a.T + C - 1) / C;
    uint8_t *ws = (uint8_t *)a.workspace;
    const int nitems = nch * a.B * a.H;
    cudaError_t e;
    if (v2) {
        auto prep_k = pro.conv_w ? chunk_prep2_kernel<true> : chunk_prep2_kernel<false>;
        e = cudaFuncSetAttribute(prep_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep2::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        mark_launch(a, st);
        const int ctas = std::min((nitems + prep2::NG - 1) / prep2::NG, num_sms());
        prep_k<<<(unsigned)ctas, prep2::NT, prep2::SMEM_BYTES, st>>>(mq, mk, mv, mg, (const __nv_bfloat16 *)a.beta, ws,
                                                                    a.T, a.H, a.B * a.H, a.fl, pro, g_wait_limit);
    } else {
        auto prep_k = pro.conv_w ? chunk_prep_kernel<true> : chunk_prep_kernel<false>;
        e = cudaFuncSetAttribute(prep_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        mark_launch(a, st);
        prep_k<<<(unsigned)std::min(nitems, num_sms()), prep::NT, prep::SMEM_BYTES, st>>>(
            mq, mk, mv, mg, (const __nv_bfloat16 *)a.beta, ws, a.T, a.H, a.B * a.H, a.fl, pro);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    mark_launch(a, st);
    if (a.out_gate) return launch_scan<D, true>(a, ws, st);
    switch (scan_slice_width(a.B * a.H, false)) {
        case 16: return launch_scan<16, false>(a, ws, st);
        case 32: return launch_scan<32, false>(a, ws, st);
        case 64: return launch_scan<64, false>(a, ws, st);
        default: return launch_scan<D, false>(a, ws, st);
    }
}

}  // namespace kda
