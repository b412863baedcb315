// kda_chunk_prep.cuh -- the split form's per-(chunk, head) prep, two items in flight per SM.
//
// Included by kda_chunk_tc2.cu after the record layout.  Everything up to the WY vectors
// depends on one chunk's inputs only (page "Kimi K3 模型结构（2）：序列维度（下），chunkwise 并行与
// 下界衰减", Q&A items on the chunkwise algorithm, the -5 decay floor and the intra-chunk matrix
// A), so the work is cut into (chunk, head) items.  A 512-thread CTA holds two independent item
// groups of 256 threads, each with its own 112 KB of shared memory, 256 TMEM columns, mbarriers
// and named barrier: while one group waits (a TMA tile, a tensor-core product, a barrier), the
// other issues.  Per item:
//
//   TMA       q, k (interleaved by 64-channel halves so [q; k] is one 128-row K-major operand),
//             g and v tiles [64 tokens x 128], 128-byte swizzle
//   tcgen05   band-local cumulative log-decay: gamma~ = L g with L = [L_band; L_band] (ones on
//             and below the diagonal inside each 16-token band; constant A operand in TMEM);
//             exact in FP32 (bf16 g times 1, FP32 sums)
//   CUDA      row norms of q and k, band totals of g (while the cumsum runs); per-channel band
//             factors e^{p_b}, e^{gamma_C - p_b}, e^{p_b' - p_b} (p_b = gamma before band b)
//   CUDA      thread = (token row, 32 channels): E = e^{gamma~} in [e^-80, 1] and 1/E, then in
//             place Q E and beta K E (the band-pair A operand), K e^gamma over g (the W product's
//             B operand), the band-pair B rows k_i e^{p_b - gamma_i} for b >= band(i), and the
//             record's Q e^gamma and K e^{gamma_C - gamma} straight to global memory
//   tcgen05   A_qk / A_kk: the ten (row band, column band) pairs as one N = 160 product
//   CUDA      A_qk -> record; Tm = (I + A_kk)^{-1} in FP32 (16x16 diagonal blocks, then 32x32)
//   tcgen05   [W; U] = [Tm' 0; 0 Tm'] [K e^gamma; V]  (Tm' = Tm diag(beta), block-diagonal A
//             operand in TMEM, one M = 128, K = 128 product)
//   CUDA      W, U -> record
//
// The record (74,240 bytes per chunk and head) has the layout the scan kernel reads.
//
// UNB (a gate without the -5 floor: Kimi Linear's softplus map, same page, Q&A on how the decay
// map differs from Kimi Linear's): the band-referenced factors of the band's own keys,
// e^{p_b - gamma_i}, have no bound.  Only the six off-diagonal band pairs stay on the tensor
// cores (N = 96), with every factor formed as one exponential of a non-positive difference;
// the four diagonal 16 x 16 blocks are FP32 position pairs, sum_c q_rc k_ic prod_{i<s<=r} alpha_sc,
// with the products of alpha = e^g taken row by row (no factor above 1, underflow harmless).
#pragma once

namespace prep2 {
constexpr int NG = 2;                  // item groups per CTA
constexpr int GT = 256;                // threads per group
constexpr int NT = NG * GT;
// shared memory of one group (bytes from its 1024-aligned base)
constexpr uint32_t OFF_X = 0;          // q, k staging [q h0][k h0][q h1][k h1] (8 KB each)
constexpr uint32_t OFF_G = 32768;      // g staging [h0][h1]; later K e^gamma
constexpr uint32_t OFF_V = 49152;      // v staging [h0][h1]
constexpr uint32_t OFF_KH = 65536;     // band-pair B operand, K-major 128-byte swizzle, 160 rows per
                                       // 64-channel half; before it: band totals; after it: the
                                       // UT inverse's A_kk^T and T (FP32)
constexpr uint32_t KH_HALF = 20480;
constexpr uint32_t OFF_TOT = OFF_KH;           // FP32 [4 bands][128]
constexpr uint32_t AS = 68;                    // row stride (floats) of the UT's FP32 tiles
constexpr uint32_t OFF_AKT = OFF_KH;           // A_kk^T [64 i][68] (A_kk[r][i] at i * AS + r)
constexpr uint32_t OFF_TMF = OFF_KH + 17408;   // T [64 r][68]
constexpr uint32_t OFF_TAB = 106496;
// per-channel band factors, FP32 rows of 128 (p_b = gamma before band b, e_b = e^{band b's total}):
// e_0..e_3, e^{p_2}, e^{p_3}, e^{gamma_C - p_0..2}, e^{p_2 - p_0}, e^{p_3 - p_1}, e^{p_3 - p_0}, ones
constexpr int R_ET = 0, R_EP2 = 4, R_EP3 = 5, R_ECP = 6, R_EM20 = 9, R_EM31 = 10, R_EM30 = 11, R_ONE = 12;
constexpr uint32_t TAB_F = 0;          // 13 rows x 512 B
constexpr uint32_t TAB_NRMP = 6656;    // FP32 sums of squares [2 halves][128 rows: q, then k]
constexpr uint32_t TAB_BET = 7680;     // FP32 beta [64]
constexpr uint32_t TAB_BAR = 7936;     // mbarriers and the abort flag
constexpr uint32_t TAB_PX = TAB_BAR + 64;   // Complex-KDA: sign parity of each warp's 32 rows [8]
constexpr uint32_t GROUP_USED = OFF_TAB + TAB_PX + 32;
constexpr uint32_t OFF_LO = OFF_KH;    // Complex-KDA: the low bf16 part of log|alpha| (g's layout)
constexpr uint32_t GROUP_STRIDE = 114688;
// UNB: alpha = e^g (FP32 [64 r][128 c]) after the band totals while the diagonal blocks are
// formed; the blocks wait in the region's last 6 KB for the readout (the six off-diagonal pairs'
// B rows are rows 0-95 of each half)
constexpr uint32_t OFF_ALPHA = OFF_KH + 2048;
constexpr uint32_t OFF_DQ = OFF_KH + 34816;    // A_qk's diagonal blocks, bf16 [4 bands][16 r][16 i]
constexpr uint32_t OFF_DK = OFF_KH + 36864;    // A_kk's diagonal blocks, FP32 [4 bands][16 r][16 i]
constexpr int NPAIR_U = 96;
// UNB band factors, FP32 rows of 128 (T_b = band b's total, p_b = T_0 + .. + T_{b-1},
// gamma_C = p_4): as logarithms T_0..T_3, T_0+T_1, T_1+T_2, T_0+T_1+T_2, gamma_C - p_0..2; then
// e^{p_1}, e^{p_2}, e^{p_3} (each <= 1)
constexpr int R_LT = 0, R_L01 = 4, R_L12 = 5, R_L012 = 6, R_LC = 7, R_EXP = 10;
constexpr uint32_t SMEM_BYTES = 1024 + GROUP_STRIDE + GROUP_USED;
static_assert(GROUP_USED <= GROUP_STRIDE, "group layout");
static_assert(OFF_TMF + 17408 <= OFF_TAB, "UT tiles inside the band-pair operand's region");
static_assert(SMEM_BYTES <= 232448 - 256, "shared memory budget");
static_assert(OFF_ALPHA + 32768 <= OFF_DQ && OFF_DK + 4096 <= OFF_TAB, "UNB staging inside the band-pair region");
static_assert(OFF_KH + KH_HALF + NPAIR_U * 128 <= OFF_DQ, "UNB B rows clear of the diagonal blocks");
// TMEM columns of a group (its 256): D = cumsum / band pairs / [W; U]; the block-diagonal
// Tm' operand; the constant cumsum operand L
constexpr uint32_t TC_D = 0, TC_TM = 160, TC_LM = 224;

struct alignas(8) GroupBars {
    uint64_t qk, g, v, m1, m2, m3;
    int abort;
};

// q / k (t = 0 / 1) unit (token row r, 8-channel group cg) in the interleaved staging
__device__ __forceinline__ uint32_t off_x(int t, int r, int cg) {
    return (uint32_t)((cg >> 3) * 16384 + t * 8192 + r * 128 + (((cg & 7) ^ (r & 7)) << 4));
}
// g / v staging (and K e^gamma over g): one tile of two 8 KB halves
__device__ __forceinline__ uint32_t off_t(int r, int cg) {
    return (uint32_t)((cg >> 3) * 8192 + r * 128 + (((cg & 7) ^ (r & 7)) << 4));
}
// band-pair B row n (0..159)
__device__ __forceinline__ uint32_t off_kh(int n, int cg) {
    return (uint32_t)((cg >> 3) * KH_HALF + n * 128 + (((cg & 7) ^ (n & 7)) << 4));
}
// factor rows: e^{p_b}, e^{gamma_C - p_b}, e^{p_b' - p_b} (b' > b)
__device__ __forceinline__ int row_ep(int b) { return b == 0 ? R_ONE : b == 1 ? R_ET + 0 : b == 2 ? R_EP2 : R_EP3; }
__device__ __forceinline__ int row_ecp(int b) { return b == 3 ? R_ET + 3 : R_ECP + b; }
__device__ __forceinline__ int row_em(int bp, int b) {
    return bp == b + 1 ? R_ET + b : (bp == 2 ? R_EM20 : b == 1 ? R_EM31 : R_EM30);
}
// UNB log rows: gamma_C - p_b, p_b' - p_b (b' > b)
__device__ __forceinline__ int lrow_c(int b) { return b == 3 ? R_LT + 3 : R_LC + b; }
__device__ __forceinline__ int lrow_m(int bp, int b) {
    return bp == b + 1 ? R_LT + b : (bp == 2 ? R_L01 : b == 1 ? R_L12 : R_L012);
}
// UNB: TMEM column block (16 columns) of the off-diagonal band pair (row band b, key band j < b)
__device__ __forceinline__ int pair_u(int b, int j) { return (j == 0 ? 0 : j == 1 ? 3 : 5) + b - j - 1; }
}  // namespace prep2

// Wait for phase `ph` of `bar` with the built-in limit, whatever the run's wait limit: used at
// exit only, so the copies and products a group has in flight land before its TMEM and shared
// memory are released, even when the run's waits were set to give up early.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t ph) {
    (void)mbar_wait_bounded(bar, ph, kWaitLimit);
}

// Group-local barrier (named barrier 1 + group, 256 threads).
__device__ __forceinline__ void gbar(int gi) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + gi), "r"(prep2::GT) : "memory");
}
// The same barrier, returning whether any of the group's threads passed p = true: every thread
// gets the same answer, so a give-up seen by one thread ends the item loop for all of them.
__device__ __forceinline__ bool gbar_or(int gi, bool p) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.or.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(1 + gi), "r"(prep2::GT)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// bf16 pair -> two floats (the low element first), one integer op each
__device__ __forceinline__ float2 bf2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t pk2(float2 v) { return pack_bf16(v.x, v.y); }
// packed FP32 pair arithmetic (one instruction per pair on sm_100)
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 dup2(float a) { return make_float2(a, a); }
// 2^x with the hardware approximation (relative error about 2^-22)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float tanh_hw(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// SiLU of a pair: x sigmoid(x), sigmoid(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh
__device__ __forceinline__ float2 silu2(float2 x) {
    const float2 h = mul2(x, dup2(0.5f));
    const float2 t = make_float2(tanh_hw(h.x), tanh_hw(h.y));
    return mul2(x, fma2(t, dup2(0.5f), dup2(0.5f)));
}
__device__ __forceinline__ uint4 ld16(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void st16(uint8_t *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}
__device__ __forceinline__ void ld4f2(const float *p, float2 (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = make_float2(a.x, a.y);
    v[1] = make_float2(a.z, a.w);
    v[2] = make_float2(b.x, b.y);
    v[3] = make_float2(b.z, b.w);
}

// The prep's work for one item group.  vc / nv: this group's index among all groups of the
// prep CTAs and their number.  MEGA: items are taken chunk-major and each record is published
// (flags[item], release) once its stores are visible; otherwise items are taken chunk-fastest
// and the scan is the next kernel.  PRO: the tiles hold the raw branch inputs and z; the short
// convolution, SiLU, the gate and beta = sigmoid(logit) run on chip first.  UNB: g has no
// lower bound (see the top of this file).
template <bool PRO, bool MEGA, bool UNB>
__device__ __forceinline__ void
prep2_group(const CUtensorMap *ptm_q, const CUtensorMap *ptm_k, const CUtensorMap *ptm_v,
            const CUtensorMap *ptm_g, const __nv_bfloat16 *__restrict__ beta, uint8_t *__restrict__ ws,
            int T, int H, int BH, KernelFlags fl, PrepPrologue pro, int gi, uint8_t *gsm, uint32_t gtm, int vc,
            int nv, int *__restrict__ flags, uint32_t wait_limit) {
    using namespace prep2;
    const uint32_t gs = smem_u32(gsm);
    float *TOT = reinterpret_cast<float *>(gsm + OFF_TOT);
    float *FT = reinterpret_cast<float *>(gsm + OFF_TAB + TAB_F);
    float *NRMP = reinterpret_cast<float *>(gsm + OFF_TAB + TAB_NRMP);
    float *BET = reinterpret_cast<float *>(gsm + OFF_TAB + TAB_BET);
    uint32_t *PX = reinterpret_cast<uint32_t *>(gsm + OFF_TAB + TAB_PX);
    float *AKT = reinterpret_cast<float *>(gsm + OFF_AKT);
    float *TMF = reinterpret_cast<float *>(gsm + OFF_TMF);
    GroupBars *gb = reinterpret_cast<GroupBars *>(gsm + OFF_TAB + TAB_BAR);
    const uint32_t b_qk = smem_u32(&gb->qk), b_g = smem_u32(&gb->g), b_v = smem_u32(&gb->v),
                   b_m1 = smem_u32(&gb->m1), b_m2 = smem_u32(&gb->m2), b_m3 = smem_u32(&gb->m3);
    volatile int *abort_f = &gb->abort;

    const int gt = threadIdx.x - gi * GT;       // thread within the group
    const int gw = gt >> 5, lane = gt & 31;     // warp within the group (TMEM quadrant gw & 3)
    const int qd = gw & 3;
    const uint32_t tl = gtm + ((uint32_t)(qd * 32) << 16);   // this warp's TMEM lanes
    const int nch = (T + C - 1) / C;
    const int nitems = nch * BH;
    constexpr uint32_t kTile = 8192;             // one 64-row x 64-channel box

    if (gt == 0) {
        mbar_init(b_qk, 1);
        mbar_init(b_g, 1);
        mbar_init(b_v, 1);
        mbar_init(b_m1, 1);
        mbar_init(b_m2, 1);
        mbar_init(b_m3, 1);
        mbar_fence_init();
        *abort_f = 0;
    }
    if (!UNB && gt < 128) FT[R_ONE * 128 + gt] = 1.f;
    // constant TMEM operands: L = [L_band; L_band] (lane m, row m & 63: ones at s <= row inside
    // the row's band), and the zero halves of the block-diagonal Tm' operand
    if (gw < 4) {
        const int m = qd * 32 + lane, rr = m & 63;
        uint32_t lv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int s0 = 2 * j, s1 = 2 * j + 1;
            const uint32_t lo = ((s0 >> 4) == (rr >> 4) && s0 <= rr) ? 0x3F80u : 0u;
            const uint32_t hi = ((s1 >> 4) == (rr >> 4) && s1 <= rr) ? 0x3F80u : 0u;
            lv[j] = lo | (hi << 16);
        }
        tmem_st32(tl + TC_LM, lv);
        uint32_t z[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = 0u;
        tmem_st32(tl + TC_TM + (qd < 2 ? 32 : 0), z);
        tmem_wait_st();
    }
    tc_fence_before();
    gbar(gi);
    tc_fence_after();

    // MN-major [K rows][N] tiles (g / K e^gamma, v): 64-channel halves 8 KB apart, 8-row groups 1 KB
    const uint64_t dT = sdesc(gs, 8192, 1024, kSwizzle128B);
    auto at = [](uint64_t base, uint32_t off) -> uint64_t { return base + (uint64_t)(off >> 4); };
    // A bounded wait by every calling thread (mbarrier try-wait polls without a sleep between
    // them: measured 2 % faster than backing off); giving up (or seeing another thread's
    // give-up) sets this thread's `bad`; the group leaves the item loop together at the next
    // gbar_or.
    bool bad = false;
    auto wait = [&](uint32_t bar, uint32_t phase) -> bool {
        for (uint32_t i = 0; i < wait_limit; ++i) {
            if (mbar_try_wait(bar, phase)) return true;
            if (*abort_f) {
                bad = true;
                return false;
            }
        }
        *abort_f = 1;
        g_kda_tc2_error = 1;
        bad = true;
        return false;
    };

    auto item_ch = [&](int item) { return MEGA ? item / BH : item % nch; };
    auto item_bh = [&](int item) { return MEGA ? item % BH : item / nch; };
    // TMA: q and k on one barrier, g and v on one each
    auto issue_qk = [&](int item) {
        const int ich = item_ch(item), ibh = item_bh(item), ib = ibh / H, ih = ibh % H, it0 = ich * C;
        mbar_arrive_expect_tx(b_qk, 4u * kTile);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(gs + OFF_X + hf * 16384, ptm_q, b_qk, hf * 64, ih, it0, ib);
            tma_load_4d(gs + OFF_X + hf * 16384 + 8192, ptm_k, b_qk, hf * 64, ih, it0, ib);
        }
    };
    auto issue_gv = [&](int item) {
        const int ich = item_ch(item), ibh = item_bh(item), ib = ibh / H, ih = ibh % H, it0 = ich * C;
        mbar_arrive_expect_tx(b_g, 2u * kTile);
        mbar_arrive_expect_tx(b_v, 2u * kTile);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(gs + OFF_G + hf * 8192, ptm_g, b_g, hf * 64, ih, it0, ib);
            tma_load_4d(gs + OFF_V + hf * 8192, ptm_v, b_v, hf * 64, ih, it0, ib);
        }
    };
    // completions issued and consumed per barrier (thread 0 of the group), for the drain:
    // qk, g, v, m1, m2, m3
    uint32_t iss[6] = {0, 0, 0, 0, 0, 0}, con[6] = {0, 0, 0, 0, 0, 0};
    if (gt == 0 && vc < nitems) {
        issue_qk(vc);
        issue_gv(vc);
        iss[0] = iss[1] = iss[2] = 1;
    }
    // beta (or its logit) of token row gt < C, one item ahead
    auto load_beta = [&](int it) -> float {
        if (gt >= C || it >= nitems) return 0.f;
        const int ich = item_ch(it), ibh = item_bh(it), t = ich * C + gt;
        if (t >= T) return 0.f;
        const size_t bth = ((size_t)(ibh / H) * T + t) * H + ibh % H;
        return PRO ? pro.b_logit[bth] : __bfloat162float(beta[bth]);
    };
    float bpre = load_beta(vc);
    uint32_t li = 0;
    for (int item = vc; item < nitems; item += nv, ++li) {
        const int ch = item_ch(item), bh = item_bh(item), b = bh / H, h = bh % H;
        const int t0 = ch * C, n = min(C, T - t0);
        const int next = item + nv;
        uint8_t *img = ws + ((size_t)bh * nch + ch) * IMG_BYTES;
        if (gt < C)
            BET[gt] = gt >= n ? 0.f : PRO ? __bfloat162float(__float2bfloat16_rn(sigmoid_fast(bpre))) : bpre;
        bpre = load_beta(next);
        const uint32_t ph = li & 1u;
        // PRO: the global-memory inputs of the convolution (the three rows before the chunk for
        // the first segment, the head's taps, A_h) are loaded before the tile wait, so their
        // latency overlaps it
        const int br = gt >> 6, pcg = ((gt >> 5) & 1) * 8 + (gt & 7), seg = (gt >> 3) & 3;
        uint4 halo[3];
        float a_h = 0.f;
        if constexpr (PRO) {
            if (br < 3) {
                const __nv_bfloat16 *rawp = br == 0 ? pro.raw_q : br == 1 ? pro.raw_k : pro.raw_v;
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    const int t = t0 - 3 + j;
                    halo[j] = (seg == 0 && t >= 0)
                                  ? *reinterpret_cast<const uint4 *>(rawp + (((size_t)b * T + t) * H + h) * D + 8 * pcg)
                                  : make_uint4(0, 0, 0, 0);
                }
            } else {
                a_h = pro.A[h];
            }
        }
        if (wait(b_qk, ph) && gt == 0) ++con[0];
        if constexpr (PRO) {
            // ---- short convolution k = 4 + SiLU of q, k, v and the bounded gate, in place.
            // Thread = (branch, 8-channel group, 16-row segment) for q, k, v (192 threads), or
            // (8-channel group, 16-row segment) for the gate (64 threads).  The three rows before
            // a segment come from the segment above (read before the barrier, so the in-place
            // writes cannot race) or, for the first segment, from global memory (zero before t = 0).
            // q and k (threads 0-127) start as soon as their tiles are in; v and the gate (threads
            // 128-255) wait for theirs, which were issued last.  Each half has its own barrier
            // for the in-place hazard (named barriers 3 + 2 gi and 4 + 2 gi, 128 threads).
            if (gbar_or(gi, bad)) break;
            if (br >= 2) {
                wait(b_g, ph);
                wait(b_v, ph);
            }
            const int sub_bar = 3 + 2 * gi + (br >= 2 ? 1 : 0);
            // lanes of a quarter-warp take the 8 channel groups of one row: conflict-free
            const int cg = pcg, r0 = 16 * seg;
            const uint32_t ubase = br == 0 ? OFF_X : br == 1 ? OFF_X + 8192 : br == 2 ? OFF_V : OFF_G;
            auto unit = [&](int r) -> uint32_t {
                return ubase + (br < 2 ? (uint32_t)((cg >> 3) * 16384) : (uint32_t)((cg >> 3) * 8192)) +
                       (uint32_t)(r * 128 + (((cg & 7) ^ (r & 7)) << 4));
            };
            if (br < 3) {
                float2 xm[3][4];   // rows r0 - 3 .. r0 - 1, channel pairs
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    const uint4 u = seg > 0 ? ld16(gsm + unit(r0 - 3 + j)) : halo[j];
                    xm[j][0] = bf2(u.x);
                    xm[j][1] = bf2(u.y);
                    xm[j][2] = bf2(u.z);
                    xm[j][3] = bf2(u.w);
                }
                float2 w[4][4];   // [tap][channel pair]: the head's taps, [c][tap] in memory
                const uint4 *wsrc = reinterpret_cast<const uint4 *>(pro.conv_w + ((size_t)br * H * D + (size_t)h * D + 8 * cg) * 4);
#pragma unroll
                for (int m = 0; m < 4; ++m) {   // channels 2m, 2m + 1
                    const uint4 u = wsrc[m];
                    const float2 a = bf2(u.x), bq = bf2(u.y), c2 = bf2(u.z), d2 = bf2(u.w);   // taps (0,1),(2,3) of 2m; of 2m+1
                    w[0][m] = make_float2(a.x, c2.x);
                    w[1][m] = make_float2(a.y, c2.y);
                    w[2][m] = make_float2(bq.x, d2.x);
                    w[3][m] = make_float2(bq.y, d2.y);
                }
                asm volatile("bar.sync %0, %1;" ::"r"(sub_bar), "r"(128) : "memory");
                const bool tail = n < C;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const int r = r0 + i;
                    const uint4 u = ld16(gsm + unit(r));
                    const float2 x3[4] = {bf2(u.x), bf2(u.y), bf2(u.z), bf2(u.w)};
                    uint32_t y[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        float2 acc = mul2(w[0][m], xm[0][m]);
                        acc = fma2(w[1][m], xm[1][m], acc);
                        acc = fma2(w[2][m], xm[2][m], acc);
                        acc = fma2(w[3][m], x3[m], acc);
                        y[m] = pk2(silu2(acc));
                        xm[0][m] = xm[1][m];
                        xm[1][m] = xm[2][m];
                        xm[2][m] = x3[m];
                    }
                    if (tail && r >= n) y[0] = y[1] = y[2] = y[3] = 0u;
                    st16(gsm + unit(r), y[0], y[1], y[2], y[3]);
                }
            } else if (pro.softplus) {
                // Kimi Linear's map g = -e^A softplus(z), softplus(z) = max(z, 0) + ln(1 + e^-|z|)
                const float ea = expf(a_h);
                constexpr float kL2E = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
                asm volatile("bar.sync %0, %1;" ::"r"(sub_bar), "r"(128) : "memory");
                const bool tail = n < C;
#pragma unroll 2
                for (int i = 0; i < 16; ++i) {
                    const int r = r0 + i;
                    const uint4 u = ld16(gsm + unit(r));
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
                    uint32_t y[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float2 z = bf2(uw[m]);
                        float l0, l1;
                        asm("lg2.approx.f32 %0, %1;" : "=f"(l0) : "f"(1.f + ex2(-fabsf(z.x) * kL2E)));
                        asm("lg2.approx.f32 %0, %1;" : "=f"(l1) : "f"(1.f + ex2(-fabsf(z.y) * kL2E)));
                        const float2 sp = make_float2(fmaxf(z.x, 0.f) + kLn2 * l0, fmaxf(z.y, 0.f) + kLn2 * l1);
                        y[m] = pk2(mul2(sp, dup2(-ea)));
                    }
                    if (tail && r >= n) y[0] = y[1] = y[2] = y[3] = 0u;
                    st16(gsm + unit(r), y[0], y[1], y[2], y[3]);
                }
            } else {
                const float2 ea = dup2(0.5f * expf(a_h));   // sigmoid(a z) = (1 + tanh(a z / 2)) / 2
                asm volatile("bar.sync %0, %1;" ::"r"(sub_bar), "r"(128) : "memory");
                const bool tail = n < C;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const int r = r0 + i;
                    const uint4 u = ld16(gsm + unit(r));
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
                    uint32_t y[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float2 hz = mul2(bf2(uw[m]), ea);
                        const float2 t = make_float2(tanh_hw(hz.x), tanh_hw(hz.y));
                        y[m] = pk2(fma2(t, dup2(-2.5f), dup2(-2.5f)));   // -5 sigmoid
                    }
                    if (tail && r >= n) y[0] = y[1] = y[2] = y[3] = 0u;
                    st16(gsm + unit(r), y[0], y[1], y[2], y[3]);
                }
            }
            fence_proxy_async();   // g and v are read by the tensor cores
            if (gt == 0) {   // by now both have landed: count them for the drain
                if (wait(b_g, ph)) ++con[1];
                if (wait(b_v, ph)) ++con[2];
            }
            if (gbar_or(gi, bad)) break;   // the gate's g is in place before the cumsum reads it
        }
        // ---- Complex-KDA: g holds the signed gate alpha.  Thread = (row r, channels 32 cq ..):
        // log|alpha| split into a bf16 high part (in place) and low part (OFF_LO), so the cumsum
        // below is exact to ~2^-17; the sign bits become this thread's prefix parity word
        // sigma_r (bit j: channel 32 cq + j) by an XOR scan over the warp's 32 rows, the carry
        // of rows 0-31 coming through PX after the barrier.  Rows past T count as alpha = 1.
        uint32_t sig = 0;
        if (fl.complex_gate) {
            if (wait(b_g, ph) && gt == 0) ++con[1];
            const int r = gt & 63, cq = gt >> 6;
            uint32_t neg = 0;
            constexpr float kLn2 = 0.6931471805599453f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int cg = 4 * cq + m;
                const uint4 u = ld16(gsm + OFF_G + off_t(r, cg));
                const uint32_t wa[4] = {u.x, u.y, u.z, u.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 a = bf2(wa[e]);
                    neg |= (a.x < 0.f ? 1u : 0u) << (8 * m + 2 * e);
                    neg |= (a.y < 0.f ? 1u : 0u) << (8 * m + 2 * e + 1);
                    float l0, l1;
                    asm("lg2.approx.f32 %0, %1;" : "=f"(l0) : "f"(fabsf(a.x)));
                    asm("lg2.approx.f32 %0, %1;" : "=f"(l1) : "f"(fabsf(a.y)));
                    const float2 lg = r < n ? mul2(make_float2(l0, l1), dup2(kLn2)) : make_float2(0.f, 0.f);
                    hi[e] = pk2(lg);
                    const float2 h2 = bf2(hi[e]);
                    lo[e] = pk2(make_float2(lg.x - h2.x, lg.y - h2.y));
                }
                st16(gsm + OFF_G + off_t(r, cg), hi[0], hi[1], hi[2], hi[3]);
                st16(gsm + OFF_LO + off_t(r, cg), lo[0], lo[1], lo[2], lo[3]);
            }
            if (r >= n) neg = 0u;
            uint32_t pfx = neg;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, pfx, o);
                if (lane >= o) pfx ^= y;
            }
            if (lane == 31) PX[gw] = pfx;
            sig = pfx;
            fence_proxy_async();   // both parts are read by the tensor cores
            if (gbar_or(gi, bad)) break;
            if (gw & 1) sig ^= PX[gw - 1];
        }
        // ---- band-local cumsum on the tensor cores: D[0,128) = [L_band; L_band] g (Complex-KDA:
        // the two parts of log|alpha|, K = 128)
        if (gt == 0) {
            const bool g_ok = PRO || fl.complex_gate || wait(b_g, ph);
            if (!PRO && !fl.complex_gate && g_ok) ++con[1];
            tc_fence_after();
            if (g_ok) {
                constexpr uint32_t id = idesc_bf16(128, 128, 0, 1, 0);
                const int nk = fl.complex_gate ? 8 : 4;
                for (int s = 0; s < nk; ++s)
                    mma_ts(gtm + TC_D, gtm + TC_LM + 8 * (s & 3),
                           at(dT, (s < 4 ? OFF_G : OFF_LO) + 2048 * (s & 3)), id, s > 0);
                mma_commit(b_m1);
                ++iss[3];
            }
        }
        // ---- meanwhile: sums of squares of the rows of [q; k] (thread = row, one 64-channel half)
        {
            const int row = gt & 127, hf = gt >> 7;
            const int t = row >> 6, r = row & 63;
            float2 ss = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const uint4 u = ld16(gsm + OFF_X + off_x(t, r, 8 * hf + m));
                float2 x = bf2(u.x);
                ss = fma2(x, x, ss);
                x = bf2(u.y);
                ss = fma2(x, x, ss);
                x = bf2(u.z);
                ss = fma2(x, x, ss);
                x = bf2(u.w);
                ss = fma2(x, x, ss);
            }
            NRMP[hf * 128 + row] = ss.x + ss.y;
        }
        if (gbar_or(gi, bad)) break;
        if (wait(b_m1, ph) && gt == 0) ++con[3];
        tc_fence_after();
        // ---- thread = (row r, channels 32 cq .. 32 cq + 31): the band-local cumsum; the last row of
        // each band holds the band totals
        const int r = 32 * (gw & 1) + lane, cq = gw >> 1, band = r >> 4;
        float gam[32];
        tmem_ld32(tl + TC_D + 32 * cq, gam);
        if ((r & 15) == 15) {
#pragma unroll
            for (int m = 0; m < 8; ++m)
                *reinterpret_cast<float4 *>(TOT + band * 128 + 32 * cq + 4 * m) =
                    make_float4(gam[4 * m], gam[4 * m + 1], gam[4 * m + 2], gam[4 * m + 3]);
        }
        gbar(gi);
        // ---- per-channel band factors (threads 0-127); UNB: as logarithms, while threads 128-255
        // form alpha = e^g for the diagonal blocks
        if (UNB) {
            constexpr float kL2E = 1.4426950408889634f;
            if (gt < 128) {
                const int c = gt;
                const float t0 = TOT[c], t1 = TOT[128 + c], t2 = TOT[256 + c], t3 = TOT[384 + c];
                FT[(R_LT + 0) * 128 + c] = t0;
                FT[(R_LT + 1) * 128 + c] = t1;
                FT[(R_LT + 2) * 128 + c] = t2;
                FT[(R_LT + 3) * 128 + c] = t3;
                const float p2 = t0 + t1, p3 = p2 + t2;
                FT[R_L01 * 128 + c] = p2;
                FT[R_L12 * 128 + c] = t1 + t2;
                FT[R_L012 * 128 + c] = p3;
                const float c2 = t2 + t3, c1 = t1 + c2, c0 = t0 + c1;
                FT[(R_LC + 0) * 128 + c] = c0;
                FT[(R_LC + 1) * 128 + c] = c1;
                FT[(R_LC + 2) * 128 + c] = c2;
                FT[(R_EXP + 0) * 128 + c] = ex2(t0 * kL2E);
                FT[(R_EXP + 1) * 128 + c] = ex2(p2 * kL2E);
                FT[(R_EXP + 2) * 128 + c] = ex2(p3 * kL2E);
                reinterpret_cast<float *>(img + IMG_GC)[c] = ex2(c0 * kL2E);
            }
            // alpha = e^g, thread = (8-channel group, rows gt / 16 + 16 m): a warp writes two
            // whole rows per store
            if (!PRO) (void)wait(b_g, ph);   // the g tile (already complete: a formality per thread)
            const int cg = gt & 15;
            float *AL = reinterpret_cast<float *>(gsm + OFF_ALPHA);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int rr = (gt >> 4) + 16 * m;
                const uint4 gu = ld16(gsm + OFF_G + off_t(rr, cg));
                const uint32_t gw4[4] = {gu.x, gu.y, gu.z, gu.w};
                float a[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 g2 = bf2(gw4[e]);
                    a[2 * e] = ex2(g2.x * kL2E);
                    a[2 * e + 1] = ex2(g2.y * kL2E);
                }
                *reinterpret_cast<float4 *>(AL + rr * 128 + 8 * cg) = make_float4(a[0], a[1], a[2], a[3]);
                *reinterpret_cast<float4 *>(AL + rr * 128 + 8 * cg + 4) = make_float4(a[4], a[5], a[6], a[7]);
            }
        } else if (gt < 128) {
            const int c = gt;
            float et[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) et[p] = __expf(fmaxf(TOT[p * 128 + c], -85.f));
            FT[(R_ET + 0) * 128 + c] = et[0];
            FT[(R_ET + 1) * 128 + c] = et[1];
            FT[(R_ET + 2) * 128 + c] = et[2];
            // Complex-KDA: K e^{gamma_C - gamma} carries sigma_C sigma_r (Gamma_C / Gamma_r), and the
            // state update sigma_C e^{gamma_C}: fold sigma_C into the e^{gamma_C - p_b} rows
            const float sc = (fl.complex_gate && (((PX[2 * (c >> 5)] ^ PX[2 * (c >> 5) + 1]) >> (c & 31)) & 1u)) ? -1.f : 1.f;
            FT[(R_ET + 3) * 128 + c] = sc * et[3];   // e_3 is used only as e^{gamma_C - p_3}
            const float e01 = et[0] * et[1], e12 = et[1] * et[2], e23 = et[2] * et[3];
            FT[R_EP2 * 128 + c] = e01;
            FT[R_EP3 * 128 + c] = e01 * et[2];
            const float eC = e01 * e23;
            FT[(R_ECP + 0) * 128 + c] = sc * eC;
            FT[(R_ECP + 1) * 128 + c] = sc * et[1] * e23;
            FT[(R_ECP + 2) * 128 + c] = sc * e23;
            FT[R_EM20 * 128 + c] = e01;
            FT[R_EM31 * 128 + c] = e12;
            FT[R_EM30 * 128 + c] = e01 * et[2];
            reinterpret_cast<float *>(img + IMG_GC)[c] = sc * eC;
        }
        gbar(gi);
        if constexpr (UNB) {
            // ---- the diagonal 16 x 16 blocks as FP32 position pairs.  Thread = (band, row pair
            // x / 15 - x, 8-channel group e); a warp takes row pairs x = 2 xh' + (lane >> 4) of
            // one band with xh' = xh, then of another band with xh' = 3 - xh, so every warp walks
            // 26 key rows.  Walking the key row i down from the row, f = prod_{i<s<=r} alpha_s
            // grows by one factor per step; sum_c q_rc k_ic f_c (and the same with k_r) for two
            // steps at a time is reduced over the 16 channel groups of a half-warp by a
            // transposing butterfly (eight values, eight shuffles).  Keys past the row (i > r) are
            // masked at the readout.
            const int xh = gw & 3, tb = gw >> 2, xl = lane >> 4, e = lane & 15;
            const float *AL = reinterpret_cast<const float *>(gsm + OFF_ALPHA);
            __nv_bfloat16 *DQ = reinterpret_cast<__nv_bfloat16 *>(gsm + OFF_DQ);
            float *DK = reinterpret_cast<float *>(gsm + OFF_DK);
            const bool b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1, b1 = (lane >> 1) & 1;
            auto norm_qk = [&](int row) -> float2 {
                return fl.l2norm ? make_float2(rsqrtf(NRMP[row] + NRMP[128 + row] + kL2Eps),
                                               rsqrtf(NRMP[64 + row] + NRMP[192 + row] + kL2Eps))
                                 : make_float2(1.f, 1.f);
            };
#pragma unroll 1
            for (int task = 0; task < 2; ++task) {
                const int xt = task == 0 ? xh : 3 - xh;
                const int ra = 2 * xt + xl, rb = 15 - ra, ilmax = 15 - 2 * xt;   // ilmax odd
                const int bnd = tb + 2 * task, bs = 16 * bnd;
                const float2 na = norm_qk(bs + ra), nb = norm_qk(bs + rb);
                float2 qa[4], ka[4], qb[4], kb[4], fa[4], fb[4], ap[4];
                {
                    const uint4 u0 = ld16(gsm + OFF_X + off_x(0, bs + ra, e));
                    const uint4 u1 = ld16(gsm + OFF_X + off_x(1, bs + ra, e));
                    const uint4 u2 = ld16(gsm + OFF_X + off_x(0, bs + rb, e));
                    const uint4 u3 = ld16(gsm + OFF_X + off_x(1, bs + rb, e));
                    const uint32_t w0[4] = {u0.x, u0.y, u0.z, u0.w}, w1[4] = {u1.x, u1.y, u1.z, u1.w};
                    const uint32_t w2[4] = {u2.x, u2.y, u2.z, u2.w}, w3[4] = {u3.x, u3.y, u3.z, u3.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        qa[m] = mul2(bf2(w0[m]), dup2(na.x));
                        ka[m] = mul2(bf2(w1[m]), dup2(na.y));
                        qb[m] = mul2(bf2(w2[m]), dup2(nb.x));
                        kb[m] = mul2(bf2(w3[m]), dup2(nb.y));
                        fa[m] = fb[m] = ap[m] = make_float2(1.f, 1.f);
                    }
                }
                // one key step: the q and k sums of rows a and b with key row i (0 where i > row)
                auto step = [&](int il, float (&v)[4]) {
                    const uint4 ku = ld16(gsm + OFF_X + off_x(1, bs + il, e));
                    const uint32_t wk[4] = {ku.x, ku.y, ku.z, ku.w};
                    float2 av[4];
                    ld4f2(AL + (bs + il) * 128 + 8 * e, av);
                    v[0] = v[1] = v[2] = v[3] = 0.f;
                    if (il <= rb) {
                        float2 aq = make_float2(0.f, 0.f), ak = aq;
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            if (il < rb) fb[m] = mul2(fb[m], ap[m]);
                            const float2 t = mul2(bf2(wk[m]), fb[m]);
                            aq = fma2(qb[m], t, aq);
                            ak = fma2(kb[m], t, ak);
                        }
                        v[0] = aq.x + aq.y;
                        v[1] = ak.x + ak.y;
                    }
                    if (il <= ra) {
                        float2 aq = make_float2(0.f, 0.f), ak = aq;
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            if (il < ra) fa[m] = mul2(fa[m], ap[m]);
                            const float2 t = mul2(bf2(wk[m]), fa[m]);
                            aq = fma2(qa[m], t, aq);
                            ak = fma2(ka[m], t, ak);
                        }
                        v[2] = aq.x + aq.y;
                        v[3] = ak.x + ak.y;
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m) ap[m] = av[m];
                };
#pragma unroll 1
                for (int il = ilmax; il > 0; il -= 2) {
                    float v0[4], v1[4];   // steps il and il - 1: (q, k) sums of row b, then row a
                    step(il, v0);
                    step(il - 1, v1);
                    // value index 4 b3 + 2 b2 + b1: step (b3), row a / b (b2), k / q (b1)
                    float w4[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float keep = b3 ? v1[j] : v0[j], send = b3 ? v0[j] : v1[j];
                        w4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                    }
                    float w2[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float keep = b2 ? w4[2 + j] : w4[j], send = b2 ? w4[j] : w4[2 + j];
                        w2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                    }
                    float w1 = (b1 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? w2[0] : w2[1], 2);
                    w1 += __shfl_xor_sync(0xffffffffu, w1, 1);
                    const int i = il - (b3 ? 1 : 0), rr = b2 ? ra : rb;
                    if ((lane & 1) == 0 && i <= rr) {
                        const float nki = fl.l2norm ? rsqrtf(NRMP[64 + bs + i] + NRMP[192 + bs + i] + kL2Eps) : 1.f;
                        const int o = (bnd * 16 + rr) * 16 + i;
                        if (b1) DK[o] = w1 * nki * BET[bs + rr];
                        else DQ[o] = __float2bfloat16_rn(w1 * nki);
                    }
                }
            }
            gbar(gi);
            tmem_ld32(tl + TC_D + 32 * cq, gam);   // gamma~ again (not kept live across the pairs)
        }

        // ---- operands (thread = row r, 32 channels): E = e^{gamma~}, 1/E; Q E and beta K E in
        // place; K e^gamma over g; the band-pair B rows k e^{p_b - gamma} for b >= band(r); the
        // record's Q e^gamma and K e^{gamma_C - gamma}.  UNB: every factor is one exponential of a
        // non-positive exponent, or a product of such: E, e^gamma = E e^{p_b}, e^{gamma_C - gamma},
        // and for the later bands' B rows e^{p_b' - gamma}; the own band's B rows are not formed.
        if constexpr (UNB) {
            const float nq = fl.l2norm ? rsqrtf(NRMP[r] + NRMP[128 + r] + kL2Eps) : 1.f;
            const float nk = fl.l2norm ? rsqrtf(NRMP[64 + r] + NRMP[192 + r] + kL2Eps) : 1.f;
            const float2 nq2 = dup2(nq), nk2 = dup2(nk), bt2 = dup2(BET[r]);
            const float *ep = FT + (R_EXP + band - 1) * 128, *lc = FT + lrow_c(band) * 128;
            constexpr float kL2E = 1.4426950408889634f;
            auto ex2p = [&](float2 x) { return make_float2(ex2(x.x * kL2E), ex2(x.y * kL2E)); };
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int cg = 4 * cq + m, c0 = 8 * cg;
                const uint4 uq = ld16(gsm + OFF_X + off_x(0, r, cg));
                const uint4 uk = ld16(gsm + OFF_X + off_x(1, r, cg));
                const uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w}, wk[4] = {uk.x, uk.y, uk.z, uk.w};
                float2 fp[4], fc[4];
                if (band > 0) {
                    ld4f2(ep + c0, fp);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) fp[e] = make_float2(1.f, 1.f);
                }
                ld4f2(lc + c0, fc);
                uint32_t o_qe[4], o_qg[4], o_ke[4], o_kg[4], o_kd[4];
                float2 kn[4], g2v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 g2 = make_float2(gam[8 * m + 2 * e], gam[8 * m + 2 * e + 1]);
                    g2v[e] = g2;
                    const float2 E = ex2p(g2);
                    const float2 G = mul2(E, fp[e]);   // e^{gamma}: both factors <= 1
                    const float2 Kf = ex2p(make_float2(fc[e].x - g2.x, fc[e].y - g2.y));
                    const float2 qn = mul2(bf2(wq[e]), nq2);
                    kn[e] = mul2(bf2(wk[e]), nk2);
                    o_qe[e] = pk2(mul2(qn, E));
                    o_qg[e] = pk2(mul2(qn, G));
                    o_ke[e] = pk2(mul2(mul2(kn[e], E), bt2));
                    o_kg[e] = pk2(mul2(kn[e], G));
                    o_kd[e] = pk2(mul2(kn[e], Kf));
                }
                st16(gsm + OFF_X + off_x(0, r, cg), o_qe[0], o_qe[1], o_qe[2], o_qe[3]);
                st16(gsm + OFF_X + off_x(1, r, cg), o_ke[0], o_ke[1], o_ke[2], o_ke[3]);
                st16(gsm + OFF_G + off_t(r, cg), o_kg[0], o_kg[1], o_kg[2], o_kg[3]);
                st16(img + IMG_QG + off_r128(r, c0), o_qg[0], o_qg[1], o_qg[2], o_qg[3]);
                st16(img + IMG_KD + off_r128(r, c0), o_kd[0], o_kd[1], o_kd[2], o_kd[3]);
                for (int bp = band + 1; bp < 4; ++bp) {
                    float2 fm[4];
                    ld4f2(FT + lrow_m(bp, band) * 128 + c0, fm);
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        o[e] = pk2(mul2(kn[e], ex2p(make_float2(fm[e].x - g2v[e].x, fm[e].y - g2v[e].y))));
                    st16(gsm + OFF_KH + off_kh(16 * pair_u(bp, band) + (r & 15), cg), o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async();
        } else {
            const float nq = fl.l2norm ? rsqrtf(NRMP[r] + NRMP[128 + r] + kL2Eps) : 1.f;
            const float nk = fl.l2norm ? rsqrtf(NRMP[64 + r] + NRMP[192 + r] + kL2Eps) : 1.f;
            const float2 nq2 = dup2(nq), nk2 = dup2(nk), bt2 = dup2(BET[r]);
            const float *ep = FT + row_ep(band) * 128, *ecp = FT + row_ecp(band) * 128;
            constexpr float kL2E = 1.4426950408889634f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int cg = 4 * cq + m, c0 = 8 * cg;
                const uint4 uq = ld16(gsm + OFF_X + off_x(0, r, cg));
                const uint4 uk = ld16(gsm + OFF_X + off_x(1, r, cg));
                uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w}, wk[4] = {uk.x, uk.y, uk.z, uk.w};
                if (fl.complex_gate) {   // sigma_r: flip the signs of q and k channel by channel
                    const uint32_t sb = sig >> (8 * m);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t mk = (((sb >> (2 * e)) & 1u) << 15) | (((sb >> (2 * e + 1)) & 1u) << 31);
                        wq[e] ^= mk;
                        wk[e] ^= mk;
                    }
                }
                float2 fp[4], fc[4];
                ld4f2(ep + c0, fp);
                ld4f2(ecp + c0, fc);
                uint32_t o_qe[4], o_qg[4], o_ke[4], o_kg[4], o_kh[4], o_kd[4];
                float2 kh[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 sg = mul2(make_float2(fmaxf(gam[8 * m + 2 * e], -85.f), fmaxf(gam[8 * m + 2 * e + 1], -85.f)),
                                           dup2(kL2E));
                    const float2 E = make_float2(ex2(sg.x), ex2(sg.y));
                    const float2 iE = make_float2(ex2(-sg.x), ex2(-sg.y));
                    const float2 qe = mul2(bf2(wq[e]), mul2(E, nq2));
                    const float2 kv = bf2(wk[e]);
                    const float2 ke = mul2(kv, mul2(E, nk2));
                    kh[e] = mul2(kv, mul2(iE, nk2));
                    o_qe[e] = pk2(qe);
                    o_qg[e] = pk2(mul2(qe, fp[e]));
                    o_ke[e] = pk2(mul2(ke, bt2));
                    o_kg[e] = pk2(mul2(ke, fp[e]));
                    o_kh[e] = pk2(kh[e]);
                    o_kd[e] = pk2(mul2(kh[e], fc[e]));
                }
                st16(gsm + OFF_X + off_x(0, r, cg), o_qe[0], o_qe[1], o_qe[2], o_qe[3]);
                st16(gsm + OFF_X + off_x(1, r, cg), o_ke[0], o_ke[1], o_ke[2], o_ke[3]);
                st16(gsm + OFF_G + off_t(r, cg), o_kg[0], o_kg[1], o_kg[2], o_kg[3]);
                st16(gsm + OFF_KH + off_kh(16 * pair_of(band, band) + (r & 15), cg), o_kh[0], o_kh[1], o_kh[2], o_kh[3]);
                st16(img + IMG_QG + off_r128(r, c0), o_qg[0], o_qg[1], o_qg[2], o_qg[3]);
                st16(img + IMG_KD + off_r128(r, c0), o_kd[0], o_kd[1], o_kd[2], o_kd[3]);
            }
            // the later bands' B rows k_i e^{p_b' - gamma_i} = (band b's own row) e^{p_b' - p_b},
            // b' > b: 6 band pairs x 16 rows x 16 channel groups, 6 per thread (a row's owner
            // alone would leave the warps of bands 2-3 idle while those of bands 0-1 form three)
            gbar(gi);
#pragma unroll
            for (int k = 0; k < 6; ++k) {
                const int it = gt + GT * k, cg = it & 15, pr = it >> 8, ri = (it >> 4) & 15;
                const int b = pr < 3 ? 0 : pr < 5 ? 1 : 2;
                const int bp = pr < 3 ? pr + 1 : pr < 5 ? pr - 1 : 3;   // (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
                const uint4 u = ld16(gsm + OFF_KH + off_kh(16 * pair_of(b, b) + ri, cg));
                float2 f[4];
                ld4f2(FT + row_em(bp, b) * 128 + 8 * cg, f);
                st16(gsm + OFF_KH + off_kh(16 * pair_of(bp, b) + ri, cg), pk2(mul2(bf2(u.x), f[0])),
                     pk2(mul2(bf2(u.y), f[1])), pk2(mul2(bf2(u.z), f[2])), pk2(mul2(bf2(u.w), f[3])));
            }
            fence_proxy_async();
        }
        tc_fence_before();
        if (gbar_or(gi, bad)) break;
        // ---- all ten band pairs: D[0,160) = [Q E; beta K E] (B rows)^T (UNB: the six off-diagonal
        // pairs, D[0,96))
        if (gt == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16(128, UNB ? NPAIR_U : 160, 0, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t da = sdesc(gs + OFF_X + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024, kSwizzle128B);
                const uint64_t db = sdesc(gs + OFF_KH + (s >> 2) * KH_HALF + (s & 3) * 32, 16, 1024, kSwizzle128B);
                mma_ss(gtm + TC_D, da, db, id, s > 0);
            }
            mma_commit(b_m2);
            ++iss[4];
        }
        const bool m2_ok = wait(b_m2, ph);
        if (gt == 0 && m2_ok) {
            ++con[4];
            if (next < nitems) {   // the q / k staging is free: the next item's tiles
                issue_qk(next);
                ++iss[0];
            }
        }
        tc_fence_after();
        // ---- A_qk -> record (lanes 0-63), A_kk -> FP32 transposed (lanes 64-127); warp gw covers
        // column bands 2h, 2h + 1 of its 32 rows
        {
            const int hh = gw >> 2, b_lo = 2 * (qd & 1);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * hh + jj;
                float v[16], v2[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = 0.f;
                if constexpr (UNB) {
                    // key bands before the row's band from the product, the own band's block
                    // from the FP32 pairs
                    if (j < b_lo) tmem_ld16(tl + TC_D + 16 * pair_u(b_lo, j), v);
                    if (j < b_lo + 1) {
                        tmem_ld16(tl + TC_D + 16 * pair_u(b_lo + 1, j), v2);
                        if (band == b_lo + 1) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) v[e] = v2[e];
                        }
                    }
                    if (j == band) {
                        const int o = (band * 16 + (r & 15)) * 16;
                        if (qd < 2) {
                            const uint4 d0 = ld16(gsm + OFF_DQ + 2 * o), d1 = ld16(gsm + OFF_DQ + 2 * o + 16);
                            const uint32_t dw[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float2 f = bf2(dw[e]);
                                v[2 * e] = f.x;
                                v[2 * e + 1] = f.y;
                            }
                        } else {
                            const float *dk = reinterpret_cast<const float *>(gsm + OFF_DK) + o;
#pragma unroll
                            for (int e4 = 0; e4 < 4; ++e4) {
                                const float4 f = *reinterpret_cast<const float4 *>(dk + 4 * e4);
                                v[4 * e4] = f.x;
                                v[4 * e4 + 1] = f.y;
                                v[4 * e4 + 2] = f.z;
                                v[4 * e4 + 3] = f.w;
                            }
                        }
                    }
                } else {
                    if (j <= b_lo) tmem_ld16(tl + TC_D + 16 * pair_of(b_lo, j), v);
                    if (j <= b_lo + 1) {
                        tmem_ld16(tl + TC_D + 16 * pair_of(b_lo + 1, j), v2);
                        if (band == b_lo + 1) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) v[e] = v2[e];
                        }
                    }
                }
                if (qd < 2) {
#pragma unroll
                    for (int g8 = 0; g8 < 2; ++g8) {
                        uint32_t y[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 16 * j + 8 * g8 + 2 * e;
                            y[e] = pk2(make_float2(i <= r ? v[8 * g8 + 2 * e] : 0.f, i + 1 <= r ? v[8 * g8 + 2 * e + 1] : 0.f));
                        }
                        st16(img + IMG_AQK + off_r64(r, 16 * j + 8 * g8), y[0], y[1], y[2], y[3]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int i = 16 * j + e;
                        AKT[i * AS + r] = (i < r) ? v[e] : 0.f;   // a warp writes 32 consecutive r
                    }
                }
            }
            if (gw == 2 || gw == 7) {
                __syncwarp();   // this warp's own A_kk^T rows
                const int blk = (gw == 2 ? 0 : 2) + (lane >> 4), base = 16 * blk, j = lane & 15;
                float x[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) x[rr] = (rr == j) ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < 15; ++i) {
                    const float xi = x[i];
                    const float *col = AKT + (base + i) * AS + base;   // A[base + rr][base + i] over rr
#pragma unroll
                    for (int r4 = ((i + 1) >> 2) << 2; r4 < 16; r4 += 4) {   // rows rr <= i hold 0
                        const float4 av = *reinterpret_cast<const float4 *>(col + r4);
                        x[r4] = fmaf(-av.x, xi, x[r4]);
                        x[r4 + 1] = fmaf(-av.y, xi, x[r4 + 1]);
                        x[r4 + 2] = fmaf(-av.z, xi, x[r4 + 2]);
                        x[r4 + 3] = fmaf(-av.w, xi, x[r4 + 3]);
                    }
                }
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) TMF[(base + rr) * AS + base + j] = x[rr];
                if ((blk & 1) == 0) {   // the zero upper-right quarter of each 32-block's T
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) TMF[(base + rr) * AS + base + 16 + j] = 0.f;
                }
            }
        }
        tc_fence_before();
        if (gbar_or(gi, bad)) break;

        // ---- Tm = (I + A_kk)^{-1} in FP32 by 32 x 32 blocks [T1 0; T21 T2]: the 16 x 16 diagonal
        // blocks D_b were swept at the end of the readout; per 32-block Z = A10 D0, X = -D1 Z;
        // then Y = A21 T1, T21 = -T2 Y.  TMF holds T (rows 0-31 hold Z, then Y, in columns 32-63).
        // Z = A10 D0 per 32-block hb (warps 0-3: block hb = gw >> 1, columns 8 (gw & 1) .. + 7;
        // 2 x 2 tiles: rows 2 rp, 2 rp + 1, columns 2 cp, 2 cp + 1)
        if (gw < 4) {
            const int hb = gw >> 1, base = 32 * hb, rp = lane >> 2, c2 = 8 * (gw & 1) + 2 * (lane & 3);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float2 a = *reinterpret_cast<const float2 *>(AKT + (base + k) * AS + base + 16 + 2 * rp);   // A10[2rp..][k]
                const float2 d = *reinterpret_cast<const float2 *>(TMF + (base + k) * AS + base + c2);            // D0[k][c2..]
                acc0 = fma2(dup2(a.x), d, acc0);
                acc1 = fma2(dup2(a.y), d, acc1);
            }
            *reinterpret_cast<float2 *>(TMF + (2 * rp) * AS + 32 + 16 * hb + c2) = acc0;
            *reinterpret_cast<float2 *>(TMF + (2 * rp + 1) * AS + 32 + 16 * hb + c2) = acc1;
        }
        gbar(gi);
        // X = -D1 Z -> rows 16-31 of the 32-block, columns 0-15 (same split)
        if (gw < 4) {
            const int hb = gw >> 1, base = 32 * hb, rp = lane >> 2, c2 = 8 * (gw & 1) + 2 * (lane & 3);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll
            for (int k4 = 0; k4 < 16; k4 += 4) {
                const float4 d0 = *reinterpret_cast<const float4 *>(TMF + (base + 16 + 2 * rp) * AS + base + 16 + k4);
                const float4 d1 = *reinterpret_cast<const float4 *>(TMF + (base + 17 + 2 * rp) * AS + base + 16 + k4);
                const float a0[4] = {d0.x, d0.y, d0.z, d0.w}, a1[4] = {d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const float2 z = *reinterpret_cast<const float2 *>(TMF + (k4 + kk) * AS + 32 + 16 * hb + c2);
                    acc0 = fma2(dup2(a0[kk]), z, acc0);
                    acc1 = fma2(dup2(a1[kk]), z, acc1);
                }
            }
            *reinterpret_cast<float2 *>(TMF + (base + 16 + 2 * rp) * AS + base + c2) = make_float2(-acc0.x, -acc0.y);
            *reinterpret_cast<float2 *>(TMF + (base + 17 + 2 * rp) * AS + base + c2) = make_float2(-acc1.x, -acc1.y);
        }
        gbar(gi);
        // Y = A21 T1 (2 x 2 tiles over 256 threads) -> rows 0-31, columns 32-63 (where Z was)
        {
            const int rp = gt >> 4, c2 = 2 * (gt & 15);   // rows 2 rp, 2 rp + 1; columns c2, c2 + 1
            float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll 8
            for (int k = 0; k < 32; ++k) {
                const float2 a = *reinterpret_cast<const float2 *>(AKT + k * AS + 32 + 2 * rp);   // A21[2rp..][k]
                const float2 t = *reinterpret_cast<const float2 *>(TMF + k * AS + c2);            // T1[k][c2..]
                acc0 = fma2(dup2(a.x), t, acc0);
                acc1 = fma2(dup2(a.y), t, acc1);
            }
            *reinterpret_cast<float2 *>(TMF + (2 * rp) * AS + 32 + c2) = acc0;
            *reinterpret_cast<float2 *>(TMF + (2 * rp + 1) * AS + 32 + c2) = acc1;
        }
        gbar(gi);
        // T21 = -T2 Y -> rows 32-63, columns 0-31
        {
            const int rp = gt >> 4, c2 = 2 * (gt & 15);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll 2
            for (int k4 = 0; k4 < 32; k4 += 4) {
                const float4 d0 = *reinterpret_cast<const float4 *>(TMF + (32 + 2 * rp) * AS + 32 + k4);   // T2[2rp][k4..]
                const float4 d1 = *reinterpret_cast<const float4 *>(TMF + (33 + 2 * rp) * AS + 32 + k4);
                const float a0[4] = {d0.x, d0.y, d0.z, d0.w}, a1[4] = {d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const float2 y = *reinterpret_cast<const float2 *>(TMF + (k4 + kk) * AS + 32 + c2);   // Y[k][c2..]
                    acc0 = fma2(dup2(a0[kk]), y, acc0);
                    acc1 = fma2(dup2(a1[kk]), y, acc1);
                }
            }
            *reinterpret_cast<float2 *>(TMF + (32 + 2 * rp) * AS + c2) = make_float2(-acc0.x, -acc0.y);
            *reinterpret_cast<float2 *>(TMF + (33 + 2 * rp) * AS + c2) = make_float2(-acc1.x, -acc1.y);
        }
        gbar(gi);
        // ---- Tm' = Tm diag(beta) -> the block-diagonal operand: lanes 0-63 get [Tm' | 0] (warps 0,
        // 1), lanes 64-127 get [0 | Tm'] (warps 6, 7); the zero halves were written once
        if (gw < 2 || gw >= 6) {
            uint32_t tv[32];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int i0 = 4 * m;
                const float4 t4 = *reinterpret_cast<const float4 *>(TMF + r * AS + i0);
                const float4 b4 = *reinterpret_cast<const float4 *>(BET + i0);
                // T's upper triangle: zero by construction except rows 0-31 x columns 32-63 (Y)
                const bool z = (r < 32 && i0 >= 32);
                tv[2 * m] = z ? 0u : pk2(mul2(make_float2(t4.x, t4.y), make_float2(b4.x, b4.y)));
                tv[2 * m + 1] = z ? 0u : pk2(mul2(make_float2(t4.z, t4.w), make_float2(b4.z, b4.w)));
            }
            tmem_st32(tl + TC_TM + (qd < 2 ? 0 : 32), tv);
            tmem_wait_st();
        }
        tc_fence_before();
        if (gbar_or(gi, bad)) break;
        // ---- [W; U] = [Tm' 0; 0 Tm'] [K e^gamma; V]
        if (gt == 0) {
            bool v_ok = true;
            if constexpr (!PRO) {
                v_ok = wait(b_v, ph);
                if (v_ok) ++con[2];
            }
            tc_fence_after();
            if (v_ok) {
                constexpr uint32_t id = idesc_bf16(128, 128, 0, 1, 0);
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t db = s < 4 ? at(dT, OFF_G + 2048 * s) : at(dT, OFF_V + 2048 * (s - 4));
                    mma_ts(gtm + TC_D, gtm + TC_TM + 8 * s, db, id, s > 0);
                }
                mma_commit(b_m3);
                ++iss[5];
            }
        }
        const bool m3_ok = wait(b_m3, ph);
        if (gt == 0 && m3_ok) {
            ++con[5];
            if (next < nitems) {   // g and v staging are free again
                issue_gv(next);
                ++iss[1];
                ++iss[2];
            }
        }
        tc_fence_after();
        // ---- W (lanes 0-63) and U (lanes 64-127) -> record, 64 channels per thread
        {
            const int hh = gw >> 2;
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
                float w[32];
                tmem_ld32(tl + TC_D + 64 * hh + 32 * hc, w);
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    const int c0 = 64 * hh + 32 * hc + 8 * g8;
                    const float *x = w + 8 * g8;
                    const uint32_t uoff = pro.u_slabs ? off_u(r, c0) : off_r128(r, c0);
                    st16(img + (qd < 2 ? IMG_W + off_r128(r, c0) : IMG_U + uoff), pk2(make_float2(x[0], x[1])),
                         pk2(make_float2(x[2], x[3])), pk2(make_float2(x[4], x[5])), pk2(make_float2(x[6], x[7])));
                }
            }
        }
        if constexpr (MEGA) __threadfence();   // this thread's record stores, before the flag
        tc_fence_before();
        const bool stop = gbar_or(gi, bad);
        tc_fence_after();
        if (stop) break;
        if (MEGA && gt == 0) flag_release(flags + item, 1);
    }
    // drain: let every copy and product this group issued land before TMEM and shared memory go
    // (each barrier has at most one completion outstanding: the one after those consumed)
    if (gt == 0) {
        const uint32_t bars[6] = {b_qk, b_g, b_v, b_m1, b_m2, b_m3};
#pragma unroll
        for (int i = 0; i < 6; ++i)
            if (iss[i] > con[i]) drain_wait(bars[i], con[i] & 1u);
    }
    tc_fence_before();
    gbar(gi);
}
