// kda_chunk_scan.cuh -- the split form's inter-chunk scan with the state and the chunk's
// intermediate products in TMEM (transposed products, A operands from TMEM).
//
// Included by kda_chunk_tc2.cu after the record layout and the two-group prep.  One CTA per
// sequence (b, h) walks its chunks in order (page "Kimi K3 模型结构（2）：序列维度（下），chunkwise
// 并行与下界衰减", Q&A items on the chunkwise algorithm: V~ = U - W S, O = (Q Gamma) S + A V~,
// S <- Diag(Gamma_C) S + (K Gamma_C / Gamma)^T V~).  Every product is taken transposed so that
// its M dimension is the head's 128 value columns (the TMEM lanes) and the state, V~ and the
// accumulators never leave TMEM / registers:
//
//   D[j][0:64)    = U^T (identity product)  -  S^T W^T     = V~^T    (lanes j = value column)
//   D[j][64:128)  = S^T (Q Gamma)^T  +  V~^T A_qk^T        = O^T
//   dS^T[j][c]    = V~^T Kd                                           (Kd = K Gamma_C / Gamma)
//   S^T[j][c]    <- sigma_C e^{gamma_C}[c] S^T[j][c] + dS^T[j][c]     (FP32 registers)
//
// S^T (bf16) and V~^T (bf16) are the A operands, read from TMEM; the record's W, Q Gamma, Kd,
// A_qk and U tiles are the B operands (or, for U, the A operand of the identity product), read
// from shared memory as the bulk copy left them.  Per chunk the tensor cores read about 72 KB
// of shared memory (the layout that keeps S and V~ in shared memory reads and writes about
// twice that), and the chain between two chunks is two tensor-core round trips and two short
// register passes.
#pragma once

namespace scan3 {
constexpr int NCW = 8;                     // CUDA warps: TMEM quadrant warp & 3, channel half warp >> 2
constexpr int MMA_WARP = NCW, LOAD_WARP = NCW + 1;
constexpr int NT = 32 * (NCW + 2);
constexpr int NSTG = 3;                    // records in flight
constexpr uint32_t STAGE = IMG_BYTES;      // one record per stage, as written by the prep
constexpr uint32_t OFF_I16 = NSTG * STAGE; // 16 x 16 bf16 identity (K-major core layout)
constexpr uint32_t SMEM_BYTES = OFF_I16 + 512 + 128;
static_assert(SMEM_BYTES <= 232448 - 512, "shared memory budget");
static_assert(STAGE % 16 == 0, "bulk copies need 16-byte alignment");
// TMEM columns: S^T bf16 operand, V~^T bf16 operand, two [V~^T | O^T] accumulators, dS^T
constexpr uint32_t TS_B = 0, TS_V = 64, TS_P0 = 128, TS_P1 = 256, TS_S = 384;
}  // namespace scan3

struct alignas(8) Scan3Bars {
    uint64_t stage[scan3::NSTG];
    uint64_t mP[2], mS, mO[2];     // tensor-core commits: V~^T done, dS^T done, O^T done
    uint64_t bV, bS;               // CUDA warps: V~^T operand written, S^T operand written
    uint64_t bE[2];                // CUDA warps: O^T of the buffer read out (emitted)
    uint32_t tmem_base;
    int abort;
    int s_done, o_done;            // MEGA: stage release counters (S updates, emits)
    int issued[scan3::NSTG + 5];   // completions issued per barrier (drain on give-up)
};

// zero_u: the chunks' U taken as zero (the segment map's linear part: S -> M S from S0 = I);
// out == nullptr: no outputs (their products are skipped), only the final state.
template <bool MEGA>
__device__ __forceinline__ void
scan3_body(const uint8_t *__restrict__ ws, const float *__restrict__ S0, __nv_bfloat16 *__restrict__ out,
           float *__restrict__ S_T, int T, int H, float scale, int cta, const int *__restrict__ flags, int nseq,
           uint32_t poll_limit, bool zero_u = false) {
    using namespace scan3;
    extern __shared__ uint8_t smem_raw[];
    __shared__ Scan3Bars sh;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = cta, b = bh / H, h = bh % H;
    const int nch = (T + C - 1) / C;
    const uint8_t *recs = ws + (size_t)bh * nch * IMG_BYTES;
    const uint32_t b_mS = smem_u32(&sh.mS), b_bV = smem_u32(&sh.bV), b_bS = smem_u32(&sh.bS);
    auto bar_mP = [&](int i) { return smem_u32(&sh.mP[i]); };
    auto bar_mO = [&](int i) { return smem_u32(&sh.mO[i]); };
    auto bar_bE = [&](int i) { return smem_u32(&sh.bE[i]); };
    auto bar_st = [&](int i) { return smem_u32(&sh.stage[i]); };

    if (tid == 0) {
        for (int i = 0; i < NSTG; ++i) mbar_init(bar_st(i), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_mP(i), 1);
            mbar_init(bar_mO(i), 1);
            mbar_init(bar_bE(i), NCW);
        }
        mbar_init(b_mS, 1);
        mbar_init(b_bV, NCW);
        mbar_init(b_bS, NCW);
        mbar_fence_init();
        sh.abort = 0;
        sh.s_done = 0;
        sh.o_done = 0;
        for (int i = 0; i < NSTG + 5; ++i) sh.issued[i] = 0;
    }
    // the 16 x 16 identity, K-major core layout: element (n, k) at (n&7)*16 + (n>>3)*256 + (k>>3)*128 + (k&7)*2
    for (int i = tid; i < 256; i += blockDim.x) {
        const int n = i >> 4, k = i & 15;
        *reinterpret_cast<uint16_t *>(smem + OFF_I16 + (n & 7) * 16 + (n >> 3) * 256 + (k >> 3) * 128 + (k & 7) * 2) =
            n == k ? 0x3F80u : 0u;
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
    auto at = [](uint64_t base, uint32_t off) -> uint64_t { return base + (uint64_t)(off >> 4); };
    const uint64_t dK = sdesc(sbase, 128, 2048, kSwizzleNone);      // K-major [128 n][128 k] (record rows)
    const uint64_t dMN = sdesc(sbase, 2048, 128, kSwizzleNone);     // MN-major [64 k][128 m] (Kd, U)
    const uint64_t dK64 = sdesc(sbase, 128, 1024, kSwizzleNone);    // K-major [64 n][64 k] (A_qk)
    const uint64_t dI = sdesc(sbase + OFF_I16, 128, 256, kSwizzleNone);
    auto fetch = [&](int ch) {
        const int s = ch % NSTG;
        ++sh.issued[s];
        mbar_arrive_expect_tx(bar_st(s), IMG_BYTES);
        bulk_load(sbase + s * STAGE, recs + (size_t)ch * IMG_BYTES, IMG_BYTES, bar_st(s));
    };
    // bounded wait by every calling thread; a give-up raises the CTA's abort flag, which ends
    // every other wait at once
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

    if (warp < NCW) {
        // ---- CUDA warps: value column j (TMEM lane), key channels c0 .. c0 + 63 of the state
        const int q = warp & 3, hh = warp >> 2, j = 32 * q + lane, c0 = 64 * hh;
        const uint32_t tl = tbase + ((uint32_t)(32 * q) << 16);
        float S[64];
        if (S0) {
            const float *src = S0 + (size_t)bh * D * D + (size_t)c0 * D + j;
#pragma unroll
            for (int i = 0; i < 64; ++i) S[i] = src[(size_t)i * D];
        } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) S[i] = 0.f;
        }
        auto store_state_operand = [&]() {
            uint32_t u[32];
#pragma unroll
            for (int p = 0; p < 32; ++p) u[p] = pack_bf16(S[2 * p], S[2 * p + 1]);
            tmem_st32(tl + TS_B + 32 * hh, u);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_bS);
        };
        store_state_operand();   // S(0)
        for (int ch = 0; ch < nch; ++ch) {
            const int buf = ch & 1;
            const uint32_t tdp = buf ? TS_P1 : TS_P0;
            const uint32_t st = (ch % NSTG) * STAGE;
            const int t0 = ch * C;
            // V~^T rows 32 hh .. 32 hh + 31 of this column -> the bf16 operand
            if (!wait(bar_mP(buf), (uint32_t)(ch >> 1) & 1u)) break;
            __syncwarp();
            tc_fence_after();
            {
                float v[32];
                tmem_ld32(tl + tdp + 32 * hh, v);
                uint32_t u[16];
#pragma unroll
                for (int p = 0; p < 16; ++p) u[p] = pack_bf16(v[2 * p], v[2 * p + 1]);
                tmem_st16(tl + TS_V + 16 * hh, u);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_bV);
            // S^T <- sigma_C e^{gamma_C} S^T + dS^T (FP32), then its bf16 operand
            if (!wait(b_mS, (uint32_t)ch & 1u)) break;
            if (!wait(bar_st(ch % NSTG), (uint32_t)(ch / NSTG) & 1u)) break;   // the record's sigma_C is visible
            __syncwarp();
            tc_fence_after();
            {
                const float *gc = reinterpret_cast<const float *>(smem + st + IMG_GC) + c0;
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    float ds[32];
                    tmem_ld32(tl + TS_S + c0 + 32 * hc, ds);
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 g4 = *reinterpret_cast<const float4 *>(gc + 32 * hc + 4 * i4);
                        const int i = 32 * hc + 4 * i4;
                        S[i] = fmaf(g4.x, S[i], ds[4 * i4]);
                        S[i + 1] = fmaf(g4.y, S[i + 1], ds[4 * i4 + 1]);
                        S[i + 2] = fmaf(g4.z, S[i + 2], ds[4 * i4 + 2]);
                        S[i + 3] = fmaf(g4.w, S[i + 3], ds[4 * i4 + 3]);
                    }
                }
            }
            store_state_operand();   // S(ch + 1)
            if (MEGA && lane == 0) smem_release_add(smem_u32(&sh.s_done), 1);   // the stage's sigma_C read
            // O^T rows 32 hh .. 32 hh + 31 of this column -> out
            if (!wait(bar_mO(buf), (uint32_t)(ch >> 1) & 1u)) break;
            __syncwarp();
            tc_fence_after();
            if (out) {
                float o[32];
                tmem_ld32(tl + tdp + 64 + 32 * hh, o);
                __nv_bfloat16 *dst = out + (((size_t)b * T + t0 + 32 * hh) * H + h) * D + j;
                const size_t rs = (size_t)H * D;
                const int nr = min(32, T - t0 - 32 * hh);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < nr) dst[(size_t)i * rs] = __float2bfloat16_rn(o[i] * scale);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar_bE(buf));
                if (MEGA) smem_release_add(smem_u32(&sh.o_done), 1);   // the stage's products are done
            }
        }
        if (S_T && !*reinterpret_cast<volatile int *>(&sh.abort)) {
            float *dst = S_T + (size_t)bh * D * D + (size_t)c0 * D + j;
#pragma unroll
            for (int i = 0; i < 64; ++i) dst[(size_t)i * D] = S[i];
        }
    } else if (warp == MMA_WARP) {
        // ---- the MMA warp: every lane waits, lane 0 issues, the warp reconverges
        if (!MEGA) {
            asm volatile("griddepcontrol.wait;" ::: "memory");   // the prep's records are complete
            if (lane == 0)
                for (int c = 0; c < NSTG && c < nch; ++c) fetch(c);
            __syncwarp();
        }
        for (int ch = 0; ch < nch; ++ch) {
            const int buf = ch & 1, sg = ch % NSTG;
            const uint32_t tdp = tbase + (buf ? TS_P1 : TS_P0);
            const uint32_t st = sg * STAGE;
            if (!wait(bar_st(sg), (uint32_t)(ch / NSTG) & 1u)) break;          // the record is in
            if (ch >= 2 && !wait(bar_bE(buf), (uint32_t)((ch - 2) >> 1) & 1u)) break;   // buffer emitted
            tc_fence_after();
            if (lane == 0 && !zero_u) {
                // U^T into the V~^T half: four M = 128, N = 16, K = 16 identity products
                constexpr uint32_t id_u = idesc_bf16(128, 16, 1, 0, 0);
#pragma unroll
                for (int s = 0; s < 4; ++s) mma_ss(tdp + 16 * s, at(dMN, st + IMG_U + 4096 * s), dI, id_u, 0);
            }
            __syncwarp();
            if (!wait(b_bS, (uint32_t)ch & 1u)) break;                          // S(ch) is in place
            tc_fence_after();
            if (lane == 0) {
                // V~^T = U^T - S^T W^T (negated A; zero_u: -S^T W^T), then O^T = S^T (Q Gamma)^T
                constexpr uint32_t id_p = idesc_bf16(128, 64, 0, 0, 1);
                constexpr uint32_t id_o = idesc_bf16(128, 64, 0, 0, 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ts(tdp, tbase + TS_B + 8 * k, at(dK, st + IMG_W + 256 * k), id_p, !zero_u || k > 0);
                mma_commit(bar_mP(buf));
                ++sh.issued[NSTG + buf];
                if (out) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_ts(tdp + 64, tbase + TS_B + 8 * k, at(dK, st + IMG_QG + 256 * k), id_o, k > 0);
                }
            }
            __syncwarp();
            // the stage of chunk ch - 1 is free once its O products are done and its sigma_C has
            // been read (S(ch) in place): refill it with chunk ch - 1 + NSTG (MEGA: the loader warp)
            if (!MEGA && ch >= 1 && ch - 1 + NSTG < nch) {
                if (!wait(bar_mO((ch - 1) & 1), (uint32_t)((ch - 1) >> 1) & 1u)) break;
                if (lane == 0) fetch(ch - 1 + NSTG);
                __syncwarp();
            }
            if (!wait(b_bV, (uint32_t)ch & 1u)) break;                          // V~^T operand in place
            tc_fence_after();
            if (lane == 0) {
                // dS^T = V~^T Kd, then O^T += V~^T A_qk^T
                constexpr uint32_t id_s = idesc_bf16(128, 128, 0, 1, 0);
                constexpr uint32_t id_q = idesc_bf16(128, 64, 0, 0, 0);
#pragma unroll
                for (int k = 0; k < 4; ++k) mma_ts(tbase + TS_S, tbase + TS_V + 8 * k, at(dMN, st + IMG_KD + 4096 * k), id_s, k > 0);
                mma_commit(b_mS);
                ++sh.issued[NSTG + 2];
                if (out) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_ts(tdp + 64, tbase + TS_V + 8 * k, at(dK64, st + IMG_AQK + 256 * k), id_q, 1);
                }
                mma_commit(bar_mO(buf));
                ++sh.issued[NSTG + 3 + buf];
            }
            __syncwarp();
        }
    } else if (MEGA && warp == LOAD_WARP) {
        // ---- MEGA: chunk c's record goes into stage c % NSTG once the prep has published it
        // (item = chunk * nseq + sequence) and, from c = NSTG on, once every reader of chunk
        // c - NSTG is done (its sigma_C and its O products: the S update and emit counters)
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const int *f = flags + (size_t)c * (size_t)nseq + bh;
                const int need = c - NSTG + 1;
                bool go = false;
                for (uint32_t i = 0; i < poll_limit; ++i) {
                    if ((need <= 0 || (smem_acquire_load(smem_u32(&sh.s_done)) >= need * NCW &&
                                       smem_acquire_load(smem_u32(&sh.o_done)) >= need * NCW)) &&
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
    }
    tc_fence_before();
    __syncthreads();
    // drain: after a give-up, copies and products may still be in flight; let each barrier reach
    // its last issued completion (built-in limit) before TMEM and shared memory go
    if (tid == 0 && *reinterpret_cast<volatile int *>(&sh.abort)) {
        uint32_t bars[NSTG + 5];
        for (int i = 0; i < NSTG; ++i) bars[i] = bar_st(i);
        bars[NSTG] = bar_mP(0);
        bars[NSTG + 1] = bar_mP(1);
        bars[NSTG + 2] = b_mS;
        bars[NSTG + 3] = bar_mO(0);
        bars[NSTG + 4] = bar_mO(1);
        for (int i = 0; i < NSTG + 5; ++i) {
            const int k = *reinterpret_cast<volatile int *>(&sh.issued[i]);
            if (k > 0) (void)mbar_wait_bounded(bars[i], (uint32_t)(k - 1) & 1u, kWaitLimit);
        }
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}
