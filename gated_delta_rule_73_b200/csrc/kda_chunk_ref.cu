// kda_chunk_ref.cu -- FP32 CUDA-core chunkwise KDA forward (two phases).
//
// This is the exact-FP32 path: it serves fp32 inputs (where tensor-core TF32
// or BF16 operands would not meet a 1e-4 relative bound) and any shape the
// tensor-core kernel does not take.  It follows the chunkwise form of page
// "Kimi K3 模型结构（2）：序列维度（下），chunkwise 并行与下界衰减" (Q&A items on
// the chunkwise algorithm and on the intra-chunk matrix A):
//
// Phase 1 (one CTA per chunk and head, all chunks in parallel):
//   gamma_r = sum_{s<=r} log|alpha_s| per key channel (chunk-local),
//   sigma_r = prod_{s<=r} sign(alpha_s) (Complex-KDA; folded into q and k),
//   A_kk[r,i] = beta_r sum_c k_rc k_ic e^{gamma_rc - gamma_ic}   (i < r)
//   A_qk[r,i] =        sum_c q_rc k_ic e^{gamma_rc - gamma_ic}   (i <= r)
//     (inside a 16-token band the factor is taken per pair; across bands as
//      e^{gamma_r - P} e^{P - gamma_i} with P = gamma just before r's band)
//   Tm = (I + A_kk)^{-1} by forward substitution (the UT transform)
//   W = Tm diag(beta) (K e^gamma),  U = Tm diag(beta) V    (WY vectors)
//   Qg = Q e^gamma,  Kd = sigma_C K e^{gamma_C - gamma},  gC = sigma_C e^{gamma_C}
// Every exponent above is <= 0, so nothing overflows in FP32.
//
// Phase 2 (one CTA per head and slice of 16 value columns, chunks in order):
//   V~ = U - W S;   O = scale (Qg S + A_qk V~);   S <- diag(gC) S + Kd^T V~
// as register-tiled products (2 x 2 and RPT x 2 outputs per thread) over shared memory.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {
constexpr int C = kChunk;
constexpr int CP = C + 1;

__device__ __forceinline__ float ldx(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ldx(const __nv_bfloat16 *p, size_t i) { return to_f32(p[i]); }

template <int DK, int DV>
struct RefLayout {
    static constexpr size_t per_chunk = (size_t)C * DK * 3 + (size_t)C * DV + (size_t)C * C + DK;
    static constexpr size_t off_W = 0;
    static constexpr size_t off_U = off_W + (size_t)C * DK;
    static constexpr size_t off_Qg = off_U + (size_t)C * DV;
    static constexpr size_t off_Kd = off_Qg + (size_t)C * DK;
    static constexpr size_t off_A = off_Kd + (size_t)C * DK;
    static constexpr size_t off_gC = off_A + (size_t)C * C;
};

template <int DK, int DV>
constexpr size_t intra_smem_bytes() {
    return sizeof(float) * ((size_t)C * (DK + 1) * 3 + (size_t)C * (DV + 1) + (size_t)C * CP * 3 +
                            C + 2 * DK + (size_t)64 * (DK + 1));
}

template <typename TQ, typename TG, typename TB, int DK, int DV>
__global__ void __launch_bounds__(256)
chunk_intra_kernel(const TQ *__restrict__ q, const TQ *__restrict__ k, const TQ *__restrict__ v,
                   const TG *__restrict__ g, const TB *__restrict__ beta, int T, int H,
                   int nchunks, KernelFlags fl, float *__restrict__ ws) {
    constexpr int DKP = DK + 1, DVP = DV + 1;
    using L = RefLayout<DK, DV>;
    extern __shared__ float sm[];
    float *Qs = sm;
    float *Ks = Qs + C * DKP;
    float *Gs = Ks + C * DKP;
    float *Vs = Gs + C * DKP;
    float *Akk = Vs + C * DVP;
    float *Aqk = Akk + C * CP;
    float *Tm = Aqk + C * CP;
    float *bs = Tm + C * CP;
    float *sgnC = bs + C;
    float *gamC = sgnC + DK;
    float *RF = gamC + DK;           // [16][DKP] row factors e^{gamma_r - P} of one row band
    float *KI = RF + 16 * DKP;       // [48][DKP] k_i e^{P - gamma_i} for the rows before it

    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int t0 = chunk * C;
    const int n = min(C, T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int idx = tid; idx < C * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        float qv = 0.f, kv = 0.f, gv = fl.complex_gate ? 1.f : 0.f;
        if (r < n) {
            const size_t row = ((size_t)b * T + t0 + r) * H + h;
            qv = ldx(q, row * DK + c);
            kv = ldx(k, row * DK + c);
            gv = ldx(g, row * DK + c);
        }
        Qs[r * DKP + c] = qv;
        Ks[r * DKP + c] = kv;
        Gs[r * DKP + c] = gv;
    }
    for (int idx = tid; idx < C * DV; idx += 256) {
        const int r = idx / DV, c = idx % DV;
        float vv = 0.f;
        if (r < n) vv = ldx(v, (((size_t)b * T + t0 + r) * H + h) * DV + c);
        Vs[r * DVP + c] = vv;
    }
    if (tid < C) bs[tid] = tid < n ? ldx(beta, ((size_t)b * T + t0 + tid) * H + h) : 0.f;
    __syncthreads();

    if (fl.l2norm) {
        for (int r = warp; r < n; r += 8) {
            float sq = 0.f, sk = 0.f;
            for (int c = lane; c < DK; c += 32) {
                sq += Qs[r * DKP + c] * Qs[r * DKP + c];
                sk += Ks[r * DKP + c] * Ks[r * DKP + c];
            }
            sq = warp_sum(sq);
            sk = warp_sum(sk);
            const float fq = rsqrtf(sq + kL2Eps), fk = rsqrtf(sk + kL2Eps);
            for (int c = lane; c < DK; c += 32) {
                Qs[r * DKP + c] *= fq;
                Ks[r * DKP + c] *= fk;
            }
        }
        __syncthreads();
    }

    // chunk-local cumulative log-decay (and sign parity for Complex-KDA)
    if (tid < DK) {
        const int c = tid;
        float gam = 0.f, sg = 1.f;
        for (int r = 0; r < n; ++r) {
            const float a = Gs[r * DKP + c];
            float lg = a;
            if (fl.complex_gate) {
                lg = logf(fabsf(a));
                if (a < 0.f) sg = -sg;
                Qs[r * DKP + c] *= sg;
                Ks[r * DKP + c] *= sg;
            }
            gam += lg;
            Gs[r * DKP + c] = gam;
        }
        for (int r = n; r < C; ++r) Gs[r * DKP + c] = gam;
        sgnC[c] = sg;
        gamC[c] = gam;
    }
    __syncthreads();

    // A_kk (strict lower, with beta_r) and A_qk (lower with diagonal), exact for any
    // gamma: a pair inside one 16-token band takes e^{gamma_r - gamma_i} directly; a pair with
    // i in an earlier band takes e^{gamma_r - P} e^{P - gamma_i}, P = gamma of the row just
    // before r's band.  gamma does not increase, so both factors are <= 1 for any g <= 0, and
    // one exponential per (row, channel) replaces one per (pair, channel) there.
    for (int p = tid; p < C * C; p += 256) {
        Akk[(p / C) * CP + p % C] = 0.f;
        Aqk[(p / C) * CP + p % C] = 0.f;
    }
    __syncthreads();
    for (int p = tid; p < 4 * 136; p += 256) {           // the four diagonal bands, i <= r
        const int band = p / 136, t = p % 136;
        int rr = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
        while ((rr + 1) * (rr + 2) / 2 <= t) ++rr;
        while (rr * (rr + 1) / 2 > t) --rr;
        const int r = 16 * band + rr, i = 16 * band + (t - rr * (rr + 1) / 2);
        if (r < n) {
            float akk = 0.f, aqk = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float e = expf(Gs[r * DKP + c] - Gs[i * DKP + c]);
                const float kk = Ks[i * DKP + c] * e;
                akk += Ks[r * DKP + c] * kk;
                aqk += Qs[r * DKP + c] * kk;
            }
            if (i < r) Akk[r * CP + i] = bs[r] * akk;
            Aqk[r * CP + i] = aqk;
        }
    }
    for (int rb = 1; rb < 4; ++rb) {                        // row band rb x earlier bands
        const int r0 = 16 * rb;
        if (r0 >= n) break;
        __syncthreads();                                    // RF / KI of the last band are read
        for (int idx = tid; idx < 16 * DK; idx += 256) {
            const int rr = idx / DK, c = idx % DK;
            RF[rr * DKP + c] = expf(Gs[(r0 + rr) * DKP + c] - Gs[(r0 - 1) * DKP + c]);
        }
        for (int idx = tid; idx < r0 * DK; idx += 256) {
            const int i = idx / DK, c = idx % DK;
            KI[i * DKP + c] = Ks[i * DKP + c] * expf(Gs[(r0 - 1) * DKP + c] - Gs[i * DKP + c]);
        }
        __syncthreads();
        const int rr = tid >> 4, ig = tid & 15, r = r0 + rr;   // columns ig, ig + 16, ...
        float aq[3] = {0.f, 0.f, 0.f}, ak[3] = {0.f, 0.f, 0.f};
        for (int c = 0; c < DK; ++c) {
            const float f = RF[rr * DKP + c];
            const float qf = Qs[r * DKP + c] * f, kf = Ks[r * DKP + c] * f;
#pragma unroll
            for (int m = 0; m < 3; ++m) {
                if (m < rb) {
                    const float ki = KI[(ig + 16 * m) * DKP + c];
                    aq[m] = fmaf(qf, ki, aq[m]);
                    ak[m] = fmaf(kf, ki, ak[m]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            if (m < rb) {
                Aqk[r * CP + ig + 16 * m] = aq[m];
                Akk[r * CP + ig + 16 * m] = bs[r] * ak[m];
            }
        }
    }
    __syncthreads();

    // Tm = (I + A_kk)^{-1}: column j solves (I + A_kk) x = e_j by forward substitution, row by
    // row; the four lanes of a column split each row's sum (lanes 4j .. 4j + 3 of one warp)
    {
        const int j = tid >> 2, part = tid & 3;
        for (int r = 0; r < C; ++r) {
            float acc = 0.f;
            for (int i = j + part; i < r; i += 4) acc = fmaf(Akk[r * CP + i], Tm[i * CP + j], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (part == 0) Tm[r * CP + j] = (r < j) ? 0.f : ((r == j) ? 1.f : 0.f) - acc;
            __syncwarp();
        }
    }

    float *wsb = ws + ((size_t)bh * nchunks + chunk) * L::per_chunk;
    for (int idx = tid; idx < C * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        const float gr = Gs[r * DKP + c];
        wsb[L::off_Qg + idx] = Qs[r * DKP + c] * expf(gr);
        wsb[L::off_Kd + idx] = sgnC[c] * Ks[r * DKP + c] * expf(gamC[c] - gr);
    }
    for (int idx = tid; idx < C * C; idx += 256) wsb[L::off_A + idx] = Aqk[(idx / C) * CP + idx % C];
    if (tid < DK) wsb[L::off_gC + tid] = sgnC[tid] * expf(gamC[tid]);
    __syncthreads();
    // EK = diag(beta) K e^gamma into the Q buffer; V <- diag(beta) V
    for (int idx = tid; idx < C * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        Qs[r * DKP + c] = bs[r] * Ks[r * DKP + c] * expf(Gs[r * DKP + c]);
    }
    for (int idx = tid; idx < C * DV; idx += 256) {
        const int r = idx / DV, c = idx % DV;
        Vs[r * DVP + c] *= bs[r];
    }
    __syncthreads();
    // W = Tm EK and U = Tm V as register tiles: thread = 4 rows (4 rg .. 4 rg + 3) x N / 16
    // columns (cg, cg + 16, ...); Tm is zero above its diagonal, so the sum may run to the
    // tile's last row.
    auto tm_product = [&](const float *X, int ldx, int N, size_t off) {
        const int rg = tid >> 4, cg = tid & 15;
        const float *t0 = Tm + (4 * rg) * CP;
        float acc[4][8];
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[m][e] = 0.f;
        const int ne = N / 16;
        for (int i = 0; i <= 4 * rg + 3; ++i) {
            const float a0 = t0[i], a1 = t0[CP + i], a2 = t0[2 * CP + i], a3 = t0[3 * CP + i];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (e < ne) {
                    const float x = X[i * ldx + cg + 16 * e];
                    acc[0][e] = fmaf(a0, x, acc[0][e]);
                    acc[1][e] = fmaf(a1, x, acc[1][e]);
                    acc[2][e] = fmaf(a2, x, acc[2][e]);
                    acc[3][e] = fmaf(a3, x, acc[3][e]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (e < ne) wsb[off + (size_t)(4 * rg + m) * N + cg + 16 * e] = acc[m][e];
    };
    tm_product(Qs, DKP, DK, L::off_W);
    tm_product(Vs, DVP, DV, L::off_U);
}

template <int DK, int DVS>
constexpr size_t scan_smem_bytes() {
    return sizeof(float) * ((size_t)C * (DK + 1) * 3 + (size_t)DK * (DVS + 1) +
                            (size_t)C * (DVS + 1) * 3 + (size_t)C * CP + DK);
}

template <typename TO, int DK, int DV, int DVS>
__global__ void __launch_bounds__(256)
chunk_scan_kernel(const float *__restrict__ ws, const float *__restrict__ S0, TO *__restrict__ out,
                  float *__restrict__ S_T, int T, int H, int nchunks, float scale) {
    constexpr int DKP = DK + 1, SP = DVS + 1;
    using L = RefLayout<DK, DV>;
    extern __shared__ float sm[];
    float *Ws = sm;
    float *Qgs = Ws + C * DKP;
    float *Kds = Qgs + C * DKP;
    float *Ss = Kds + C * DKP;      // DK x SP
    float *Vt = Ss + DK * SP;       // C x SP
    float *Os = Vt + C * SP;
    float *Us = Os + C * SP;
    float *Aq = Us + C * SP;        // C x CP
    float *gCs = Aq + C * CP;       // DK

    const int bh = blockIdx.x, j0 = blockIdx.y * DVS;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x;

    for (int idx = tid; idx < DK * DVS; idx += 256) {
        const int c = idx / DVS, j = idx % DVS;
        Ss[c * SP + j] = S0 ? S0[((size_t)bh * DK + c) * DV + j0 + j] : 0.f;
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * C;
        const int n = min(C, T - t0);
        const float *wsb = ws + ((size_t)bh * nchunks + ch) * L::per_chunk;
        {
            // the chunk's record: every 16-byte load of a matrix is issued before any of its
            // stores, so each thread keeps NV loads of three matrices in flight (offsets and the
            // record size are multiples of 4 floats, so every float4 is aligned)
            constexpr int NV = C * DK / 4 / 256;
            const float4 *w4 = reinterpret_cast<const float4 *>(wsb + L::off_W);
            const float4 *q4 = reinterpret_cast<const float4 *>(wsb + L::off_Qg);
            const float4 *k4 = reinterpret_cast<const float4 *>(wsb + L::off_Kd);
            float4 a[NV], bq[NV], bk[NV];
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                a[m] = w4[tid + 256 * m];
                bq[m] = q4[tid + 256 * m];
                bk[m] = k4[tid + 256 * m];
            }
            const int ur = tid >> 2, up = tid & 3;                  // U: 64 rows x 16 columns
            const float4 u = *reinterpret_cast<const float4 *>(wsb + L::off_U + (size_t)ur * DV + j0 + 4 * up);
            float4 av[4];
            const float4 *a4 = reinterpret_cast<const float4 *>(wsb + L::off_A);
#pragma unroll
            for (int m = 0; m < 4; ++m) av[m] = a4[tid + 256 * m];
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                const int e0 = 4 * (tid + 256 * m), r = e0 / DK, c = e0 % DK;
                float *dw = Ws + r * DKP + c, *dq = Qgs + r * DKP + c, *dk = Kds + r * DKP + c;
                dw[0] = a[m].x; dw[1] = a[m].y; dw[2] = a[m].z; dw[3] = a[m].w;
                dq[0] = bq[m].x; dq[1] = bq[m].y; dq[2] = bq[m].z; dq[3] = bq[m].w;
                dk[0] = bk[m].x; dk[1] = bk[m].y; dk[2] = bk[m].z; dk[3] = bk[m].w;
            }
            float *du = Us + ur * SP + 4 * up;
            du[0] = u.x; du[1] = u.y; du[2] = u.z; du[3] = u.w;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int e0 = 4 * (tid + 256 * m), r = e0 / C, c = e0 % C;
                float *da = Aq + r * CP + c;
                da[0] = av[m].x; da[1] = av[m].y; da[2] = av[m].z; da[3] = av[m].w;
            }
            if (tid < DK) gCs[tid] = wsb[L::off_gC + tid];
        }
        __syncthreads();
        // Register tiles: thread = (row pair 2rg, 2rg+1; column pair 2jg, 2jg+1) of the
        // 64 x DVS products, and (RPT key rows, column pair) of the DK x DVS state update.
        const int rg = tid >> 3, jg = tid & 7, ja = 2 * jg;
        static_assert(DVS == 16, "the tiles cover 64 x 16 outputs with 256 threads");
        {
            // V~ = U - W S,  O = Qg S
            float w[2][2] = {}, o[2][2] = {};
            const float *w0 = Ws + (2 * rg) * DKP, *w1 = w0 + DKP;
            const float *q0 = Qgs + (2 * rg) * DKP, *q1 = q0 + DKP;
#pragma unroll 4
            for (int c = 0; c < DK; ++c) {
                const float s0 = Ss[c * SP + ja], s1 = Ss[c * SP + ja + 1];
                const float a0 = w0[c], a1 = w1[c], b0 = q0[c], b1 = q1[c];
                w[0][0] = fmaf(a0, s0, w[0][0]); w[0][1] = fmaf(a0, s1, w[0][1]);
                w[1][0] = fmaf(a1, s0, w[1][0]); w[1][1] = fmaf(a1, s1, w[1][1]);
                o[0][0] = fmaf(b0, s0, o[0][0]); o[0][1] = fmaf(b0, s1, o[0][1]);
                o[1][0] = fmaf(b1, s0, o[1][0]); o[1][1] = fmaf(b1, s1, o[1][1]);
            }
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = 2 * rg + m, j = ja + e;
                    Vt[r * SP + j] = Us[r * SP + j] - w[m][e];
                    Os[r * SP + j] = o[m][e];
                }
        }
        __syncthreads();
        {
            // out = scale (O + A_qk V~); A_qk is zero above the diagonal
            float acc[2][2];
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int e = 0; e < 2; ++e) acc[m][e] = Os[(2 * rg + m) * SP + ja + e];
            const float *a0 = Aq + (2 * rg) * CP, *a1 = a0 + CP;
            for (int i = 0; i <= 2 * rg + 1; ++i) {
                const float v0 = Vt[i * SP + ja], v1 = Vt[i * SP + ja + 1];
                const float x0 = a0[i], x1 = a1[i];
                acc[0][0] = fmaf(x0, v0, acc[0][0]); acc[0][1] = fmaf(x0, v1, acc[0][1]);
                acc[1][0] = fmaf(x1, v0, acc[1][0]); acc[1][1] = fmaf(x1, v1, acc[1][1]);
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int r = 2 * rg + m;
                if (r < n) {
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        out[(((size_t)b * T + t0 + r) * H + h) * DV + j0 + ja + e] = from_f32<TO>(scale * acc[m][e]);
                }
            }
        }
        {
            // S <- diag(gC) S + Kd^T V~ (each thread reads and writes only its own entries)
            constexpr int RPT = DK / 32;
            const int cb = RPT * rg;
            float acc[RPT][2];
#pragma unroll
            for (int m = 0; m < RPT; ++m)
#pragma unroll
                for (int e = 0; e < 2; ++e) acc[m][e] = gCs[cb + m] * Ss[(cb + m) * SP + ja + e];
            for (int r = 0; r < n; ++r) {
                const float v0 = Vt[r * SP + ja], v1 = Vt[r * SP + ja + 1];
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    const float kd = Kds[r * DKP + cb + m];
                    acc[m][0] = fmaf(kd, v0, acc[m][0]);
                    acc[m][1] = fmaf(kd, v1, acc[m][1]);
                }
            }
#pragma unroll
            for (int m = 0; m < RPT; ++m)
#pragma unroll
                for (int e = 0; e < 2; ++e) Ss[(cb + m) * SP + ja + e] = acc[m][e];
        }
        __syncthreads();
    }
    if (S_T) {
        for (int idx = tid; idx < DK * DVS; idx += 256) {
            const int c = idx / DVS, j = idx % DVS;
            S_T[((size_t)bh * DK + c) * DV + j0 + j] = Ss[c * SP + j];
        }
    }
}

template <typename TQ, typename TG, typename TB, int DK, int DV>
cudaError_t launch_intra(const ChunkArgs &a, int nchunks, float *ws, cudaStream_t st) {
    auto kern = chunk_intra_kernel<TQ, TG, TB, DK, DV>;
    const size_t smem = intra_smem_bytes<DK, DV>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    mark_launch(a, st);
    dim3 grid(nchunks, a.B * a.H);
    kern<<<grid, 256, smem, st>>>((const TQ *)a.q, (const TQ *)a.k, (const TQ *)a.v, (const TG *)a.g,
                                  (const TB *)a.beta, a.T, a.H, nchunks, a.fl, ws);
    return cudaGetLastError();
}

template <typename TO, int DK, int DV>
cudaError_t launch_scan(const ChunkArgs &a, int nchunks, const float *ws, cudaStream_t st) {
    constexpr int DVS = 16;
    auto kern = chunk_scan_kernel<TO, DK, DV, DVS>;
    const size_t smem = scan_smem_bytes<DK, DVS>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    mark_launch(a, st);
    dim3 grid(a.B * a.H, DV / DVS);
    kern<<<grid, 256, smem, st>>>(ws, a.S0, (TO *)a.out, a.S_T, a.T, a.H, nchunks, a.fl.scale);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_ref_dims(const ChunkArgs &a, cudaStream_t st) {
    const int nchunks = (a.T + C - 1) / C;
    float *ws = (float *)a.workspace;
    cudaError_t e;
    // phase 1: input element types
    if (a.t_qkv == Elt::BF16 && a.t_g == Elt::BF16 && a.t_beta == Elt::BF16)
        e = launch_intra<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16, DK, DV>(a, nchunks, ws, st);
    else if (a.t_qkv == Elt::F32 && a.t_g == Elt::F32 && a.t_beta == Elt::F32)
        e = launch_intra<float, float, float, DK, DV>(a, nchunks, ws, st);
    else
        return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    // phase 2: output element type
    if (a.t_out == Elt::BF16) e = launch_scan<__nv_bfloat16, DK, DV>(a, nchunks, ws, st);
    else e = launch_scan<float, DK, DV>(a, nchunks, ws, st);
    return e;
}
}  // namespace

size_t chunk_ref_workspace_bytes(int B, int T, int H, int dk, int dv) {
    const size_t nchunks = ((size_t)T + C - 1) / C;
    const size_t per = (size_t)C * dk * 3 + (size_t)C * dv + (size_t)C * C + dk;
    return sizeof(float) * per * nchunks * (size_t)B * (size_t)H;
}

cudaError_t launch_chunk_ref(const ChunkArgs &a, cudaStream_t st) {
    if (a.dk == 128 && a.dv == 128) return launch_ref_dims<128, 128>(a, st);
    if (a.dk == 128 && a.dv == 64) return launch_ref_dims<128, 64>(a, st);
    if (a.dk == 64 && a.dv == 128) return launch_ref_dims<64, 128>(a, st);
    return launch_ref_dims<64, 64>(a, st);
}

}  // namespace kda
