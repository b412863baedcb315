// kda_decode.cu -- one recurrent KDA step per sequence (decode).
//
// Page "Kimi K3 模型结构（2）：序列维度（下），chunkwise 并行与下界衰减", Q&A item
// on train/prefill vs decode: decode uses the recurrent form, one token per
// call.  The update is the recurrence of page "Kimi K3 の KDA(1)" section
// 1.2.1 (decay, erase, write, then read the post-write state).  Every value
// column of S evolves independently under the shared transition (same page,
// section 2.3.2), which is what lets one CTA stream its (n, h) state through
// registers exactly once:
//
//   read S (64 KiB FP32 for dk = dv = 128) -> St = Diag(alpha) S
//   column sums  p_k[j] = sum_i k_i St[i,j],  p_q[j] = sum_i q_i St[i,j]
//   u_j = beta (v_j - p_k[j]);   o_j = scale (p_q[j] + (q.k) u_j)
//   write S_t = St + k u^T
//
// The step is bound by HBM: 2 * dk * dv * 4 bytes of state traffic per
// (n, h) against 7 dk dv FLOPs.  Each thread owns a 4-column x RPT-row patch
// (float4 loads, 512 contiguous bytes per warp and row); loads are issued
// first so that the small q/k/g/v set-up overlaps the state's latency.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

// Decode prologue (page "Kimi K3 の KDA(1)" section 1.2.1 for the short convolution, SiLU and
// beta = sigmoid(b); page "Kimi K3 模型结构（2）", Q&A on the decay function, for the gate):
// the new token's raw q, k, v go through the causal k = 4 convolution whose three earlier
// inputs are the conv state, which is then shifted by one token.
struct DecodePro {
    const void *conv_w;
    void *conv_state;
    const float *A, *b_logit;
    int H;
    int gate_softplus;   // g = -exp(A_h) softplus(z) (Kimi Linear) instead of -5 sigmoid(exp(A_h) z)
};

// the four taps of one channel (contiguous) as one vector load
__device__ __forceinline__ void load_taps(const float *p, float (&w)[4]) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
}
__device__ __forceinline__ void load_taps(const __nv_bfloat16 *p, float (&w)[4]) {
    const uint2 t = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.y));
    w[0] = a.x; w[1] = a.y; w[2] = b.x; w[3] = b.y;
}

template <typename T, int DK, int DV, bool PRO>
__global__ void __launch_bounds__(256)
decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const T *__restrict__ g, const T *__restrict__ beta, float *__restrict__ S,
                   T *__restrict__ out, KernelFlags fl, DecodePro pro) {
    constexpr int NT = 256;
    constexpr int CG = DV / 4;        // column groups (float4 each)
    constexpr int RG = NT / CG;       // row groups
    constexpr int RPT = DK / RG;      // rows per thread
    static_assert(RG * CG == NT && RPT * RG == DK, "tiling");

    __shared__ float qs[DK], ks[DK], as[DK], vs[DV], us[DV];
    __shared__ float4 red_k[RG][CG], red_q[RG][CG];
    __shared__ float scal[4];

    const size_t unit = blockIdx.x;
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4 *Sp = reinterpret_cast<float4 *>(S + unit * (size_t)(DK * DV));

    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = __ldcs(&Sp[(size_t)(rg * RPT + r) * CG + cg]);

    float bt;
    if constexpr (PRO) {
        static_assert(DK == DV, "the decode prologue needs dk == dv");
        const int H = pro.H, h = (int)(unit % H);
        const size_t n = unit / H, HD = (size_t)H * DK, ch = (size_t)h * DK + tid;
        const T *w = static_cast<const T *>(pro.conv_w);
        T *cs = static_cast<T *>(pro.conv_state) + n * 9 * HD;   // [3 branches][3 taps][H * d]
        if (tid < DK) {
            // every load first (one round of latency, overlapping the state's), then the math,
            // then the shifted conv state
            float taps[3][4], hist[3][3], x[3];
#pragma unroll
            for (int br = 0; br < 3; ++br) {
                load_taps(w + (br * HD + ch) * 4, taps[br]);
#pragma unroll
                for (int j = 0; j < 3; ++j) hist[br][j] = to_f32(cs[(br * 3 + j) * HD + ch]);
            }
            x[0] = to_f32(q[unit * DK + tid]);
            x[1] = to_f32(k[unit * DK + tid]);
            x[2] = to_f32(v[unit * DV + tid]);
            const float zv = to_f32(g[unit * DK + tid]), a_h = pro.A[h];
            float y[3];
#pragma unroll
            for (int br = 0; br < 3; ++br) {
                const float acc = taps[br][0] * hist[br][0] + taps[br][1] * hist[br][1] +
                                  taps[br][2] * hist[br][2] + taps[br][3] * x[br];
                y[br] = acc / (1.f + expf(-acc));
            }
            qs[tid] = y[0];
            ks[tid] = y[1];
            vs[tid] = y[2];
            // alpha = e^g; softplus(z) = max(z, 0) + log1p(e^-|z|)
            as[tid] = pro.gate_softplus
                          ? expf(-expf(a_h) * (fmaxf(zv, 0.f) + log1pf(expf(-fabsf(zv)))))
                          : expf(-5.f / (1.f + expf(-expf(a_h) * zv)));
#pragma unroll
            for (int br = 0; br < 3; ++br) {
                cs[(br * 3 + 0) * HD + ch] = from_f32<T>(hist[br][1]);
                cs[(br * 3 + 1) * HD + ch] = from_f32<T>(hist[br][2]);
                cs[(br * 3 + 2) * HD + ch] = from_f32<T>(x[br]);
            }
        }
        bt = 1.f / (1.f + expf(-pro.b_logit[unit]));
    } else {
        if (tid < DK) {
            qs[tid] = to_f32(q[unit * DK + tid]);
            ks[tid] = to_f32(k[unit * DK + tid]);
            const float gv = to_f32(g[unit * DK + tid]);
            as[tid] = fl.complex_gate ? gv : expf(gv);
        }
        if (tid < DV) vs[tid] = to_f32(v[unit * DV + tid]);
        bt = to_f32(beta[unit]);
    }
    __syncthreads();
    const int warp = tid >> 5, lane = tid & 31;
    if (warp < 3) {
        float acc = 0.f;
        for (int i = lane; i < DK; i += 32) {
            const float a = warp == 1 ? ks[i] : qs[i];
            const float b = warp == 0 ? qs[i] : ks[i];
            acc += a * b;
        }
        acc = warp_sum(acc);
        if (lane == 0) scal[warp] = acc;   // 0: |q|^2, 1: |k|^2, 2: q.k
    }
    __syncthreads();
    const float fq = fl.l2norm ? rsqrtf(scal[0] + kL2Eps) : 1.f;
    const float fk = fl.l2norm ? rsqrtf(scal[1] + kL2Eps) : 1.f;
    const float qk = scal[2] * fq * fk;

    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float a = as[i], kk = ks[i], qq = qs[i];
        s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
        pk.x += kk * s[r].x; pk.y += kk * s[r].y; pk.z += kk * s[r].z; pk.w += kk * s[r].w;
        pq.x += qq * s[r].x; pq.y += qq * s[r].y; pq.z += qq * s[r].z; pq.w += qq * s[r].w;
    }
    red_k[rg][cg] = pk;
    red_q[rg][cg] = pq;
    __syncthreads();
    if (tid < DV) {
        const int j = tid, c4 = j >> 2, e = j & 3;
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            const float *rk = reinterpret_cast<const float *>(&red_k[r][c4]);
            const float *rq = reinterpret_cast<const float *>(&red_q[r][c4]);
            sk += rk[e];
            sq += rq[e];
        }
        const float u = bt * (vs[j] - fk * sk);
        us[j] = u;
        out[unit * DV + j] = from_f32<T>(fl.scale * (fq * sq + qk * u));
    }
    __syncthreads();
    const float4 u4 = reinterpret_cast<const float4 *>(us)[cg];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rg * RPT + r;
        const float kk = fk * ks[i];
        float4 o = s[r];
        o.x += kk * u4.x; o.y += kk * u4.y; o.z += kk * u4.z; o.w += kk * u4.w;
        __stcs(&Sp[(size_t)i * CG + cg], o);
    }
}

template <typename T, int DK, int DV, bool PRO>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t st) {
    decode_step_kernel<T, DK, DV, PRO><<<(unsigned)a.units, 256, 0, st>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.g, (const T *)a.beta, a.S,
        (T *)a.out, a.fl, DecodePro{a.conv_w, a.conv_state, a.A, a.b_logit, a.H, a.gate_softplus});
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_decode_d(const DecodeArgs &a, cudaStream_t st) {
    if (a.conv_w) {   // the prologue needs dk == dv (checked by the host)
        if (a.dk == 128) return launch_decode_t<T, 128, 128, true>(a, st);
        return launch_decode_t<T, 64, 64, true>(a, st);
    }
    if (a.dk == 128 && a.dv == 128) return launch_decode_t<T, 128, 128, false>(a, st);
    if (a.dk == 128 && a.dv == 64) return launch_decode_t<T, 128, 64, false>(a, st);
    if (a.dk == 64 && a.dv == 128) return launch_decode_t<T, 64, 128, false>(a, st);
    return launch_decode_t<T, 64, 64, false>(a, st);
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
    return a.bf16 ? launch_decode_d<__nv_bfloat16>(a, st) : launch_decode_d<float>(a, st);
}

}  // namespace kda
