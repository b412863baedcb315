// kda_chunk_bwd.cu -- backward of the KDA forward (chunk_kda training): gradients of
// L = <dO, O> + <dS_T, S_T> with respect to q, k, v, g, beta and S0.
//
// The forward is the recurrence of page "Kimi K3 の KDA(1)", section 1.2.1 (decay, erase,
// write, read the post-write state) with per-channel decay (page "GDN, KDA の整理", section
// "Kimi Delta Attention").  With St = Diag(alpha_t) S_{t-1}, r = v_t - St^T k_t and
// G = dS_t + q_t (scale do_t)^T, its reverse pass per token is
//
//   dq_t = S_t (scale do_t)      a = G^T k_t       dbeta_t = a . r      dv_t = beta_t a
//   dk_t = beta_t G r - St dv_t  dSt = G - k_t dv_t^T   dalpha_t = rowsum(dSt * S_{t-1})
//   dS_{t-1} = Diag(alpha_t) dSt
//
// then dg = alpha * dalpha (alpha = e^g; Complex-KDA: dg = dalpha) and the L2 norm's
// backward dx = (dx_hat - x_hat (x_hat . dx_hat)) / n.
//
// Layout of the work.  The value columns of S evolve independently (column j sees only
// v_{t,j}), and so do the columns of dS; a CTA owns NS = 16 columns of one (b, h): 8 warps, two
// columns per warp (two independent reduction chains per warp), each lane 4 (or 2) key rows of
// both in registers.
//
// The reverse recursion dS_{t-1} = Diag(alpha_t)(G - beta_t k_t (k_t . G)), G = dS_t + q_t do_t^T,
// needs no state.  So two sequential sweeps over the tokens, one launch side by side, give every
// 8-token window both of its boundary values: the forward sweep writes S at every window
// start, the reverse sweep dS at every window end (and dS0).  Then every window's local work
// is independent, and a second launch runs all windows of all heads at once, one thread-block
// cluster of DV / NS CTAs per (window, b, h):
//   1. recompute the window's pre-token states S_{t-1} into shared memory, with r_t;
//   2. reverse pass over the window from its end's dS: G = dS + q do, a = k . G (a warp
//      reduction), dv = beta a, dS <- alpha (G - k dv); it records dv_t and a_t r_t per column;
//   3. post-pass: every (token, key row) sum over the CTA's columns -- dq (S_t do), dk
//      (beta G r - St dv), dalpha (dSt * S_{t-1}) -- re-running the elementwise dS recursion
//      from the window's end with the recorded dv (no reduction on it), thread = (key row,
//      column group);
//   4. the CTAs of the cluster sum those partial sums through distributed shared memory; the
//      CTA that finishes a token row applies the L2-norm and gate backward and writes it.
// No atomics anywhere; the result is deterministic.
#include <cooperative_groups.h>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace cg = cooperative_groups;

namespace kda {

namespace {
constexpr int WL = 8;           // tokens per window (one checkpoint each)
constexpr int NS = 16;          // value columns per CTA
constexpr int NW = 8;           // warps per CTA, two columns each
constexpr int NT = NW * 32;     // threads per CTA
static_assert(WL == NW, "staging gives one warp per token row of a window");

// The inputs of one window of tokens, staged in shared memory.
template <int DK>
struct WinIn {
    float qs[WL][DK], ks[WL][DK], as[WL][DK];   // normalised q, k and alpha
    float vs[WL][NS], dos[WL][NS];              // v and scale * dO of this CTA's columns
    float bs[WL], nq[WL], nk[WL];               // beta and the reciprocal norms of q and k
};

template <int DK>
struct BwdSmem {
    static constexpr int JQ = NT / DK;           // column groups of the post-pass
    WinIn<DK> in;
    float win[WL][NS][DK];      // S_{t-1} of each token of the window, per column
    float part[3][JQ][WL][DK];  // post-pass sums (dq, dk, dalpha) per column group
    float dsb[NS][DK];          // dS at the window's end (the post-pass restarts from it)
    float rr[WL][NS], drr[WL][NS], ab[WL][NS];   // r, dv and a*r per token and column
};


// RPL consecutive FP32 values (RPL = 4 or 2) of 16- or 8-byte aligned memory, and the store.
template <int RPL>
__device__ __forceinline__ void ld_rows(const float *p, float (&x)[RPL]) {
    if constexpr (RPL == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        x[0] = t.x; x[1] = t.y;
    }
}
template <int RPL>
__device__ __forceinline__ void st_rows(float *p, const float (&x)[RPL]) {
    if constexpr (RPL == 4) *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
}

// RPL consecutive input values as one vector load, kept packed until they are used.
template <typename T, int RPL> struct RowVec;
template <> struct RowVec<__nv_bfloat16, 4> {
    uint2 u;
    __device__ void unpack(float (&x)[4]) const {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    }
};
template <> struct RowVec<__nv_bfloat16, 2> {
    uint32_t u;
    __device__ void unpack(float (&x)[2]) const {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
        x[0] = a.x; x[1] = a.y;
    }
};
template <> struct RowVec<float, 4> {
    float4 u;
    __device__ void unpack(float (&x)[4]) const { x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; }
};
template <> struct RowVec<float, 2> {
    float2 u;
    __device__ void unpack(float (&x)[2]) const { x[0] = u.x; x[1] = u.y; }
};
template <typename T, int RPL>
__device__ __forceinline__ void ldg_rows(RowVec<T, RPL> &r, const T *p) {
    r.u = *reinterpret_cast<const decltype(r.u) *>(p);
}

// A window's inputs as one warp's token row holds them between its global loads and its
// shared-memory writes (so the loads of the next window can be in flight during this one).
// Lane l holds channels RPL l .. RPL l + RPL - 1.
template <typename T, int DK>
struct RowIn {
    RowVec<T, DK / 32> q, k, g;
    T v, dout, beta;
};

// Load token row ta + (warp index) of the sequence whose token t sits at row row0 + t * H, if
// it is one of the m rows of the window; the CTA's value columns are [col0, col0 + NS).
template <typename T, int DK, int DV>
__device__ __forceinline__ void load_row(RowIn<T, DK> &r, const T *q, const T *k, const T *v, const T *g,
                                         const T *beta, const T *dout, size_t row0, int H, int ta,
                                         int m, int col0) {
    constexpr int RPL = DK / 32;
    const int tt = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (tt >= m) return;
    const size_t row = row0 + (size_t)(ta + tt) * H;
    ldg_rows<T, RPL>(r.q, q + row * DK + RPL * lane);
    ldg_rows<T, RPL>(r.k, k + row * DK + RPL * lane);
    ldg_rows<T, RPL>(r.g, g + row * DK + RPL * lane);
    if (lane < NS) {
        r.v = v[row * DV + col0 + lane];
        r.dout = dout[row * DV + col0 + lane];
    }
    if (lane == 0) r.beta = beta[row];
}

// Normalise q and k, form alpha and write the row to the window in shared memory.
template <typename T, int DK>
__device__ __forceinline__ void commit_row(WinIn<DK> &in, const RowIn<T, DK> &r, int m,
                                           const KernelFlags &fl) {
    constexpr int RPL = DK / 32;
    const int tt = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (tt >= m) return;
    float qv[RPL], kv[RPL], gv[RPL], sq = 0.f, sk = 0.f;
    r.q.unpack(qv);
    r.k.unpack(kv);
    r.g.unpack(gv);
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        sq += qv[i] * qv[i];
        sk += kv[i] * kv[i];
        gv[i] = fl.complex_gate ? gv[i] : expf(gv[i]);
    }
    float fq = 1.f, fk = 1.f;
    if (fl.l2norm) {
        fq = rsqrtf(warp_sum(sq) + kL2Eps);
        fk = rsqrtf(warp_sum(sk) + kL2Eps);
    }
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        qv[i] *= fq;
        kv[i] *= fk;
    }
    st_rows<RPL>(&in.as[tt][RPL * lane], gv);
    st_rows<RPL>(&in.qs[tt][RPL * lane], qv);
    st_rows<RPL>(&in.ks[tt][RPL * lane], kv);
    if (lane < NS) {
        in.vs[tt][lane] = to_f32(r.v);
        in.dos[tt][lane] = fl.scale * to_f32(r.dout);
    }
    if (lane == 0) {
        in.bs[tt] = to_f32(r.beta);
        in.nq[tt] = fq;
        in.nk[tt] = fk;
    }
}

// Stage tokens [ta, ta + m): one warp per token row.
template <typename T, int DK, int DV>
__device__ __forceinline__ void stage_window(WinIn<DK> &in, const T *q, const T *k, const T *v,
                                             const T *g, const T *beta, const T *dout, size_t row0,
                                             int H, int ta, int m, int col0, const KernelFlags &fl) {
    RowIn<T, DK> r;
    load_row<T, DK, DV>(r, q, k, v, g, beta, dout, row0, H, ta, m, col0);
    commit_row<T, DK>(in, r, m, fl);
}

__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }

// One forward step of the warp's two columns lc0, lc0 + 1 (s[i] holds row RPL lane + i of
// both, as one packed pair): S <- alpha S, r = v - S^T k, S += beta k r^T.  With win / rr,
// S_{t-1} and r are recorded.
template <int DK>
__device__ __forceinline__ void fwd_step(const WinIn<DK> &in, int tt, int lc0, int lane,
                                         float2 (&s)[DK / 32], float (*win)[NS][DK],
                                         float (*rr)[NS]) {
    constexpr int RPL = DK / 32;
    const int c0 = RPL * lane;
    if (win) {
        float x0[RPL], x1[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            x0[i] = s[i].x;
            x1[i] = s[i].y;
        }
        st_rows<RPL>(&win[tt][lc0][c0], x0);
        st_rows<RPL>(&win[tt][lc0 + 1][c0], x1);
    }
    float a[RPL], kk[RPL];
    ld_rows<RPL>(&in.as[tt][c0], a);
    ld_rows<RPL>(&in.ks[tt][c0], kk);
    float2 d = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        s[i] = __fmul2_rn(s[i], f2(a[i]));
        d = __ffma2_rn(f2(kk[i]), s[i], d);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        d = __fadd2_rn(d, make_float2(__shfl_xor_sync(0xffffffffu, d.x, o),
                                      __shfl_xor_sync(0xffffffffu, d.y, o)));
    const float r0 = in.vs[tt][lc0] - d.x, r1 = in.vs[tt][lc0 + 1] - d.y;
    if (rr && lane == 0) {
        rr[tt][lc0] = r0;
        rr[tt][lc0 + 1] = r1;
    }
    const float bt = in.bs[tt];
    const float2 br = make_float2(bt * r0, bt * r1);
#pragma unroll
    for (int i = 0; i < RPL; ++i) s[i] = __ffma2_rn(f2(kk[i]), br, s[i]);
}

// One reverse step of the warp's two columns: G = dS + q do, d = k . G, dv = beta d,
// dS <- alpha (G - k dv).  Returns d and dv of both columns.
template <int DK>
__device__ __forceinline__ void rev_step(const WinIn<DK> &in, int tt, int lc0, int lane,
                                         float2 (&dS)[DK / 32], float2 &d, float2 &dr) {
    constexpr int RPL = DK / 32;
    const int c0 = RPL * lane;
    const float2 dov = make_float2(in.dos[tt][lc0], in.dos[tt][lc0 + 1]);
    const float bt = in.bs[tt];
    float qq[RPL], kk[RPL], a[RPL];
    ld_rows<RPL>(&in.qs[tt][c0], qq);
    ld_rows<RPL>(&in.ks[tt][c0], kk);
    ld_rows<RPL>(&in.as[tt][c0], a);
    float2 G[RPL];
    d = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        G[i] = __ffma2_rn(f2(qq[i]), dov, dS[i]);
        d = __ffma2_rn(f2(kk[i]), G[i], d);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        d = __fadd2_rn(d, make_float2(__shfl_xor_sync(0xffffffffu, d.x, o),
                                      __shfl_xor_sync(0xffffffffu, d.y, o)));
    dr = __fmul2_rn(f2(bt), d);
    const float2 ndr = make_float2(-dr.x, -dr.y);
#pragma unroll
    for (int i = 0; i < RPL; ++i) dS[i] = __fmul2_rn(f2(a[i]), __ffma2_rn(f2(kk[i]), ndr, G[i]));
}

// A lane's RPL rows of the warp's two columns from / to a column-major checkpoint.
template <int RPL>
__device__ __forceinline__ void ck_load(const float *ck, int DK, int lane, float2 (&x)[RPL]) {
    float a[RPL], b[RPL];
    ld_rows<RPL>(ck + RPL * lane, a);
    ld_rows<RPL>(ck + DK + RPL * lane, b);
#pragma unroll
    for (int i = 0; i < RPL; ++i) x[i] = make_float2(a[i], b[i]);
}
template <int RPL>
__device__ __forceinline__ void ck_store(float *ck, int DK, int lane, const float2 (&x)[RPL]) {
    float a[RPL], b[RPL];
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        a[i] = x[i].x;
        b[i] = x[i].y;
    }
    st_rows<RPL>(ck + RPL * lane, a);
    st_rows<RPL>(ck + DK + RPL * lane, b);
}

// Checkpoint of window wi of sequence-head bh, value column j: DK FP32 values (column-major).
__device__ __forceinline__ size_t ck_off(int bh, int nwin, int wi, int j, int DK, int DV) {
    return (((size_t)bh * nwin + wi) * DV + j) * DK;
}

// Launch 1: the two sequential sweeps.  CTAs [0, n) run the forward recurrence and write S at
// every window start to ckpt; CTAs [n, 2n) run the reverse recursion from dS_T and write dS at
// every window end to dckpt, then dS0.  n = B * H * (DV / NS).
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, 4)
chunk_bwd_sweep_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       const T *__restrict__ g, const T *__restrict__ beta,
                       const float *__restrict__ S0, const T *__restrict__ dout,
                       const float *__restrict__ dST, float *__restrict__ dS0,
                       float *__restrict__ ckpt, float *__restrict__ dckpt, int T_, int H, int nwin,
                       KernelFlags fl) {
    constexpr int RPL = DK / 32;
    constexpr int CS = DV / NS;
    __shared__ __align__(16) WinIn<DK> in;
    const int n = (int)gridDim.x / 2;
    const bool reverse = (int)blockIdx.x >= n;
    const int cta = (int)blockIdx.x - (reverse ? n : 0);
    const int bh = cta / CS, rank = cta % CS;
    const int b = bh / H, h = bh % H;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lc0 = 2 * w, j0 = rank * NS + lc0;
    const size_t row0 = (size_t)b * T_ * H + h;
    const size_t sbase = (size_t)bh * DK * DV;

    float2 s[RPL];
    const float *init = reverse ? dST : S0;
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        const size_t rowc = sbase + (size_t)(RPL * lane + i) * DV + j0;
        s[i] = init ? *reinterpret_cast<const float2 *>(&init[rowc]) : make_float2(0.f, 0.f);
    }
    auto put = [&](float *base, int wi) { ck_store<RPL>(base + ck_off(bh, nwin, wi, j0, DK, DV), DK, lane, s); };

    // Window wi covers tokens [wi WL, min(wi WL + WL, T)).  Each pass stages window wi from
    // registers loaded during the previous window's steps, then loads the next window's rows.
    RowIn<T, DK> r;
    if (!reverse) {
        const int nw = nwin - 1;                // the last window's state is its start's
        if (nw > 0) load_row<T, DK, DV>(r, q, k, v, g, beta, dout, row0, H, 0, WL, rank * NS);
        for (int wi = 0; wi < nw; ++wi) {
            put(ckpt, wi);
            __syncthreads();
            commit_row<T, DK>(in, r, WL, fl);
            if (wi + 1 < nw)
                load_row<T, DK, DV>(r, q, k, v, g, beta, dout, row0, H, (wi + 1) * WL, WL, rank * NS);
            __syncthreads();
#pragma unroll
            for (int tt = 0; tt < WL; ++tt) fwd_step<DK>(in, tt, lc0, lane, s, nullptr, nullptr);
        }
        put(ckpt, nwin - 1);
        return;
    }
    load_row<T, DK, DV>(r, q, k, v, g, beta, dout, row0, H, (nwin - 1) * WL, T_ - (nwin - 1) * WL,
                        rank * NS);
    for (int wi = nwin - 1; wi >= 0; --wi) {
        put(dckpt, wi);
        if (wi == 0 && !dS0) return;
        const int ta = wi * WL, m = min(WL, T_ - ta);
        __syncthreads();
        commit_row<T, DK>(in, r, m, fl);
        if (wi > 0) load_row<T, DK, DV>(r, q, k, v, g, beta, dout, row0, H, (wi - 1) * WL, WL, rank * NS);
        __syncthreads();
        float2 d, dr;
        if (m == WL) {
#pragma unroll
            for (int tt = WL - 1; tt >= 0; --tt) rev_step<DK>(in, tt, lc0, lane, s, d, dr);
        } else {
            for (int tt = m - 1; tt >= 0; --tt) rev_step<DK>(in, tt, lc0, lane, s, d, dr);
        }
    }
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        const size_t rowc = sbase + (size_t)(RPL * lane + i) * DV + j0;
        *reinterpret_cast<float2 *>(&dS0[rowc]) = s[i];
    }
}

// Launch 2: one cluster of DV / NS CTAs per (window, b, h); cluster ci is window ci / (B H) of
// sequence-head ci % (B H).
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, 2)
chunk_bwd_block_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       const T *__restrict__ g, const T *__restrict__ beta, const T *__restrict__ dout,
                       float *__restrict__ dq, float *__restrict__ dkk, float *__restrict__ dvv,
                       float *__restrict__ dg, float *__restrict__ dbeta,
                       const float *__restrict__ ckpt, const float *__restrict__ dckpt, int T_, int H,
                       int BH, int nwin, KernelFlags fl) {
    constexpr int RPL = DK / 32;            // key rows per lane
    constexpr int CS = DV / NS;             // CTAs per cluster
    constexpr int JQ = BwdSmem<DK>::JQ;     // post-pass column groups
    constexpr int CPJ = NS / JQ;            // columns per post-pass thread
    constexpr int TPC = (WL + CS - 1) / CS; // token rows each CTA finishes per window
    static_assert(CPJ % 4 == 0, "the post-pass reads r, dv and dO four columns at a time");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem<DK> &sm = *reinterpret_cast<BwdSmem<DK> *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();

    const int rank = (int)cluster.block_rank();
    const int ci = (int)blockIdx.x / CS;
    const int bh = ci % BH, wi = ci / BH;
    const int b = bh / H, h = bh % H;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lc0 = 2 * w;                  // this warp's local columns lc0, lc0 + 1
    const int j0 = rank * NS + lc0;         // and global columns j0, j0 + 1
    const size_t row0 = (size_t)b * T_ * H + h;
    auto row_of = [&](int t) { return row0 + (size_t)t * H; };

    auto load = [&](const float *base, float2 (&x)[RPL]) {
        ck_load<RPL>(base + ck_off(bh, nwin, wi, j0, DK, DV), DK, lane, x);
    };
    float2 dS[RPL];
    load(dckpt, dS);

    auto window = [&](int ta, int m, float2 (&st)[RPL]) {
        __syncthreads();
        stage_window<T, DK, DV>(sm.in, q, k, v, g, beta, dout, row0, H, ta, m, rank * NS, fl);
        __syncthreads();
        if (m == WL) {      // a full window: token loops unrolled
#pragma unroll
            for (int tt = 0; tt < WL; ++tt) fwd_step<DK>(sm.in, tt, lc0, lane, st, sm.win, sm.rr);
        } else {
            for (int tt = 0; tt < m; ++tt) fwd_step<DK>(sm.in, tt, lc0, lane, st, sm.win, sm.rr);
        }
        {
            float x0[RPL], x1[RPL];
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                x0[i] = dS[i].x;
                x1[i] = dS[i].y;
            }
            st_rows<RPL>(&sm.dsb[lc0][RPL * lane], x0);
            st_rows<RPL>(&sm.dsb[lc0 + 1][RPL * lane], x1);
        }
        __syncwarp();
        // 2. reverse pass (sequential in t)
        auto rev = [&](int tt) {
            float2 d, dr;
            rev_step<DK>(sm.in, tt, lc0, lane, dS, d, dr);
            if (lane == 0) {
                sm.drr[tt][lc0] = dr.x;
                sm.drr[tt][lc0 + 1] = dr.y;
                sm.ab[tt][lc0] = d.x * sm.rr[tt][lc0];
                sm.ab[tt][lc0 + 1] = d.y * sm.rr[tt][lc0 + 1];
                *reinterpret_cast<float2 *>(&dvv[row_of(ta + tt) * DV + j0]) = dr;
            }
        };
        if (m == WL) {
#pragma unroll
            for (int tt = WL - 1; tt >= 0; --tt) rev(tt);
        } else {
            for (int tt = m - 1; tt >= 0; --tt) rev(tt);
        }
        __syncthreads();
        // 3. post-pass: thread = (key row c, column group jq), the columns in packed pairs
        {
            constexpr int CP = CPJ / 2;
            const int c = threadIdx.x % DK, jq = threadIdx.x / DK;
            float2 dl[CP];
#pragma unroll
            for (int p = 0; p < CP; ++p)
                dl[p] = make_float2(sm.dsb[jq * CPJ + 2 * p][c], sm.dsb[jq * CPJ + 2 * p + 1][c]);
            auto post = [&](int tt) {
                const float a = sm.in.as[tt][c], kc = sm.in.ks[tt][c], qc = sm.in.qs[tt][c];
                const float bt = sm.in.bs[tt];
                float2 r[CP], dr[CP], dov[CP];
#pragma unroll
                for (int j4 = 0; j4 < CP; j4 += 2) {
                    const int jl = jq * CPJ + 2 * j4;
                    *reinterpret_cast<float4 *>(&r[j4]) = *reinterpret_cast<const float4 *>(&sm.rr[tt][jl]);
                    *reinterpret_cast<float4 *>(&dr[j4]) = *reinterpret_cast<const float4 *>(&sm.drr[tt][jl]);
                    *reinterpret_cast<float4 *>(&dov[j4]) = *reinterpret_cast<const float4 *>(&sm.in.dos[tt][jl]);
                }
                const float2 a2 = f2(a), btk = f2(bt * kc), q2 = f2(qc), b2 = f2(bt), nk = f2(-kc);
                float2 sq = make_float2(0.f, 0.f), sk = sq, sa = sq;
#pragma unroll
                for (int p = 0; p < CP; ++p) {
                    const int jl = jq * CPJ + 2 * p;
                    const float2 sp = make_float2(sm.win[tt][jl][c], sm.win[tt][jl + 1][c]);
                    const float2 St = __fmul2_rn(a2, sp);
                    const float2 post = __ffma2_rn(btk, r[p], St);
                    const float2 G = __ffma2_rn(q2, dov[p], dl[p]);
                    sq = __ffma2_rn(post, dov[p], sq);
                    sk = __ffma2_rn(__fmul2_rn(b2, G), r[p], sk);
                    sk = __ffma2_rn(make_float2(-St.x, -St.y), dr[p], sk);
                    const float2 dSt = __ffma2_rn(nk, dr[p], G);
                    sa = __ffma2_rn(dSt, sp, sa);
                    dl[p] = __fmul2_rn(a2, dSt);
                }
                sm.part[0][jq][tt][c] = sq.x + sq.y;
                sm.part[1][jq][tt][c] = sk.x + sk.y;
                sm.part[2][jq][tt][c] = sa.x + sa.y;
            };
            if (m == WL) {
#pragma unroll
                for (int tt = WL - 1; tt >= 0; --tt) post(tt);
            } else {
                for (int tt = m - 1; tt >= 0; --tt) post(tt);
            }
        }
        __syncthreads();
        cluster.sync();
        // 4. token rows tt = rank, rank + CS, ... of the window: sum over the cluster's CTAs
        //    and column groups, finish and write
        for (int item = w; item < TPC * 4; item += NW) {
            const int tt = rank + CS * (item / 4), qty = item % 4;
            if (tt >= m) continue;
            const size_t row = row_of(ta + tt);
            if (qty == 3) {
                float sb = 0.f;
                if (lane < NS)
                    for (int rk = 0; rk < CS; ++rk) sb += *cluster.map_shared_rank(&sm.ab[tt][lane], rk);
                sb = warp_sum(sb);
                if (lane == 0) dbeta[row] = sb;
                continue;
            }
            float val[RPL];
#pragma unroll
            for (int i = 0; i < RPL; ++i) val[i] = 0.f;
            for (int rk = 0; rk < CS; ++rk) {
#pragma unroll
                for (int jq = 0; jq < JQ; ++jq) {
                    const float *rp = cluster.map_shared_rank(&sm.part[qty][jq][tt][0], rk);
#pragma unroll
                    for (int i = 0; i < RPL; ++i) val[i] += rp[lane + 32 * i];
                }
            }
            if (qty == 2) {
#pragma unroll
                for (int i = 0; i < RPL; ++i) {
                    const int c = lane + 32 * i;
                    dg[row * DK + c] = fl.complex_gate ? val[i] : sm.in.as[tt][c] * val[i];
                }
            } else {
                const float *xh = qty == 0 ? &sm.in.qs[tt][0] : &sm.in.ks[tt][0];
                const float inv = qty == 0 ? sm.in.nq[tt] : sm.in.nk[tt];
                float proj = 0.f;
                if (fl.l2norm) {
                    float d = 0.f;
#pragma unroll
                    for (int i = 0; i < RPL; ++i) d += xh[lane + 32 * i] * val[i];
                    proj = warp_sum(d);
                }
                float *dst = qty == 0 ? dq : dkk;
#pragma unroll
                for (int i = 0; i < RPL; ++i) {
                    const int c = lane + 32 * i;
                    dst[row * DK + c] = fl.l2norm ? (val[i] - xh[c] * proj) * inv : val[i];
                }
            }
        }
        cluster.sync();
    };

    float2 st[RPL];
    load(ckpt, st);
    window(wi * WL, min(WL, T_ - wi * WL), st);
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const BwdArgs &a, cudaStream_t st) {
    constexpr int CS = DV / NS;
    const int nwin = (a.T + WL - 1) / WL, BH = a.B * a.H;
    float *ckpt = (float *)a.workspace;
    float *dckpt = ckpt + (size_t)BH * nwin * DK * DV;
    if (a.events && a.n_events > 0) cudaEventRecord(a.events[0], st);
    chunk_bwd_sweep_kernel<T, DK, DV><<<2 * CS * BH, NT, 0, st>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.g, (const T *)a.beta, a.S0,
        (const T *)a.dout, a.dS_T, a.dS0, ckpt, dckpt, a.T, a.H, nwin, a.fl);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    const size_t smem = sizeof(BwdSmem<DK>);
    auto kern = chunk_bwd_block_kernel<T, DK, DV>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((size_t)CS * BH * nwin));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.events && a.n_events > 1) cudaEventRecord(a.events[1], st);
    return cudaLaunchKernelEx(&cfg, kern, (const T *)a.q, (const T *)a.k, (const T *)a.v,
                              (const T *)a.g, (const T *)a.beta, (const T *)a.dout, a.dq, a.dk, a.dv,
                              a.dg, a.dbeta, (const float *)ckpt, (const float *)dckpt, a.T, a.H, BH,
                              nwin, a.fl);
}

template <typename T>
cudaError_t launch_d(const BwdArgs &a, cudaStream_t st) {
    if (a.dk_ == 128 && a.dv_ == 128) return launch_t<T, 128, 128>(a, st);
    if (a.dk_ == 128 && a.dv_ == 64) return launch_t<T, 128, 64>(a, st);
    if (a.dk_ == 64 && a.dv_ == 128) return launch_t<T, 64, 128>(a, st);
    return launch_t<T, 64, 64>(a, st);
}
}  // namespace

// S at every window start and dS at every window end, FP32.
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    const size_t nwin = ((size_t)T + WL - 1) / WL;
    return 2 * (size_t)B * H * nwin * dk * dv * sizeof(float);
}

cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t st) {
    return a.bf16 ? launch_d<__nv_bfloat16>(a, st) : launch_d<float>(a, st);
}

}  // namespace kda
