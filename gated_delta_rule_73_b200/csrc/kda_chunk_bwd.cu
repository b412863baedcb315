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
// v_{t,j}), so a CTA owns NS = 16 columns of one (b, h): 8 warps, two columns per warp (two
// independent reduction chains per warp), each lane 4 (or 2) key rows of both in registers.
// The DV / NS CTAs of a sequence form one thread-block cluster.
//
// States are needed in reverse order.  Phase 1 runs the recurrence forward and writes the
// state at the start of every 16-token block to the workspace (FP32, column-major).  Phase 2
// walks the blocks backward, each as two 8-token windows, upper window first:
//   1. recompute the window's pre-token states S_{t-1} into shared memory, with r_t;
//   2. reverse pass over the window, the only sequential part: G = dS + q do,
//      a = k . G (a warp reduction), dv = beta a, dS <- alpha (G - k dv).  It needs no
//      state, only r_t; it records dv_t and a_t r_t per column;
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
constexpr int BL = 16;          // tokens per checkpoint block
constexpr int WL = 8;           // tokens per window (half a block)
constexpr int NS = 16;          // value columns per CTA
constexpr int NW = 8;           // warps per CTA, two columns each
constexpr int NT = NW * 32;     // threads per CTA
static_assert(WL == NW, "staging gives one warp per token row of a window");

template <int DK>
struct BwdSmem {
    static constexpr int JQ = NT / DK;           // column groups of the post-pass
    float win[WL][NS][DK];      // S_{t-1} of each token of the window, per column
    float part[3][JQ][WL][DK];  // post-pass sums (dq, dk, dalpha) per column group
    float qs[WL][DK], ks[WL][DK], as[WL][DK];    // normalised q, k and alpha of the window
    float dsb[NS][DK];          // dS at the window's end (the post-pass restarts from it)
    float rr[WL][NS], drr[WL][NS], ab[WL][NS];   // r, dv and a*r per token and column
    float vs[WL][NS], dos[WL][NS];               // v and scale * dO of this CTA's columns
    float bs[WL], nq[WL], nk[WL];
};

__device__ __forceinline__ float ldf(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, 2)
chunk_bwd_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const T *__restrict__ g, const T *__restrict__ beta, const float *__restrict__ S0,
                 const T *__restrict__ dout, const float *__restrict__ dST,
                 float *__restrict__ dq, float *__restrict__ dkk, float *__restrict__ dvv,
                 float *__restrict__ dg, float *__restrict__ dbeta, float *__restrict__ dS0,
                 float *__restrict__ ckpt, int T_, int H, int nblk, KernelFlags fl) {
    constexpr int RPL = DK / 32;            // key rows per lane
    constexpr int CS = DV / NS;             // CTAs per sequence (cluster size)
    constexpr int JQ = BwdSmem<DK>::JQ;     // post-pass column groups
    constexpr int CPJ = NS / JQ;            // columns per post-pass thread
    constexpr int TPC = (WL + CS - 1) / CS; // token rows each CTA finishes per window
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem<DK> &sm = *reinterpret_cast<BwdSmem<DK> *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();

    const int rank = (int)cluster.block_rank();
    const int bh = blockIdx.x / CS;
    const int b = bh / H, h = bh % H;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lc0 = 2 * w;                  // this warp's local columns lc0, lc0 + 1
    const int j0 = rank * NS + lc0;         // and global columns j0, j0 + 1

    auto row_of = [&](int t) { return ((size_t)b * T_ + t) * H + h; };

    // One warp per token row: normalised q, k (and 1/n), alpha, beta, this CTA's v and dO.
    auto stage = [&](int ta, int m) {
        const int tt = w;
        if (tt < m) {
            const size_t row = row_of(ta + tt);
            float qv[RPL], kv[RPL], sq = 0.f, sk = 0.f;
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int c = lane + 32 * i;
                qv[i] = ldf(q, row * DK + c);
                kv[i] = ldf(k, row * DK + c);
                sq += qv[i] * qv[i];
                sk += kv[i] * kv[i];
                const float gv = ldf(g, row * DK + c);
                sm.as[tt][c] = fl.complex_gate ? gv : expf(gv);
            }
            float fq = 1.f, fk = 1.f;
            if (fl.l2norm) {
                fq = rsqrtf(warp_sum(sq) + kL2Eps);
                fk = rsqrtf(warp_sum(sk) + kL2Eps);
            }
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                sm.qs[tt][lane + 32 * i] = qv[i] * fq;
                sm.ks[tt][lane + 32 * i] = kv[i] * fk;
            }
            if (lane < NS) {
                sm.vs[tt][lane] = ldf(v, row * DV + rank * NS + lane);
                sm.dos[tt][lane] = fl.scale * ldf(dout, row * DV + rank * NS + lane);
            }
            if (lane == 0) {
                sm.bs[tt] = ldf(beta, row);
                sm.nq[tt] = fq;
                sm.nk[tt] = fk;
            }
        }
    };

    // one forward step of both columns; with WIN, S_{t-1} goes to the window and r to rr
    auto fwd_step = [&](int tt, float (&s)[2][RPL], bool store) {
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const int c = lane + 32 * i;
            if (store) {
                sm.win[tt][lc0][c] = s[0][i];
                sm.win[tt][lc0 + 1][c] = s[1][i];
            }
            const float a = sm.as[tt][c], kc = sm.ks[tt][c];
            s[0][i] *= a;
            s[1][i] *= a;
            d0 = fmaf(kc, s[0][i], d0);
            d1 = fmaf(kc, s[1][i], d1);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            d0 += __shfl_xor_sync(0xffffffffu, d0, o);
            d1 += __shfl_xor_sync(0xffffffffu, d1, o);
        }
        const float r0 = sm.vs[tt][lc0] - d0, r1 = sm.vs[tt][lc0 + 1] - d1;
        if (store && lane == 0) {
            sm.rr[tt][lc0] = r0;
            sm.rr[tt][lc0 + 1] = r1;
        }
        const float bt = sm.bs[tt];
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const float kc = sm.ks[tt][lane + 32 * i];
            s[0][i] = fmaf(kc, bt * r0, s[0][i]);
            s[1][i] = fmaf(kc, bt * r1, s[1][i]);
        }
    };

    const size_t sbase = (size_t)bh * DK * DV;
    auto load_ckpt = [&](int blk, float (&s)[2][RPL]) {
        const float *ck = ckpt + (((size_t)bh * nblk + blk) * DV + j0) * DK;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            s[0][i] = ck[lane + 32 * i];
            s[1][i] = ck[DK + lane + 32 * i];
        }
    };

    float s[2][RPL];
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        const size_t rowc = sbase + (size_t)(lane + 32 * i) * DV + j0;
        s[0][i] = S0 ? S0[rowc] : 0.f;
        s[1][i] = S0 ? S0[rowc + 1] : 0.f;
    }

    // ---- phase 1: forward, checkpoint at every block start
    for (int blk = 0; blk < nblk; ++blk) {
        float *ck = ckpt + (((size_t)bh * nblk + blk) * DV + j0) * DK;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            ck[lane + 32 * i] = s[0][i];
            ck[DK + lane + 32 * i] = s[1][i];
        }
        if (blk == nblk - 1) break;
        for (int half = 0; half < 2; ++half) {
            const int ta = blk * BL + half * WL, m = min(WL, T_ - ta);
            __syncthreads();
            stage(ta, m);
            __syncthreads();
            for (int tt = 0; tt < m; ++tt) fwd_step(tt, s, false);
        }
    }

    // ---- phase 2: blocks in reverse, each as its upper then its lower window
    float dS[2][RPL];
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        const size_t rowc = sbase + (size_t)(lane + 32 * i) * DV + j0;
        dS[0][i] = dST ? dST[rowc] : 0.f;
        dS[1][i] = dST ? dST[rowc + 1] : 0.f;
    }

    auto window = [&](int ta, int m, float (&st)[2][RPL]) {
        __syncthreads();
        stage(ta, m);
        __syncthreads();
        for (int tt = 0; tt < m; ++tt) fwd_step(tt, st, true);
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            sm.dsb[lc0][lane + 32 * i] = dS[0][i];
            sm.dsb[lc0 + 1][lane + 32 * i] = dS[1][i];
        }
        __syncwarp();
        // 2. reverse pass (sequential in t)
        for (int tt = m - 1; tt >= 0; --tt) {
            const float do0 = sm.dos[tt][lc0], do1 = sm.dos[tt][lc0 + 1], bt = sm.bs[tt];
            float G0[RPL], G1[RPL], d0 = 0.f, d1 = 0.f;
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int c = lane + 32 * i;
                const float qc = sm.qs[tt][c], kc = sm.ks[tt][c];
                G0[i] = fmaf(qc, do0, dS[0][i]);
                G1[i] = fmaf(qc, do1, dS[1][i]);
                d0 = fmaf(kc, G0[i], d0);
                d1 = fmaf(kc, G1[i], d1);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                d0 += __shfl_xor_sync(0xffffffffu, d0, o);
                d1 += __shfl_xor_sync(0xffffffffu, d1, o);
            }
            const float dr0 = bt * d0, dr1 = bt * d1;
            if (lane == 0) {
                sm.drr[tt][lc0] = dr0;
                sm.drr[tt][lc0 + 1] = dr1;
                sm.ab[tt][lc0] = d0 * sm.rr[tt][lc0];
                sm.ab[tt][lc0 + 1] = d1 * sm.rr[tt][lc0 + 1];
                *reinterpret_cast<float2 *>(&dvv[row_of(ta + tt) * DV + j0]) = make_float2(dr0, dr1);
            }
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int c = lane + 32 * i;
                const float a = sm.as[tt][c], kc = sm.ks[tt][c];
                dS[0][i] = a * fmaf(-kc, dr0, G0[i]);
                dS[1][i] = a * fmaf(-kc, dr1, G1[i]);
            }
        }
        __syncthreads();
        // 3. post-pass: thread = (key row c, column group jq)
        {
            const int c = threadIdx.x % DK, jq = threadIdx.x / DK;
            float dl[CPJ];
#pragma unroll
            for (int jj = 0; jj < CPJ; ++jj) dl[jj] = sm.dsb[jq * CPJ + jj][c];
            for (int tt = m - 1; tt >= 0; --tt) {
                const float a = sm.as[tt][c], kc = sm.ks[tt][c], qc = sm.qs[tt][c], bt = sm.bs[tt];
                float sq = 0.f, sk = 0.f, sa = 0.f;
#pragma unroll
                for (int jj = 0; jj < CPJ; ++jj) {
                    const int jl = jq * CPJ + jj;
                    const float sp = sm.win[tt][jl][c];
                    const float St = a * sp;
                    const float r = sm.rr[tt][jl], dr = sm.drr[tt][jl], dov = sm.dos[tt][jl];
                    const float post = fmaf(bt * kc, r, St);
                    const float G = fmaf(qc, dov, dl[jj]);
                    sq = fmaf(post, dov, sq);
                    sk += bt * G * r - St * dr;
                    const float dSt = fmaf(-kc, dr, G);
                    sa = fmaf(dSt, sp, sa);
                    dl[jj] = a * dSt;
                }
                sm.part[0][jq][tt][c] = sq;
                sm.part[1][jq][tt][c] = sk;
                sm.part[2][jq][tt][c] = sa;
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
                    dg[row * DK + c] = fl.complex_gate ? val[i] : sm.as[tt][c] * val[i];
                }
            } else {
                const float *xh = qty == 0 ? &sm.qs[tt][0] : &sm.ks[tt][0];
                const float inv = qty == 0 ? sm.nq[tt] : sm.nk[tt];
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

    for (int blk = nblk - 1; blk >= 0; --blk) {
        const int t0 = blk * BL, n = min(BL, T_ - t0);
        float st[2][RPL];
        load_ckpt(blk, st);
        if (n > WL) {
            __syncthreads();
            stage(t0, WL);
            __syncthreads();
            for (int tt = 0; tt < WL; ++tt) fwd_step(tt, st, false);
            window(t0 + WL, n - WL, st);
            load_ckpt(blk, st);
        }
        window(t0, min(n, WL), st);
    }
    if (dS0) {
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const size_t rowc = sbase + (size_t)(lane + 32 * i) * DV + j0;
            *reinterpret_cast<float2 *>(&dS0[rowc]) = make_float2(dS[0][i], dS[1][i]);
        }
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const BwdArgs &a, cudaStream_t st) {
    constexpr int CS = DV / NS;
    const size_t smem = sizeof(BwdSmem<DK>);
    auto kern = chunk_bwd_kernel<T, DK, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nblk = (a.T + BL - 1) / BL;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(CS * a.B * a.H));
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
    return cudaLaunchKernelEx(&cfg, kern, (const T *)a.q, (const T *)a.k, (const T *)a.v,
                              (const T *)a.g, (const T *)a.beta, a.S0, (const T *)a.dout, a.dS_T,
                              a.dq, a.dk, a.dv, a.dg, a.dbeta, a.dS0, (float *)a.workspace, a.T,
                              a.H, nblk, a.fl);
}

template <typename T>
cudaError_t launch_d(const BwdArgs &a, cudaStream_t st) {
    if (a.dk_ == 128 && a.dv_ == 128) return launch_t<T, 128, 128>(a, st);
    if (a.dk_ == 128 && a.dv_ == 64) return launch_t<T, 128, 64>(a, st);
    if (a.dk_ == 64 && a.dv_ == 128) return launch_t<T, 64, 128>(a, st);
    return launch_t<T, 64, 64>(a, st);
}
}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    const size_t nblk = ((size_t)T + BL - 1) / BL;
    return (size_t)B * H * nblk * dk * dv * sizeof(float);
}

cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t st) {
    return a.bf16 ? launch_d<__nv_bfloat16>(a, st) : launch_d<float>(a, st);
}

}  // namespace kda
