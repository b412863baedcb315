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
// v_{t,j}), so a CTA owns NS = 16 columns of one (b, h), one warp per column, each lane 4
// (or 2) key rows of it in registers.  The DV / NS CTAs of a sequence form one thread-block
// cluster.  Per-token sums over value columns (dq, dk, dalpha, dbeta) are accumulated in
// each CTA's shared memory and then summed across the cluster through distributed shared
// memory, one 16-token block at a time; the CTA that finishes a token row also applies the
// L2-norm and gate backward and writes it.  No global atomics; the result is deterministic.
//
// States are needed in reverse order: phase 1 runs the recurrence forward and writes the
// state at the start of every 16-token block to the workspace (FP32, column-major per
// block); phase 2 walks the blocks backward, recomputes the block's 16 pre-token states
// from its checkpoint into shared memory, and runs the reverse pass over them.
#include <cooperative_groups.h>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace cg = cooperative_groups;

namespace kda {

namespace {
constexpr int BL = 16;          // tokens per block (checkpoint interval)
constexpr int NS = 16;          // value columns per CTA (one warp each)
constexpr int NT = NS * 32;     // threads per CTA
static_assert(BL == NS, "staging gives one warp per token row of a block");

template <int DK>
struct BwdSmem {
    float win[BL][NS][DK];      // S_{t-1} of each token of the block, per column (warp)
    float qs[BL][DK], ks[BL][DK], as[BL][DK];   // normalised q, k and alpha of the block
    float accq[BL][DK], acck[BL][DK], acca[BL][DK];   // this CTA's column sums
    float rr[BL][NS];           // residual r = v - St^T k per token and column
    float vs[BL][NS], dos[BL][NS];   // v and scale * dO of this CTA's columns
    float bs[BL], nq[BL], nk[BL], accb[BL];
};

__device__ __forceinline__ float ldf(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, 1)
chunk_bwd_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const T *__restrict__ g, const T *__restrict__ beta, const float *__restrict__ S0,
                 const T *__restrict__ dout, const float *__restrict__ dST,
                 float *__restrict__ dq, float *__restrict__ dkk, float *__restrict__ dvv,
                 float *__restrict__ dg, float *__restrict__ dbeta, float *__restrict__ dS0,
                 float *__restrict__ ckpt, int T_, int H, int nblk, KernelFlags fl) {
    constexpr int RPL = DK / 32;            // key rows per lane
    constexpr int CS = DV / NS;             // CTAs per sequence (cluster size)
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem<DK> &sm = *reinterpret_cast<BwdSmem<DK> *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();

    const int rank = (int)cluster.block_rank();
    const int bh = blockIdx.x / CS;
    const int b = bh / H, h = bh % H;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = rank * NS + w;            // this warp's value column

    auto row_of = [&](int t) { return ((size_t)b * T_ + t) * H + h; };

    // One warp per token row: normalised q, k (and 1/n), alpha, beta, and this CTA's v, dO.
    auto stage = [&](int t0, int n) {
        const int tt = w;
        if (tt < n) {
            const size_t row = row_of(t0 + tt);
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

    // state column j, rows lane + 32 i
    float s[RPL];
    const size_t sbase = (size_t)bh * DK * DV;
#pragma unroll
    for (int i = 0; i < RPL; ++i) s[i] = S0 ? S0[sbase + (size_t)(lane + 32 * i) * DV + j] : 0.f;

    // ---- phase 1: forward, checkpoint at every block start
    for (int blk = 0; blk < nblk; ++blk) {
        const int t0 = blk * BL, n = min(BL, T_ - t0);
        float *ck = ckpt + (((size_t)bh * nblk + blk) * DV + j) * DK;
#pragma unroll
        for (int i = 0; i < RPL; ++i) ck[lane + 32 * i] = s[i];
        if (blk == nblk - 1) break;
        __syncthreads();
        stage(t0, n);
        __syncthreads();
        for (int tt = 0; tt < n; ++tt) {
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int c = lane + 32 * i;
                s[i] *= sm.as[tt][c];
                dot += sm.ks[tt][c] * s[i];
            }
            const float r = sm.vs[tt][w] - warp_sum(dot);
            const float br = sm.bs[tt] * r;
#pragma unroll
            for (int i = 0; i < RPL; ++i) s[i] += sm.ks[tt][lane + 32 * i] * br;
        }
    }

    // zero the accumulators once; each block re-zeroes them after its reduction
    for (int idx = threadIdx.x; idx < BL * DK; idx += NT) {
        (&sm.accq[0][0])[idx] = 0.f;
        (&sm.acck[0][0])[idx] = 0.f;
        (&sm.acca[0][0])[idx] = 0.f;
    }
    if (threadIdx.x < BL) sm.accb[threadIdx.x] = 0.f;

    // ---- phase 2: blocks in reverse
    float dS[RPL];
#pragma unroll
    for (int i = 0; i < RPL; ++i) dS[i] = dST ? dST[sbase + (size_t)(lane + 32 * i) * DV + j] : 0.f;

    for (int blk = nblk - 1; blk >= 0; --blk) {
        const int t0 = blk * BL, n = min(BL, T_ - t0);
        __syncthreads();
        stage(t0, n);
        __syncthreads();
        const float *ck = ckpt + (((size_t)bh * nblk + blk) * DV + j) * DK;
#pragma unroll
        for (int i = 0; i < RPL; ++i) s[i] = ck[lane + 32 * i];
        // recompute the block's pre-token states and residuals
        for (int tt = 0; tt < n; ++tt) {
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int c = lane + 32 * i;
                sm.win[tt][w][c] = s[i];
                s[i] *= sm.as[tt][c];
                dot += sm.ks[tt][c] * s[i];
            }
            const float r = sm.vs[tt][w] - warp_sum(dot);
            if (lane == 0) sm.rr[tt][w] = r;
            const float br = sm.bs[tt] * r;
#pragma unroll
            for (int i = 0; i < RPL; ++i) s[i] += sm.ks[tt][lane + 32 * i] * br;
        }
        __syncwarp();
        // reverse pass over the block
        for (int tt = n - 1; tt >= 0; --tt) {
            const float dov = sm.dos[tt][w], r = sm.rr[tt][w], bt = sm.bs[tt];
            float G[RPL], St[RPL], sp[RPL];
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int c = lane + 32 * i;
                sp[i] = sm.win[tt][w][c];
                const float kc = sm.ks[tt][c];
                St[i] = sm.as[tt][c] * sp[i];
                const float post = St[i] + bt * kc * r;
                G[i] = dS[i] + sm.qs[tt][c] * dov;
                atomicAdd(&sm.accq[tt][c], post * dov);
                dot += kc * G[i];
            }
            const float a = warp_sum(dot);
            const float dr = bt * a;
            if (lane == 0) {
                atomicAdd(&sm.accb[tt], a * r);
                dvv[row_of(t0 + tt) * DV + j] = dr;
            }
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int c = lane + 32 * i;
                const float kc = sm.ks[tt][c];
                atomicAdd(&sm.acck[tt][c], bt * G[i] * r - St[i] * dr);
                const float dSt = G[i] - kc * dr;
                atomicAdd(&sm.acca[tt][c], dSt * sp[i]);
                dS[i] = sm.as[tt][c] * dSt;
            }
        }
        __syncthreads();
        cluster.sync();
        // token rows tt = rank, rank + CS, ...: sum the CS CTAs' column sums, finish, write
        constexpr int TPC = BL / CS;                 // token rows per CTA
        for (int item = w; item < TPC * 3; item += NS) {
            const int tt = rank + CS * (item / 3), qty = item % 3;
            if (tt >= n) continue;
            float *src = qty == 0 ? &sm.accq[tt][0] : qty == 1 ? &sm.acck[tt][0] : &sm.acca[tt][0];
            float val[RPL];
#pragma unroll
            for (int i = 0; i < RPL; ++i) val[i] = 0.f;
            for (int rk = 0; rk < CS; ++rk) {
                const float *rp = cluster.map_shared_rank(src, rk);
#pragma unroll
                for (int i = 0; i < RPL; ++i) val[i] += rp[lane + 32 * i];
            }
            const size_t row = row_of(t0 + tt);
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
        if (w == NS - 1 && lane < BL && lane % CS == rank && lane < n) {
            float sb = 0.f;
            for (int rk = 0; rk < CS; ++rk) sb += *cluster.map_shared_rank(&sm.accb[lane], rk);
            dbeta[row_of(t0 + lane)] = sb;
        }
        cluster.sync();
        for (int idx = threadIdx.x; idx < BL * DK; idx += NT) {
            (&sm.accq[0][0])[idx] = 0.f;
            (&sm.acck[0][0])[idx] = 0.f;
            (&sm.acca[0][0])[idx] = 0.f;
        }
        if (threadIdx.x < BL) sm.accb[threadIdx.x] = 0.f;
    }
    if (dS0) {
#pragma unroll
        for (int i = 0; i < RPL; ++i) dS0[sbase + (size_t)(lane + 32 * i) * DV + j] = dS[i];
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
