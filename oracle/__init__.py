"""FP64 CPU oracle for the Kimi Delta Attention (KDA) hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``gated_delta_rule_73_b200``) and never imports it; the
library never imports this package.

Pages cited (titles as published; the section, figure or Q&A item follows):

* "Kimi K3 の KDA(1): KDA が Gated MLA と AttnRes とどのように連携するか"
  (news.ainew.jp) -- cited as *Kimi K3 KDA(1)*.
* "Kimi K3 模型结构（2）：序列维度（下），chunkwise 并行与下界衰减"
  (xhh.club) -- cited as *Kimi K3 structure (2)*.
* "Complex KDA: 理解并增强 Kimi Delta Attention 的表达能力" (ai-feeds.com)
  -- cited as *Complex KDA summary*.
* "GDN, KDA の整理" (taxfree.dev) -- cited as *GDN, KDA notes*.
* "[논문리뷰] Complex KDA: Understanding and Enhancing the Expressivity of
  Kimi Delta Attention" (blog.secrett2633.cloud) -- cited as *CKDA review*.

Functions
---------
``recurrence_c``      plain C FP64 token recurrence (threaded over sequences).
``recurrence_np``     numpy FP64 twin of the same recurrence (vectorised over
                      sequences, loop over tokens).
``recurrence_loops``  pure-Python loops, for tiny cases only.
``recurrence_bwd_np`` FP64 reverse-mode gradient of the token recurrence
                      (dq, dk, dv, dg, dbeta, dS0 from dO and dS_T).
``chunkwise_bwd_np``  the same gradient through the chunkwise form: a reverse scan
                      of dS over chunks, then the WY / UT and decay derivatives
                      inside each chunk.
``transition_product_np``  dense product of a segment's per-token transitions.
``affine_combine_np`` fold of (M, B) segment pairs onto a start state.
``chunkwise_np``      FP64 chunkwise-algebra form (cumulative decay, A_kk,
                      UT inverse, WY vectors, inter-chunk state update).
``conv_silu_np``      causal depthwise short convolution + SiLU.
``bounded_log_decay`` g = -5 * sigmoid(exp(A_h) * z).
``softplus_log_decay`` g = -exp(A_h) * softplus(z) (Kimi Linear's unbounded gate).
``sigmoid``           beta = sigmoid(b).
``prologue_np``       the three together (raw inputs -> q, k, v, g, beta).
``rmsnorm_gate_np``   the output epilogue RMSNorm(o) * w * sigmoid(g_out).

Every function is pinned by tests in ``tests/test_oracle_pins.py`` against
closed forms, special cases, brute force and the worked example printed on the
pages.  No function here is "parity unpinned".

Conventions shared with the library's ABI (but not its code): layouts are
``q, k, g: [B, T, H, dk]``, ``v, out: [B, T, H, dv]``, ``beta: [B, T, H]``,
``S: [B, H, dk, dv]`` with rows = key channels; ``o_t = scale * S_t^T q_t``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")

L2NORM_EPS = 1e-6   # reading: epsilon inside the square root (pages give none)
G_MIN = -5.0        # Kimi K3 structure (2), Q&A on the -5 lower bound


def build() -> str:
    """Compile the C oracle into ``oracle/libkda_oracle.so`` (gcc, -O2)."""
    if (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", _LIB, _SRC,
             "-lm", "-lpthread"])
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.kda_oracle_recurrence.argtypes = [dp] * 8 + [ctypes.c_long] * 5 + [
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.kda_oracle_recurrence.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def recurrence_c(q, k, v, g, beta, S0=None, *, l2norm=True, complex_gate=False,
                 scale=1.0, eps=L2NORM_EPS, nthreads=None):
    """FP64 token recurrence in plain C (``kda_oracle.c``).

    Decay, then erase, then write, then read the post-write state:
    Kimi K3 KDA(1) section 1.2.1; GDN, KDA notes section "Kimi Delta
    Attention".  Returns ``(out [B,T,H,dv], S_T [B,H,dk,dv])``.
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and g.shape == q.shape
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    S0a = None if S0 is None else _f64(S0)
    if S0a is not None:
        assert S0a.shape == (B, H, dk, dv)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    S_T = np.zeros((B, H, dk, dv), dtype=np.float64)
    nt = nthreads if nthreads is not None else (os.cpu_count() or 1)
    rc = _load().kda_oracle_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0a), _ptr(out), _ptr(S_T),
        B, T, H, dk, dv, int(bool(l2norm)), int(bool(complex_gate)), float(scale),
        float(eps), int(nt))
    if rc != 0:
        raise ValueError("kda_oracle_recurrence rejected its arguments")
    return out, S_T


def _normalise(x, eps):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def recurrence_np(q, k, v, g, beta, S0=None, *, l2norm=True, complex_gate=False,
                  scale=1.0, eps=L2NORM_EPS):
    """numpy FP64 twin of :func:`recurrence_c` (same definition, vectorised
    over the independent (b, h) sequences, loop over tokens)."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if l2norm:
        q, k = _normalise(q, eps), _normalise(k, eps)
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0).copy()
    out = np.zeros((B, T, H, dv))
    alpha = g if complex_gate else np.exp(g)
    for t in range(T):
        St = alpha[:, t, :, :, None] * S                       # decay rows
        pred = np.einsum("bhij,bhi->bhj", St, k[:, t])          # St^T k
        r = v[:, t] - pred
        S = St + beta[:, t, :, None, None] * k[:, t, :, :, None] * r[:, :, None, :]
        out[:, t] = scale * np.einsum("bhij,bhi->bhj", S, q[:, t])
    return out, S


def recurrence_bwd_np(q, k, v, g, beta, S0, dO, dS_T=None, *, l2norm=True,
                      complex_gate=False, scale=1.0, eps=L2NORM_EPS):
    """FP64 gradient of ``L = <dO, O> + <dS_T, S_T>`` with respect to every input of the
    recurrence: returns ``(dq, dk, dv, dg, dbeta, dS0)`` with the shapes of q, k, v, g,
    beta and S (dS0 is returned even when ``S0`` is None, meaning zero).

    The forward is the recurrence of :func:`recurrence_np` (Kimi K3 KDA(1) section 1.2.1:
    decay, erase, write, read the post-write state; GDN, KDA notes section "Kimi Delta
    Attention").  Its reverse pass, token by token from t = T down to 1, with
    ``St = Diag(alpha_t) S_{t-1}``, ``r = v_t - St^T k_t`` and ``G = dS_t + scale q_t do_t^T``
    (dS_t: the gradient reaching S_t from later tokens, dS_T at the end):

      dq_t = scale S_t do_t            a = G^T k_t        dbeta_t = a . r
      dv_t = beta_t a                  dk_t = beta_t G r - St dv_t
      dSt  = G - k_t dv_t^T            dalpha_t = rowsum(dSt * S_{t-1})
      dS_{t-1} = Diag(alpha_t) dSt

    then ``dg = alpha * dalpha`` (alpha = e^g) or ``dalpha`` (Complex-KDA, g = alpha), and
    through the in-kernel L2 norm ``x_hat = x / n``, ``n = sqrt(|x|^2 + eps)``:
    ``dx = (dx_hat - x_hat (x_hat . dx_hat)) / n``.  Every state S_0..S_T is kept (tiny and
    moderate sizes only).
    """
    q, k, v, g, beta, dO = map(_f64, (q, k, v, g, beta, dO))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if l2norm:
        nq = np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + eps)
        nk = np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + eps)
        qh, kh = q / nq, k / nk
    else:
        qh, kh = q, k
    alpha = g if complex_gate else np.exp(g)
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0).copy()
    states = [S]
    resid = []
    for t in range(T):
        St = alpha[:, t, :, :, None] * S
        r = v[:, t] - np.einsum("bhij,bhi->bhj", St, kh[:, t])
        S = St + beta[:, t, :, None, None] * kh[:, t, :, :, None] * r[:, :, None, :]
        states.append(S)
        resid.append(r)
    dS = np.zeros((B, H, dk, dv)) if dS_T is None else _f64(dS_T).copy()
    dqh, dkh, dalpha = np.zeros_like(q), np.zeros_like(k), np.zeros_like(g)
    dvv, dbeta = np.zeros_like(v), np.zeros_like(beta)
    for t in range(T - 1, -1, -1):
        Sp, St_post, r = states[t], states[t + 1], resid[t]
        a_t, k_t, q_t, b_t = alpha[:, t], kh[:, t], qh[:, t], beta[:, t]
        do = scale * dO[:, t]
        St = a_t[..., None] * Sp
        G = dS + q_t[..., :, None] * do[..., None, :]
        dqh[:, t] = np.einsum("bhij,bhj->bhi", St_post, do)
        a = np.einsum("bhij,bhi->bhj", G, k_t)
        dbeta[:, t] = np.sum(a * r, axis=-1)
        dr = b_t[..., None] * a
        dvv[:, t] = dr
        dkh[:, t] = (b_t[..., None] * np.einsum("bhij,bhj->bhi", G, r)
                     - np.einsum("bhij,bhj->bhi", St, dr))
        dSt = G - k_t[..., :, None] * dr[..., None, :]
        dalpha[:, t] = np.sum(dSt * Sp, axis=-1)
        dS = a_t[..., None] * dSt
    dg = dalpha if complex_gate else alpha * dalpha
    if l2norm:
        dq = (dqh - qh * np.sum(qh * dqh, axis=-1, keepdims=True)) / nq
        dk_ = (dkh - kh * np.sum(kh * dkh, axis=-1, keepdims=True)) / nk
    else:
        dq, dk_ = dqh, dkh
    return dq, dk_, dvv, dg, dbeta, dS


def chunkwise_bwd_np(q, k, v, g, beta, S0, dO, dS_T=None, *, C=64, l2norm=True,
                     complex_gate=False, scale=1.0, eps=L2NORM_EPS, chunk_stages=False):
    """FP64 gradient of ``L = <dO, O> + <dS_T, S_T>`` through the chunkwise form of
    :func:`chunkwise_np`; returns what :func:`recurrence_bwd_np` returns.

    Kimi K3 structure (2), Q&A items on the chunkwise algorithm (training runs this form).
    Per chunk, with the forward's Gamma, Kg = K*Gamma, Ki = K/Gamma, Qg = Q*Gamma,
    A_kk, Tm = (I + A_kk)^{-1}, X = diag(beta) Kg, Y = diag(beta) V, W = Tm X, U = Tm Y,
    V~ = U - W S, A_qk = tril(Qg Ki^T), Kd = K * Gamma_C / Gamma, the adjoint steps are,
    chunks in reverse (dS' = the gradient at the chunk's end, dO scaled by ``scale``):

      dV~ = A_qk^T dO + Kd dS'
      dS  = diag(Gamma_C) dS' + Qg^T dO - W^T dV~          (to the previous chunk)
      dA_qk = tril(dO V~^T),  dW = -dV~ S^T,  dU = dV~,  dKd = V~ dS'^T
      dX = Tm^T dW,  dY = Tm^T dU,  dA_kk = strict_tril(-Tm^T (dW X^T + dU Y^T) Tm^T)

    then the products back to Q, K, V, beta and Gamma, Gamma_C = Gamma[last], and
    Gamma = cumprod(alpha) (dg_s = sum_{r >= s} dGamma_r Gamma_r / alpha_s * dalpha_s/dg_s).
    FP64 holds exp(+-320), so the plain K / Gamma is used, as in the forward.

    With ``chunk_stages=True`` it also returns the two sequences a chunked kernel produces
    between its stages, each [B, H, n_chunks + 1, dk, dv]: the state at the start of every
    chunk (the last entry is S_T) and dL/dS there (the reverse scan's output; the last
    entry is dS_T, the first dS0).
    """
    q, k, v, g, beta, dO = map(_f64, (q, k, v, g, beta, dO))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if l2norm:
        nq = np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + eps)
        nk = np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + eps)
        qh, kh = q / nq, k / nk
    else:
        qh, kh = q, k
    alpha = g if complex_gate else np.exp(g)
    dqh, dkh, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dalpha, dbeta = np.zeros_like(g), np.zeros_like(beta)
    dS0 = np.zeros((B, H, dk, dv))
    starts = list(range(0, T, C))
    st_all = np.zeros((B, H, len(starts) + 1, dk, dv))
    gr_all = np.zeros((B, H, len(starts) + 1, dk, dv))
    for b in range(B):
        for h in range(H):
            # forward, keeping each chunk's start state
            S = np.zeros((dk, dv)) if S0 is None else _f64(S0)[b, h].copy()
            states = []
            for s in starts:
                e = min(s + C, T)
                states.append(S)
                Q, K, V = qh[b, s:e, h], kh[b, s:e, h], v[b, s:e, h]
                bt = beta[b, s:e, h]
                Gam = np.cumprod(alpha[b, s:e, h], axis=0)
                Kg, Ki = K * Gam, K / Gam
                Akk = np.tril(bt[:, None] * (Kg @ Ki.T), -1)
                Tm = np.linalg.inv(np.eye(e - s) + Akk)
                Vt = Tm @ (bt[:, None] * V) - Tm @ (bt[:, None] * Kg) @ S
                GC = Gam[-1]
                S = GC[:, None] * S + (K * (GC[None, :] / Gam)).T @ Vt
            st_all[b, h, :len(states)] = states
            st_all[b, h, len(states)] = S
            dS = np.zeros((dk, dv)) if dS_T is None else _f64(dS_T)[b, h].copy()
            gr_all[b, h, len(starts)] = dS
            for ci, s, S in zip(reversed(range(len(starts))), reversed(starts), reversed(states)):
                e = min(s + C, T)
                n = e - s
                Q, K, V = qh[b, s:e, h], kh[b, s:e, h], v[b, s:e, h]
                bt = beta[b, s:e, h]
                al = alpha[b, s:e, h]
                Gam = np.cumprod(al, axis=0)
                GC = Gam[-1]
                Kg, Ki, Qg = K * Gam, K / Gam, Q * Gam
                KK = Kg @ Ki.T
                Akk = np.tril(bt[:, None] * KK, -1)
                Tm = np.linalg.inv(np.eye(n) + Akk)
                X, Y = bt[:, None] * Kg, bt[:, None] * V
                W, U = Tm @ X, Tm @ Y
                Vt = U - W @ S
                Aqk = np.tril(Qg @ Ki.T)
                Kd = K * (GC[None, :] / Gam)
                dOs = scale * dO[b, s:e, h]
                # adjoint of the chunk
                dVt = Aqk.T @ dOs + Kd @ dS
                dS_prev = GC[:, None] * dS + Qg.T @ dOs - W.T @ dVt
                dAqk = np.tril(dOs @ Vt.T)
                dQg = dOs @ S.T + dAqk @ Ki
                dKi = dAqk.T @ Qg
                dW, dU = -dVt @ S.T, dVt
                dKd = Vt @ dS.T
                dGC = np.sum(S * dS, axis=1) + np.sum(K / Gam * dKd, axis=0)
                dX, dY = Tm.T @ dW, Tm.T @ dU
                dTm = dW @ X.T + dU @ Y.T
                dAkk = np.tril(-Tm.T @ dTm @ Tm.T, -1)
                bA = bt[:, None] * dAkk
                dKg = bA @ Ki + bt[:, None] * dX
                dKi = dKi + bA.T @ Kg
                dbeta[b, s:e, h] = (np.sum(dAkk * KK, axis=1) + np.sum(Kg * dX, axis=1)
                                    + np.sum(V * dY, axis=1))
                dvv[b, s:e, h] = bt[:, None] * dY
                dqh[b, s:e, h] = Gam * dQg
                dkh[b, s:e, h] = Gam * dKg + dKi / Gam + (GC[None, :] / Gam) * dKd
                dGam = Q * dQg + K * dKg - Ki * dKi / Gam - Kd * dKd / Gam
                dGam[-1] += dGC
                # Gamma_r = prod_{s <= r} alpha_s:  dalpha_s = sum_{r >= s} dGam_r Gamma_r / alpha_s
                rc = np.cumsum((dGam * Gam)[::-1], axis=0)[::-1]
                dalpha[b, s:e, h] = rc / al
                dS = dS_prev
                gr_all[b, h, ci] = dS
            dS0[b, h] = dS
    dg = dalpha if complex_gate else alpha * dalpha
    if l2norm:
        dq = (dqh - qh * np.sum(qh * dqh, axis=-1, keepdims=True)) / nq
        dk_ = (dkh - kh * np.sum(kh * dkh, axis=-1, keepdims=True)) / nk
    else:
        dq, dk_ = dqh, dkh
    if chunk_stages:
        return (dq, dk_, dvv, dg, dbeta, dS0), st_all, gr_all
    return dq, dk_, dvv, dg, dbeta, dS0


def transition_product_np(k, g, beta, *, l2norm=True, complex_gate=False, eps=L2NORM_EPS):
    """M = T_T ... T_2 T_1 with T_t = (I - beta_t k_t k_t^T) Diag(alpha_t), [B, H, dk, dk].

    Kimi K3 KDA(1) section 2.3 (the algebraic view): every token acts on the state by the
    affine map S -> T_t S + beta_t k_t v_t^T, and a segment of tokens composes to one
    affine map S -> M S + B (the monoid of affine pairs), so a long sequence can be cut
    into segments whose pairs are combined in order.  M is formed here as the explicit
    product of dense dk x dk matrices; B is the segment's final state from S = 0.
    """
    k, g, beta = map(_f64, (k, g, beta))
    B, T, H, dk = k.shape
    if l2norm:
        k = _normalise(k, eps)
    alpha = g if complex_gate else np.exp(g)
    M = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
    eye = np.eye(dk)
    for t in range(T):
        kt = k[:, t]
        E = eye - beta[:, t, :, None, None] * kt[..., :, None] * kt[..., None, :]
        Tt = E * alpha[:, t, :, None, :]            # (I - b k k^T) Diag(alpha): scale columns
        M = np.einsum("bhij,bhjk->bhik", Tt, M)
    return M


def affine_combine_np(Ms, Bs, S0=None):
    """Apply the segment pairs in order to a start state: S <- M_r S + B_r for
    r = 0, 1, ..., returning S (Kimi K3 KDA(1) section 2.3, composition of affine pairs).
    ``Ms``: [R, B, H, dk, dk]; ``Bs``: [R, B, H, dk, dv]; ``S0``: [B, H, dk, dv] or None."""
    Ms, Bs = _f64(Ms), _f64(Bs)
    S = np.zeros(Bs.shape[1:]) if S0 is None else _f64(S0).copy()
    for M, Bm in zip(Ms, Bs):
        S = np.einsum("bhij,bhjk->bhik", M, S) + Bm
    return S


def recurrence_loops(q, k, v, g, beta, S0=None, *, l2norm=True, complex_gate=False,
                     scale=1.0, eps=L2NORM_EPS):
    """Pure-Python scalar loops of the same recurrence (tiny cases only)."""
    import math
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = [[0.0] * dv for _ in range(dk)] if S0 is None else \
                [[float(S0[b, h, i, j]) for j in range(dv)] for i in range(dk)]
            for t in range(T):
                qt = [float(x) for x in q[b, t, h]]
                kt = [float(x) for x in k[b, t, h]]
                if l2norm:
                    nq = math.sqrt(sum(x * x for x in qt) + eps)
                    nk = math.sqrt(sum(x * x for x in kt) + eps)
                    qt = [x / nq for x in qt]
                    kt = [x / nk for x in kt]
                for i in range(dk):
                    a = float(g[b, t, h, i]) if complex_gate else math.exp(float(g[b, t, h, i]))
                    for j in range(dv):
                        S[i][j] *= a
                for j in range(dv):
                    p = sum(S[i][j] * kt[i] for i in range(dk))
                    rj = float(v[b, t, h, j]) - p
                    for i in range(dk):
                        S[i][j] += float(beta[b, t, h]) * kt[i] * rj
                for j in range(dv):
                    out[b, t, h, j] = scale * sum(S[i][j] * qt[i] for i in range(dk))
            S_T[b, h] = np.array(S)
    return out, S_T


def chunkwise_np(q, k, v, g, beta, S0=None, *, C=64, l2norm=True, complex_gate=False,
                 scale=1.0, eps=L2NORM_EPS):
    """FP64 chunkwise-parallel form, written from the pages' chunk algebra.

    Kimi K3 structure (2), Q&A items on the chunkwise algorithm and on the
    intra-chunk matrix A: chunks of C tokens, one state update per chunk, a
    UT transform (one C x C triangular inverse) for the WY auxiliary vectors,
    ``A = Tril[(Q * Gamma)(K / Gamma)^T]`` with the diagonal kept (Kimi K3
    KDA(1) section 1.2.1: the read sees the token's own write) and
    ``O = (Gamma * Q) S + A V~``.  The forms of A_kk, W, U and V~ are derived
    from the recurrence (the pages name them without formulas):

      Gamma_r = prod_{s<=r} alpha_s                 (within the chunk)
      A_kk    = tril(beta_r (K*Gamma)(K/Gamma)^T, -1)
      Tm      = (I + A_kk)^{-1}
      W = Tm diag(beta) (K*Gamma),   U = Tm diag(beta) V
      V~ = U - W S
      O  = (Q*Gamma) S + tril((Q*Gamma)(K/Gamma)^T) V~
      S <- diag(Gamma_C) S + (K * Gamma_C/Gamma)^T V~

    FP64 holds exp(+-320), so the plain K/Gamma is used (no sub-tiling).
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if l2norm:
        q, k = _normalise(q, eps), _normalise(k, eps)
    alpha = g if complex_gate else np.exp(g)
    out = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else _f64(S0)[b, h].copy()
            for s in range(0, T, C):
                e = min(s + C, T)
                n = e - s
                Q, K, V = q[b, s:e, h], k[b, s:e, h], v[b, s:e, h]
                bt = beta[b, s:e, h]
                Gam = np.cumprod(alpha[b, s:e, h], axis=0)            # n x dk
                Kg, Ki, Qg = K * Gam, K / Gam, Q * Gam
                Akk = np.tril(bt[:, None] * (Kg @ Ki.T), -1)
                Tm = np.linalg.inv(np.eye(n) + Akk)
                W = Tm @ (bt[:, None] * Kg)
                U = Tm @ (bt[:, None] * V)
                Vt = U - W @ S
                Aqk = np.tril(Qg @ Ki.T)
                out[b, s:e, h] = scale * (Qg @ S + Aqk @ Vt)
                GC = Gam[-1]
                S = GC[:, None] * S + (K * (GC[None, :] / Gam)).T @ Vt
            S_T[b, h] = S
    return out, S_T


def sigmoid(x):
    x = _f64(x)
    return 1.0 / (1.0 + np.exp(-x))


def bounded_log_decay(z, A):
    """g = G_MIN * sigmoid(exp(A_h) * z), G_MIN = -5.

    Kimi K3 structure (2), Q&A "衰减函数与 Kimi Linear 的负 softplus 有何不同";
    GDN, KDA notes section "Kimi Delta Attention" (-5 < g < 0).
    ``z``: [..., H, dk]; ``A``: [H] (the per-head log-scale).
    """
    z = _f64(z)
    A = _f64(A)
    return G_MIN * sigmoid(np.exp(A)[:, None] * z)


def softplus_log_decay(z, A):
    """g = -exp(A_h) * softplus(z), softplus(z) = log(1 + e^z); range (-inf, 0).

    Kimi K3 structure (2), Q&A "衰减函数与 Kimi Linear 的负 softplus 有何不同": the
    gate Kimi Linear uses, with no lower bound, against which the pages set K3's
    bounded map.  ``log1p(exp(.))`` is evaluated as ``logaddexp(0, z)`` (no overflow).
    ``z``: [..., H, dk]; ``A``: [H].
    """
    z = _f64(z)
    A = _f64(A)
    return -np.exp(A)[:, None] * np.logaddexp(0.0, z)


def conv_silu_np(x, w):
    """Causal depthwise short convolution (kernel 4, no bias, zero history)
    followed by SiLU.

    Kimi K3 KDA(1) section 1.2.1: ``ShortConvolution(hidden_size=12288,
    kernel_size=4, activation='silu')``, each channel independent, the current
    token and the three before it.  Tap order follows a causal Conv1d weight
    ``[channels, 4]``: ``y_t = sum_j w[c, j] * x_{t-3+j}`` (tap 3 = current).
    ``x``: [B, T, Cch]; ``w``: [Cch, 4].
    """
    x = _f64(x)
    w = _f64(w)
    B, T, Cch = x.shape
    Kw = w.shape[1]
    y = np.zeros_like(x)
    for j in range(Kw):
        shift = Kw - 1 - j            # x_{t - shift}
        if shift == 0:
            y += w[None, None, :, j] * x
        elif shift < T:
            y[:, shift:, :] += w[None, None, :, j] * x[:, :T - shift, :]
    return y * sigmoid(y)


def prologue_np(q_pre, k_pre, v_pre, conv_w, z, A, b_logit, *, gate="bounded"):
    """Raw branch inputs -> (q, k, v, g, beta), FP64.

    ``gate``: ``"bounded"`` (K3: :func:`bounded_log_decay`) or ``"softplus"``
    (Kimi Linear: :func:`softplus_log_decay`).

    ``q_pre, k_pre``: [B, T, H, dk]; ``v_pre``: [B, T, H, dv];
    ``conv_w``: [3, H*dk, 4] (q, k, v taps; requires dk == dv);
    ``z``: [B, T, H, dk]; ``A``: [H]; ``b_logit``: [B, T, H].
    The L2 norm of q and k is left to the recurrence (``l2norm=True``).
    """
    q_pre, k_pre, v_pre = map(_f64, (q_pre, k_pre, v_pre))
    B, T, H, dk = q_pre.shape
    cw = _f64(conv_w)
    outs = []
    for i, x in enumerate((q_pre, k_pre, v_pre)):
        d = x.shape[-1]
        y = conv_silu_np(x.reshape(B, T, H * d), cw[i])
        outs.append(y.reshape(B, T, H, d))
    if gate == "bounded":
        g = bounded_log_decay(z, A)
    elif gate == "softplus":
        g = softplus_log_decay(z, A)
    else:
        raise ValueError(f"unknown gate {gate!r}")
    beta = sigmoid(b_logit)
    return outs[0], outs[1], outs[2], g, beta


def rmsnorm_gate_np(o, gate, w=None, eps=1e-5):
    """Output epilogue of a KDA branch (*Kimi K3 KDA(1)* section 1.2.1, the full-rank output
    gate: ``o = FusedRMSNormGated(o, g) = RMSNorm(o) * sigmoid(g)``, the RMS per (token,
    head) over the head_dim values, the norm before the gate).  Readings: the RMSNorm weight
    ``w`` is one head_dim vector shared by the heads (None = ones) and ``eps`` sits inside
    the square root.  ``o``, ``gate``: [..., d]."""
    o = _f64(o)
    gate = _f64(gate)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    y = o / np.sqrt(ms + eps)
    if w is not None:
        y = y * _f64(w)
    return y * sigmoid(gate)
