"""The backward's decay factors in range: a band-referenced factorization of the chunkwise
gradient, checked against the oracle's plain chunkwise form (which divides by Gamma).

Under the -5 floor a 64-token chunk's cumulative decay reaches e^-320, so K / Gamma
overflows even FP32.  The forward kernels cut a chunk into four 16-token bands with
reference p_b = gamma just before band b: a row carries E_r = e^{gamma_r - p_b} <= 1 and a
key row i <= band end carries k_i e^{p_b - gamma_i} <= e^80.  This file writes every term
of the gradient that way -- the pairwise-factor sums of dq and dk as per-band products, the
decay gradient as products of values and their gradients (no division by Gamma) -- and
requires it to equal the plain form, so a chunked backward kernel can follow it.
Unsigned gates (the bounded map) only; a CPU test of the algebra, not of a kernel.
"""
import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle


def _band_chunk_backward(Q, K, V, bt, g, S, dS, dO):
    """One chunk (n <= 64 tokens, unit-norm Q, K) from its start state S, with dS the
    gradient at its end and dO the (scaled) output gradient; returns dq, dk, dv, dg, dbeta
    of the chunk and the gradient at its start."""
    n, dk = K.shape
    gam = np.cumsum(g, axis=0)                       # gamma_r, non-increasing
    gC = gam[-1]
    nb = (n + 15) // 16
    band = np.arange(n) // 16
    P = np.array([np.zeros(dk) if b == 0 else gam[16 * b - 1] for b in range(nb)])   # p_b
    E = np.exp(gam - P[band])                        # row factors, <= 1
    Kt = [K[:16 * b + 16] * np.exp(P[b] - gam[:16 * b + 16]) for b in range(nb)]   # <= e^80
    # forward quantities of the chunk, every factor in range
    Aqk = np.zeros((n, n))
    Akk = np.zeros((n, n))
    for r in range(n):
        b = band[r]
        Aqk[r, :r + 1] = (Q[r] * E[r]) @ Kt[b][:r + 1].T
        Akk[r, :r] = bt[r] * ((K[r] * E[r]) @ Kt[b][:r].T)
    Gam = np.exp(gam)                                # <= 1 (may underflow: harmless)
    Tm = np.linalg.inv(np.eye(n) + Akk)
    X, Y = bt[:, None] * K * Gam, bt[:, None] * V
    Wm, U = Tm @ X, Tm @ Y
    Vt = U - Wm @ S
    Kd = K * np.exp(gC - gam)                        # <= 1
    # adjoint of the state and output steps
    dVt = Aqk.T @ dO + Kd @ dS
    dS_prev = np.exp(gC)[:, None] * dS + (Q * Gam).T @ dO - Wm.T @ dVt
    dAqk = np.tril(dO @ Vt.T)
    dWm, dU = -dVt @ S.T, dVt
    dKd = Vt @ dS.T
    dX, dY = Tm.T @ dWm, Tm.T @ dU
    dAkk = np.tril(-Tm.T @ (dWm @ X.T + dU @ Y.T) @ Tm.T, -1)
    # pairwise-factor sums by bands: row side (query or erasing key) and column side (key)
    dq_row = np.zeros((n, dk))
    dk_row = np.zeros((n, dk))
    dk_col = np.zeros((n, dk))
    for b in range(nb):
        rows = np.where(band == b)[0]
        lim = 16 * b + 16
        dq_row[rows] = E[rows] * (dAqk[rows, :lim] @ Kt[b])
        dk_row[rows] = bt[rows, None] * E[rows] * (dAkk[rows, :lim] @ Kt[b])
        # column side: key rows i <= band end see row band b through e^{p_b - gamma_i}
        lhs = dAqk[rows, :lim].T @ (Q[rows] * E[rows]) + \
            dAkk[rows, :lim].T @ (bt[rows, None] * K[rows] * E[rows])
        dk_col[:lim] += np.exp(P[b] - gam[:lim]) * lhs
    dq = Gam * (dO @ S.T) + dq_row
    dkk = dk_row + dk_col + bt[:, None] * Gam * dX + np.exp(gC - gam) * dKd
    dv = bt[:, None] * dY
    # beta: A_kk rows (without their beta), X and Y
    raw_kk = np.zeros((n, n))
    for r in range(n):
        raw_kk[r, :r] = (K[r] * E[r]) @ Kt[band[r]][:r].T
    dbeta = np.sum(dAkk * raw_kk, axis=1) + np.sum(K * Gam * dX, axis=1) + np.sum(V * dY, axis=1)
    # decay: d/dgamma_r of each term is value x gradient (query side +, key side -)
    dgam = (Q * Gam * (dO @ S.T) + Q * dq_row + K * dk_row - K * dk_col
            + bt[:, None] * K * Gam * dX - K * np.exp(gC - gam) * dKd)
    dgam[-1] += np.sum(K * np.exp(gC - gam) * dKd, axis=0) + np.exp(gC) * np.sum(S * dS, axis=1)
    dg = np.cumsum(dgam[::-1], axis=0)[::-1]        # gamma_r = sum_{s <= r} g_s
    return dq, dkk, dv, dg, dbeta, dS_prev


def _band_backward(q, k, v, g, beta, S0, dO, dST, C=64, eps=oracle.L2NORM_EPS):
    q, k, v, g, beta, dO = (np.asarray(x, np.float64) for x in (q, k, v, g, beta, dO))
    B, T, H, dk = q.shape
    nq = np.sqrt(np.sum(q * q, -1, keepdims=True) + eps)
    nk = np.sqrt(np.sum(k * k, -1, keepdims=True) + eps)
    qh, kh = q / nq, k / nk
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(g),
           np.zeros_like(beta)]
    dS0 = np.zeros(S0.shape)
    for b in range(B):
        for h in range(H):
            starts = list(range(0, T, C))
            S = S0[b, h].copy()
            states = []
            for s in starts:                          # chunk start states (plain forward)
                e = min(s + C, T)
                states.append(S)
                sl = lambda x: x[b:b + 1, s:e, h:h + 1]
                _, S = oracle.recurrence_np(sl(qh), sl(kh), sl(v), sl(g), sl(beta), S[None, None],
                                            l2norm=False)
                S = S[0, 0]
            dS = dST[b, h].copy()
            for s, S in zip(reversed(starts), reversed(states)):
                e = min(s + C, T)
                r = _band_chunk_backward(qh[b, s:e, h], kh[b, s:e, h], v[b, s:e, h], beta[b, s:e, h],
                                         g[b, s:e, h], S, dS, dO[b, s:e, h])
                for o, x in zip(out, r[:5]):
                    o[b, s:e, h] = x
                dS = r[5]
            dS0[b, h] = dS
    dqh, dkh = out[0], out[1]
    dq = (dqh - qh * np.sum(qh * dqh, -1, keepdims=True)) / nq
    dkk = (dkh - kh * np.sum(kh * dkh, -1, keepdims=True)) / nk
    return dq, dkk, out[2], out[3], out[4], dS0


@pytest.mark.parametrize("T", [16, 64, 100, 150])
def test_band_referenced_backward_equals_plain_chunkwise(T):
    x = W.chunk_inputs(1, T, 2, 32, 8, dtype=torch.float32, seed=T)
    gr = W.grad_inputs(1, T, 2, 32, 8, dtype=torch.float32, seed=T)
    a = {n: x[n].double().numpy() for n in ("q", "k", "v", "g", "beta", "S0")}
    dO, dST = gr["dout"].double().numpy(), gr["dS_T"].double().numpy()
    ref = oracle.chunkwise_bwd_np(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], dO, dST)
    got = _band_backward(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], dO, dST)
    for name, u, w in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), got, ref):
        assert np.max(np.abs(u - w)) <= 1e-10 * max(np.max(np.abs(w)), 1e-30), name


def test_band_factors_stay_in_range():
    """Under the -5 floor every factor the band form exponentiates lies in [e^-80, e^80]
    or below 1 -- what keeps it representable in bf16 / FP32 where K / Gamma is not."""
    x = W.chunk_inputs(1, 64, 4, 32, 8, seed=5)
    g = x["g"].double().numpy()[0, :, :, :]            # [T, H, dk]
    gam = np.cumsum(g, axis=0)
    for b in range(1, 4):
        p = gam[16 * b - 1]
        assert np.all(gam[16 * b:16 * b + 16] - p <= 0) and np.all(gam[16 * b:16 * b + 16] - p >= -80)
        assert np.all(p - gam[:16 * b + 16] <= 80)
    assert np.max(-gam[-1]) > 88.7                     # so 1 / Gamma itself overflows FP32
