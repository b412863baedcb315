"""The backward's split into windows: boundary values from two independent sweeps, then
every window on its own, checked against the oracle's token-level reverse pass.

The state gradient's recursion dS_{t-1} = Diag(alpha_t)(G - beta_t k_t (k_t . G)),
G = dS_t + scale q_t do_t^T, never reads the state, so one sweep backward from dS_T gives the
gradient at every window end while another, forward from S0, gives the state at every window
start.  From those two values a window's reverse pass (the per-token formulas of the
recurrence's adjoint: Kimi K3 KDA(1) section 1.2.1 for the forward it differentiates) needs
nothing outside the window, which is what lets the backward kernels run all windows at once.
A CPU test of the algebra, not of a kernel; plain FP64 loops.
"""
import numpy as np
import pytest

import kda_workloads as W
import oracle

WL = 8   # tokens per window


def _window_split_backward(q, k, v, g, beta, S0, dO, dS_T, *, complex_gate=False, scale=1.0,
                           eps=oracle.L2NORM_EPS):
    q, k, v, g, beta, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta, dO))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    nq = np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + eps)
    nk = np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + eps)
    qh, kh = q / nq, k / nk
    alpha = g if complex_gate else np.exp(g)
    nwin = (T + WL - 1) // WL
    out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(g),
           np.zeros_like(beta), np.zeros((B, H, dk, dv))]
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], dtype=np.float64)
            dS = np.zeros((dk, dv)) if dS_T is None else np.array(dS_T[b, h], dtype=np.float64)
            A, K, Q = alpha[b, :, h], kh[b, :, h], qh[b, :, h]
            V, Bt, dOs = v[b, :, h], beta[b, :, h], scale * dO[b, :, h]
            # sweep 1: the state at every window start
            S_start = []
            for t in range(T):
                if t % WL == 0:
                    S_start.append(S.copy())
                St = A[t][:, None] * S
                S = St + Bt[t] * np.outer(K[t], V[t] - St.T @ K[t])
            # sweep 2: the state gradient at every window end (no state read), then dS0
            dS_end = [None] * nwin
            for t in range(T - 1, -1, -1):
                if t == T - 1 or t % WL == WL - 1:
                    dS_end[t // WL] = dS.copy()
                G = dS + np.outer(Q[t], dOs[t])
                dS = A[t][:, None] * (G - Bt[t] * np.outer(K[t], G.T @ K[t]))
            out[5][b, h] = dS
            # every window on its own, from its two boundary values
            for wi in range(nwin):
                t0, t1 = wi * WL, min(T, wi * WL + WL)
                S = S_start[wi]
                prev, Sts, rs = [], [], []
                for t in range(t0, t1):
                    prev.append(S)
                    St = A[t][:, None] * S
                    r = V[t] - St.T @ K[t]
                    S = St + Bt[t] * np.outer(K[t], r)
                    Sts.append(St)
                    rs.append(r)
                dS = dS_end[wi]
                for t in range(t1 - 1, t0 - 1, -1):
                    i = t - t0
                    S_t = Sts[i] + Bt[t] * np.outer(K[t], rs[i])
                    G = dS + np.outer(Q[t], dOs[t])
                    a = G.T @ K[t]
                    dvt = Bt[t] * a
                    out[0][b, t, h] = S_t @ dOs[t]
                    out[1][b, t, h] = Bt[t] * (G @ rs[i]) - Sts[i] @ dvt
                    out[2][b, t, h] = dvt
                    out[4][b, t, h] = a @ rs[i]
                    dSt = G - np.outer(K[t], dvt)
                    dalpha = np.sum(dSt * prev[i], axis=1)
                    out[3][b, t, h] = dalpha if complex_gate else A[t] * dalpha
                    dS = A[t][:, None] * dSt
    # through the L2 norm
    for i, (xh, n) in enumerate(((qh, nq), (kh, nk))):
        d = out[i]
        out[i] = (d - xh * np.sum(xh * d, axis=-1, keepdims=True)) / n
    return tuple(out)


@pytest.mark.parametrize("T", [1, 7, 8, 9, 16, 29])
@pytest.mark.parametrize("complex_gate", [False, True], ids=["kda", "ckda"])
def test_window_split_equals_reverse_pass(T, complex_gate):
    x = W.chunk_inputs(1, T, 2, 16, 8, seed=40 + T, complex_gate=complex_gate)
    gr = W.grad_inputs(1, T, 2, 16, 8, seed=T)
    f = lambda t: None if t is None else t.double().numpy()
    args = [f(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")] + [f(gr["dout"]), f(gr["dS_T"])]
    got = _window_split_backward(*args, complex_gate=complex_gate, scale=0.9)
    ref = oracle.recurrence_bwd_np(*args, complex_gate=complex_gate, scale=0.9)
    for name, a, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), got, ref):
        assert np.allclose(a, r, rtol=1e-10, atol=1e-12), name


def test_state_gradient_sweep_ignores_the_state():
    """The reverse sweep's dS at a window end is the same whatever the start state and v:
    the oracle's dS0 for two different (S0, v) agree, while dq (which reads the state)
    does not."""
    x = W.chunk_inputs(1, 20, 1, 16, 8, seed=3)
    gr = W.grad_inputs(1, 20, 1, 16, 8, seed=4)
    f = lambda t: None if t is None else t.double().numpy()
    base = [f(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")]
    other = list(base)
    other[2] = base[2] * -1.7 + 0.3
    other[5] = base[5] + 0.5
    r1 = oracle.recurrence_bwd_np(*base, f(gr["dout"]), f(gr["dS_T"]))
    r2 = oracle.recurrence_bwd_np(*other, f(gr["dout"]), f(gr["dS_T"]))
    assert np.allclose(r1[5], r2[5], rtol=1e-12, atol=1e-14)
    assert not np.allclose(r1[0], r2[0])
