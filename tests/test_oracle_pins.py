"""Pins of the FP64 oracle against what the pages and the mathematics fix.

Each test is chosen so that a plausible mistake in the oracle (erase before
decay, read before write, decay on the value side, a dropped beta, a sign
error, a transposed state) fails at least one of them.  All run on the CPU.
"""
import math
import os

import numpy as np
import pytest

import oracle
import kda_workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL = 1e-12

ALL_ORACLES = {
    "c": oracle.recurrence_c,
    "np": oracle.recurrence_np,
    "loops": oracle.recurrence_loops,
    "chunk4": lambda *a, **kw: oracle.chunkwise_np(*a, C=4, **kw),
}


def _rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_case(rng, B=2, T=9, H=2, dk=5, dv=3, complex_gate=False):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    if complex_gate:
        g = np.tanh(rng.standard_normal((B, T, H, dk)))
        g = np.sign(g) * np.maximum(np.abs(g), math.exp(-5))
        beta = 2.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    else:
        g = -5.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dk))))
        beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.3 * rng.standard_normal((B, H, dk, dv))
    return q, k, v, g, beta, S0


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


def _one_step_transition(fn, k, alpha, beta, complex_gate=True):
    """Extract T_t from one oracle step: S0 = I, v = 0 gives S_1 = T_t S0."""
    n = k.shape[0]
    q = np.zeros((1, 1, 1, n)); q[..., 0] = 1.0
    g = alpha if complex_gate else np.log(alpha)
    _, S1 = fn(q, k.reshape(1, 1, 1, n), np.zeros((1, 1, 1, n)), g.reshape(1, 1, 1, n),
               np.array([[[beta]]]), np.eye(n).reshape(1, 1, n, n), l2norm=False,
               complex_gate=complex_gate)
    return S1[0, 0]


# ---------------------------------------------------------------- worked example
@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_golden_ckda_rotation(name):
    """CKDA review, Figure 1: (I - 2kk^T)Diag(-1,1), k=(1,1)/sqrt2, is a 90-degree rotation."""
    fx = _read_golden("ckda_rotation_2d.txt")
    fn = ALL_ORACLES[name]
    T_exp = fx["T"].reshape(2, 2)
    T_got = _one_step_transition(fn, fx["k"], fx["alpha"], float(fx["beta"][0]))
    assert np.max(np.abs(T_got - T_exp)) < 1e-15
    # four rotations by 90 degrees give back the start state, for any S0
    rng = np.random.default_rng(1)
    S0 = rng.standard_normal((1, 1, 2, 3))
    k4 = np.tile(fx["k"], (1, 4, 1, 1))
    g4 = np.tile(fx["alpha"], (1, 4, 1, 1))
    q4 = rng.standard_normal((1, 4, 1, 2))
    out, S4 = fn(q4, k4, np.zeros((1, 4, 1, 3)), g4, np.full((1, 4, 1), 2.0), S0,
                 l2norm=False, complex_gate=True)
    assert np.max(np.abs(S4 - S0)) < 1e-14
    # the read-out of step 1 is (R S0)^T q_1
    R = T_exp
    assert np.max(np.abs(out[0, 0, 0] - (R @ S0[0, 0]).T @ q4[0, 0, 0])) < 1e-14


# ---------------------------------------------------------------- closed forms of one transition
@pytest.mark.parametrize("complex_gate", [False, True])
def test_transition_det_norm_spectrum(complex_gate):
    """det T = (1-beta) prod(alpha) (matrix determinant lemma, unit k);
    ||T||_2 <= 1 (CKDA review: non-expansiveness; Kimi K3 KDA(1) 1.2.1: the
    L2 norm bounds the erase operator); the spectrum is real unless the gate
    is signed and beta > 1 (CKDA review, section 2 and Figure 11)."""
    rng = np.random.default_rng(7)
    n_complex = 0
    for trial in range(400):
        n = int(rng.integers(2, 7))
        k = _unit(rng.standard_normal(n))
        if complex_gate:
            alpha = rng.uniform(-1, 1, n)
            beta = float(rng.uniform(0, 2))
        else:
            alpha = np.exp(rng.uniform(-5, 0, n))
            beta = float(rng.uniform(0, 1))
        Tm = _one_step_transition(oracle.recurrence_c, k, alpha, beta, complex_gate)
        assert abs(np.linalg.det(Tm) - (1 - beta) * np.prod(alpha)) < 1e-12
        assert np.linalg.norm(Tm, 2) <= 1 + 1e-12
        ev = np.linalg.eigvals(Tm)
        if not (alpha.min() < 0 and beta > 1):
            assert np.max(np.abs(ev.imag)) < 1e-9
        else:
            n_complex += int(np.max(np.abs(ev.imag)) > 1e-9)
    if complex_gate:
        assert n_complex > 0     # signed gate + beta > 1 does reach complex eigenvalues


# ---------------------------------------------------------------- special cases of the recurrence
@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_beta_one_recall(name):
    """GDN, KDA notes, section "局所損失": with ||k||=1 and beta=1 the read-out
    along the key just written returns its value; with q = k, o_t = v_t."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = _rand_case(rng, T=7)
    beta[:] = 1.0
    kn = _unit(k)
    out, _ = ALL_ORACLES[name](kn, kn, v, g, beta, S0, l2norm=False)
    assert _rel(out, v) < 1e-12


@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_beta_general_residual(name):
    """Same section: after the update the residual along k_t is (1 - beta_t)
    times the residual before it (sign flips for beta > 1).  Checked through
    read-outs only: the pre-update residual is taken from a run with beta_t = 0."""
    rng = np.random.default_rng(4)
    q, k, v, g, beta, S0 = _rand_case(rng, B=1, H=1, T=5, complex_gate=True)
    fn = ALL_ORACLES[name]
    kn = _unit(k)
    b0 = beta.copy(); b0[:, -1] = 0.0
    out_after, _ = fn(kn, kn, v, g, beta, S0, l2norm=False, complex_gate=True)  # S_T^T k_T
    out_before, _ = fn(kn, kn, v, g, b0, S0, l2norm=False, complex_gate=True)   # St^T k_T
    r_after = v[0, -1, 0] - out_after[0, -1, 0]
    r_before = v[0, -1, 0] - out_before[0, -1, 0]
    assert _rel(r_after, (1 - beta[0, -1, 0]) * r_before) < 1e-12


@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_decay_only(name):
    """beta = 0 leaves decay only (GDN, KDA notes: beta_t = 0 writes nothing):
    S_T = Diag(exp(sum g)) S0 and o_t = S0^T (exp(cumsum g)_t * q_t).  dk != dv
    so that decaying the value side instead of the key side fails."""
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = _rand_case(rng, dk=6, dv=3, T=8)
    beta[:] = 0.0
    out, ST = ALL_ORACLES[name](q, k, v, g, beta, S0)
    qn = _unit(q) * (1.0 / np.sqrt(1.0 + oracle.L2NORM_EPS / np.sum(q * q, -1, keepdims=True)))
    Gam = np.exp(np.cumsum(g, axis=1))
    exp_S = np.exp(g.sum(axis=1))[..., None] * S0
    exp_o = np.einsum("bhij,bthi->bthj", S0, Gam * qn)
    assert _rel(ST, exp_S) < 1e-12
    assert _rel(out, exp_o) < 1e-12


@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_frozen_state_alpha1_beta0(name):
    """alpha = 1, beta = 0 (taken literally): nothing decays or is written,
    so S_T = S0 and o_t = S0^T q_t."""
    rng = np.random.default_rng(6)
    q, k, v, g, beta, S0 = _rand_case(rng)
    g[:] = 0.0
    beta[:] = 0.0
    out, ST = ALL_ORACLES[name](q, k, v, g, beta, S0, l2norm=False)
    assert _rel(ST, S0) < 1e-15
    assert _rel(out, np.einsum("bhij,bthi->bthj", S0, q)) < 1e-12


@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_linear_attention_reduction(name):
    """alpha = 1, S0 = 0 and mutually orthonormal keys: the erase never meets
    an earlier write, so o_t = sum_{i<=t} beta_i (q_t . k_i) v_i -- causal
    linear attention with beta weights (GDN, KDA notes, additive update;
    Kimi K3 KDA(1) 2.1).  The diagonal i = t is included: the read sees the
    token's own write (Kimi K3 KDA(1) 1.2.1)."""
    rng = np.random.default_rng(8)
    B, T, H, dk, dv = 1, 6, 2, 8, 4
    q = rng.standard_normal((B, T, H, dk))
    k = np.zeros((B, T, H, dk))
    for h in range(H):
        Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
        k[0, :, h] = Qm[:, :T].T
    v = rng.standard_normal((B, T, H, dv))
    g = np.zeros((B, T, H, dk))
    beta = rng.uniform(0.1, 1.0, (B, T, H))
    out, _ = ALL_ORACLES[name](q, k, v, g, beta, None, l2norm=False)
    exp = np.zeros_like(out)
    for h in range(H):
        M = np.tril(q[0, :, h] @ k[0, :, h].T) * beta[0, :, h][None, :]
        exp[0, :, h] = M @ v[0, :, h]
    assert _rel(out, exp) < 1e-12


@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_scalar_gate_is_gated_deltanet(name):
    """GDN, KDA notes: D_t = alpha_t I gives Gated DeltaNet.  A scalar gate
    commutes with the erase, so with gamma_t = prod_{s<=t} alpha_s the run
    equals gamma_t times an undecayed delta-rule run on v_t / gamma_t and
    S0 (an identity that only holds for the scalar-gate special case)."""
    rng = np.random.default_rng(9)
    q, k, v, g, beta, S0 = _rand_case(rng, T=6, dk=4, dv=3)
    gs = rng.uniform(-0.5, 0, (2, 6, 2))
    g = np.repeat(gs[..., None], 4, axis=-1)
    gam = np.exp(np.cumsum(gs, axis=1))                      # [B,T,H]
    out, ST = ALL_ORACLES[name](q, k, v, g, beta, S0)
    out0, ST0 = ALL_ORACLES[name](q, k, v / gam[..., None], np.zeros_like(g), beta, S0)
    assert _rel(out, gam[..., None] * out0) < 1e-12
    assert _rel(ST, gam[:, -1, :, None, None] * ST0) < 1e-12


@pytest.mark.parametrize("name", list(ALL_ORACLES))
@pytest.mark.parametrize("complex_gate", [False, True])
def test_brute_force_transition_products(name, complex_gate):
    """Kimi K3 KDA(1) 2.3.3-2.3.5: S_T = T_T...T_1 S0 + sum_i T_T...T_{i+1}
    beta_i k_i v_i^T with T_t = (I - beta_t k_t k_t^T) Diag(alpha_t), and
    o_t = S_t^T q_t; dense matrices on tiny sizes."""
    rng = np.random.default_rng(10)
    for T in range(1, 5):
        q, k, v, g, beta, S0 = _rand_case(rng, B=1, H=1, T=T, dk=3, dv=2,
                                          complex_gate=complex_gate)
        kn, qn = _unit(k), _unit(q)
        out, ST = ALL_ORACLES[name](qn, kn, v, g, beta, S0, l2norm=False,
                                    complex_gate=complex_gate)
        S = S0[0, 0]
        for t in range(T):
            a = g[0, t, 0] if complex_gate else np.exp(g[0, t, 0])
            kt = kn[0, t, 0][:, None]
            Tt = (np.eye(3) - beta[0, t, 0] * kt @ kt.T) @ np.diag(a)
            S = Tt @ S + beta[0, t, 0] * kt @ v[0, t, 0][None, :]
            assert _rel(out[0, t, 0], S.T @ qn[0, t, 0]) < 1e-12
        assert _rel(ST[0, 0], S) < 1e-12


# ---------------------------------------------------------------- algebraic structure
@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_split_is_exact_and_empty_is_identity(name):
    """Kimi K3 KDA(1) 2.3.4: the per-token affine maps form a monoid; the empty
    sequence is the identity and a sequence may be split and recombined."""
    rng = np.random.default_rng(11)
    q, k, v, g, beta, S0 = _rand_case(rng, T=11)
    fn = ALL_ORACLES[name]
    out, ST = fn(q, k, v, g, beta, S0)
    for T1 in (0, 1, 5, 11):
        o1, S1 = fn(q[:, :T1], k[:, :T1], v[:, :T1], g[:, :T1], beta[:, :T1], S0)
        o2, S2 = fn(q[:, T1:], k[:, T1:], v[:, T1:], g[:, T1:], beta[:, T1:], S1)
        assert _rel(np.concatenate([o1, o2], axis=1), out) < 1e-12
        assert _rel(S2, ST) < 1e-12
    o0, S_empty = fn(q[:, :0], k[:, :0], v[:, :0], g[:, :0], beta[:, :0], S0)
    assert o0.shape[1] == 0 and np.array_equal(S_empty, S0)


@pytest.mark.parametrize("name", list(ALL_ORACLES))
def test_value_columns_are_independent(name):
    """Kimi K3 KDA(1) 2.3.2: the dv columns of S evolve independently under one
    shared transition, so permuting value channels permutes O and S columns."""
    rng = np.random.default_rng(12)
    q, k, v, g, beta, S0 = _rand_case(rng, dv=5)
    perm = rng.permutation(5)
    fn = ALL_ORACLES[name]
    out, ST = fn(q, k, v, g, beta, S0)
    out_p, ST_p = fn(q, k, v[..., perm], g, beta, S0[..., perm])
    assert _rel(out_p, out[..., perm]) < 1e-13
    assert _rel(ST_p, ST[..., perm]) < 1e-13


def test_token_order_matters():
    """Kimi K3 KDA(1) 2.3.4.6: decays commute but rank-one updates do not, so
    swapping two tokens changes the state (non-commutative monoid)."""
    rng = np.random.default_rng(13)
    q, k, v, g, beta, S0 = _rand_case(rng, T=2, B=1, H=1)
    _, ST = oracle.recurrence_c(q, k, v, g, beta, S0)
    sw = lambda x: x[:, ::-1].copy()
    _, ST2 = oracle.recurrence_c(sw(q), sw(k), sw(v), sw(g), sw(beta), S0)
    assert _rel(ST2, ST) > 1e-3


# ---------------------------------------------------------------- the oracles agree
@pytest.mark.parametrize("complex_gate", [False, True])
def test_c_numpy_loops_agree(complex_gate):
    rng = np.random.default_rng(14)
    q, k, v, g, beta, S0 = _rand_case(rng, T=13, complex_gate=complex_gate)
    ref = oracle.recurrence_loops(q, k, v, g, beta, S0, complex_gate=complex_gate, scale=0.7)
    for fn in (oracle.recurrence_c, oracle.recurrence_np):
        got = fn(q, k, v, g, beta, S0, complex_gate=complex_gate, scale=0.7)
        assert _rel(got[0], ref[0]) < RTOL and _rel(got[1], ref[1]) < RTOL


@pytest.mark.parametrize("C", [4, 16, 64])
@pytest.mark.parametrize("complex_gate", [False, True])
def test_chunkwise_algebra_equals_recurrence(C, complex_gate):
    """Kimi K3 structure (2): the chunkwise form (WY/UT transform, A_qk with its
    diagonal, one state update per chunk) reaches the recurrence's result;
    T is not a multiple of C so a ragged tail chunk is included."""
    rng = np.random.default_rng(15 + C)
    T = 2 * C + 3 if C < 64 else 150
    q, k, v, g, beta, S0 = _rand_case(rng, B=1, H=2, T=T, dk=8, dv=6,
                                      complex_gate=complex_gate)
    ref = oracle.recurrence_c(q, k, v, g, beta, S0, complex_gate=complex_gate)
    got = oracle.chunkwise_np(q, k, v, g, beta, S0, C=C, complex_gate=complex_gate)
    assert _rel(got[0], ref[0]) < 1e-11
    assert _rel(got[1], ref[1]) < 1e-11


def test_zero_vector_l2norm_is_finite():
    """L2 norm with epsilon inside the root: a zero query reads zero."""
    rng = np.random.default_rng(16)
    q, k, v, g, beta, S0 = _rand_case(rng, T=3)
    q[:] = 0.0
    out, _ = oracle.recurrence_c(q, k, v, g, beta, S0)
    assert np.all(out == 0.0)


# ---------------------------------------------------------------- bounds of the workloads
def test_generated_gate_bounds():
    """Kimi K3 structure (2), Q&A on the -5 floor: g in (-5, 0), so over any 16
    tokens the cumulative log-decay is >= -80 and e^80 < bf16 max; CKDA gate in
    [-1, 1] with |alpha| >= e^-5 and beta in [0, 2] (Complex KDA summary)."""
    x = W.chunk_inputs(2, 300, 3, 16, 8, seed=3)
    g = x["g"].double().numpy()
    assert g.max() < 0.0 and g.min() > -5.0
    c = np.cumsum(g, axis=1)
    win = c[:, 16:] - c[:, :-16]
    assert win.min() >= -80.0
    assert math.exp(80.0) < 3.3895313892515355e38     # largest finite bf16
    b = x["beta"].double().numpy()
    assert b.min() > 0.0 and b.max() < 1.0
    xc = W.chunk_inputs(2, 300, 3, 16, 8, seed=3, complex_gate=True)
    a = xc["g"].double().numpy()
    assert np.abs(a).max() <= 1.0 and np.abs(a).min() >= math.exp(-5.0) * (1 - 2 ** -8)
    assert (a < 0).any() and (a > 0).any()
    bc = xc["beta"].double().numpy()
    assert bc.min() >= 0.0 and bc.max() <= 2.0 and bc.max() > 1.0


# ---------------------------------------------------------------- prologue pieces
def test_conv_impulse_response_and_causality():
    """Kimi K3 KDA(1) 1.2.1: each channel is independent and sees the current
    token and the three before it.  An impulse at t0 returns the taps in
    reverse order (tap 3 = current token) through SiLU; nothing before t0."""
    rng = np.random.default_rng(17)
    B, T, Cch = 1, 10, 5
    w = rng.uniform(-0.5, 0.5, (Cch, 4))
    x = np.zeros((B, T, Cch))
    t0, amp = 4, 1.7
    x[0, t0, :] = amp
    y = oracle.conv_silu_np(x, w)
    silu = lambda a: a / (1 + np.exp(-a))
    assert np.all(y[0, :t0] == 0.0)
    for s in range(4):
        assert np.allclose(y[0, t0 + s], silu(amp * w[:, 3 - s]), rtol=0, atol=1e-15)
    assert np.all(y[0, t0 + 4:] == 0.0)
    # constant input: partial sums at the start (zero history), full sum after
    y1 = oracle.conv_silu_np(np.ones((1, 6, Cch)), w)
    for t in range(6):
        assert np.allclose(y1[0, t], silu(w[:, max(0, 3 - t):].sum(axis=1)), atol=1e-15)


def test_silu_sigmoid_and_gate_values():
    """Textbook values: sigmoid(0) = 1/2, sigmoid(1) = 0.7310585786300049,
    so SiLU(1) = 0.7310585786300049; g(z=0) = -5/2 for any A_h; g -> -5 as
    exp(A_h) z -> +inf and -> 0 as it -> -inf; g is decreasing in z."""
    assert oracle.sigmoid(0.0) == 0.5
    assert abs(oracle.sigmoid(1.0) - 0.7310585786300049) < 1e-16
    y = oracle.conv_silu_np(np.ones((1, 1, 1)) * 1.0, np.array([[0.0, 0.0, 0.0, 1.0]]))
    assert abs(y[0, 0, 0] - 0.7310585786300049) < 1e-16
    A = np.array([-0.3, 0.0])
    z = np.zeros((1, 1, 2, 3))
    assert np.all(oracle.bounded_log_decay(z, A) == -2.5)
    big = oracle.bounded_log_decay(np.full((1, 1, 2, 1), 60.0), A)
    small = oracle.bounded_log_decay(np.full((1, 1, 2, 1), -60.0), A)
    assert np.all(np.abs(big + 5.0) < 1e-15) and np.all(np.abs(small) < 1e-15)
    zs = np.linspace(-4, 4, 9).reshape(1, 9, 1, 1) * np.ones((1, 9, 2, 1))
    gz = oracle.bounded_log_decay(zs, A)[0, :, :, 0]
    assert np.all(np.diff(gz, axis=0) < 0)
    # A_h scales the slope: g(z; A) = g(exp(A) z; 0)
    assert np.allclose(oracle.bounded_log_decay(zs, A)[0, :, 0, 0],
                       oracle.bounded_log_decay(zs * math.exp(-0.3), np.zeros(2))[0, :, 0, 0],
                       atol=1e-15)


def test_prologue_composes_the_pieces():
    rng = np.random.default_rng(18)
    B, T, H, d = 1, 7, 2, 3
    qp, kp, vp = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    cw = rng.uniform(-0.5, 0.5, (3, H * d, 4))
    z = rng.standard_normal((B, T, H, d))
    A = rng.uniform(-1, 0, H)
    b = rng.standard_normal((B, T, H))
    q, k, v, g, beta = oracle.prologue_np(qp, kp, vp, cw, z, A, b)
    # channel c of head h is flattened as h*d + c
    for h in range(H):
        for c in range(d):
            ch = h * d + c
            xq = qp[0, :, h, c]
            yq = np.array([sum(cw[0, ch, j] * (xq[t - 3 + j] if t - 3 + j >= 0 else 0.0)
                               for j in range(4)) for t in range(T)])
            assert np.allclose(q[0, :, h, c], yq / (1 + np.exp(-yq)), atol=1e-14)
    assert np.all((g < 0) & (g > -5))
    assert np.allclose(beta, 1 / (1 + np.exp(-b)), atol=1e-16)


def test_rmsnorm_gate_hand_values():
    """Output epilogue pinned by hand arithmetic: o = (3, 4) has mean square 12.5, so with
    eps = 0 the norm gives (3, 4) / sqrt(12.5) = (0.848528..., 1.131370...); a gate of 0
    halves it; w scales channel-wise; a very negative gate closes it."""
    o = np.array([[3.0, 4.0]])
    r = np.sqrt(12.5)
    got = oracle.rmsnorm_gate_np(o, np.array([[40.0, 40.0]]), eps=0.0)
    assert np.allclose(got, [[3.0 / r, 4.0 / r]], rtol=1e-12)
    got = oracle.rmsnorm_gate_np(o, np.zeros((1, 2)), w=np.array([2.0, -1.0]), eps=0.0)
    assert np.allclose(got, [[0.5 * 2.0 * 3.0 / r, 0.5 * -1.0 * 4.0 / r]], rtol=1e-12)
    got = oracle.rmsnorm_gate_np(o, np.array([[-60.0, -60.0]]), eps=0.0)
    assert np.all(np.abs(got) < 1e-25)


def test_rmsnorm_gate_invariances():
    """RMSNorm is scale invariant (eps = 0), gives unit mean square, and the norm is taken
    per row over the last axis only; eps damps small rows toward 0."""
    rng = np.random.default_rng(4)
    o = rng.normal(size=(5, 3, 128))
    big = 1e9                                    # sigmoid(big) = 1: the gate is open
    y = oracle.rmsnorm_gate_np(o, np.full_like(o, big), eps=0.0)
    assert np.allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-12)
    assert np.allclose(oracle.rmsnorm_gate_np(7.5 * o, np.full_like(o, big), eps=0.0), y, rtol=1e-12)
    o2 = o.copy()
    o2[0, 0] *= 100.0                            # another row changing leaves this one alone
    y2 = oracle.rmsnorm_gate_np(o2, np.full_like(o, big), eps=0.0)
    assert np.allclose(y2[1:], y[1:], rtol=1e-12) and np.allclose(y2[0, 1:], y[0, 1:], rtol=1e-12)
    tiny = 1e-6 * o[0, 0]
    damped = oracle.rmsnorm_gate_np(tiny, np.full_like(tiny, big), eps=1.0)
    assert np.max(np.abs(damped)) < 1e-5


def test_softplus_gate_values():
    """Kimi Linear's gate g = -exp(A_h) softplus(z), pinned by textbook facts: softplus(0) =
    ln 2 (so g = -exp(A_h) ln 2 at z = 0); softplus(z) - softplus(-z) = z; its slope is the
    logistic sigmoid (central differences); softplus(z) -> z for large z and -> e^z for very
    negative z; the map has no lower bound (it passes -5 once exp(A_h) softplus(z) > 5)."""
    A = np.array([-0.3, 0.0, math.log(16.0)])
    z0 = np.zeros((1, 1, 3, 2))
    g0 = oracle.softplus_log_decay(z0, A)
    assert np.allclose(g0[0, 0, :, 0], -np.exp(A) * math.log(2.0), rtol=1e-15)
    zs = np.linspace(-6, 6, 25).reshape(1, 25, 1, 1) * np.ones((1, 25, 3, 1))
    sp = -oracle.softplus_log_decay(zs, A) / np.exp(A)[:, None]
    spm = -oracle.softplus_log_decay(-zs, A) / np.exp(A)[:, None]
    assert np.allclose(sp - spm, zs, atol=1e-13)
    h = 1e-5
    slope = (oracle.softplus_log_decay(zs + h, A) - oracle.softplus_log_decay(zs - h, A)) / (2 * h)
    assert np.allclose(slope, -np.exp(A)[:, None] / (1 + np.exp(-zs)), atol=1e-8)
    big = -oracle.softplus_log_decay(np.full((1, 1, 3, 1), 800.0), A)[0, 0, :, 0]
    assert np.allclose(big, 800.0 * np.exp(A), rtol=1e-15)      # no overflow in e^z
    tail = -oracle.softplus_log_decay(np.full((1, 1, 3, 1), -40.0), A)[0, 0, :, 0]
    assert np.allclose(tail, math.exp(-40.0) * np.exp(A), rtol=1e-12)
    assert np.all(oracle.softplus_log_decay(zs, A) < 0)
    assert oracle.softplus_log_decay(np.full((1, 1, 3, 1), 3.0), A)[0, 0, 2, 0] < -5.0
    # the prologue takes the gate it is asked for and nothing else changes
    rng = np.random.default_rng(5)
    B, T, H, d = 1, 5, 3, 2
    qp, kp, vp, z = (rng.standard_normal((B, T, H, d)) for _ in range(4))
    cw = rng.uniform(-0.5, 0.5, (3, H * d, 4))
    b = rng.standard_normal((B, T, H))
    p1 = oracle.prologue_np(qp, kp, vp, cw, z, A, b)
    p2 = oracle.prologue_np(qp, kp, vp, cw, z, A, b, gate="softplus")
    for x1, x2 in zip(p1[:3] + p1[4:], p2[:3] + p2[4:]):
        assert np.array_equal(x1, x2)
    assert np.array_equal(p2[3], oracle.softplus_log_decay(z, A))
    with pytest.raises(ValueError):
        oracle.prologue_np(qp, kp, vp, cw, z, A, b, gate="relu")


# ---------------------------------------------------------------- backward
def _loss(fwd_inputs, dO, dST, **kw):
    o, s = oracle.recurrence_np(*fwd_inputs, **kw)
    return float(np.sum(o * dO) + np.sum(s * dST))


@pytest.mark.parametrize("complex_gate,l2norm,scale", [(False, True, 1.0), (False, False, 0.7),
                                                       (True, True, 1.0), (True, False, 1.3)])
def test_backward_equals_finite_differences(complex_gate, l2norm, scale):
    """Every gradient of the oracle's backward agrees with central differences of the
    forward oracle (an independent route: only the forward definition is used), for
    every element of q, k, v, g, beta and S0, including a token past a chunk-sized
    stretch and both gates."""
    rng = np.random.default_rng(11 + int(complex_gate) + 2 * int(l2norm))
    q, k, v, g, beta, S0 = _rand_case(rng, B=1, T=6, H=2, dk=4, dv=3, complex_gate=complex_gate)
    dO = rng.standard_normal((1, 6, 2, 3))
    dST = rng.standard_normal((1, 2, 4, 3))
    kw = dict(l2norm=l2norm, complex_gate=complex_gate, scale=scale)
    grads = oracle.recurrence_bwd_np(q, k, v, g, beta, S0, dO, dST, **kw)
    inputs = [q, k, v, g, beta, S0]
    h = 1e-6
    for idx, (x, gx) in enumerate(zip(inputs, grads)):
        assert gx.shape == x.shape
        fd = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[pos] += h
            xm[pos] -= h
            ip = list(inputs); ip[idx] = xp
            im = list(inputs); im[idx] = xm
            fd[pos] = (_loss(ip, dO, dST, **kw) - _loss(im, dO, dST, **kw)) / (2 * h)
        assert np.max(np.abs(fd - gx)) <= 1e-7 * max(1.0, np.max(np.abs(fd))), idx


def test_backward_frozen_state_closed_form():
    """beta = 0 freezes the write: o_t = scale S0^T (Gamma_t * q_t) with Gamma_t the
    decay accumulated from the start and S_T = Diag(Gamma_T) S0.  So by hand:
    dq_t = scale Diag(Gamma_t) S0 do_t, dv = 0, dS0 = sum_t scale Diag(Gamma_t) q_t do_t^T
    + Diag(Gamma_T) dS_T, and dg_{t,c} = sum_{s >= t} (the terms of o_s and S_T on channel c),
    i.e. the reverse cumulative sum of Gamma_s,c q_s,c (S0 scale do_s)_c (+ the S_T term)."""
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 1, 5, 1, 4, 3
    q, k, v, g, beta, S0 = _rand_case(rng, B=B, T=T, H=H, dk=dk, dv=dv)
    beta = np.zeros_like(beta)
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    sc = 0.9
    dq, dk_, dvv, dg, db, dS0 = oracle.recurrence_bwd_np(q, k, v, g, beta, S0, dO, dST,
                                                         l2norm=False, scale=sc)
    Gam = np.exp(np.cumsum(g[0, :, 0], axis=0))          # [T, dk], from the start
    S = S0[0, 0]
    for t in range(T):
        assert np.allclose(dq[0, t, 0], sc * Gam[t] * (S @ dO[0, t, 0]), atol=1e-13)
    assert np.all(dvv == 0) and np.all(dk_ == 0)
    want_S0 = sum(sc * (Gam[t] * q[0, t, 0])[:, None] * dO[0, t, 0][None, :] for t in range(T))
    want_S0 = want_S0 + Gam[-1][:, None] * dST[0, 0]
    assert np.allclose(dS0[0, 0], want_S0, atol=1e-13)
    per_t = np.array([sc * Gam[t] * q[0, t, 0] * (S @ dO[0, t, 0]) for t in range(T)])
    per_t[-1] += Gam[-1] * np.sum(S * dST[0, 0], axis=1)
    want_g = np.cumsum(per_t[::-1], axis=0)[::-1]
    assert np.allclose(dg[0, :, 0], want_g, atol=1e-13)


# ---------------------------------------------------------------- segments (affine pairs)
@pytest.mark.parametrize("complex_gate", [False, True])
def test_segment_pair_reproduces_the_recurrence(complex_gate):
    """A segment acts on its start state as S -> M S + B: M from the dense transition
    product, B = the recurrence's final state from S = 0; M S0 + B must equal the
    recurrence run from S0, and M must equal the recurrence's final state from S0 = I
    with v = 0 (each column of the state evolves on its own)."""
    rng = np.random.default_rng(21 + int(complex_gate))
    q, k, v, g, beta, S0 = _rand_case(rng, B=2, T=11, H=2, dk=4, dv=3, complex_gate=complex_gate)
    M = oracle.transition_product_np(k, g, beta, complex_gate=complex_gate)
    _, Bseg = oracle.recurrence_c(q, k, v, g, beta, None, complex_gate=complex_gate)
    _, ST = oracle.recurrence_c(q, k, v, g, beta, S0, complex_gate=complex_gate)
    assert _rel(np.einsum("bhij,bhjk->bhik", M, S0) + Bseg, ST) < RTOL
    eye = np.broadcast_to(np.eye(4), (2, 2, 4, 4)).copy()
    _, MI = oracle.recurrence_c(q, k, np.zeros((2, 11, 2, 4)), g, beta, eye,
                                complex_gate=complex_gate)
    assert _rel(M, MI) < RTOL


def test_affine_combine_is_the_sequential_run():
    """Cut one sequence into segments of lengths 5, 1, 7 and 3: folding the segments'
    (M, B) pairs onto S0 gives the state after the whole sequence, every prefix fold gives
    the state at that segment's start, and an empty fold returns S0."""
    rng = np.random.default_rng(31)
    q, k, v, g, beta, S0 = _rand_case(rng, B=1, T=16, H=2, dk=5, dv=3)
    cuts = [0, 5, 6, 13, 16]
    Ms, Bs = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sl = lambda x: x[:, a:b]
        Ms.append(oracle.transition_product_np(sl(k), sl(g), sl(beta)))
        Bs.append(oracle.recurrence_c(sl(q), sl(k), sl(v), sl(g), sl(beta), None)[1])
    for r, c in enumerate(cuts):
        want = S0 if c == 0 else oracle.recurrence_c(q[:, :c], k[:, :c], v[:, :c], g[:, :c],
                                                     beta[:, :c], S0)[1]
        got = oracle.affine_combine_np(np.array(Ms[:r]).reshape(r, 1, 2, 5, 5),
                                       np.array(Bs[:r]).reshape(r, 1, 2, 5, 3), S0)
        assert _rel(got, want) < RTOL


@pytest.mark.parametrize("C", [4, 5, 16])
@pytest.mark.parametrize("complex_gate,l2norm", [(False, True), (False, False), (True, True)])
def test_chunkwise_backward_equals_recurrence_backward(C, complex_gate, l2norm):
    """The gradient through the chunkwise form (reverse scan of dS over chunks, WY / UT and
    decay derivatives inside each chunk) equals the token-level reverse pass (itself pinned
    by finite differences above), with ragged last chunks and scale != 1."""
    rng = np.random.default_rng(40 + C + 3 * int(complex_gate) + int(l2norm))
    q, k, v, g, beta, S0 = _rand_case(rng, B=2, T=13, H=2, dk=5, dv=3, complex_gate=complex_gate)
    dO = rng.standard_normal((2, 13, 2, 3))
    dST = rng.standard_normal((2, 2, 5, 3))
    kw = dict(complex_gate=complex_gate, l2norm=l2norm, scale=0.8)
    ref = oracle.recurrence_bwd_np(q, k, v, g, beta, S0, dO, dST, **kw)
    got = oracle.chunkwise_bwd_np(q, k, v, g, beta, S0, dO, dST, C=C, **kw)
    for a, b in zip(got, ref):
        assert _rel(a, b) < 1e-12


def test_chunkwise_backward_stage_outputs():
    """The chunked backward's intermediate sequences, pinned without the chunk algebra: the
    state at chunk start c is the recurrence run over tokens [0, 16c); dL/dS there is the
    dS0 of the token-level reverse pass over the suffix [16c, T) started from that state
    (the adjoint of the suffix is the gradient the prefix hands back)."""
    rng = np.random.default_rng(77)
    T, C = 37, 16
    q, k, v, g, beta, S0 = _rand_case(rng, B=1, T=T, H=2, dk=4, dv=3)
    dO = rng.standard_normal((1, T, 2, 3))
    dST = rng.standard_normal((1, 2, 4, 3))
    grads, states, sgrads = oracle.chunkwise_bwd_np(q, k, v, g, beta, S0, dO, dST, C=C,
                                                    chunk_stages=True)
    starts = [0, 16, 32, T]
    assert states.shape == (1, 2, 4, 4, 3) and sgrads.shape == (1, 2, 4, 4, 3)
    for ci, t in enumerate(starts):
        want = S0 if t == 0 else oracle.recurrence_c(q[:, :t], k[:, :t], v[:, :t], g[:, :t],
                                                     beta[:, :t], S0)[1]
        assert _rel(states[:, :, ci], want) < RTOL
        if t == T:
            assert np.array_equal(sgrads[:, :, ci], dST)
            continue
        suffix = oracle.recurrence_bwd_np(q[:, t:], k[:, t:], v[:, t:], g[:, t:], beta[:, t:],
                                          want, dO[:, t:], dST)[5]
        assert _rel(sgrads[:, :, ci], suffix) < 1e-12
    assert np.array_equal(sgrads[:, :, 0], grads[5])


def test_generated_inputs_follow_their_recipes():
    """The seeded inputs of the newer workloads are what DESIGN's input table says: Kimi
    Linear's softplus gate has A_h = log U(1, 16) and no floor (a large share of g below -5,
    all of it below 0); the prologue inputs take the same A_h law; the upstream gradients
    of the backward have the run dtype (dout) and FP32 (dS_T); one seed, one draw."""
    x = W.chunk_inputs(1, 512, 4, 32, 16, seed=9, gate="softplus")
    g = x["g"].double().numpy()
    assert g.max() < 0.0 and g.min() < -20.0 and (g < -5.0).mean() > 0.2
    p = W.prologue_inputs(1, 5, 64, 8, 8, seed=2, gate="softplus")
    A = p["A"].double().numpy()
    assert A.min() >= 0.0 and A.max() <= math.log(16.0) + 1e-6 and A.std() > 0.3
    pb = W.prologue_inputs(1, 5, 64, 8, 8, seed=2)
    assert pb["A"].max() <= 0.0 and pb["A"].min() >= -1.0
    with pytest.raises(ValueError):
        W.chunk_inputs(1, 4, 1, 8, 8, gate="relu")
    gr = W.grad_inputs(2, 7, 3, 16, 8, seed=4)
    assert gr["dout"].shape == (2, 7, 3, 8) and gr["dout"].dtype.is_floating_point
    assert str(gr["dout"].dtype) == "torch.bfloat16" and str(gr["dS_T"].dtype) == "torch.float32"
    assert gr["dS_T"].shape == (2, 3, 16, 8) and 0.005 < float(gr["dS_T"].std()) < 0.02
    assert W.grad_inputs(1, 3, 1, 8, 8, dST_std=0.0)["dS_T"] is None
    again = W.grad_inputs(2, 7, 3, 16, 8, seed=4)
    assert bool((again["dout"] == gr["dout"]).all()) and bool((again["dS_T"] == gr["dS_T"]).all())
