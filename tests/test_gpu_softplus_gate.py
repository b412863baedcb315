"""GPU parity of the unbounded-decay variant: Kimi Linear's gate g = -exp(A_h) softplus(z),
which has no -5 floor, through the prologue entry points (``KDA_GATE_SOFTPLUS``) and through
``kda_chunk_fwd`` with ``KDA_UNBOUNDED_DECAY``, against the FP64 oracle."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from tests._util import cuda, f64, rel_err, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from gated_delta_rule_73_b200 import build
    build.build()
    import gated_delta_rule_73_b200 as K
    return K


def _oracle_prologue(x):
    B, T, H, d = x["q_pre"].shape
    cw = f64(x["conv_w"])
    outs, states = [], []
    for h in range(H):
        sl = lambda n: f64(x[n][:, :, h:h + 1])
        q, k, v, g, beta = oracle.prologue_np(sl("q_pre"), sl("k_pre"), sl("v_pre"),
                                              cw[:, h * d:(h + 1) * d], sl("z"),
                                              f64(x["A"])[h:h + 1], sl("b_logit"), gate="softplus")
        S0 = None if x["S0"] is None else f64(x["S0"][:, h:h + 1])
        o, s = oracle.recurrence_c(q, k, v, g, beta, S0)
        outs.append(o[:, :, 0])
        states.append(s[:, 0])
    return np.stack(outs, axis=2), np.stack(states, axis=1)


@pytest.mark.parametrize("T", [5, 67, 200])
@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_chunk_prologue_softplus(K, T, d, dtype):
    x = W.prologue_inputs(2, T, 3, d, d, dtype=dtype, seed=300 + T, gate="softplus")
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    out, S_T = K.chunk_fwd_prologue(c["q_pre"], c["k_pre"], c["v_pre"], c["conv_w"], c["z"],
                                    c["A"], c["b_logit"], c["S0"], gate_softplus=True)
    torch.cuda.synchronize()
    ref_o, ref_s = _oracle_prologue(x)
    assert rel_err(f64(out), ref_o) <= tol_for(dtype)
    assert rel_err(f64(S_T), ref_s) <= tol_for(dtype)


def _chunk_oracle(x, complex_gate=False):
    return oracle.recurrence_c(*(f64(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")),
                               complex_gate=complex_gate)


@pytest.mark.parametrize("B,T,H", [(2, 64, 3), (2, 130, 3), (1, 512, 96), (1, 4096, 16)])
def test_chunk_unbounded_decay_bf16(K, B, T, H):
    """bf16 d=128 with g far below -5 (down to about -60 per token): the split tensor-core form
    with the diagonal 16-token blocks as FP32 position pairs; two launches (2 x 3 heads, 96 heads)
    and the one-launch form (16 heads x 4096 tokens)."""
    x = W.chunk_inputs(B, T, H, 128, 128, seed=400 + T + H, gate="softplus")
    g = x["g"].float()
    assert g.min() < -20 and (g < -5).float().mean() > 0.2     # the floor really is absent
    out, S_T = K.chunk_fwd(*(cuda(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")),
                           unbounded=True)
    torch.cuda.synchronize()
    ref_o, ref_s = _chunk_oracle(x)
    assert rel_err(f64(out), ref_o) <= 2e-2
    assert rel_err(f64(S_T), ref_s) <= 2e-2


def test_unbounded_decay_extreme_gates(K):
    """Gates no band reference could hold: a whole 16-token band at -200 per token, single
    tokens at -3000 on a third of the channels, a band with g = 0, and a ragged last chunk.
    Every factor of the unbounded prep is one exponential of a non-positive exponent or a
    product of such, so underflow only ever yields the (negligible) true value."""
    x = W.chunk_inputs(1, 200, 4, 128, 128, seed=450, gate="softplus")
    g = x["g"].float()
    g[:, 10:26] = -200.0
    g[:, 40, :, ::3] = -3000.0
    g[:, 64:80] = 0.0
    x["g"] = g.to(torch.bfloat16)
    out, S_T = K.chunk_fwd(*(cuda(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")),
                           unbounded=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(S_T).all()
    ref_o, ref_s = _chunk_oracle(x)
    assert rel_err(f64(out), ref_o) <= 2e-2
    assert rel_err(f64(S_T), ref_s) <= 2e-2


def test_unbounded_decay_complex_gate_fp32_path(K):
    """Complex-KDA with KDA_UNBOUNDED_DECAY: the signed-gate steps of the tensor-core prep rely
    on the floor, so the call takes the exact-FP32 path; it still matches the oracle."""
    x = W.chunk_inputs(1, 130, 2, 128, 128, seed=460, complex_gate=True)
    out, S_T = K.chunk_fwd(*(cuda(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")),
                           complex_gate=True, unbounded=True)
    torch.cuda.synchronize()
    ref_o, ref_s = _chunk_oracle(x, complex_gate=True)
    assert rel_err(f64(out), ref_o) <= 2e-2
    assert rel_err(f64(S_T), ref_s) <= 2e-2


@pytest.mark.parametrize("H", [3, 32])
def test_unbounded_decay_output_epilogue(K, H):
    """kda_chunk_fwd_gated with the unbounded gate: the epilogue as a pass (2 x 3 heads) and
    inside the whole-row scan (2 x 32 heads), both after the unbounded prep."""
    T = 130
    x = W.chunk_inputs(2, T, H, 128, 128, seed=470 + H, gate="softplus")
    gen = torch.Generator().manual_seed(471 + H)
    gate = torch.randn((2, T, H, 128), generator=gen).to(torch.bfloat16)
    w = (1.0 + 0.5 * torch.randn(128, generator=gen)).float()
    q, k, v, g, beta = (cuda(x[n]) for n in ("q", "k", "v", "g", "beta"))
    S0 = cuda(x["S0"])
    out, S_T = K.chunk_fwd_gated(q, k, v, g, beta, S0, cuda(gate), cuda(w), norm_eps=1e-5,
                                 unbounded=True)
    plain, _ = K.chunk_fwd(q, k, v, g, beta, S0, unbounded=True)
    torch.cuda.synchronize()
    o, s = _chunk_oracle(x)
    assert rel_err(f64(plain), o) <= 2e-2
    mine = oracle.rmsnorm_gate_np(f64(plain), f64(gate), f64(w), eps=1e-5)
    assert rel_err(f64(out), mine) <= 2e-2
    assert rel_err(f64(S_T), s) <= 2e-2


def test_chunk_prologue_softplus_long(K):
    """The softplus gate inside the split form's prep (prologue fused) over several chunks and
    heads, with a ragged tail: 2 x 1000 tokens x 8 heads."""
    x = W.prologue_inputs(2, 1000, 8, 128, 128, dtype=torch.bfloat16, seed=480, gate="softplus")
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    out, S_T = K.chunk_fwd_prologue(c["q_pre"], c["k_pre"], c["v_pre"], c["conv_w"], c["z"],
                                    c["A"], c["b_logit"], c["S0"], gate_softplus=True)
    torch.cuda.synchronize()
    ref_o, ref_s = _oracle_prologue(x)
    assert rel_err(f64(out), ref_o) <= 2e-2
    assert rel_err(f64(S_T), ref_s) <= 2e-2


@pytest.mark.parametrize("T0", [0, 70])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prefill_then_decode_softplus(K, T0, dtype):
    """Prefill with the softplus gate, hand the conv state over, decode the next tokens with
    the same gate: one sequence, equal to the oracle over all of it."""
    m, d = 4, 128
    x = W.prologue_inputs(2, T0 + m, 3, d, d, dtype=dtype, seed=500 + T0, gate="softplus")
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    pre = lambda n: c[n][:, :T0].contiguous()
    _, S = K.chunk_fwd_prologue(pre("q_pre"), pre("k_pre"), pre("v_pre"), c["conv_w"], pre("z"),
                                c["A"], pre("b_logit"), c["S0"], gate_softplus=True)
    state = K.conv_state_from_prefill(pre("q_pre"), pre("k_pre"), pre("v_pre"))
    outs = []
    for t in range(T0, T0 + m):
        at = lambda n: c[n][:, t].contiguous()
        outs.append(K.recurrent_step_prologue(at("q_pre"), at("k_pre"), at("v_pre"), c["conv_w"],
                                              state, at("z"), c["A"], at("b_logit"), S,
                                              gate_softplus=True))
    torch.cuda.synchronize()
    ref_o, ref_s = _oracle_prologue(x)
    got_o = np.stack([f64(o) for o in outs], axis=1)
    assert rel_err(got_o, ref_o[:, T0:]) <= tol_for(dtype)
    assert rel_err(f64(S), ref_s) <= tol_for(dtype)
