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


@pytest.mark.parametrize("T", [64, 130])
def test_chunk_unbounded_decay_bf16(K, T):
    """bf16 d=128 with g far below -5 (down to about -60 per token): the call takes the
    exact-FP32 chunk path and matches the oracle."""
    x = W.chunk_inputs(2, T, 3, 128, 128, seed=400 + T, gate="softplus")
    g = x["g"].float()
    assert g.min() < -20 and (g < -5).float().mean() > 0.2     # the floor really is absent
    out, S_T = K.chunk_fwd(*(cuda(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")),
                           unbounded=True)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.recurrence_c(*(f64(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")))
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
