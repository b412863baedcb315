"""GPU parity of the decode prologue (``kda_recurrent_step_prologue``) and of the
prefill -> decode handoff (``kda_conv_state_from_prefill``): a prefill over the first
T0 tokens followed by decode steps must continue one sequence, i.e. equal the FP64
oracle (prologue + token recurrence) on all T0 + m tokens."""
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


def _oracle_full(x):
    """Prologue + recurrence over the whole sequence, per head (every step is per channel
    or per head, so slicing the inputs by head is exact)."""
    B, T, H, d = x["q_pre"].shape
    cw = f64(x["conv_w"])
    outs, states = [], []
    for h in range(H):
        sl = lambda n: f64(x[n][:, :, h:h + 1])
        q, k, v, g, beta = oracle.prologue_np(sl("q_pre"), sl("k_pre"), sl("v_pre"),
                                              cw[:, h * d:(h + 1) * d], sl("z"),
                                              f64(x["A"])[h:h + 1], sl("b_logit"))
        S0 = None if x["S0"] is None else f64(x["S0"][:, h:h + 1])
        o, s = oracle.recurrence_c(q, k, v, g, beta, S0)
        outs.append(o[:, :, 0])
        states.append(s[:, 0])
    return np.stack(outs, axis=2), np.stack(states, axis=1)


@pytest.mark.parametrize("T0", [0, 1, 2, 70])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prefill_then_decode_continues_the_sequence(K, T0, d, dtype):
    m = 5
    x = W.prologue_inputs(2, T0 + m, 3, d, d, dtype=dtype, seed=7 + T0 + d)
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    pre = lambda n: c[n][:, :T0].contiguous()
    # prefill over the first T0 tokens, then hand the conv state over
    _, S = K.chunk_fwd_prologue(pre("q_pre"), pre("k_pre"), pre("v_pre"), c["conv_w"], pre("z"),
                                c["A"], pre("b_logit"), c["S0"])
    state = K.conv_state_from_prefill(pre("q_pre"), pre("k_pre"), pre("v_pre"))
    outs = []
    for t in range(T0, T0 + m):
        at = lambda n: c[n][:, t].contiguous()
        outs.append(K.recurrent_step_prologue(at("q_pre"), at("k_pre"), at("v_pre"), c["conv_w"],
                                              state, at("z"), c["A"], at("b_logit"), S))
    torch.cuda.synchronize()
    ref_o, ref_s = _oracle_full(x)
    tol = tol_for(dtype)
    got_o = np.stack([f64(o) for o in outs], axis=1)
    assert rel_err(got_o, ref_o[:, T0:]) <= tol
    assert rel_err(f64(S), ref_s) <= tol


def test_conv_state_is_the_last_three_raw_rows(K):
    """The handoff copies raw inputs bit for bit, zero before t = 0."""
    x = W.prologue_inputs(2, 2, 3, 128, 128, dtype=torch.bfloat16, seed=3)
    q, k, v = (cuda(x[n]) for n in ("q_pre", "k_pre", "v_pre"))
    st = K.conv_state_from_prefill(q, k, v)
    torch.cuda.synchronize()
    st = st.cpu().view(2, 3, 3, 3, 128)   # [B, branch, tap, H, d]
    for br, src in enumerate((x["q_pre"], x["k_pre"], x["v_pre"])):
        assert torch.equal(st[:, br, 0], torch.zeros_like(st[:, br, 0]))   # token T - 3 = -1
        assert torch.equal(st[:, br, 1], src[:, 0])
        assert torch.equal(st[:, br, 2], src[:, 1])
