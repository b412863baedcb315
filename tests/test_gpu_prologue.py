"""GPU parity of ``kda_chunk_fwd_prologue`` (short conv + SiLU + L2 norm + gate + beta,
then the chunk forward) against the FP64 oracle."""
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


def _oracle_heads(x, heads):
    """Prologue + recurrence for the listed heads (all batches); every step is per
    channel or per head, so slicing the inputs by head is exact."""
    B, T, H, d = x["q_pre"].shape
    outs, states = [], []
    cw = f64(x["conv_w"])
    for h in heads:
        sl = lambda n: f64(x[n][:, :, h:h + 1])
        cwh = cw[:, h * d:(h + 1) * d]
        q, k, v, g, beta = oracle.prologue_np(sl("q_pre"), sl("k_pre"), sl("v_pre"), cwh,
                                              sl("z"), f64(x["A"])[h:h + 1], sl("b_logit"))
        S0 = None if x["S0"] is None else f64(x["S0"][:, h:h + 1])
        o, s = oracle.recurrence_c(q, k, v, g, beta, S0)
        outs.append(o[:, :, 0])
        states.append(s[:, 0])
    return np.stack(outs, axis=2), np.stack(states, axis=1)


def _run(K, x, **kw):
    args = [cuda(x[n]) for n in ("q_pre", "k_pre", "v_pre", "conv_w", "z", "A", "b_logit")]
    out, S_T = K.chunk_fwd_prologue(*args, cuda(x["S0"]), **kw)
    torch.cuda.synchronize()
    return out, S_T


@pytest.mark.parametrize("T", [1, 3, 5, 64, 67, 200])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prologue_small(K, T, dtype):
    x = W.prologue_inputs(2, T, 3, 64, 64, dtype=dtype, seed=T)
    out, S_T = _run(K, x)
    ref = _oracle_heads(x, range(3))
    tol = tol_for(dtype)
    assert rel_err(f64(out), ref[0]) <= tol
    assert rel_err(f64(S_T), ref[1]) <= tol


@pytest.mark.parametrize("T", [1, 3, 5, 64, 67, 130, 200])
@pytest.mark.parametrize("fused", [None, True], ids=["prologue-in-prep", "fused-kernel"])
def test_prologue_tensor_core(K, T, fused):
    """bf16 d=128: the split form applies the convolution to TMA tiles with a 3-row halo
    inside its prep kernel (rows before t = 0, or of the previous batch, must read as
    zeros); the fused form runs the standalone prologue kernel first."""
    x = W.prologue_inputs(2, T, 3, 128, 128, dtype=torch.bfloat16, seed=100 + T)
    out, S_T = _run(K, x, fused=fused)
    ref = _oracle_heads(x, range(3))
    assert rel_err(f64(out), ref[0]) <= 2e-2
    assert rel_err(f64(S_T), ref[1]) <= 2e-2


def test_prologue_one_launch_form(K):
    """Few long sequences (B=1, T=2048, H=8): the prologue inside the prep of the one-launch
    form, whose prep CTAs take items chunk-major."""
    x = W.prologue_inputs(1, 2048, 8, 128, 128, dtype=torch.bfloat16, seed=90)
    out, S_T = _run(K, x, fused=False)
    ref = _oracle_heads(x, range(8))
    assert rel_err(f64(out), ref[0]) <= 2e-2
    assert rel_err(f64(S_T), ref[1]) <= 2e-2


def test_sweep_T2048_full(K):
    """length-sweep workload, T = 2048, B=1, H=96, d=128: every head."""
    x = W.sweep_inputs(2048)
    out, S_T = _run(K, x)
    ref = _oracle_heads(x, range(96))
    assert rel_err(f64(out), ref[0]) <= 2e-2
    assert rel_err(f64(S_T), ref[1]) <= 2e-2


@pytest.mark.parametrize("T", [8192, 32768, 65536])
def test_sweep_long_sampled(K, T):
    """length-sweep workload at T = 8192, 32768 and 65536 (every length the benchmark times
    beyond the fully checked T = 2048), sampled heads."""
    x = W.sweep_inputs(T)
    out, S_T = _run(K, x)
    heads = [0, 47, 95]
    ref = _oracle_heads(x, heads)
    o = f64(out[:, :, heads])
    s = f64(S_T[:, heads])
    assert rel_err(o, ref[0]) <= 2e-2
    assert rel_err(s, ref[1]) <= 2e-2
