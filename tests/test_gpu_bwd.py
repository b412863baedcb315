"""GPU parity of ``kda_chunk_bwd`` (the gradients of the chunk forward) against the FP64
oracle's reverse pass, itself pinned by finite differences of the forward oracle."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from tests._util import cuda, f64, rel_err, tol_for

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")


@pytest.fixture(scope="module")
def K():
    from gated_delta_rule_73_b200 import build
    build.build()
    import gated_delta_rule_73_b200 as K
    return K


def _check(K, x, gr, tol, heads=None, **kw):
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    got = K.chunk_bwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S0"], cuda(gr["dout"]),
                      cuda(gr["dS_T"]), **kw)
    torch.cuda.synchronize()
    if heads is None:
        heads = range(x["q"].shape[2])
    heads = list(heads)
    sl = lambda t: None if t is None else f64(t[:, :, heads])
    slS = lambda t: None if t is None else f64(t[:, heads])
    ref = oracle.recurrence_bwd_np(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["beta"]),
                                   slS(x["S0"]), sl(gr["dout"]), slS(gr["dS_T"]), **kw)
    for name, a, b in zip(NAMES, got, ref):
        a = f64(a[:, heads]) if name == "dS0" else f64(a[:, :, heads])
        assert rel_err(a, b) <= tol, (name, rel_err(a, b))


@pytest.mark.parametrize("T", [1, 15, 16, 17, 64, 100])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_small(K, T, dtype):
    x = W.chunk_inputs(2, T, 3, 128, 128, dtype=dtype, seed=600 + T)
    gr = W.grad_inputs(2, T, 3, 128, 128, dtype=dtype, seed=T)
    _check(K, x, gr, tol_for(dtype))


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128)])
def test_bwd_head_dims(K, dk, dv):
    x = W.chunk_inputs(2, 37, 3, dk, dv, dtype=torch.float32, seed=dk + dv)
    gr = W.grad_inputs(2, 37, 3, dk, dv, dtype=torch.float32, seed=1)
    _check(K, x, gr, 1e-4)


@pytest.mark.parametrize("kw", [dict(complex_gate=True), dict(l2norm=False, scale=0.7)],
                         ids=["complex", "no-l2norm-scaled"])
def test_bwd_options(K, kw):
    x = W.chunk_inputs(1, 50, 4, 128, 128, dtype=torch.float32, seed=7,
                       complex_gate=kw.get("complex_gate", False))
    gr = W.grad_inputs(1, 50, 4, 128, 128, dtype=torch.float32, seed=2)
    _check(K, x, gr, 1e-4, **kw)


def test_bwd_optional_tensors(K):
    """S0 = NULL (zero), dS_T = NULL (zero), grad_S0 = NULL (skipped)."""
    x = W.chunk_inputs(1, 33, 2, 128, 128, dtype=torch.float32, S0_std=0.0, seed=8)
    gr = W.grad_inputs(1, 33, 2, 128, 128, dtype=torch.float32, dST_std=0.0, seed=3)
    _check(K, x, gr, 1e-4)
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    got = K.chunk_bwd(c["q"], c["k"], c["v"], c["g"], c["beta"], None, cuda(gr["dout"]), None,
                      want_dS0=False)
    torch.cuda.synchronize()
    assert got[5] is None


def test_bwd_unbounded_decay(K):
    """The backward is exact FP32 for any g <= 0: Kimi Linear's softplus gate."""
    x = W.chunk_inputs(1, 80, 3, 128, 128, dtype=torch.float32, seed=9, gate="softplus")
    gr = W.grad_inputs(1, 80, 3, 128, 128, dtype=torch.float32, seed=4)
    _check(K, x, gr, 1e-4)


def test_bwd_empty_sequence(K):
    """T = 0 is the identity: grad_S0 = dS_T."""
    x = W.chunk_inputs(2, 0, 3, 128, 128, dtype=torch.float32, seed=1)
    gr = W.grad_inputs(2, 0, 3, 128, 128, dtype=torch.float32, seed=5)
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    got = K.chunk_bwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S0"], cuda(gr["dout"]),
                      cuda(gr["dS_T"]))
    torch.cuda.synchronize()
    assert torch.equal(got[5].cpu(), gr["dS_T"])


def test_bwd_prefill_workload_sampled(K):
    """Full prefill workload (B=1, T=4096, H=16, d=128, bf16) through the same launch the
    benchmark times; two heads checked against the oracle's reverse pass."""
    x = W.workload_inputs("prefill")
    gr = W.grad_inputs(1, 4096, 16, 128, 128, dtype=torch.bfloat16, seed=0)
    _check(K, x, gr, 2e-2, heads=[0, 11])
