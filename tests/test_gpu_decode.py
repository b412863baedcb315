"""GPU parity of ``kda_recurrent_step`` (decode) against the FP64 oracle."""
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


def _oracle_step(x, S, units=None, **kw):
    """One oracle token per sequence: the decode step is the recurrence at T = 1."""
    a = {n: f64(x[n]) for n in ("q", "k", "v", "g", "beta")}
    if units is not None:
        a = {n: np.stack([a[n][i, h] for i, h in units]) [:, None] for n in a}   # [U,1,...]
        return oracle.recurrence_c(a["q"][:, None], a["k"][:, None], a["v"][:, None],
                                   a["g"][:, None], a["beta"][:, None], S, **kw)
    return oracle.recurrence_c(a["q"][:, None], a["k"][:, None], a["v"][:, None],
                               a["g"][:, None], a["beta"][:, None], S, **kw)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("complex_gate", [False, True])
def test_decode_small_three_steps(K, dk, dv, dtype, complex_gate):
    N, H = 5, 3
    S = W.decode_state(N, H, dk, dv, S_std=0.05, seed=dk + dv)
    S_gpu = cuda(S)
    S_ref = S.double().numpy()
    for step in range(3):
        x = W.decode_step_inputs(N, H, dk, dv, step, dtype=dtype)
        if complex_gate:
            xc = W.chunk_inputs(N, 1, H, dk, dv, dtype=dtype, seed=step, complex_gate=True)
            x["g"] = xc["g"][:, 0].contiguous()
            x["beta"] = xc["beta"][:, 0].contiguous()
        out = K.recurrent_step(*(cuda(x[n]) for n in ("q", "k", "v", "g", "beta")), S_gpu,
                               complex_gate=complex_gate)
        torch.cuda.synchronize()
        o_ref, S_ref = _oracle_step(x, S_ref, complex_gate=complex_gate)
        tol = tol_for(dtype)
        assert rel_err(f64(out), o_ref[:, 0]) <= tol
        assert rel_err(f64(S_gpu), S_ref) <= tol


def test_decode_workload_64_steps_sampled(K):
    """decode workload at full size: N=256, H=96, d=128, 64 separate calls with
    the FP32 state carried in HBM; sampled (sequence, head) units checked at
    every step and at the end."""
    D = W.DECODE
    N, H, dk, dv = D["N"], D["H"], D["dk"], D["dv"]
    S = W.decode_state(N, H, dk, dv, S_std=D["S_std"])
    units = [(0, 0), (17, 5), (128, 64), (255, 95), (200, 1)]
    S_ref = np.stack([S[i, h].double().numpy() for i, h in units])[:, None]
    S_gpu = cuda(S)
    del S
    A = W.decode_log_scale(H)
    out = torch.empty((N, H, dv), dtype=torch.bfloat16, device="cuda")
    for step in range(D["steps"]):
        x = W.decode_step_inputs(N, H, dk, dv, step, A=A)
        K.recurrent_step(*(cuda(x[n]) for n in ("q", "k", "v", "g", "beta")), S_gpu, out=out)
        o_ref, S_ref = _oracle_step(x, S_ref.reshape(len(units), 1, dk, dv), units)
        S_ref = S_ref.reshape(len(units), 1, dk, dv)
        o = f64(out)
        got = np.stack([o[i, h] for i, h in units])
        assert rel_err(got, o_ref[:, 0, 0]) <= 2e-2
    torch.cuda.synchronize()
    Sg = f64(torch.stack([S_gpu[i, h] for i, h in units]))
    assert rel_err(Sg, S_ref[:, 0]) <= 2e-2
