"""Closed-form special cases run on the GPU through the C ABI (dk = dv = 128).

These are the oracle's pins replayed on the CUDA path: each has an answer
fixed by the pages or by the mathematics, independent of both implementations.
"""
import math

import numpy as np
import pytest
import torch

import kda_workloads as W
from tests._util import cuda, f64, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from gated_delta_rule_73_b200 import build
    build.build()
    import gated_delta_rule_73_b200 as K
    return K


def _chunk(K, q, k, v, g, beta, S0, **kw):
    out, S_T = K.chunk_fwd(cuda(q), cuda(k), cuda(v), cuda(g), cuda(beta), cuda(S0), **kw)
    torch.cuda.synchronize()
    return f64(out), f64(S_T)


def test_rotation_example_on_gpu(K):
    """CKDA review, Figure 1 embedded in dk = 128: k = (e0 + e1)/sqrt2, alpha =
    (-1, 1, 1, ...), beta = 2, v = 0 rotates rows 0-1 of S by 90 degrees and
    leaves the others; four steps give S0 back."""
    d, T = 128, 4
    k = torch.zeros(1, T, 1, d); k[..., 0] = k[..., 1] = 1 / math.sqrt(2)
    g = torch.ones(1, T, 1, d); g[..., 0] = -1.0
    q = torch.randn(1, T, 1, d, generator=torch.Generator().manual_seed(0))
    S0 = torch.randn(1, 1, d, d, generator=torch.Generator().manual_seed(1))
    v = torch.zeros(1, T, 1, d)
    beta = torch.full((1, T, 1), 2.0)
    for dtype in (torch.float32, torch.bfloat16):
        out, ST = _chunk(K, q.to(dtype), k.to(dtype), v.to(dtype), g.to(dtype), beta.to(dtype),
                         S0, l2norm=False, complex_gate=True)
        S0n = S0.double().numpy()[0, 0]
        tol = 1e-5 if dtype == torch.float32 else 2e-2
        assert rel_err(ST[0, 0], S0n) <= tol
        R = np.eye(d); R[:2, :2] = [[0, -1], [1, 0]]
        qb = f64(q.to(dtype))[0, 0, 0]
        assert rel_err(out[0, 0, 0], (R @ S0n).T @ qb) <= tol


def test_beta_one_recall_on_gpu(K):
    """GDN, KDA notes: beta = 1, unit k, q = k returns o_t = v_t."""
    x = W.chunk_inputs(1, 150, 2, 128, 128, dtype=torch.float32, seed=21)
    x["beta"][:] = 1.0
    out, _ = _chunk(K, x["k"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    # the in-kernel norm uses eps = 1e-6, so |k| is 1 to ~1e-8 for these k
    assert rel_err(out, f64(x["v"])) <= 1e-4


def test_decay_only_on_gpu(K):
    """beta = 0: S_T = Diag(exp(sum g)) S0 and o_t = S0^T (exp(cumsum g)_t * q_t)."""
    x = W.chunk_inputs(1, 130, 2, 128, 128, dtype=torch.float32, seed=22)
    x["beta"][:] = 0.0
    x["g"] = (x["g"] * 0.02).contiguous()   # keep exp(sum g) inside the FP32 range
    out, ST = _chunk(K, x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    g = f64(x["g"])
    S0 = f64(x["S0"])
    q = f64(x["q"])
    qn = q / np.sqrt(np.sum(q * q, -1, keepdims=True) + 1e-6)
    assert rel_err(ST, np.exp(g.sum(axis=1))[..., None] * S0) <= 1e-4
    assert rel_err(out, np.einsum("bhij,bthi->bthj", S0, np.exp(np.cumsum(g, 1)) * qn)) <= 1e-4


def test_linear_attention_on_gpu(K):
    """alpha = 1, S0 = 0, orthonormal keys: causal linear attention with beta weights."""
    T, d, H = 100, 128, 2
    rng = np.random.default_rng(23)
    k = np.zeros((1, T, H, d)); q = rng.standard_normal((1, T, H, d))
    for h in range(H):
        Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
        k[0, :, h] = Qm[:, :T].T
    v = rng.standard_normal((1, T, H, d))
    beta = rng.uniform(0.1, 1.0, (1, T, H))
    t = lambda a: torch.tensor(a, dtype=torch.float32)
    out, _ = _chunk(K, t(q), t(k), t(v), torch.zeros(1, T, H, d), t(beta), None, l2norm=False)
    exp = np.zeros_like(out)
    for h in range(H):
        M = np.tril(q[0, :, h] @ k[0, :, h].T) * beta[0, :, h][None, :]
        exp[0, :, h] = M @ v[0, :, h]
    assert rel_err(out, exp) <= 1e-4


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_split_prefill_and_prefill_then_decode(K, dtype):
    """Kimi K3 KDA(1) 2.3.4: splitting a sequence is exact; prefill(T) then one
    decode step equals prefill(T + 1)."""
    x = W.chunk_inputs(2, 201, 2, 128, 128, dtype=dtype, seed=24)
    n = lambda s: {k: (v[:, s] if k not in ("S0",) and v is not None else v) for k, v in x.items()}
    full_o, full_S = _chunk(K, *(x[n_] for n_ in ("q", "k", "v", "g", "beta", "S0")))
    a = n(slice(0, 77))
    o1, S1 = _chunk(K, *(a[n_] for n_ in ("q", "k", "v", "g", "beta", "S0")))
    b = n(slice(77, 200))
    o2, S2 = _chunk(K, *(b[n_] for n_ in ("q", "k", "v", "g", "beta")), torch.tensor(S1, dtype=torch.float32))
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    assert rel_err(np.concatenate([o1, o2], axis=1), full_o[:, :200]) <= tol
    # one decode step from S at T = 200 gives token 200 of the full run
    S = torch.tensor(S2, dtype=torch.float32, device="cuda")
    last = {k_: cuda(x[k_][:, 200]) for k_ in ("q", "k", "v", "g", "beta")}
    o = K.recurrent_step(last["q"], last["k"], last["v"], last["g"], last["beta"], S)
    torch.cuda.synchronize()
    assert rel_err(f64(o), full_o[:, 200]) <= tol
    assert rel_err(f64(S), full_S) <= tol


def test_value_permutation_on_gpu(K):
    """Kimi K3 KDA(1) 2.3.2: permuting the value channels permutes O and S."""
    x = W.chunk_inputs(1, 150, 2, 128, 128, dtype=torch.float32, seed=25)
    perm = torch.randperm(128, generator=torch.Generator().manual_seed(3))
    o, S = _chunk(K, *(x[n] for n in ("q", "k", "v", "g", "beta", "S0")))
    op, Sp = _chunk(K, x["q"], x["k"], x["v"][..., perm], x["g"], x["beta"], x["S0"][..., perm])
    assert rel_err(op, o[..., perm.numpy()]) <= 1e-5
    assert rel_err(Sp, S[..., perm.numpy()]) <= 1e-5


def test_generated_decay_stays_in_bf16_range(K):
    """Kimi K3 structure (2): with g in (-5, 0) a 16-token window's decay is >= e^-80,
    whose reciprocal e^80 is finite in bf16; the workloads' g satisfy it."""
    x = W.workload_inputs("prefill")
    g = x["g"].double()
    assert g.max() < 0 and g.min() > -5
    c = torch.cumsum(g, dim=1)
    assert (c[:, 16:] - c[:, :-16]).min() >= -80
    assert torch.isfinite(torch.tensor(math.exp(80.0), dtype=torch.bfloat16))
