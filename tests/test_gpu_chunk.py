"""GPU parity of ``kda_chunk_fwd`` against the FP64 oracle (through the C ABI)."""
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


def _run(K, x, **kw):
    q, k, v, g, beta = (cuda(x[n]) for n in ("q", "k", "v", "g", "beta"))
    S0 = cuda(x["S0"])
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    out = torch.full((B, T, H, dv), float("nan"), dtype=q.dtype, device="cuda")
    S_T = torch.full((B, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda")
    K.chunk_fwd(q, k, v, g, beta, S0, out=out, S_T=S_T, **kw)
    torch.cuda.synchronize()
    return out, S_T


def _oracle(x, heads=None, **kw):
    """Oracle on all heads, or on the listed (b, h) pairs only (stacked as B=1, H=len)."""
    arr = {n: f64(x[n]) for n in ("q", "k", "v", "g", "beta")}
    S0 = f64(x["S0"])
    if heads is None:
        return oracle.recurrence_c(arr["q"], arr["k"], arr["v"], arr["g"], arr["beta"], S0, **kw)
    sel = lambda a: np.stack([a[b, :, h] for b, h in heads], axis=1)[None]
    S0s = None if S0 is None else np.stack([S0[b, h] for b, h in heads])[None]
    return oracle.recurrence_c(*(sel(arr[n]) for n in ("q", "k", "v", "g")),
                               np.stack([arr["beta"][b, :, h] for b, h in heads], axis=1)[None],
                               S0s, **kw)


def _check(out, S_T, ref, dtype, heads=None):
    o, s = f64(out), f64(S_T)
    if heads is not None:
        o = np.stack([o[b, :, h] for b, h in heads], axis=1)[None]
        s = np.stack([s[b, h] for b, h in heads])[None]
    tol = tol_for(dtype)
    eo, es = rel_err(o, ref[0]), rel_err(s, ref[1])
    assert eo <= tol and es <= tol, (eo, es, tol)
    return eo, es


def test_tiny_fp32_workload(K):
    """tiny workload: B=1, T=256, H=2, d=64, fp32, S0 = 0; bound 1e-4."""
    x = W.workload_inputs("tiny")
    out, S_T = _run(K, x)
    _check(out, S_T, _oracle(x), torch.float32)


def test_prefill_workload_full(K):
    """prefill workload at full size: B=1, T=4096, H=16, d=128, bf16; every output."""
    x = W.workload_inputs("prefill")
    out, S_T = _run(K, x)
    _check(out, S_T, _oracle(x), torch.bfloat16)


@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 130, 200])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ragged_lengths(K, T, dtype):
    x = W.chunk_inputs(2, T, 3, 128, 128, dtype=dtype, seed=T)
    out, S_T = _run(K, x)
    _check(out, S_T, _oracle(x), dtype)


@pytest.mark.parametrize("H", [8, 12, 24, 40])
@pytest.mark.parametrize("T", [1, 200])
def test_split_scan_value_slices(K, H, T):
    """The split form's scan runs each head as 128/NS value-column slices, NS picked from B*H
    and the SM count.  On a 148-SM B200, B*H = 16, 24, 48, 80 take NS = 16, 32, 64, 128."""
    x = W.chunk_inputs(2, T, H, 128, 128, dtype=torch.bfloat16, seed=70 + H + T)
    out, S_T = _run(K, x, fused=False)
    _check(out, S_T, _oracle(x), torch.bfloat16)


@pytest.mark.parametrize("complex_gate", [False, True])
@pytest.mark.parametrize("B,T,H", [(1, 2048, 8), (1, 4096, 16)], ids=["ns32", "ns64"])
def test_one_launch_form(K, B, T, H, complex_gate):
    """Few long sequences run prep and scan CTAs side by side in one cooperative launch, the
    scan reading each record once the prep has published it.  On a 148-SM B200 these shapes
    take slice widths 32 (8 heads) and 64 (16 heads); every output is checked."""
    x = W.chunk_inputs(B, T, H, 128, 128, dtype=torch.bfloat16, seed=80 + H, complex_gate=complex_gate)
    out, S_T = _run(K, x, complex_gate=complex_gate, fused=False)
    _check(out, S_T, _oracle(x, complex_gate=complex_gate), torch.bfloat16)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_head_dims(K, dk, dv, dtype):
    x = W.chunk_inputs(1, 150, 2, dk, dv, dtype=dtype, seed=dk + dv)
    out, S_T = _run(K, x)
    _check(out, S_T, _oracle(x), dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_complex_kda_small(K, dtype):
    x = W.chunk_inputs(2, 190, 2, 128, 128, dtype=dtype, seed=5, complex_gate=True)
    out, S_T = _run(K, x, complex_gate=True)
    _check(out, S_T, _oracle(x, complex_gate=True), dtype)


@pytest.mark.parametrize("fused", [None, False], ids=["auto", "split"])
def test_complex_kda_workload_sampled(K, fused):
    """Complex-KDA workload at full size (B=8, T=8192, H=32, d=128), sampled heads, through
    the path the library picks (fused on a 148-SM B200) and through the split path."""
    x = W.workload_inputs("ckda")
    out, S_T = _run(K, x, complex_gate=True, fused=fused)
    heads = [(0, 0), (3, 17), (7, 31)]
    _check(out, S_T, _oracle(x, heads, complex_gate=True), torch.bfloat16, heads)


def test_options_no_l2norm_scale_and_no_S0(K):
    x = W.chunk_inputs(1, 100, 2, 128, 128, dtype=torch.float32, seed=9, S0_std=0.0)
    # without the in-kernel norm the inputs must be normalised by the caller
    for n in ("q", "k"):
        x[n] = (x[n] / x[n].norm(dim=-1, keepdim=True)).contiguous()
    out, S_T = _run(K, x, l2norm=False, scale=0.5)
    _check(out, S_T, _oracle(x, l2norm=False, scale=0.5), torch.float32)


def test_empty_sequence_is_identity(K):
    """T = 0: S_T = S0 (the empty chunk is the identity of the monoid)."""
    x = W.chunk_inputs(2, 0, 3, 128, 128, seed=1)
    S0 = cuda(x["S0"])
    S_T = torch.full_like(S0, float("nan"))
    opts = K.make_opts(torch.bfloat16)
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device="cuda")
    K.kda_chunk_fwd(e(2, 0, 3, 128), e(2, 0, 3, 128), e(2, 0, 3, 128), e(2, 0, 3, 128),
                    e(2, 0, 3), S0, e(2, 0, 3, 128), S_T, opts)
    torch.cuda.synchronize()
    assert torch.equal(S_T, S0)


@pytest.mark.parametrize("T", [1, 64, 130, 333])
@pytest.mark.parametrize("complex_gate", [False, True])
def test_fused_single_kernel_path(K, T, complex_gate):
    """KDA_FUSED: the one-kernel-per-sequence tensor-core path (no workspace)."""
    x = W.chunk_inputs(2, T, 3, 128, 128, dtype=torch.bfloat16, seed=40 + T, complex_gate=complex_gate)
    out, S_T = _run(K, x, complex_gate=complex_gate, fused=True)
    _check(out, S_T, _oracle(x, complex_gate=complex_gate), torch.bfloat16)


def test_prefill_workload_fused(K):
    """prefill workload through the fused path, every output."""
    x = W.workload_inputs("prefill")
    out, S_T = _run(K, x, fused=True)
    _check(out, S_T, _oracle(x), torch.bfloat16)


def _check_epilogue(out, plain, gate, w, eps, ref_o, tol):
    """RMSNorm rescales every (token, head) row to unit size, so a row whose o is small
    carries the chunk kernel's error magnified.  Two checks: (1) the epilogue itself, against
    the oracle epilogue applied to the same call's plain output; (2) end to end against the
    oracle on rows holding at least a fifth of the largest row norm (a tenth of the rows
    or more on these inputs)."""
    got = f64(out)
    mine = oracle.rmsnorm_gate_np(f64(plain), f64(gate), None if w is None else f64(w), eps=eps)
    assert rel_err(got, mine) <= tol
    ref = oracle.rmsnorm_gate_np(ref_o, f64(gate), None if w is None else f64(w), eps=eps)
    norms = np.sqrt(np.sum(ref_o * ref_o, axis=-1))
    keep = norms >= 0.2 * norms.max()
    assert keep.sum() >= 0.1 * keep.size
    assert rel_err(got[keep], ref[keep]) <= tol


@pytest.mark.parametrize("fused,H", [(False, 3), (False, 32), (True, 3)],
                         ids=["split-pass", "split-in-scan", "fused"])
@pytest.mark.parametrize("T", [64, 130])
def test_output_epilogue_bf16(K, fused, H, T):
    """kda_chunk_fwd_gated: out = RMSNorm(o) * w * sigmoid(g_out).  The split form applies
    it inside the scan kernel when B*H >= 64 (here 2 x 32) and as a pass otherwise; the
    fused form always as a pass."""
    x = W.chunk_inputs(2, T, H, 128, 128, dtype=torch.bfloat16, seed=60 + T)
    gen = torch.Generator().manual_seed(61 + T)
    gate = torch.randn((2, T, H, 128), generator=gen).to(torch.bfloat16)
    w = (1.0 + 0.5 * torch.randn(128, generator=gen)).float()
    q, k, v, g, beta = (cuda(x[n]) for n in ("q", "k", "v", "g", "beta"))
    S0 = cuda(x["S0"])
    out, S_T = K.chunk_fwd_gated(q, k, v, g, beta, S0, cuda(gate), cuda(w), norm_eps=1e-5, fused=fused)
    plain, _ = K.chunk_fwd(q, k, v, g, beta, S0, fused=fused)
    torch.cuda.synchronize()
    o, s = _oracle(x)
    _check_epilogue(out, plain, gate, w, 1e-5, o, 2e-2)
    assert rel_err(f64(S_T), s) <= 2e-2


def test_output_epilogue_fp32_and_no_weight(K):
    """The FP32 path applies the epilogue as its own pass; weight NULL means ones."""
    x = W.chunk_inputs(1, 100, 2, 64, 64, dtype=torch.float32, seed=62)
    gen = torch.Generator().manual_seed(63)
    gate = torch.randn((1, 100, 2, 64), generator=gen)
    q, k, v, g, beta = (cuda(x[n]) for n in ("q", "k", "v", "g", "beta"))
    out, _ = K.chunk_fwd_gated(q, k, v, g, beta, cuda(x["S0"]), cuda(gate), None, norm_eps=1e-6)
    plain, _ = K.chunk_fwd(q, k, v, g, beta, cuda(x["S0"]))
    torch.cuda.synchronize()
    o, _ = _oracle(x)
    _check_epilogue(out, plain, gate, None, 1e-6, o, 1e-4)


@pytest.mark.parametrize("fused,H", [(False, 3), (False, 32), (True, 3)],
                         ids=["split-pass", "split-in-scan", "fused"])
def test_output_epilogue_all_rows(K, fused, H):
    """kda_chunk_fwd_gated end to end on every (token, head) row, on inputs whose output rows
    all have sizeable norms: q = k and beta in [0.5, 1] make o_t = (1 - beta) S~^T k_t + beta v_t
    (up to the normalisation), so RMSNorm divides by no small row.  The precondition is checked
    on the oracle's outputs before the comparison."""
    T = 130
    x = W.chunk_inputs(2, T, H, 128, 128, dtype=torch.bfloat16, seed=64)
    gen = torch.Generator().manual_seed(65)
    beta = (0.5 + 0.5 * torch.sigmoid(torch.randn((2, T, H), generator=gen))).to(torch.bfloat16)
    x = dict(x, q=x["k"].clone(), beta=beta)
    gate = torch.randn((2, T, H, 128), generator=gen).to(torch.bfloat16)
    w = (1.0 + 0.5 * torch.randn(128, generator=gen)).float()
    o, s = _oracle(x)
    norms = np.sqrt(np.sum(o * o, axis=-1))
    assert norms.min() >= 0.2 * norms.max()
    q, k, v, g, bt = (cuda(x[n]) for n in ("q", "k", "v", "g", "beta"))
    out, S_T = K.chunk_fwd_gated(q, k, v, g, bt, cuda(x["S0"]), cuda(gate), cuda(w), norm_eps=1e-5, fused=fused)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm_gate_np(o, f64(gate), f64(w), eps=1e-5)
    assert rel_err(f64(out), ref) <= 2e-2
    assert rel_err(f64(S_T), s) <= 2e-2
