"""GPU parity of the segment pairs behind context parallelism over T (``kda_segment_pair``,
``kda_affine_combine``) against the FP64 oracle, and the whole split forward emulated on
one GPU: segments of one sequence run one after another with the start states the folds
give, and their outputs, joined, must equal the oracle's run over the whole sequence."""
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


@pytest.mark.parametrize("T", [0, 1, 64, 150])
@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_segment_pair(K, T, d, dtype):
    """The pair of a segment.  Under the bounded gate the product M of 64+ transitions is
    about e^-160 (below the FP32 range, so it is 0 on the GPU), so the pair is checked by
    what it is for, M S0 + B = the final state from S0 (against the oracle's run), and M
    itself on a slow-decay copy of the inputs (g scaled by 1/100), where it stays O(1)."""
    x = W.chunk_inputs(2, T, 3, d, d, dtype=dtype, seed=800 + T)
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    M, Bm = K.segment_pair(c["q"], c["k"], c["v"], c["g"], c["beta"])
    torch.cuda.synchronize()
    if T == 0:
        assert torch.equal(M.cpu(), torch.eye(d).expand(2, 3, d, d))
        assert torch.count_nonzero(Bm).item() == 0
        return
    a = {n: f64(x[n]) for n in ("q", "k", "v", "g", "beta")}
    S0 = f64(x["S0"])
    ref_ST = oracle.recurrence_c(a["q"], a["k"], a["v"], a["g"], a["beta"], S0)[1]
    got_ST = np.einsum("bhij,bhjk->bhik", f64(M), S0) + f64(Bm)
    assert rel_err(got_ST, ref_ST) <= tol_for(dtype)
    ref_B = oracle.recurrence_c(a["q"], a["k"], a["v"], a["g"], a["beta"], None)[1]
    assert rel_err(f64(Bm), ref_B) <= tol_for(dtype)
    # M on a slow-decay copy: g / 100 (alpha in (e^-0.05, 1))
    gs = (x["g"].float() / 100).to(dtype).contiguous()
    Ms, _ = K.segment_pair(c["q"], c["k"], c["v"], cuda(gs), c["beta"])
    torch.cuda.synchronize()
    ref_M = oracle.transition_product_np(a["k"], f64(gs), a["beta"])
    assert np.max(np.abs(ref_M)) > 1e-3
    assert rel_err(f64(Ms), ref_M) <= tol_for(dtype)


def _seg_workspace(K, q, **flags):
    B, T, H, d = q.shape
    n = K.kda_segment_pair_workspace_bytes(B, T, H, d, d, K.make_opts(q.dtype, **flags))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)


@pytest.mark.parametrize("kind", ["bf16", "complex", "unbounded", "fp32-d64"])
def test_segment_forward_from_records(K, kind):
    """kda_segment_forward after kda_segment_pair on the same inputs and workspace: the scan
    alone over the pair's records (bf16 d=128, Complex-KDA, the unbounded gate) or the whole
    chunk forward (fp32 d=64), from a given start state; equal to the oracle from that state,
    and the pair itself still right (M S0 + B = the final state)."""
    d, dtype = (64, torch.float32) if kind == "fp32-d64" else (128, torch.bfloat16)
    flags = dict(complex_gate=kind == "complex", unbounded=kind == "unbounded")
    x = W.chunk_inputs(2, 200, 3, d, d, dtype=dtype, seed=820, complex_gate=flags["complex_gate"],
                       gate="softplus" if flags["unbounded"] else "bounded")
    c = {n: (None if x[n] is None else cuda(x[n])) for n in x}
    ws = _seg_workspace(K, c["q"], **flags)
    args = [c[n] for n in ("q", "k", "v", "g", "beta")]
    M, Bm = K.segment_pair(*args, workspace=ws, **flags)
    out, S_T = K.segment_forward(*args, c["S0"], ws, **flags)
    torch.cuda.synchronize()
    a = [f64(x[n]) for n in ("q", "k", "v", "g", "beta")]
    ref_o, ref_s = oracle.recurrence_c(*a, f64(x["S0"]), complex_gate=flags["complex_gate"])
    tol = tol_for(dtype)
    assert rel_err(f64(out), ref_o) <= tol and rel_err(f64(S_T), ref_s) <= tol
    got_ST = np.einsum("bhij,bhjk->bhik", f64(M), f64(x["S0"])) + f64(Bm)
    assert rel_err(got_ST, ref_s) <= tol


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
def test_affine_combine(K, dk, dv):
    gen = torch.Generator().manual_seed(dk + dv)
    R, BH = 5, 6
    Ms = torch.randn((R, BH, dk, dk), generator=gen) / dk ** 0.5
    Bs = torch.randn((R, BH, dk, dv), generator=gen)
    S0 = torch.randn((BH, dk, dv), generator=gen)
    for n in (0, 1, 3, 5):
        got = K.affine_combine(cuda(Ms), cuda(Bs), n, cuda(S0))
        torch.cuda.synchronize()
        ref = oracle.affine_combine_np(f64(Ms[:n]).reshape(n, 1, BH, dk, dk),
                                       f64(Bs[:n]).reshape(n, 1, BH, dk, dv), f64(S0)[None])[0]
        assert rel_err(f64(got), ref) <= 1e-5
    got = K.affine_combine(cuda(Ms), cuda(Bs), 2, None)
    torch.cuda.synchronize()
    ref = oracle.affine_combine_np(f64(Ms[:2]).reshape(2, 1, BH, dk, dk),
                                   f64(Bs[:2]).reshape(2, 1, BH, dk, dv), None)[0]
    assert rel_err(f64(got), ref) <= 1e-5


@pytest.mark.parametrize("cuts", [[0, 1000, 1500, 2900, 4096], [0, 64, 64, 4096]],
                         ids=["four-ragged", "with-empty"])
def test_split_sequence_emulated(K, cuts):
    """Prefill-shaped sequence (H=16, d=128, bf16) cut into segments, run as the ranks of a
    context-parallel group would (pairs, ordered fold, forward from the fold's state)."""
    x = W.workload_inputs("prefill")
    c = {n: cuda(x[n]) for n in x}
    segs = [(a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    sl = lambda n, a, b: c[n][:, a:b].contiguous()
    wss = [_seg_workspace(K, sl("q", a, b)) for a, b in segs]
    pairs = [K.segment_pair(*(sl(n, a, b) for n in ("q", "k", "v", "g", "beta")), workspace=ws)
             for (a, b), ws in zip(segs, wss)]
    Ms = torch.stack([p[0] for p in pairs])
    Bs = torch.stack([p[1] for p in pairs])
    outs = []
    for r, (a, b) in enumerate(segs):
        S_start = K.affine_combine(Ms, Bs, r, c["S0"])
        o, _ = K.segment_forward(*(sl(n, a, b) for n in ("q", "k", "v", "g", "beta")), S_start, wss[r])
        outs.append(o)
    S_T = K.affine_combine(Ms, Bs, len(segs), c["S0"])
    torch.cuda.synchronize()
    heads = [0, 9]
    a = {n: f64(x[n][:, :, heads]) for n in ("q", "k", "v", "g", "beta")}
    ref_o, ref_s = oracle.recurrence_c(a["q"], a["k"], a["v"], a["g"], a["beta"],
                                       f64(x["S0"][:, heads]))
    out = torch.cat(outs, dim=1)
    assert rel_err(f64(out[:, :, heads]), ref_o) <= 2e-2
    assert rel_err(f64(S_T[:, heads]), ref_s) <= 2e-2
