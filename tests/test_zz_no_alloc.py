"""kda_chunk_fwd_noalloc through the C ABI: against the FP64 oracle and against kda_chunk_fwd.

The no-allocation entry point serves callers that cannot call cudaMalloc
(code that must not synchronise the device, loops that forbid allocation,
hosts that own the device pool).  It uses the library's fixed device scratch,
so this file checks two calls in a row (the second must not see the first
one's leftovers), each against the oracle at the tolerance of its dtype and
against the allocating entry point, and the size limit.  It sits last in
collection order.
"""
import ctypes

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


def _both(K, x, dtype, complex_gate=False):
    q, k, v, g, beta = (cuda(x[n]) for n in ("q", "k", "v", "g", "beta"))
    S0 = cuda(x["S0"])
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    ref_out, ref_S = K.chunk_fwd(q, k, v, g, beta, S0, complex_gate=complex_gate)
    out = torch.full((B, T, H, dv), float("nan"), dtype=dtype, device="cuda")
    S_T = torch.full((B, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda")
    opts = K.make_opts(dtype, complex_gate=complex_gate)
    K.kda_chunk_fwd_noalloc(q, k, v, g, beta, S0, out, S_T, opts)
    torch.cuda.synchronize()
    return f64(out), f64(S_T), f64(ref_out), f64(ref_S)


def _oracle(x, complex_gate=False):
    a = {n: (None if x[n] is None else f64(x[n])) for n in ("q", "k", "v", "g", "beta", "S0")}
    return oracle.recurrence_c(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"],
                               complex_gate=complex_gate)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_oracle_and_chunk_fwd_twice(K, dtype):
    tol = tol_for(dtype)
    # call 1, then call 2 with other inputs and shape: no leftovers may leak in
    x1 = W.chunk_inputs(2, 333, 3, 128, 128, dtype=dtype, seed=101)
    o, s, ro, rs = _both(K, x1, dtype)
    oo, os_ = _oracle(x1)
    assert rel_err(o, oo) <= tol and rel_err(s, os_) <= tol
    assert rel_err(o, ro) <= tol and rel_err(s, rs) <= tol
    x2 = W.chunk_inputs(1, 190, 2, 128, 64, dtype=dtype, seed=102, complex_gate=True)
    o, s, ro, rs = _both(K, x2, dtype, complex_gate=True)
    oo, os_ = _oracle(x2, complex_gate=True)
    assert rel_err(o, oo) <= tol and rel_err(s, os_) <= tol
    assert rel_err(o, ro) <= tol and rel_err(s, rs) <= tol


def test_noalloc_rejects_sizes_beyond_the_scratch(K):
    # Every pointer is NULL: the size check comes first and returns KDA_ERR_WORKSPACE; were the
    # checks ever reordered, the NULL check would refuse the call (KDA_ERR_ARG) before any
    # launch, so no kernel can see a made-up address.
    opts = K.make_opts(torch.bfloat16)
    p = ctypes.c_void_p(0)
    # 4096 tokens x 16 heads at d = 128 needs ~150 MB of scratch > 32 MiB
    st = K.kda._lib.kda_chunk_fwd_noalloc(p, p, p, p, p, p, p, p, 1, 4096, 16, 128, 128,
                                          ctypes.byref(opts), None)
    assert st == -7
