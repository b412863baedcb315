"""Failure handling on the GPU without a fault: the library's bounded waits give up when
nothing arrives, report KDA_ERR_TIMEOUT to the host, and leave the context usable."""
import pytest
import torch

import kda_workloads as W
import oracle
from tests._util import cuda, f64, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from gated_delta_rule_73_b200 import build
    build.build()
    import gated_delta_rule_73_b200 as K
    return K


@pytest.mark.parametrize("limit", [0, 1, 1000])
def test_bounded_waits_give_up_and_the_context_survives(K, limit):
    assert K.kda_selftest_bounded_wait(limit) == -6          # KDA_ERR_TIMEOUT
    # the next call on the same context still computes the right answer
    x = W.chunk_inputs(1, 70, 2, 128, 128, seed=5)
    out, S_T = K.chunk_fwd(*(cuda(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")))
    torch.cuda.synchronize()
    ro, rs = oracle.recurrence_c(*(f64(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")))
    assert rel_err(f64(out), ro) <= 2e-2 and rel_err(f64(S_T), rs) <= 2e-2


@pytest.mark.parametrize("form", ["split", "one_launch"])
def test_chunk_kernels_give_up_report_timeout_and_recover(K, form):
    """The product kernels' own waits: with the wait limit at 0 the split form's prep gives up at
    its first wait (and, in the one-launch form, the scan CTAs at their first poll for a
    published record); the call drains what it has in flight and returns, and
    kda_device_status reports KDA_ERR_TIMEOUT once.  With the limit restored the same call on
    the same context matches the oracle."""
    # 16 heads x 4096 tokens takes the one-launch form; 96 heads x 512 tokens the two launches
    B, T, H = (1, 4096, 16) if form == "one_launch" else (1, 512, 96)
    x = W.chunk_inputs(B, T, H, 128, 128, seed=7)
    args = [cuda(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")]
    assert K.kda_device_status() == 0
    prev = K.kda_set_wait_limit(0)
    try:
        K.chunk_fwd(*args, fused=False)
        assert K.kda_device_status() == -6          # KDA_ERR_TIMEOUT, read and cleared
        assert K.kda_device_status() == 0
    finally:
        K.kda_set_wait_limit(prev)
    assert prev == K.KDA_WAIT_LIMIT_DEFAULT
    out, S_T = K.chunk_fwd(*args, fused=False)
    assert K.kda_device_status() == 0
    ro, rs = oracle.recurrence_c(*(f64(x[n]) for n in ("q", "k", "v", "g", "beta", "S0")))
    assert rel_err(f64(out), ro) <= 2e-2 and rel_err(f64(S_T), rs) <= 2e-2
