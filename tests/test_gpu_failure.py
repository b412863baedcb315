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
