"""Failure detection on the GPU without a fault: a bounded device-side wait that runs
out reports KDA_ERR_TIMEOUT through the status word, and the context stays usable.

The wait is the same bounded mbarrier wait the tensor-core prefill uses on its MMA
completions and TMA loads; here nothing ever completes the barrier's phase.
"""
import time

import pytest
import torch

import gated_delta_rule_122_b200 as kda
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_F32, o_err, oracle_full, s_err, to_device

pytestmark = pytest.mark.gpu

KDA_ERR_TIMEOUT = 8


def test_completed_wait_reports_ok():
    assert kda.selftest_bounded_wait(True, limit_us=20000) == 0


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert kda.selftest_bounded_wait(False, limit_us=20000) == KDA_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.019 < elapsed < 2.0, elapsed
    assert kda.status_string(KDA_ERR_TIMEOUT) == "a bounded device-side wait timed out"
    # the context is still usable: a prefill right after matches the oracle
    x = make_inputs(WORKLOADS["tiny"].scaled(B=1, H=2, T=40))
    d = to_device(x)
    o, S = kda.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], scale=x["scale"], check_status=True)
    o_ref, s_ref = oracle_full(x)
    assert o_err(o, o_ref) < TOL_F32 and s_err(S, s_ref) < TOL_F32


@pytest.mark.parametrize("limit_us", [0, 2000001])
def test_wait_limit_out_of_range_rejected(limit_us):
    with pytest.raises(kda.KDAError) as e:
        kda.selftest_bounded_wait(False, limit_us=limit_us)
    assert e.value.code == 2   # KDA_ERR_SHAPE
