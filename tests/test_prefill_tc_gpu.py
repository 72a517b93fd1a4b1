"""The tensor-core chunk prefill (d_k = d_v = 128, bf16 inputs) against the oracle.

Covers single tokens, a chunk boundary +-1, ragged tails, several chunks, both
decay regimes of the workloads (near-one retention with zero initial state;
30% strong-forget channels with a random initial state), agreement with the
token-by-token GPU schedule, and the device status word.
"""
import pytest
import torch

import gated_delta_rule_122_b200 as kda
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, o_err, oracle_full, s_err, to_device

pytestmark = pytest.mark.gpu


def _run(fn, x, **kw):
    return fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], initial_state=x["s0"],
              scale=x["scale"], **kw)


@pytest.mark.parametrize("name", ["prefill", "long"])
@pytest.mark.parametrize("B,H,T", [(1, 1, 1), (1, 2, 31), (2, 2, 32), (1, 2, 33), (1, 3, 100),
                                   (2, 2, 257)])
def test_tc_prefill_matches_oracle(name, B, H, T):
    x = make_inputs(WORKLOADS[name].scaled(B=B, H=H, T=T))
    o_ref, s_ref = oracle_full(x)
    o, S = _run(kda.forward, to_device(x), check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


@pytest.mark.parametrize("name", ["prefill", "long"])
def test_tc_chunked_agrees_with_sequential(name):
    x = to_device(make_inputs(WORKLOADS[name].scaled(B=1, H=4, T=1000)))
    o1, s1 = _run(kda.forward, x, check_status=True)
    o2, s2 = _run(kda.forward_sequential, x)
    eo = o_err(o1, o2.double().cpu().numpy())
    es = s_err(s1, s2.double().cpu().numpy())
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


def test_tc_out_bf16_is_rounded_fp32():
    x = to_device(make_inputs(WORKLOADS["long"].scaled(B=1, H=2, T=70)))
    o32, _ = _run(kda.forward, x)
    o16, _ = _run(kda.forward, x, out_dtype=torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_tc_continuation():
    x = to_device(make_inputs(WORKLOADS["long"].scaled(B=1, H=2, T=96)))
    o, S = _run(kda.forward, x)
    part = lambda a, b: {k: (v[:, a:b].contiguous() if k in ("q", "k", "v", "alpha", "beta") else v)
                         for k, v in x.items()}
    x1, x2 = part(0, 40), part(40, 96)
    o1, S1 = _run(kda.forward, x1)
    x2["s0"] = S1
    o2, S2 = _run(kda.forward, x2)
    assert o_err(torch.cat([o1, o2], 1), o.double().cpu().numpy()) < TOL_BF16
    assert s_err(S2, S.double().cpu().numpy()) < TOL_BF16


def test_tc_no_final_state_and_reused_workspace():
    x = to_device(make_inputs(WORKLOADS["prefill"].scaled(B=1, H=2, T=64)))
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    o_a, _ = _run(kda.forward, x, workspace=ws)
    o_b, none = _run(kda.forward, x, workspace=ws, output_final_state=False, check_status=True)
    assert none is None and torch.equal(o_a, o_b)
