"""Fused input preprocessing on the GPU (kda_forward_raw, kda_decode_step_raw) against
the oracle's fp64 preprocessing followed by the recurrence.

Raw inputs: q and k un-normalised (the kernels divide each row by its L2 norm),
gate logits x with alpha = exp(-softplus(x)), beta logits y with beta = sigmoid(y).
Covers the tensor-core prefill (d = 128, bf16), the CUDA-core prefill (fp32 and
d = 64), a zero key row, and the decode step.
"""
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_decode_inputs, make_inputs
from tests.helpers import TOL_BF16, TOL_F32, o_err, s_err

pytestmark = pytest.mark.gpu


def _raw(x, seed):
    """Raw projections with the workload's shapes: rows of q, k rescaled by random
    positive factors, and the logits that map back to the workload's alpha and beta."""
    g = torch.Generator().manual_seed(seed)
    q, k = x["q"].float(), x["k"].float()
    cq = torch.exp(torch.randn(*q.shape[:-1], 1, generator=g))
    ck = torch.exp(torch.randn(*k.shape[:-1], 1, generator=g))
    a = x["alpha"].double().clamp(1e-30, 1 - 1e-7)
    b = x["beta"].double().clamp(1e-7, 1 - 1e-7)
    return dict(q=(cq * q).to(x["q"].dtype), k=(ck * k).to(x["k"].dtype), v=x["v"],
                x=torch.log((1 - a) / a).to(x["alpha"].dtype), y=torch.log(b / (1 - b)).to(x["beta"].dtype))


@pytest.mark.parametrize("name,over,tol", [
    ("prefill", dict(B=1, H=3, T=133), TOL_BF16),
    ("long", dict(B=2, H=2, T=96), TOL_BF16),
    ("small", dict(B=2, H=2, T=97, qkv_dtype=torch.float32), TOL_F32),
    ("small", dict(B=1, H=2, T=70), TOL_BF16),
])
def test_forward_raw_matches_oracle(name, over, tol):
    w = WORKLOADS[name].scaled(**over)
    x = make_inputs(w)
    r = _raw(x, 17)
    if name == "long":
        r["k"][0, 5, 1] = 0          # a zero key row stays zero
    o_ref, s_ref = oracle.forward_raw(r["q"], r["k"], r["v"], r["x"], r["y"], s0=x["s0"], scale=x["scale"])
    c = lambda t: t.cuda()
    o, S = kda.forward_raw(c(r["q"]), c(r["k"]), c(r["v"]), c(r["x"]), c(r["y"]),
                           initial_state=None if x["s0"] is None else c(x["s0"]), scale=x["scale"],
                           check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < tol and es < tol, f"o {eo:.3e} state {es:.3e}"


def test_decode_step_raw_matches_oracle():
    w = WORKLOADS["decode"].scaled(B=6, H=4)
    y = make_decode_inputs(w)
    r = _raw(y, 23)
    s0 = y["state"].clone()
    state = y["state"].cuda()
    o = kda.decode_step_raw(r["q"].cuda(), r["k"].cuda(), r["v"].cuda(), r["x"].cuda(), r["y"].cuda(), state,
                            scale=y["scale"])
    u = lambda t: t.unsqueeze(1)
    o_ref, s_ref = oracle.forward_raw(u(r["q"]), u(r["k"]), u(r["v"]), u(r["x"]), u(r["y"]), s0=s0,
                                      scale=y["scale"])
    eo, es = o_err(o, o_ref[:, 0]), s_err(state, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"
