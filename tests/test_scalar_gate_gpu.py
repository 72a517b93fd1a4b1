"""One retention factor per head (Gated DeltaNet) against KDA with alpha broadcast.

The scalar gate is KDA with alpha_t repeated over the key channels, so the
per-head entry points must give exactly the per-channel ones on the broadcast
tensor (same kernels, same arithmetic), and the oracle on the broadcast tensor.
Covers the tensor-core prefill (d = 128, bf16; gates staged by TMA boxes when H is a
multiple of 8, read per token otherwise), the CUDA-core prefill (fp32, d = 64) and the
decode step.
"""
import pytest
import torch

import gated_delta_rule_122_b200 as kda
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, TOL_F32, o_err, oracle_full, s_err, to_device

pytestmark = pytest.mark.gpu


def _head_gate(B, T, H, dtype, seed):
    """alpha = exp(-softplus(x)), one per (token, head), the workloads' near-one recipe."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, H, generator=g)
    return torch.exp(-0.1 * torch.nn.functional.softplus(x)).to(dtype)


@pytest.mark.parametrize("name,over,tol", [("prefill", dict(B=2, H=3, T=133), TOL_BF16),
                                           ("prefill", dict(B=2, H=8, T=133), TOL_BF16),    # gates staged by TMA
                                           ("long", dict(B=1, H=16, T=65), TOL_BF16),
                                           ("small", dict(B=1, H=2, T=97, qkv_dtype=torch.float32), TOL_F32)])
def test_scalar_gate_prefill(name, over, tol):
    w = WORKLOADS[name].scaled(**over)
    x = make_inputs(w)
    ah = _head_gate(w.B, w.T, w.H, x["alpha"].dtype, 5)
    x["alpha"] = ah.unsqueeze(-1).expand(w.B, w.T, w.H, w.dk).contiguous()
    o_ref, s_ref = oracle_full(x)
    d = to_device(x)
    o_b, s_b = kda.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], initial_state=d["s0"],
                           scale=x["scale"], check_status=True)
    o_h, s_h = kda.forward_scalar_gate(d["q"], d["k"], d["v"], ah.cuda(), d["beta"], initial_state=d["s0"],
                                       scale=x["scale"], check_status=True)
    assert torch.equal(o_h, o_b) and torch.equal(s_h, s_b)
    eo, es = o_err(o_h, o_ref), s_err(s_h, s_ref)
    assert eo < tol and es < tol, f"o {eo:.3e} state {es:.3e}"


def test_scalar_gate_decode():
    w = WORKLOADS["decode"].scaled(B=8, H=4)
    from gated_delta_rule_122_b200.inputs import make_decode_inputs
    y = make_decode_inputs(w, device="cuda")
    ah = _head_gate(1, w.B, w.H, y["alpha"].dtype, 9)[0].cuda()
    a_full = ah.unsqueeze(-1).expand(w.B, w.H, w.dk).contiguous()
    s1, s2 = y["state"].clone(), y["state"].clone()
    o1 = kda.decode_step(y["q"], y["k"], y["v"], a_full, y["beta"], s1, scale=y["scale"])
    o2 = kda.decode_step_scalar_gate(y["q"], y["k"], y["v"], ah, y["beta"], s2, scale=y["scale"])
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
