"""GDN-2 (decoupled erase and write gates) on the GPU against the oracle.

"From Fast Weight Programmers to KDA", section "Gated DeltaNet-2": the erase
gate b_t (per key channel) scales the retrieval key, the write gate w_t (per
value channel) scales the written value.  Checks the chunked prefill and the
decode step against the fp64 oracle, and that b = w = beta reproduces the KDA
entry points on the same inputs.
"""
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_decode_inputs, make_inputs
from tests.helpers import TOL_BF16, TOL_F32, o_err, s_err, to_device

pytestmark = pytest.mark.gpu


def _gates(shape_k, shape_v, dtype, seed):
    """Erase and write gates as sigmoids of standard normals (values in (0, 1))."""
    g = torch.Generator().manual_seed(seed)
    return (torch.sigmoid(torch.randn(*shape_k, generator=g)).to(dtype),
            torch.sigmoid(torch.randn(*shape_v, generator=g)).to(dtype))


@pytest.mark.parametrize("name,over,tol", [
    ("small", dict(B=2, H=2, T=97, qkv_dtype=torch.float32), TOL_F32),
    ("small", dict(B=1, H=3, T=64, dk=32, dv=16, qkv_dtype=torch.float32), TOL_F32),
    ("prefill", dict(B=1, H=2, T=133), TOL_BF16),
])
def test_gdn2_prefill_matches_oracle(name, over, tol):
    w = WORKLOADS[name].scaled(**over)
    x = make_inputs(w)
    b, wr = _gates(x["k"].shape, x["v"].shape, x["alpha"].dtype, 11)
    o_ref, s_ref = oracle.forward_gdn2(x["q"], x["k"], x["v"], x["alpha"], b, wr, s0=x["s0"], scale=x["scale"])
    d = to_device(x)
    o, S = kda.forward_gdn2(d["q"], d["k"], d["v"], d["alpha"], b.cuda(), wr.cuda(), initial_state=d["s0"],
                            scale=x["scale"], check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < tol and es < tol, f"o {eo:.3e} state {es:.3e}"


def test_gdn2_tied_gates_match_kda():
    w = WORKLOADS["small"].scaled(B=1, H=2, T=70, qkv_dtype=torch.float32)
    x = make_inputs(w)
    beta = x["beta"]
    b = beta.unsqueeze(-1).expand(*x["k"].shape).contiguous()
    wr = beta.unsqueeze(-1).expand(*x["v"].shape).contiguous()
    d = to_device(x)
    o1, s1 = kda.forward_gdn2(d["q"], d["k"], d["v"], d["alpha"], b.cuda(), wr.cuda(), initial_state=d["s0"],
                              scale=x["scale"], check_status=True)
    o2, s2 = kda.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], initial_state=d["s0"],
                         scale=x["scale"], check_status=True)
    # the same kernel family with beta folded at a different point: equal to rounding
    assert o_err(o1, o2.cpu().double().numpy()) < 1e-5
    assert s_err(s1, s2.cpu().double().numpy()) < 1e-5


def test_gdn2_decode_matches_oracle():
    w = WORKLOADS["decode"].scaled(B=6, H=4)
    y = make_decode_inputs(w, device="cuda")
    b, wr = _gates(y["k"].shape, y["v"].shape, y["alpha"].dtype, 13)
    b, wr = b.cuda(), wr.cuda()
    s0 = y["state"].clone()
    o = kda.decode_step_gdn2(y["q"], y["k"], y["v"], y["alpha"], b, wr, y["state"], scale=y["scale"])
    u = lambda t: t.cpu().unsqueeze(1)   # [N, H, d] -> [N, 1, H, d]
    o_ref, s_ref = oracle.forward_gdn2(u(y["q"]), u(y["k"]), u(y["v"]), u(y["alpha"]), u(b), u(wr),
                                       s0=s0.cpu(), scale=y["scale"])
    eo, es = o_err(o, o_ref[:, 0]), s_err(y["state"], s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


def test_gdn2_empty_sequence_copies_state():
    w = WORKLOADS["small"].scaled(B=1, H=2, T=1, qkv_dtype=torch.float32)
    x = to_device(make_inputs(w))
    sl = lambda t: t[:, :0].contiguous()
    b = torch.ones_like(x["k"])
    o, S = kda.forward_gdn2(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]), sl(b), sl(torch.ones_like(x["v"])),
                            initial_state=x["s0"], scale=x["scale"], check_status=True)
    assert o.numel() == 0 and torch.equal(S, x["s0"])


# --- the tensor-core prefill (d_k = d_v = 128, bf16 inputs and gates) ----------------------
@pytest.mark.parametrize("name", ["prefill", "long"])
@pytest.mark.parametrize("B,H,T", [(1, 1, 1), (1, 2, 31), (2, 2, 64), (1, 3, 100), (2, 1, 257)])
def test_gdn2_tc_prefill_matches_oracle(name, B, H, T):
    x = make_inputs(WORKLOADS[name].scaled(B=B, H=H, T=T))
    b, wr = _gates(x["k"].shape, x["v"].shape, x["alpha"].dtype, 21 + T)
    o_ref, s_ref = oracle.forward_gdn2(x["q"], x["k"], x["v"], x["alpha"], b, wr, s0=x["s0"], scale=x["scale"])
    d = to_device(x)
    o, S = kda.forward_gdn2(d["q"], d["k"], d["v"], d["alpha"], b.cuda(), wr.cuda(), initial_state=d["s0"],
                            scale=x["scale"], check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


def test_gdn2_tc_strong_decay_runs_token_by_token():
    """alpha = 0 on two tokens of one half chunk and a small retention held on some
    channels: those chunks run token by token with the erase and write gates."""
    x = make_inputs(WORKLOADS["long"].scaled(B=1, H=2, T=130))
    x["alpha"][0, 40, :, :] = 0.0
    x["alpha"][0, 44, :, :] = 0.0
    x["alpha"][0, 80:112, 1, 5:30] = 1e-3
    b, wr = _gates(x["k"].shape, x["v"].shape, x["alpha"].dtype, 31)
    o_ref, s_ref = oracle.forward_gdn2(x["q"], x["k"], x["v"], x["alpha"], b, wr, s0=x["s0"], scale=x["scale"])
    d = to_device(x)
    o, S = kda.forward_gdn2(d["q"], d["k"], d["v"], d["alpha"], b.cuda(), wr.cuda(), initial_state=d["s0"],
                            scale=x["scale"], check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


def test_gdn2_tc_tied_gates_match_kda():
    """b = w = beta on the tensor-core path equals the KDA prefill up to the rounding of the
    split operands (beta enters the products at different points)."""
    x = make_inputs(WORKLOADS["long"].scaled(B=1, H=2, T=100))
    beta = x["beta"]
    b = beta.unsqueeze(-1).expand(*x["k"].shape).contiguous()
    wr = beta.unsqueeze(-1).expand(*x["v"].shape).contiguous()
    d = to_device(x)
    o1, s1 = kda.forward_gdn2(d["q"], d["k"], d["v"], d["alpha"], b.cuda(), wr.cuda(), initial_state=d["s0"],
                              scale=x["scale"], check_status=True)
    o2, s2 = kda.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], initial_state=d["s0"],
                         scale=x["scale"], check_status=True)
    assert o_err(o1, o2.cpu().double().numpy()) < 1e-3
    assert s_err(s1, s2.cpu().double().numpy()) < 1e-3
