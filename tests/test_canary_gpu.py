"""Canary-padded outputs: every kernel writes exactly its own output rows and states.

The outputs are views into larger buffers filled with a canary value; after the call the
padding before and after the view must still hold it, and the view must hold no canary
(every element written).  Covers the tensor-core prefill (a ragged last chunk), the
CUDA-core prefill, the decode step and the multi-token decode.
"""
import pytest
import torch

import gated_delta_rule_122_b200 as kda
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_decode_inputs, make_inputs
from tests.helpers import to_device

pytestmark = pytest.mark.gpu

CANARY = 1234.5
PAD = 4096   # elements of padding on each side (16 KiB of fp32)


def _padded(shape):
    n = 1
    for s in shape:
        n *= s
    buf = torch.full((PAD + n + PAD,), CANARY, device="cuda")
    return buf, buf[PAD:PAD + n].view(*shape)


def _check(buf, view):
    assert torch.all(buf[:PAD] == CANARY) and torch.all(buf[-PAD:] == CANARY)
    assert not torch.any(view == CANARY)


@pytest.mark.parametrize("name,over", [("prefill", dict(B=2, H=3, T=77)),
                                       ("small", dict(B=2, H=2, T=45, qkv_dtype=torch.float32))])
def test_prefill_writes_only_its_outputs(name, over):
    w = WORKLOADS[name].scaled(**over)
    d = to_device(make_inputs(w))
    ob, o = _padded((w.B, w.T, w.H, w.dv))
    sb, S = _padded((w.B, w.H, w.dk, w.dv))
    kda.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], initial_state=d["s0"], scale=d["scale"],
                out=o, final_state=S, check_status=True)
    torch.cuda.synchronize()
    _check(ob, o)
    _check(sb, S)


def test_decode_writes_only_its_outputs():
    w = WORKLOADS["decode"].scaled(B=5, H=3)
    y = make_decode_inputs(w, device="cuda")
    ob, o = _padded((w.B, w.H, w.dv))
    pb, pool = _padded((w.B, w.H, w.dk, w.dv))
    pool.copy_(y["state"])
    kda.decode_step(y["q"], y["k"], y["v"], y["alpha"], y["beta"], pool, scale=y["scale"], out=o)
    torch.cuda.synchronize()
    _check(ob, o)
    assert torch.all(pb[:PAD] == CANARY) and torch.all(pb[-PAD:] == CANARY)


def test_decode_tokens_writes_only_its_outputs():
    N, T, H = 3, 4, 2
    w = WORKLOADS["decode"].scaled(B=N, T=T, H=H, decode=False, init_state=False)
    x = to_device(make_inputs(w))
    pool = 0.1 * torch.randn(N, H, 128, 128, device="cuda")
    ob, o = _padded((N, T, H, 128))
    tb, ts = _padded((N, T, H, 128, 128))
    kda.decode_tokens(x["q"], x["k"], x["v"], x["alpha"], x["beta"], pool, token_states=ts, out=o,
                      scale=x["scale"], check_status=True)
    torch.cuda.synchronize()
    _check(ob, o)
    _check(tb, ts)
