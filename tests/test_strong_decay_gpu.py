"""Strong decays on the tensor-core prefill (d_k = d_v = 128, bf16 inputs) against the oracle.

A retention factor of zero clears the old state exactly ("From Fast Weight Programmers to
KDA", section "Gated Delta Networks"), and the C ABI accepts alpha in [0, 1].  In a
32-token chunk the tensor-core kernel forms pairwise decays from factors anchored in the
middle of the chunk; when some channel decays by more than 2^-100 over a 16-token half,
those factors leave the fp32 range and the chunk is computed token by token instead.
These cases put such decays on either side of the anchor, in the first and last chunk,
in consecutive chunks, in a ragged tail, held over many tokens on a subset of channels,
and through the raw-input, scalar-gate and packed-sequence entry points.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, o_err, oracle_full, s_err, to_device

pytestmark = pytest.mark.gpu


def _run(fn, x, **kw):
    return fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], initial_state=x["s0"],
              scale=x["scale"], **kw)


def _check(x, fn=kda.forward):
    o_ref, s_ref = oracle_full(x)
    o, S = _run(fn, to_device(x), check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


def _inputs(T, B=1, H=2, name="long"):
    return make_inputs(WORKLOADS[name].scaled(B=B, H=H, T=T))


@pytest.mark.parametrize("rows", [(3, 9), (18, 27), (14, 17), (0, 31)])
def test_two_zero_retentions_in_one_chunk(rows):
    """alpha = 0 on two tokens of one chunk, every channel: both in the first half, both in
    the second, straddling the anchor, at the chunk's ends."""
    x = _inputs(T=130)
    for r in rows:
        x["alpha"][0, 64 + r, :, :] = 0.0
    _check(x)


def test_zero_retention_on_some_channels():
    x = _inputs(T=200, H=3)
    x["alpha"][0, 37, 1, 5:40] = 0.0
    x["alpha"][0, 41, 1, 20:60] = 0.0
    x["alpha"][0, 100, 0, 0] = 0.0
    x["alpha"][0, 105, 0, 0] = 0.0
    _check(x)


def test_small_retention_held_on_a_subset_of_channels():
    """alpha = 1e-3 for 32 tokens (about 6.9 nats per token) on 24 channels."""
    x = _inputs(T=160)
    x["alpha"][0, 50:82, 0, 10:34] = 1e-3
    x["alpha"][0, 90:122, 1, 100:124] = 1e-3
    _check(x)


def test_strong_decay_first_last_and_consecutive_chunks():
    x = _inputs(T=160)
    x["alpha"][0, 2:5, :, :64] = 0.0          # chunk 0
    x["alpha"][0, 70:100, 0, :] = 1e-4         # chunks 2 and 3
    x["alpha"][0, 150:153, 1, 7] = 0.0         # the last chunk (final state written from it)
    _check(x)


@pytest.mark.parametrize("T", [33, 77, 100])
def test_strong_decay_in_a_ragged_tail(T):
    x = _inputs(T=T, B=2)
    x["alpha"][:, T - 3:T, :, :] = 0.0
    x["alpha"][1, T - 20:T - 18, 0, :] = 0.0
    _check(x)


def test_strong_decay_zero_initial_state_near_one_workload():
    x = make_inputs(WORKLOADS["prefill"].scaled(B=1, H=2, T=96))
    x["alpha"][0, 40, :, :] = 0.0
    x["alpha"][0, 45, :, :] = 0.0
    _check(x)


def test_whole_sequence_of_zero_retention():
    """alpha = 0 everywhere: every token sees only its own write."""
    x = _inputs(T=70)
    x["alpha"].zero_()
    _check(x)


def test_strong_decay_raw_inputs():
    """Gate logits of 100 (alpha = e^-100 after the softplus) on two tokens of a chunk."""
    x = _inputs(T=96)
    a = x["alpha"].double().clamp(1e-30, 1 - 1e-7)
    b = x["beta"].double().clamp(1e-7, 1 - 1e-7)
    gl = torch.log((1 - a) / a)
    gl[0, 40:42] = 100.0
    gl[0, 70, 1, :30] = 100.0
    gl = gl.to(x["alpha"].dtype)
    bl = torch.log(b / (1 - b)).to(x["beta"].dtype)
    o_ref, s_ref = oracle.forward_raw(x["q"], x["k"], x["v"], gl, bl, s0=x["s0"], scale=x["scale"])
    c = lambda t: t.cuda()
    o, S = kda.forward_raw(c(x["q"]), c(x["k"]), c(x["v"]), c(gl), c(bl), initial_state=c(x["s0"]),
                           scale=x["scale"], check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


@pytest.mark.parametrize("H", [8, 3])   # gates staged by TMA (H % 8 == 0) or read from memory
def test_strong_decay_scalar_gate(H):
    x = _inputs(T=100, H=H)
    ah = x["alpha"][..., 0].contiguous()
    ah[0, 10] = 0.0
    ah[0, 12] = 0.0
    ah[0, 60:70, 1] = 1e-4
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], ah.unsqueeze(-1).expand_as(x["alpha"]).contiguous(),
                                  x["beta"], s0=x["s0"], scale=x["scale"])
    d = to_device(x)
    o, S = kda.forward_scalar_gate(d["q"], d["k"], d["v"], ah.cuda(), d["beta"], initial_state=d["s0"],
                                   scale=x["scale"], check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


def test_strong_decay_packed_sequences():
    lengths = [50, 33, 0, 96, 7]
    total = sum(lengths)
    x = make_inputs(WORKLOADS["long"].scaled(B=1, H=2, T=total))
    x["alpha"][0, 20:22] = 0.0            # sequence 0
    x["alpha"][0, 60, 1, :] = 0.0         # sequence 1
    x["alpha"][0, 62, 1, :] = 0.0
    x["alpha"][0, 100:131, 0, 3:9] = 1e-3  # sequence 3
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    g = torch.Generator().manual_seed(5)
    s0 = 0.1 * torch.randn(len(lengths), 2, 128, 128, generator=g)
    p = {n: x[n][0].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
    outs, states = [], []
    for i in range(len(lengths)):
        a, b = int(cu[i]), int(cu[i + 1])
        sl = lambda t: t[a:b].unsqueeze(0)
        o_i, S_i = oracle.forward(sl(p["q"]), sl(p["k"]), sl(p["v"]), sl(p["alpha"]), sl(p["beta"]),
                                  s0=s0[i:i + 1], scale=x["scale"])
        outs.append(o_i[0])
        states.append(S_i[0])
    o_ref, s_ref = np.concatenate(outs, 0), np.stack(states, 0)
    d = {n: t.cuda() for n, t in p.items()}
    o, S = kda.forward_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], torch.from_numpy(cu).cuda(),
                              initial_state=s0.cuda(), scale=x["scale"], check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"
