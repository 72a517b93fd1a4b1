"""GPU parity: the CUDA entry points against the fp64 oracle on the same seeded inputs.

Tolerances: fp32 inputs 1e-4, bf16 inputs 5e-3, for max|do|/RMS(o_ref) and the
final state's relative Frobenius error.  Worked examples with dyadic values
must match exactly.
"""
import json
import os

import numpy as np
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_decode_inputs, make_inputs
from tests.helpers import (TOL_BF16, TOL_F32, o_err, oracle_full, oracle_heads, s_err, to_device,
                           tol_for)

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PREFILL_FNS = {"chunked": kda.forward, "sequential": kda.forward_sequential}


def _run(fn, x, **kw):
    return fn(x["q"], x["k"], x["v"], x["alpha"], x["beta"], initial_state=x["s0"],
              scale=x["scale"], **kw)


# --- Module 03, section 4 worked example, padded to d = 16 --------------------------------
def _worked_example_tensors(T=1):
    g = json.load(open(os.path.join(GOLDEN, "module03_worked_example.json")))
    d = 16
    S = torch.zeros(1, 1, d, d)
    S[0, 0, :2, :2] = torch.tensor(g["S_prev"])
    k = torch.zeros(1, T, 1, d)
    k[0, :, 0, :2] = torch.tensor(g["k"])
    v = torch.zeros(1, T, 1, d)
    v[0, :, 0, :2] = torch.tensor(g["v"])
    q = torch.zeros(1, T, 1, d)
    q[0, :, 0, 0] = 1.0
    alpha = torch.ones(1, T, 1, d)
    beta = torch.full((1, T, 1), g["beta"])
    exp = torch.zeros(d, d)
    exp[:2, :2] = torch.tensor(g["expected_S"])
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, s0=S, scale=1.0), exp


@pytest.mark.parametrize("schedule", ["chunked", "sequential"])
def test_worked_example_prefill_exact(schedule):
    x, exp = _worked_example_tensors()
    x = to_device(x)
    o, S = _run(PREFILL_FNS[schedule], x)
    torch.cuda.synchronize()
    assert torch.equal(S[0, 0].cpu(), exp)
    assert torch.equal(o[0, 0, 0].cpu(), exp[0])


def test_worked_example_decode_exact():
    x, exp = _worked_example_tensors()
    x = to_device(x)
    state = x["s0"].clone()
    o = kda.decode_step(x["q"][:, 0], x["k"][:, 0], x["v"][:, 0], x["alpha"][:, 0],
                        x["beta"][:, 0], state, scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(state[0, 0].cpu(), exp)
    assert torch.equal(o[0, 0].cpu(), exp[0])


# --- decode ---------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [16, 64, 128])
def test_decode_parity_small(dtype, d):
    w = WORKLOADS["decode"].scaled(B=6, H=3, dk=d, dv=d, qkv_dtype=dtype, gate_dtype=dtype)
    x = make_decode_inputs(w)
    o_ref, s_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["state"],
                                      scale=x["scale"])
    xd = to_device(x)
    o = kda.decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], xd["state"],
                        scale=x["scale"])
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert o_err(o, o_ref) < tol
    assert s_err(xd["state"], s_ref) < tol


def test_decode_parity_full_size_sampled():
    """The decode workload (256 sequences x 64 heads, d = 128) in the bench's launch shape."""
    x = make_decode_inputs("decode", device="cuda")
    pairs = [(0, 0), (255, 63), (17, 5), (128, 40), (200, 1), (3, 62)]
    before = {p: x["state"][p].cpu().clone() for p in pairs}
    o = kda.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["state"],
                        scale=x["scale"])
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    for (n, h) in pairs:
        sl = lambda t: t[n:n + 1, h:h + 1].cpu()
        o_ref, s_ref = oracle.decode_step(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]),
                                          sl(x["beta"]), before[(n, h)][None, None],
                                          scale=x["scale"])
        assert o_err(o[n, h], o_ref[0, 0]) < TOL_BF16
        assert s_err(x["state"][n, h], s_ref[0, 0]) < TOL_BF16


def test_decode_out_bf16_is_rounded_fp32():
    x = to_device(make_decode_inputs(WORKLOADS["decode"].scaled(B=4, H=2)))
    s1, s2 = x["state"].clone(), x["state"].clone()
    args = (x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    o32 = kda.decode_step(*args, s1, scale=x["scale"])
    o16 = kda.decode_step(*args, s2, scale=x["scale"], out_dtype=torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(s1, s2)


# --- prefill: small workloads, both schedules ------------------------------------------------
@pytest.mark.parametrize("schedule", ["chunked", "sequential"])
@pytest.mark.parametrize("name", ["tiny", "small"])
def test_prefill_parity(schedule, name):
    x = make_inputs(name)
    o_ref, s_ref = oracle_full(x)
    o, S = _run(PREFILL_FNS[schedule], to_device(x))
    tol = tol_for(x)
    assert o_err(o, o_ref) < tol
    assert s_err(S, s_ref) < tol


@pytest.mark.parametrize("T", [1, 31, 33, 100])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (128, 16), (64, 128)])
def test_prefill_ragged_shapes_fp32(T, dk, dv):
    w = WORKLOADS["tiny"].scaled(B=2, H=3, T=T, dk=dk, dv=dv, init_state=True)
    x = make_inputs(w)
    o_ref, s_ref = oracle_full(x)
    for fn in PREFILL_FNS.values():
        o, S = _run(fn, to_device(x))
        assert o_err(o, o_ref) < TOL_F32
        assert s_err(S, s_ref) < TOL_F32


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(48, 48), (80, 80), (96, 96), (112, 112), (48, 112), (112, 48), (80, 32)])
def test_prefill_multiple_of_16_head_sizes(dtype, dk, dv):
    """Every multiple of 16 up to 128 is a supported head size: both schedules against the
    oracle, a ragged last chunk and an initial state."""
    w = WORKLOADS["tiny"].scaled(B=2, H=2, T=77, dk=dk, dv=dv, init_state=True, qkv_dtype=dtype,
                                 gate_dtype=dtype)
    x = make_inputs(w)
    o_ref, s_ref = oracle_full(x)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    for fn in PREFILL_FNS.values():
        o, S = _run(fn, to_device(x))
        assert o_err(o, o_ref) < tol
        assert s_err(S, s_ref) < tol


@pytest.mark.parametrize("dk,dv", [(48, 48), (112, 112), (80, 96)])
def test_decode_multiple_of_16_head_sizes(dk, dv):
    w = WORKLOADS["decode"].scaled(B=5, H=3, dk=dk, dv=dv)
    x = make_decode_inputs(w)
    o_ref, s_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["state"],
                                      scale=x["scale"])
    xd = to_device(x)
    o = kda.decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], xd["state"], scale=x["scale"])
    assert o_err(o, o_ref) < TOL_BF16
    assert s_err(xd["state"], s_ref) < TOL_BF16


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_chunked_agrees_with_sequential(name):
    x = to_device(make_inputs(name))
    o1, s1 = _run(kda.forward, x)
    o2, s2 = _run(kda.forward_sequential, x)
    tol = tol_for(x)
    assert o_err(o1, o2.double().cpu().numpy()) < tol
    assert s_err(s1, s2.double().cpu().numpy()) < tol


def test_zero_and_tiny_retention_fp32():
    w = WORKLOADS["tiny"].scaled(B=1, H=2, T=96, dk=32, dv=32, init_state=True)
    x = make_inputs(w)
    x["alpha"][0, 5, 0, :] = 0.0
    x["alpha"][0, 40:50, 1, 3:9] = 1e-30
    x["alpha"][0, 70, :, 0] = 0.0
    o_ref, s_ref = oracle_full(x)
    for fn in PREFILL_FNS.values():
        o, S = _run(fn, to_device(x))
        assert o_err(o, o_ref) < TOL_F32
        assert s_err(S, s_ref) < TOL_F32


# --- state as the resume point ---------------------------------------------------------------
@pytest.mark.parametrize("split", [1, 32, 50])
def test_prefill_continuation(split):
    w = WORKLOADS["small"].scaled(T=128, H=2)
    x = to_device(make_inputs(w))
    o, S = _run(kda.forward, x)
    cut = lambda t, a, b: t[:, a:b].contiguous()
    x1 = {k: (cut(v, 0, split) if k in "q k v alpha beta".split() else v) for k, v in x.items()}
    x2 = {k: (cut(v, split, 128) if k in "q k v alpha beta".split() else v) for k, v in x.items()}
    o1, S1 = _run(kda.forward, x1)
    x2["s0"] = S1
    o2, S2 = _run(kda.forward, x2)
    assert o_err(torch.cat([o1, o2], 1), o.double().cpu().numpy()) < TOL_BF16
    assert s_err(S2, S.double().cpu().numpy()) < TOL_BF16


def test_in_place_continuation_final_aliases_initial():
    x = to_device(make_inputs(WORKLOADS["small"].scaled(T=64, H=2)))
    o, S = _run(kda.forward, x)
    s_buf = x["s0"].clone()
    o2, S2 = kda.forward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], initial_state=s_buf,
                         final_state=s_buf, scale=x["scale"])
    assert torch.equal(S2, S) and torch.equal(o2, o)


def test_decode_continues_prefill():
    w = WORKLOADS["small"].scaled(T=67, H=3)
    x = to_device(make_inputs(w))
    o_all, S_all = _run(kda.forward, x)
    pre = {k: (v[:, :64].contiguous() if k in "q k v alpha beta".split() else v) for k, v in x.items()}
    _, state = _run(kda.forward, pre)
    for t in range(64, 67):
        tok = lambda name: x[name][:, t].contiguous()
        o_t = kda.decode_step(tok("q"), tok("k"), tok("v"), tok("alpha"), tok("beta"), state,
                              scale=x["scale"])
        assert o_err(o_t, o_all[:, t].double().cpu().numpy()) < TOL_BF16
    assert s_err(state, S_all.double().cpu().numpy()) < TOL_BF16


def test_empty_sequence_returns_initial_state():
    x = to_device(make_inputs(WORKLOADS["small"].scaled(T=4, H=2)))
    cut = {k: (v[:, :0].contiguous() if k in "q k v alpha beta".split() else v) for k, v in x.items()}
    o, S = _run(kda.forward, cut)
    assert o.numel() == 0 and torch.equal(S, x["s0"])
    cut["s0"] = None
    _, S0 = _run(kda.forward, cut)
    assert torch.count_nonzero(S0) == 0


def test_prefill_out_bf16_is_rounded_fp32():
    x = to_device(make_inputs(WORKLOADS["small"].scaled(T=100, H=2)))
    o32, _ = _run(kda.forward, x)
    o16, _ = _run(kda.forward, x, out_dtype=torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_host_buffers_round_trip():
    x = make_inputs(WORKLOADS["small"].scaled(T=80, H=2))
    o_h, S_h = _run(kda.forward, x)
    o_d, S_d = _run(kda.forward, to_device(x))
    assert o_h.device.type == "cpu" and torch.equal(o_h, o_d.cpu()) and torch.equal(S_h, S_d.cpu())


@pytest.mark.parametrize("gate", ["channel", "head"])
def test_host_buffers_pipelined_match_device(gate):
    """Host tensors of at least two 1024-token segments take the pipelined host path
    (copies overlapped with the kernel, state carried between segments).  It matches the
    oracle like the device path, and the device path closely: the carried state is
    written out in fp32 and split again into bf16 hi/lo planes (about 16 significant
    bits) when the next segment starts, so the two differ by a few parts in 1e5."""
    w = WORKLOADS["prefill"].scaled(B=2, H=8, T=2100, init_state=True)
    x = make_inputs(w)
    if gate == "head":
        x["alpha"] = x["alpha"][..., 0].contiguous()
    fn = kda.forward if gate == "channel" else kda.forward_scalar_gate
    hx = {n: x[n].pin_memory() for n in ("q", "k", "v", "alpha", "beta", "s0")}
    o_h, s_h = fn(hx["q"], hx["k"], hx["v"], hx["alpha"], hx["beta"], initial_state=hx["s0"], scale=x["scale"])
    assert o_h.device.type == "cpu" and s_h.device.type == "cpu"
    d = to_device(x)
    o_d, s_d = fn(d["q"], d["k"], d["v"], d["alpha"], d["beta"], initial_state=d["s0"], scale=x["scale"])
    assert o_err(o_h, o_d.cpu().double().numpy()) < 2e-4
    assert s_err(s_h, s_d.cpu().double().numpy()) < 2e-4
    if gate == "channel":
        for (b, h), (o_ref, s_ref) in oracle_heads(x, [(0, 0), (1, 7)]).items():
            assert o_err(o_h[b, :, h], o_ref) < TOL_BF16 and s_err(s_h[b, h], s_ref) < TOL_BF16


def test_status_errors_raise():
    x = to_device(make_inputs(WORKLOADS["tiny"].scaled(T=8, dk=40, dv=16)))
    with pytest.raises(kda.KDAError, match="head size"):
        _run(kda.forward, x)


# --- full-size workloads, sampled heads ------------------------------------------------------
@pytest.mark.parametrize("name", ["prefill", "long"])
def test_full_size_prefill_sampled_heads(name):
    x = make_inputs(name, device="cuda")
    o, S = _run(kda.forward, x)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    w = x["workload"]
    pairs = [(0, 0), (w.B - 1, w.H - 1), (0, 37)]
    ref = oracle_heads(x, pairs)
    for (b, h), (o_ref, s_ref) in ref.items():
        assert o_err(o[b, :, h], o_ref) < TOL_BF16, (b, h)
        assert s_err(S[b, h], s_ref) < TOL_BF16, (b, h)


def test_decode_step_host_inputs_match_device():
    """Host token vectors and host o with the state resident on the device (the host-buffer
    decode entry point) give the device path's results exactly."""
    x = make_decode_inputs(WORKLOADS["decode"].scaled(B=5, H=3))
    s_host_path = x["state"].cuda()
    s_dev_path = x["state"].cuda()
    hx = {n: x[n].pin_memory() for n in ("q", "k", "v", "alpha", "beta")}
    o_h = kda.decode_step(hx["q"], hx["k"], hx["v"], hx["alpha"], hx["beta"], s_host_path, scale=x["scale"])
    d = to_device(x)
    o_d = kda.decode_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], s_dev_path, scale=x["scale"])
    torch.cuda.synchronize()
    assert o_h.device.type == "cpu" and torch.equal(o_h, o_d.cpu()) and torch.equal(s_host_path, s_dev_path)
