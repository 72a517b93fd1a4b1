"""The column-scan prefill (token by token, one 8-lane group per value column) against
the oracle.

The scan is the schedule the library picks for workloads with few (sequence, head)
pairs, such as the small workload (B=1 H=4 T=2048 d=64).  Checked here: the worked
example exactly, the tiny and small workloads in full, ragged lengths and every
multiple-of-16 head size, all input/gate dtype pairs, the per-head gate, packed
sequences (empty ones too), continuation across calls and in place, the
automatic choice (bit-identical to the kernel it names), agreement with the chunkwise
schedule, and the host-buffer entry point.
"""
import json
import os

import numpy as np
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, TOL_F32, o_err, oracle_full, s_err, to_device, tol_for

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fwd(x, **kw):
    return kda.forward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], initial_state=x.get("s0"),
                       scale=x["scale"], check_status=True, **kw)


def test_worked_example_exact():
    """Module 03's worked example (dyadic values): one token, exact to the bit."""
    g = json.load(open(os.path.join(GOLDEN, "module03_worked_example.json")))
    d = 16
    S = torch.zeros(1, 1, d, d)
    S[0, 0, :2, :2] = torch.tensor(g["S_prev"])
    k = torch.zeros(1, 1, 1, d)
    k[0, 0, 0, :2] = torch.tensor(g["k"])
    v = torch.zeros(1, 1, 1, d)
    v[0, 0, 0, :2] = torch.tensor(g["v"])
    q = torch.zeros(1, 1, 1, d)
    q[0, 0, 0, 0] = 1.0
    x = to_device(dict(q=q, k=k, v=v, alpha=torch.ones(1, 1, 1, d), beta=torch.full((1, 1, 1), g["beta"]),
                       s0=S, scale=1.0))
    exp = torch.zeros(d, d)
    exp[:2, :2] = torch.tensor(g["expected_S"])
    with kda.schedule("scan"):
        o, S1 = _fwd(x)
    assert torch.equal(S1[0, 0].cpu(), exp)
    assert torch.equal(o[0, 0, 0].cpu(), exp[0])


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_workload_parity(name):
    x = make_inputs(name)
    o_ref, s_ref = oracle_full(x)
    with kda.schedule("scan"):
        o, S = _fwd(to_device(x))
    tol = tol_for(x)
    assert o_err(o, o_ref) < tol and s_err(S, s_ref) < tol


@pytest.mark.parametrize("T", [1, 31, 32, 33, 95])
@pytest.mark.parametrize("dk,dv", [(16, 16), (48, 80), (112, 32), (128, 128), (96, 64)])
def test_ragged_lengths_and_head_sizes(T, dk, dv):
    w = WORKLOADS["tiny"].scaled(B=2, H=3, T=T, dk=dk, dv=dv)
    x = make_inputs(w)
    o_ref, s_ref = oracle_full(x)
    with kda.schedule("scan"):
        o, S = _fwd(to_device(x))
    assert o_err(o, o_ref) < TOL_F32 and s_err(S, s_ref) < TOL_F32


@pytest.mark.parametrize("H,d", [(4, 64), (4, 32), (20, 64), (40, 64)])
def test_launch_forms(H, d):
    """The launch forms: one column a group of 16 lanes (d = 64: H d/2 = 128 warps, within
    4 a SM) or 8 lanes (d = 32), two columns a group of 8 lanes with one warp a block
    (H d/8 = 160 warps) and with two (320 warps, at least two a SM)."""
    w = WORKLOADS["small"].scaled(T=45, H=H, dk=d, dv=d)
    x = make_inputs(w)
    o_ref, s_ref = oracle_full(x)
    with kda.schedule("scan"):
        o, S = _fwd(to_device(x))
    assert o_err(o, o_ref) < TOL_BF16 and s_err(S, s_ref) < TOL_BF16


@pytest.mark.parametrize("qkv", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", [torch.float32, torch.bfloat16])
def test_dtype_pairs(qkv, gate):
    w = WORKLOADS["small"].scaled(T=77, H=2, qkv_dtype=qkv, gate_dtype=gate)
    x = make_inputs(w)
    o_ref, s_ref = oracle_full(x)
    d = to_device(x)
    with kda.schedule("scan"):
        o, S = _fwd(d)
        o16, S16 = _fwd(d, out_dtype=torch.bfloat16)
    tol = tol_for(x)
    assert o_err(o, o_ref) < tol and s_err(S, s_ref) < tol
    # the bf16 output is the fp32 output rounded; the state does not depend on it
    assert torch.equal(o16, o.to(torch.bfloat16)) and torch.equal(S16, S)


def test_scalar_gate():
    w = WORKLOADS["small"].scaled(B=2, H=3, T=70)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(12)
    ah = torch.exp(-0.1 * torch.nn.functional.softplus(torch.randn(w.B, w.T, w.H, generator=g)))
    ah = ah.to(x["alpha"].dtype)
    x["alpha"] = ah.unsqueeze(-1).expand(w.B, w.T, w.H, w.dk).contiguous()
    o_ref, s_ref = oracle_full(x)
    d = to_device(x)
    with kda.schedule("scan"):
        o_h, s_h = kda.forward_scalar_gate(d["q"], d["k"], d["v"], ah.cuda(), d["beta"], initial_state=d["s0"],
                                           scale=x["scale"], check_status=True)
        o_b, s_b = _fwd(d)
    # the per-head gate is the per-channel one broadcast: the same arithmetic
    assert torch.equal(o_h, o_b) and torch.equal(s_h, s_b)
    assert o_err(o_h, o_ref) < TOL_BF16 and s_err(s_h, s_ref) < TOL_BF16


def test_packed_sequences():
    lengths = [40, 0, 1, 33, 64, 5]
    total, H = sum(lengths), 2
    w = WORKLOADS["small"].scaled(B=1, H=H, T=total)
    x = make_inputs(w)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    g = torch.Generator().manual_seed(31)
    s0 = (0.1 * torch.randn(len(lengths), H, w.dk, w.dv, generator=g)).float()
    p = {n: x[n][0].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
    d = {n: t.cuda() for n, t in p.items()}
    with kda.schedule("scan"):
        o, S = kda.forward_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], torch.from_numpy(cu).cuda(),
                                  initial_state=s0.cuda(), scale=x["scale"], check_status=True)
    for i in range(len(lengths)):
        a, b = int(cu[i]), int(cu[i + 1])
        sl = lambda t: t[a:b].unsqueeze(0)
        o_ref, s_ref = oracle.forward(sl(p["q"]), sl(p["k"]), sl(p["v"]), sl(p["alpha"]), sl(p["beta"]),
                                      s0=s0[i:i + 1], scale=x["scale"])
        assert s_err(S[i], s_ref[0]) < TOL_BF16
        if b > a:
            assert o_err(o[a:b], o_ref[0]) < TOL_BF16


@pytest.mark.parametrize("split", [1, 32, 50])
def test_continuation(split):
    """Two calls with the state passed on equal one call; the second call writes the
    state in place."""
    x = to_device(make_inputs(WORKLOADS["small"].scaled(T=100, H=2)))
    with kda.schedule("scan"):
        o, S = _fwd(x)
        first = {n: (t[:, :split].contiguous() if n in ("q", "k", "v", "alpha", "beta") else t)
                 for n, t in x.items()}
        rest = {n: (t[:, split:].contiguous() if n in ("q", "k", "v", "alpha", "beta") else t)
                for n, t in x.items()}
        o1, S1 = _fwd(first)
        rest["s0"] = S1
        o2, S2 = kda.forward(rest["q"], rest["k"], rest["v"], rest["alpha"], rest["beta"], initial_state=S1,
                             final_state=S1, scale=x["scale"], check_status=True)
    assert S2.data_ptr() == S1.data_ptr()
    # token by token, the split changes nothing: bit-identical
    assert torch.equal(torch.cat([o1, o2], 1), o) and torch.equal(S2, S)


def test_one_sequence_of_the_pack_empty():
    """A sequence with no tokens inside a packed batch goes through the kernel: its
    final state is its initial state, bit for bit."""
    H = 2
    w = WORKLOADS["small"].scaled(B=1, H=H, T=40)
    x = make_inputs(w)
    cu = torch.tensor([0, 0, 40, 40], dtype=torch.int32)
    s0 = (0.1 * torch.randn(3, H, w.dk, w.dv, generator=torch.Generator().manual_seed(4))).float().cuda()
    d = {n: x[n][0].contiguous().cuda() for n in ("q", "k", "v", "alpha", "beta")}
    with kda.schedule("scan"):
        _, S = kda.forward_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu.cuda(), initial_state=s0,
                                  scale=x["scale"], check_status=True)
    assert torch.equal(S[0], s0[0]) and torch.equal(S[2], s0[2])


def test_automatic_choice():
    """The automatic schedule runs the scan on the small workload (d = 64: no tensor-core
    kernel) and the tensor-core chunk kernel on the prefill workload's shape:
    bit-identical to the schedule it picks."""
    small = to_device(make_inputs(WORKLOADS["small"].scaled(T=300)))
    wide = to_device(make_inputs(WORKLOADS["prefill"].scaled(B=1, H=2, T=70)))
    res = {}
    for sched in ("auto", "scan", "chunked"):
        with kda.schedule(sched):
            res[sched] = (_fwd(small), _fwd(wide))
    (oa, sa), (owa, swa) = res["auto"]
    assert torch.equal(oa, res["scan"][0][0]) and torch.equal(sa, res["scan"][0][1])
    assert torch.equal(owa, res["chunked"][1][0]) and torch.equal(swa, res["chunked"][1][1])


def test_agrees_with_chunkwise_on_small_workload():
    x = to_device(make_inputs("small"))
    with kda.schedule("scan"):
        o_s, s_s = _fwd(x)
    with kda.schedule("chunked"):
        o_c, s_c = _fwd(x)
    assert o_err(o_s, o_c.double().cpu().numpy()) < TOL_BF16
    assert s_err(s_s, s_c.double().cpu().numpy()) < TOL_BF16


def test_host_buffers_match_device():
    x = make_inputs(WORKLOADS["small"].scaled(T=200))
    with kda.schedule("auto"):
        o_h, s_h = _fwd(x)                # host tensors: the host-buffer entry point
        o_d, s_d = _fwd(to_device(x))
    assert o_h.device.type == "cpu"
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(s_h, s_d.cpu())


def test_unknown_schedule_rejected():
    with pytest.raises(ValueError):
        kda.set_schedule("fastest")
    assert kda.library().kda_set_schedule(3) == 10   # KDA_ERR_VALUE, setting unchanged


def test_variants_without_a_scan_stay_chunkwise():
    """Raw inputs and GDN-2 gates have no column-scan form: with the scan forced they run
    the chunk kernels, bit-identical to the chunkwise schedule."""
    x = to_device(make_inputs(WORKLOADS["small"].scaled(T=70, H=2)))
    a = x["alpha"].float().clamp(1e-30, 1 - 1e-7)
    gl = torch.log((1 - a) / a).to(x["alpha"].dtype)
    bt = x["beta"].float().clamp(1e-7, 1 - 1e-7)
    bl = torch.log(bt / (1 - bt)).to(x["beta"].dtype)
    er = torch.sigmoid(torch.randn(x["k"].shape, generator=torch.Generator().manual_seed(3))).to(x["alpha"].dtype).cuda()
    wr = torch.sigmoid(torch.randn(x["v"].shape, generator=torch.Generator().manual_seed(4))).to(x["alpha"].dtype).cuda()
    res = {}
    for sched in ("scan", "chunked"):
        with kda.schedule(sched):
            raw = kda.forward_raw(x["q"], x["k"], x["v"], gl, bl, initial_state=x["s0"], scale=x["scale"],
                                  check_status=True)
            g2 = kda.forward_gdn2(x["q"], x["k"], x["v"], x["alpha"], er, wr, initial_state=x["s0"],
                                  scale=x["scale"], check_status=True)
        res[sched] = (raw, g2)
    for i in range(2):
        for j in range(2):
            assert torch.equal(res["scan"][i][j], res["chunked"][i][j])
