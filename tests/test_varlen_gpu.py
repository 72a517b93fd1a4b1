"""Packed variable-length prefill (kda_forward_varlen) against the oracle.

Each sequence of the packed batch is checked against the oracle run on its own
rows from its own initial state: the tensor-core path (d = 128, bf16) and the
CUDA-core path (fp32, d = 64), empty and one-token sequences, lengths at a chunk
boundary +-1, agreement with the dense entry point when every length is equal,
rows outside every sequence left untouched, and invalid offsets reported
through the status word.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, TOL_F32, o_err, s_err

pytestmark = pytest.mark.gpu


def _packed(name, lengths, H, seed_offset=0, **over):
    """A packed batch: the workload's draws for one sequence of sum(lengths) tokens, cut
    into the given lengths, plus a seeded initial state per sequence."""
    total = sum(lengths)
    w = WORKLOADS[name].scaled(B=1, H=H, T=max(total, 1), **over)
    x = make_inputs(w, seed=w.seed + seed_offset)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    g = torch.Generator().manual_seed(77 + seed_offset)
    s0 = 0.1 * torch.randn(len(lengths), H, w.dk, w.dv, generator=g)
    p = {n: x[n][0, :total].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
    return p, cu, s0.float(), x["scale"]


def _oracle(p, cu, s0, scale):
    outs, states = [], []
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        sl = lambda t: t[a:b].unsqueeze(0)
        o, S = oracle.forward(sl(p["q"]), sl(p["k"]), sl(p["v"]), sl(p["alpha"]), sl(p["beta"]),
                              s0=s0[i:i + 1], scale=scale)
        outs.append(o[0])
        states.append(S[0])
    return np.concatenate(outs, 0), np.stack(states, 0)


def _run(p, cu, s0, scale, **kw):
    d = {n: t.cuda() for n, t in p.items()}
    return kda.forward_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                              torch.from_numpy(cu).cuda(), initial_state=s0.cuda(), scale=scale, **kw)


@pytest.mark.parametrize("name,lengths", [
    ("prefill", [5, 0, 32, 1, 33, 31, 64, 100]),
    ("long", [200, 17, 96, 0, 65]),
])
def test_varlen_tc_matches_oracle(name, lengths):
    p, cu, s0, scale = _packed(name, lengths, H=3)
    o_ref, s_ref = _oracle(p, cu, s0, scale)
    o, S = _run(p, cu, s0, scale, check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_BF16 and es < TOL_BF16, f"o {eo:.3e} state {es:.3e}"


def test_varlen_simt_matches_oracle():
    lengths = [40, 1, 0, 63, 64, 65, 9]
    p, cu, s0, scale = _packed("small", lengths, H=2, dk=64, dv=64, qkv_dtype=torch.float32)
    o_ref, s_ref = _oracle(p, cu, s0, scale)
    o, S = _run(p, cu, s0, scale, check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < TOL_F32 and es < TOL_F32, f"o {eo:.3e} state {es:.3e}"


def test_varlen_equal_lengths_match_dense():
    B, T, H = 3, 80, 2
    w = WORKLOADS["long"].scaled(B=B, H=H, T=T)
    x = make_inputs(w)
    d = {n: x[n].cuda() for n in ("q", "k", "v", "alpha", "beta")}
    s0 = x["s0"].cuda()
    o_dense, S_dense = kda.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], initial_state=s0,
                                   scale=x["scale"], check_status=True)
    flat = {n: t.reshape(B * T, *t.shape[2:]).contiguous() for n, t in d.items()}
    cu = torch.arange(0, B * T + 1, T, dtype=torch.int32, device="cuda")
    o_var, S_var = kda.forward_varlen(flat["q"], flat["k"], flat["v"], flat["alpha"], flat["beta"], cu,
                                      initial_state=s0, scale=x["scale"], check_status=True)
    assert torch.equal(o_var.reshape(B, T, H, -1), o_dense)
    assert torch.equal(S_var, S_dense)


def test_varlen_leaves_rows_outside_sequences():
    p, cu, s0, scale = _packed("prefill", [20, 45], H=2)
    d = {n: t.cuda() for n, t in p.items()}
    cu_short = torch.tensor([0, 20, 50], dtype=torch.int32, device="cuda")   # rows 50..64 belong to nobody
    out = torch.full((65, 2, 128), 7.0, device="cuda")
    kda.forward_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], cu_short, initial_state=s0.cuda(),
                       scale=scale, out=out, check_status=True)
    assert torch.all(out[50:] == 7.0)
    assert not torch.any(out[:50] == 7.0)


@pytest.mark.parametrize("bad", [[0, 30, 20], [0, 10, 70], [-1, 5, 10]])
def test_varlen_invalid_offsets_reported(bad):
    p, cu, s0, scale = _packed("prefill", [30, 35], H=2)
    d = {n: t.cuda() for n, t in p.items()}
    with pytest.raises(kda.KDAError) as e:
        kda.forward_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                           torch.tensor(bad, dtype=torch.int32, device="cuda"), initial_state=s0.cuda(),
                           scale=scale, check_status=True)
    assert e.value.code == 2   # KDA_ERR_SHAPE


def _packed_extra(name, lengths, H, seed, **over):
    p, cu, s0, scale = _packed(name, lengths, H, **over)
    g = torch.Generator().manual_seed(seed)
    return p, cu, s0, scale, g


@pytest.mark.parametrize("name,lengths,over,tol", [
    ("long", [40, 0, 33, 1, 96, 31], {}, TOL_BF16),                          # tensor cores
    ("small", [20, 0, 33, 5], dict(qkv_dtype=torch.float32), TOL_F32),       # CUDA cores
])
def test_varlen_raw_matches_oracle(name, lengths, over, tol):
    """Raw inputs over packed sequences: rows of q, k rescaled, gate and beta logits whose
    maps give the workload's alpha and beta; each sequence against the oracle's fp64
    preprocessing and recurrence."""
    p, cu, s0, scale, g = _packed_extra(name, lengths, 3, 41, **over)
    cq = torch.exp(torch.randn(*p["q"].shape[:-1], 1, generator=g))
    ck = torch.exp(torch.randn(*p["k"].shape[:-1], 1, generator=g))
    a = p["alpha"].double().clamp(1e-30, 1 - 1e-7)
    bb = p["beta"].double().clamp(1e-7, 1 - 1e-7)
    r = dict(q=(cq * p["q"].float()).to(p["q"].dtype), k=(ck * p["k"].float()).to(p["k"].dtype), v=p["v"],
             x=torch.log((1 - a) / a).to(p["alpha"].dtype), y=torch.log(bb / (1 - bb)).to(p["beta"].dtype))
    outs, states = [], []
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        sl = lambda t: t[lo:hi].unsqueeze(0)
        o_i, S_i = oracle.forward_raw(sl(r["q"]), sl(r["k"]), sl(r["v"]), sl(r["x"]), sl(r["y"]),
                                      s0=s0[i:i + 1], scale=scale)
        outs.append(o_i[0])
        states.append(S_i[0])
    o_ref, s_ref = np.concatenate(outs, 0), np.stack(states, 0)
    c = lambda t: t.cuda()
    o, S = kda.forward_varlen_raw(c(r["q"]), c(r["k"]), c(r["v"]), c(r["x"]), c(r["y"]),
                                  torch.from_numpy(cu).cuda(), initial_state=s0.cuda(), scale=scale,
                                  check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < tol and es < tol, f"o {eo:.3e} state {es:.3e}"


@pytest.mark.parametrize("name,lengths,over,tol", [
    ("long", [50, 0, 32, 1, 100, 7], {}, TOL_BF16),                          # tensor cores
    ("small", [20, 0, 33, 5], dict(qkv_dtype=torch.float32), TOL_F32),       # CUDA cores
])
def test_varlen_gdn2_matches_oracle(name, lengths, over, tol):
    p, cu, s0, scale, g = _packed_extra(name, lengths, 2, 43, **over)
    er = torch.sigmoid(torch.randn(*p["k"].shape, generator=g)).to(p["alpha"].dtype)
    wr = torch.sigmoid(torch.randn(*p["v"].shape, generator=g)).to(p["alpha"].dtype)
    outs, states = [], []
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        sl = lambda t: t[lo:hi].unsqueeze(0)
        o_i, S_i = oracle.forward_gdn2(sl(p["q"]), sl(p["k"]), sl(p["v"]), sl(p["alpha"]), sl(er), sl(wr),
                                       s0=s0[i:i + 1], scale=scale)
        outs.append(o_i[0])
        states.append(S_i[0])
    o_ref, s_ref = np.concatenate(outs, 0), np.stack(states, 0)
    d = {n: t.cuda() for n, t in p.items()}
    o, S = kda.forward_varlen_gdn2(d["q"], d["k"], d["v"], d["alpha"], er.cuda(), wr.cuda(),
                                   torch.from_numpy(cu).cuda(), initial_state=s0.cuda(), scale=scale,
                                   check_status=True)
    eo, es = o_err(o, o_ref), s_err(S, s_ref)
    assert eo < tol and es < tol, f"o {eo:.3e} state {es:.3e}"
