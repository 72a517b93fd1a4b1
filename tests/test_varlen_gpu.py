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
