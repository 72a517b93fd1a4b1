"""Serving operations on the GPU: multi-token decode over a slot pool, per-token states,
speculative rollback and whole-state copies, against the oracle.

"Module 03 -- KDA I: The Delta-Rule Recurrence", section 5 "State vs. checkpoint
weights": a state is request-scoped, cached per slot, and copied or restored on a
fork or a speculative rollback.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, TOL_F32, o_err, s_err

pytestmark = pytest.mark.gpu


def _draft(N, T, H, dk=128, dv=128, seed_offset=0, **over):
    """T tokens for each of N sequences (the decode workload's recipe), [N,T,H,d]."""
    w = WORKLOADS["decode"].scaled(B=N, T=T, H=H, dk=dk, dv=dv, decode=False, init_state=False, **over)
    x = make_inputs(w, seed=w.seed + seed_offset)
    g = torch.Generator().manual_seed(91 + seed_offset)
    s0 = 0.1 * torch.randn(N, H, dk, dv, generator=g)
    return x, s0.float()


def _args(x):
    return [x[n].cuda() for n in ("q", "k", "v", "alpha", "beta")]


@pytest.mark.parametrize("T,dk,dv,over,tol", [
    (4, 128, 128, {}, TOL_BF16),
    (1, 128, 128, {}, TOL_BF16),
    (7, 64, 32, dict(qkv_dtype=torch.float32, gate_dtype=torch.float32), TOL_F32),
])
def test_decode_tokens_matches_oracle(T, dk, dv, over, tol):
    x, s0 = _draft(5, T, 3, dk, dv, **over)
    pool = s0.cuda().clone()
    o, ts = kda.decode_tokens(*_args(x), pool, token_states=True, scale=x["scale"], check_status=True)
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], s0=s0, scale=x["scale"])
    ts_ref = oracle.token_states(x["q"], x["k"], x["v"], x["alpha"], x["beta"], s0=s0, scale=x["scale"])
    eo, es, et = o_err(o, o_ref), s_err(pool, s_ref), s_err(ts, ts_ref)
    assert eo < tol and es < tol and et < tol, f"o {eo:.3e} state {es:.3e} token states {et:.3e}"
    assert torch.equal(ts[:, -1], pool)


def test_decode_tokens_equals_sequential_schedule():
    # the same kernel as the token-by-token prefill: identical bits
    x, s0 = _draft(4, 5, 2)
    pool = s0.cuda().clone()
    o, _ = kda.decode_tokens(*_args(x), pool, scale=x["scale"])
    o2, s2 = kda.forward_sequential(*_args(x), initial_state=s0.cuda(), scale=x["scale"])
    assert torch.equal(o, o2) and torch.equal(pool, s2)


def test_decode_tokens_without_commit_leaves_pool():
    x, s0 = _draft(3, 4, 2)
    pool = s0.cuda().clone()
    o1, ts = kda.decode_tokens(*_args(x), pool, commit=False, token_states=True, scale=x["scale"])
    assert torch.equal(pool, s0.cuda())
    o2, _ = kda.decode_tokens(*_args(x), pool, commit=True, scale=x["scale"])
    assert torch.equal(o1, o2) and torch.equal(ts[:, -1], pool)


def test_decode_tokens_slot_pool():
    N, T, H, slots = 4, 3, 2, 9
    x, s0 = _draft(N, T, H, seed_offset=1)
    g = torch.Generator().manual_seed(5)
    pool0 = 0.1 * torch.randn(slots, H, 128, 128, generator=g)
    slot_of = [7, 2, -1, 5]                       # sequence 2 is padding
    for n, s in enumerate(slot_of):
        if s >= 0:
            pool0[s] = s0[n]
    pool = pool0.cuda().clone()
    out = torch.full((N, T, H, 128), 3.0, device="cuda")
    kda.decode_tokens(*_args(x), pool, state_slots=torch.tensor(slot_of, dtype=torch.int32, device="cuda"),
                      out=out, scale=x["scale"], check_status=True)
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], s0=s0, scale=x["scale"])
    live = [n for n, s in enumerate(slot_of) if s >= 0]
    assert o_err(out[live], o_ref[live]) < TOL_BF16
    assert s_err(pool[[slot_of[n] for n in live]], s_ref[live]) < TOL_BF16
    assert torch.all(out[2] == 3.0)
    untouched = [s for s in range(slots) if s not in slot_of]
    assert torch.equal(pool[untouched], pool0[untouched].cuda())


def test_decode_tokens_slot_out_of_range_reported():
    x, s0 = _draft(2, 2, 2)
    pool = s0.cuda().clone()
    with pytest.raises(kda.KDAError) as e:
        kda.decode_tokens(*_args(x), pool, state_slots=torch.tensor([1, 2], dtype=torch.int32, device="cuda"),
                          scale=x["scale"], check_status=True)
    assert e.value.code == 2   # KDA_ERR_SHAPE
    assert torch.equal(pool[0], s0[0].cuda())


def test_speculative_rollback():
    # verify T draft tokens without committing, accept a prefix per sequence, roll the
    # pool forward to the state after the last accepted token
    N, T, H = 5, 4, 2
    x, s0 = _draft(N, T, H, seed_offset=2)
    pool = s0.cuda().clone()
    _, ts = kda.decode_tokens(*_args(x), pool, commit=False, token_states=True, scale=x["scale"])
    accepted = [0, 1, 4, 2, 3]
    src = torch.tensor([n * T + a - 1 if a > 0 else -1 for n, a in enumerate(accepted)],
                       dtype=torch.int32, device="cuda")
    kda.state_copy(ts.view(N * T, H, 128, 128), pool, src_index=src,
                   dst_index=torch.arange(N, dtype=torch.int32, device="cuda"), check_status=True)
    for n, a in enumerate(accepted):
        sl = lambda t: t[n:n + 1, :a]
        _, s_ref = oracle.forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]), sl(x["beta"]),
                                  s0=s0[n:n + 1], scale=x["scale"])
        assert s_err(pool[n:n + 1], s_ref) < TOL_BF16, n
    assert torch.equal(pool[0], s0[0].cuda())


@pytest.mark.parametrize("H,dk,dv", [(64, 128, 128), (3, 16, 32)])
def test_state_copy_matches_oracle(H, dk, dv):
    g = torch.Generator().manual_seed(H)
    src = torch.randn(6, H, dk, dv, generator=g)
    dst = torch.randn(5, H, dk, dv, generator=g)
    si, di = [5, 0, -1, 3, 2], [1, 4, 0, 0, 2]
    d_gpu = dst.cuda()
    kda.state_copy(src.cuda(), d_gpu, src_index=torch.tensor(si, dtype=torch.int32, device="cuda"),
                   dst_index=torch.tensor(di, dtype=torch.int32, device="cuda"), check_status=True)
    ref, bad = oracle.state_copy(src.numpy(), dst.numpy(), si, di)
    assert not bad and np.array_equal(d_gpu.cpu().numpy(), ref.astype(np.float32))


def test_state_copy_fork_in_one_pool_and_identity():
    pool = torch.randn(4, 2, 64, 64, device="cuda")
    before = pool.clone()
    kda.state_copy(pool, pool, src_index=torch.tensor([0, 1], dtype=torch.int32, device="cuda"),
                   dst_index=torch.tensor([3, 2], dtype=torch.int32, device="cuda"))
    assert torch.equal(pool[3], before[0]) and torch.equal(pool[2], before[1])
    assert torch.equal(pool[:2], before[:2])
    other = torch.zeros(3, 2, 64, 64, device="cuda")
    kda.state_copy(pool, other)                   # identity index over min(slots)
    assert torch.equal(other, pool[:3])


def test_state_copy_index_out_of_range_reported():
    src = torch.randn(2, 1, 16, 16, device="cuda")
    dst = torch.zeros(2, 1, 16, 16, device="cuda")
    with pytest.raises(kda.KDAError) as e:
        kda.state_copy(src, dst, src_index=torch.tensor([0, 2], dtype=torch.int32, device="cuda"),
                       dst_index=torch.tensor([1, 0], dtype=torch.int32, device="cuda"), check_status=True)
    assert e.value.code == 2
    assert torch.equal(dst[1], src[0]) and torch.all(dst[0] == 0)
