"""The further entry points at full size, in the launch shapes bench.py times, checked on
sampled (sequence, head) pairs against the oracle: scalar gate, raw inputs, packed
sequences and GDN-2 on the prefill workload (B=2, T=8192, H=64, d=128); the
multi-token decode and the state copy on the decode workload (256 x 64 heads).
"""
import itertools

import numpy as np
import pytest
import torch

import gated_delta_rule_122_b200 as kda
import oracle
from gated_delta_rule_122_b200.inputs import make_decode_inputs, make_inputs
from tests.helpers import TOL_BF16, o_err, s_err

pytestmark = pytest.mark.gpu

PAIRS = [(0, 0), (1, 63), (0, 37)]
LENGTHS = [4096, 1000, 3000, 200, 5000, 1084, 1500, 504]   # bench.py's packed layout


def _head(t, b, h):
    """[B,T,H,...] -> the (b, h) slice as a [1,T,1,...] CPU tensor."""
    return t[b:b + 1, :, h:h + 1].cpu()


def _check(o, S, pairs, ref_fn):
    for b, h in pairs:
        o_ref, s_ref = ref_fn(b, h)
        assert o_err(o[b, :, h], o_ref[0, :, 0]) < TOL_BF16, (b, h)
        assert s_err(S[b, h], s_ref[0, 0]) < TOL_BF16, (b, h)


def test_full_size_scalar_gate():
    x = make_inputs("prefill", device="cuda")
    ah = x["alpha"][..., 0].contiguous()
    o, S = kda.forward_scalar_gate(x["q"], x["k"], x["v"], ah, x["beta"], scale=x["scale"], check_status=True)
    torch.cuda.synchronize()

    def ref(b, h):
        a = ah[b:b + 1, :, h:h + 1].cpu().unsqueeze(-1).expand(1, -1, 1, 128)
        return oracle.forward(_head(x["q"], b, h), _head(x["k"], b, h), _head(x["v"], b, h), a,
                              _head(x["beta"], b, h), scale=x["scale"])
    _check(o, S, PAIRS, ref)


def test_full_size_raw_inputs():
    x = make_inputs("prefill", device="cuda")
    g = torch.Generator(device="cuda").manual_seed(3)
    q = (x["q"].float() * torch.exp(torch.randn(*x["q"].shape[:-1], 1, generator=g, device="cuda"))).bfloat16()
    k = (x["k"].float() * torch.exp(torch.randn(*x["k"].shape[:-1], 1, generator=g, device="cuda"))).bfloat16()
    a = x["alpha"].double().clamp(1e-30, 1 - 1e-7)
    bt = x["beta"].double().clamp(1e-7, 1 - 1e-7)
    gl, bl = torch.log((1 - a) / a).bfloat16(), torch.log(bt / (1 - bt)).bfloat16()
    del a, bt
    o, S = kda.forward_raw(q, k, x["v"], gl, bl, scale=x["scale"], check_status=True)
    torch.cuda.synchronize()
    _check(o, S, PAIRS, lambda b, h: oracle.forward_raw(_head(q, b, h), _head(k, b, h), _head(x["v"], b, h),
                                                        _head(gl, b, h), _head(bl, b, h), scale=x["scale"]))


def test_full_size_packed_sequences():
    x = make_inputs("prefill", device="cuda")
    B, T, H = 2, 8192, 64
    flat = {n: x[n].reshape(B * T, *x[n].shape[2:]) for n in ("q", "k", "v", "alpha", "beta")}
    starts = [0] + list(itertools.accumulate(LENGTHS))
    cu = torch.tensor(starts, dtype=torch.int32, device="cuda")
    o, S = kda.forward_varlen(flat["q"], flat["k"], flat["v"], flat["alpha"], flat["beta"], cu,
                              scale=x["scale"], check_status=True)
    torch.cuda.synchronize()
    for i, h in [(0, 0), (4, 63), (3, 10), (7, 5), (1, 31)]:
        a, e = starts[i], starts[i + 1]
        sl = lambda t: t[a:e, h:h + 1].unsqueeze(0).cpu()
        o_ref, s_ref = oracle.forward(sl(flat["q"]), sl(flat["k"]), sl(flat["v"]), sl(flat["alpha"]),
                                      sl(flat["beta"]), scale=x["scale"])
        assert o_err(o[a:e, h], o_ref[0, :, 0]) < TOL_BF16, (i, h)
        assert s_err(S[i, h], s_ref[0, 0]) < TOL_BF16, (i, h)


def test_full_size_gdn2():
    x = make_inputs("prefill", device="cuda")
    g = torch.Generator(device="cuda").manual_seed(7)
    er = torch.sigmoid(torch.randn(x["k"].shape, generator=g, device="cuda")).bfloat16()
    wr = torch.sigmoid(torch.randn(x["v"].shape, generator=g, device="cuda")).bfloat16()
    o, S = kda.forward_gdn2(x["q"], x["k"], x["v"], x["alpha"], er, wr, scale=x["scale"], check_status=True)
    torch.cuda.synchronize()
    _check(o, S, PAIRS[:2], lambda b, h: oracle.forward_gdn2(
        _head(x["q"], b, h), _head(x["k"], b, h), _head(x["v"], b, h), _head(x["alpha"], b, h),
        _head(er, b, h), _head(wr, b, h), scale=x["scale"]))


def test_full_size_decode_tokens_and_rollback():
    y = make_decode_inputs("decode", device="cuda")
    N, H, d, Td = 256, 64, 128, 4
    g = torch.Generator(device="cuda").manual_seed(11)
    # four draft tokens per sequence: the decode token and three more from the same recipe
    more = make_decode_inputs("decode", device="cuda", seed=4242)
    draft = {}
    for n in ("q", "k", "v", "alpha", "beta"):
        perm = [y[n]] + [more[n][torch.randperm(N, generator=g, device="cuda")] for _ in range(Td - 1)]
        draft[n] = torch.stack(perm, 1).contiguous()
    del more
    s0 = y["state"].clone()
    ts = torch.empty((N, Td, H, d, d), device="cuda")
    o, _ = kda.decode_tokens(draft["q"], draft["k"], draft["v"], draft["alpha"], draft["beta"], y["state"],
                             commit=False, token_states=ts, scale=y["scale"], check_status=True)
    torch.cuda.synchronize()
    assert torch.equal(y["state"], s0)
    accepted = torch.randint(0, Td + 1, (N,), generator=g, device="cuda")
    src = torch.where(accepted > 0, torch.arange(N, device="cuda") * Td + accepted - 1,
                      torch.full_like(accepted, -1)).to(torch.int32)
    kda.state_copy(ts.view(N * Td, H, d, d), y["state"], src_index=src,
                   dst_index=torch.arange(N, dtype=torch.int32, device="cuda"), check_status=True)
    acc = accepted.cpu().numpy()
    for n, h in [(0, 0), (255, 63), (17, 5), (128, 40)]:
        sl = lambda t: t[n:n + 1, :, h:h + 1].cpu()
        s_in = s0[n:n + 1, h:h + 1].cpu()
        o_ref, _ = oracle.forward(sl(draft["q"]), sl(draft["k"]), sl(draft["v"]), sl(draft["alpha"]),
                                  sl(draft["beta"]), s0=s_in, scale=y["scale"])
        ts_ref = oracle.token_states(sl(draft["q"]), sl(draft["k"]), sl(draft["v"]), sl(draft["alpha"]),
                                     sl(draft["beta"]), s0=s_in, scale=y["scale"])
        assert o_err(o[n, :, h], o_ref[0, :, 0]) < TOL_BF16, (n, h)
        assert s_err(ts[n, :, h], ts_ref[0, :, 0]) < TOL_BF16, (n, h)
        want = s_in[0, 0].double().numpy() if acc[n] == 0 else ts_ref[0, acc[n] - 1, 0]
        assert s_err(y["state"][n, h], want) < TOL_BF16, (n, h, int(acc[n]))


def test_full_size_state_copy_is_exact():
    y = make_decode_inputs("decode", device="cuda")
    N = y["state"].shape[0]
    g = torch.Generator(device="cuda").manual_seed(5)
    src = torch.randperm(N, generator=g, device="cuda").to(torch.int32)
    src[::7] = -1
    pool = torch.zeros_like(y["state"])
    kda.state_copy(y["state"], pool, src_index=src, dst_index=torch.arange(N, dtype=torch.int32, device="cuda"),
                   check_status=True)
    keep = (src >= 0).cpu().numpy()
    idx = np.nonzero(keep)[0]
    assert torch.equal(pool[idx], y["state"][src[idx].long()])
    assert torch.all(pool[np.nonzero(~keep)[0]] == 0)
