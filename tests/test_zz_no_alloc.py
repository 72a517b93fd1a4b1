"""kda_forward_noalloc: the prefill entry point for callers that cannot allocate.

Some callers have no way to allocate device memory (an allocator-less runtime,
a plugin that must not touch its host process's memory pool), so they cannot
pass kda_forward its workspace.  kda_forward_noalloc takes only inputs and
outputs and uses a fixed scratch array owned by the library.  This test calls it
through the C ABI twice in a row and checks each result against kda_forward's on
the same inputs, within the bf16-input tolerance of the parity tests.  It lives
in its own file, collected last.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_122_b200 as kda
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, o_err, s_err

pytestmark = pytest.mark.gpu


def _noalloc(lib, x, o, S):
    vp = ctypes.c_void_p
    w = x["workload"]
    return lib.kda_forward_noalloc(
        vp(x["q"].data_ptr()), vp(x["k"].data_ptr()), vp(x["v"].data_ptr()),
        vp(x["alpha"].data_ptr()), vp(x["beta"].data_ptr()),
        None if x["s0"] is None else vp(x["s0"].data_ptr()), vp(o.data_ptr()), vp(S.data_ptr()),
        w.B, w.T, w.H, w.dk, w.dv, float(x["scale"]), 1, 1, 0,
        vp(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name", ["long", "prefill"])
def test_noalloc_matches_forward_twice(name):
    lib = kda.library()
    x = make_inputs(WORKLOADS[name].scaled(B=2, H=3, T=200), device="cuda")
    o_ref, s_ref = kda.forward(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                               initial_state=x["s0"], scale=x["scale"])
    ref_o, ref_s = o_ref.double().cpu().numpy(), s_ref.double().cpu().numpy()
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(s_ref, float("nan"))
        assert _noalloc(lib, x, o, S) == 0
        torch.cuda.synchronize()
        assert o_err(o, ref_o) < TOL_BF16 and s_err(S, ref_s) < TOL_BF16
