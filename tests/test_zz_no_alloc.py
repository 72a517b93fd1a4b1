"""kda_forward_noalloc: the prefill entry point for callers that cannot allocate.

Some callers have no way to allocate device memory (an allocator-less runtime,
a plugin that must not touch its host process's memory pool), so they cannot
pass kda_forward its workspace.  kda_forward_noalloc takes only inputs and
outputs and uses a fixed scratch array owned by the library; kda_noalloc_status
reads the status word the kernel leaves in that array.  This test calls both
through the C ABI, twice in a row, and checks each result element by element
against the fp64 oracle on the same inputs, within the bf16-input tolerance of
the parity tests, and that the status reads KDA_OK after each call.  It lives in
its own file, collected last.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_122_b200 as kda
from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
from tests.helpers import TOL_BF16, o_err, oracle_full, s_err

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
def test_noalloc_matches_oracle_twice(name):
    lib = kda.library()
    x = make_inputs(WORKLOADS[name].scaled(B=2, H=3, T=200), device="cuda")
    ref_o, ref_s = oracle_full(x)
    w = x["workload"]
    for _ in range(2):
        o = torch.full((w.B, w.T, w.H, w.dv), float("nan"), device="cuda")
        S = torch.full((w.B, w.H, w.dk, w.dv), float("nan"), device="cuda")
        assert _noalloc(lib, x, o, S) == 0
        assert lib.kda_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        assert o_err(o, ref_o) < TOL_BF16 and s_err(S, ref_s) < TOL_BF16
