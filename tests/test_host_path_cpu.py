"""Argument checks of the pipelined host-buffer prefill, which run before any device is
touched (so they are testable without a GPU)."""
import pytest
import torch

import gated_delta_rule_122_b200 as kda

T = 2048   # two 1024-token segments: the pipelined host path


def _host(B=1, H=2, d=16, T=T):
    q = torch.zeros(B, T, H, d)
    return q, q.clone(), torch.zeros(B, T, H, d), torch.ones(B, T, H, d), torch.zeros(B, T, H)


def test_mismatched_key_shape_raises():
    q, k, v, a, b = _host()
    with pytest.raises(ValueError, match="shapes"):
        kda.forward(q, k[:, :-1].contiguous(), v, a, b)


def test_per_head_gate_shape_checked():
    q, k, v, a, b = _host()
    with pytest.raises(ValueError, match=r"alpha \[B,T,H\]"):
        kda.forward_scalar_gate(q, k, v, a, b)   # a per-channel alpha given to the per-head entry


def test_mixed_host_and_device_arguments_rejected():
    q, k, v, a, b = _host()
    with pytest.raises(ValueError, match="host tensor"):
        kda.forward(q, k, v, a, b, out=torch.empty(1, T, 2, 16, device="meta"))


def test_output_shape_checked():
    q, k, v, a, b = _host()
    with pytest.raises(ValueError, match=r"out must be \[B,T,H,dv\]"):
        kda.forward(q, k, v, a, b, out=torch.empty(1, T, 2, 8))
