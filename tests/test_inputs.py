"""The seeded generators draw what the workload table states (CPU, small sizes)."""
import torch

from gated_delta_rule_122_b200.inputs import WORKLOADS, make_decode_inputs, make_inputs


def test_prefill_inputs_shapes_dtypes_and_ranges():
    w = WORKLOADS["long"].scaled(T=256, H=8)
    x = make_inputs(w)
    assert x["q"].shape == (1, 256, 8, 128) and x["q"].dtype == torch.bfloat16
    assert x["beta"].shape == (1, 256, 8) and x["s0"].dtype == torch.float32
    qn = x["q"].float().norm(dim=-1)
    assert torch.allclose(qn, torch.ones_like(qn), atol=1e-2)
    a = x["alpha"].float()
    assert (a > 0).all() and (a <= 1).all()
    # strong-forget channels are fixed per (head, channel): mean log-decay splits in two groups
    mean_g = torch.log(a).mean(dim=(0, 1))                 # [H, dk]
    strong = mean_g < -1.0
    frac = strong.float().mean().item()
    assert 0.15 < frac < 0.45
    assert abs(x["s0"].std().item() - 0.1) < 0.01


def test_inputs_are_reproducible():
    w = WORKLOADS["small"].scaled(T=64)
    a, b = make_inputs(w), make_inputs(w)
    for key in ("q", "k", "v", "alpha", "beta", "s0"):
        assert torch.equal(a[key], b[key])
    assert a["alpha"].dtype == torch.float32 and a["q"].dtype == torch.bfloat16


def test_decode_inputs():
    w = WORKLOADS["decode"].scaled(B=4, H=2)
    x = make_decode_inputs(w)
    assert x["state"].shape == (4, 2, 128, 128) and x["q"].shape == (4, 2, 128)
    assert x["beta"].shape == (4, 2)


def test_long_workload_decays_stay_inside_the_anchored_range():
    """The tensor-core prefill computes a chunk token by token when some key channel decays
    by more than 2^-100 over a 16-token half.  The long workload's strong-forget channels
    (about 2.1 nats per token) stay well inside that bound, so its chunks all take the
    tensor-core schedule: the largest 16-token decay is checked on the host."""
    import numpy as np
    x = make_inputs(WORKLOADS["long"].scaled(B=1, H=64, T=4096))
    g = torch.log(x["alpha"].double().clamp_min(1e-300))[0]          # [T, H, d]
    T = g.shape[0]
    halves = g[: T // 16 * 16].reshape(T // 16, 16, *g.shape[1:]).sum(1)
    assert float(halves.min()) > -100 * np.log(2)
