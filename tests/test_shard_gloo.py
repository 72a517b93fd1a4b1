"""The multi-rank path on CPU: two gloo ranks shard the sequences, run the oracle on
their shard, and the gathered result equals one run over the whole batch; the
timing reduction is a max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_122_b200.shard import max_over_ranks, shard_bounds


def test_shard_bounds_cover_exactly_once():
    for n in (0, 1, 5, 128, 131):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = shard_bounds(n, r, world)
                assert 0 <= a <= b <= n
                seen.extend(range(a, b))
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        shard_bounds(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
        x = make_inputs(WORKLOADS["small"].scaled(B=5, H=2, T=24, dk=16, dv=16))
        a, b = shard_bounds(5, rank, world)
        sl = lambda t: t[a:b]
        o, S = oracle.forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]), sl(x["beta"]),
                              s0=sl(x["s0"]), scale=x["scale"], n_threads=1)
        parts = [None] * world
        dist.all_gather_object(parts, (a, b, o, S))
        t = max_over_ranks([float(rank + 1), 10.0 - rank])
        if rank == 0:
            out.put((parts, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_single_run():
    import oracle
    from gated_delta_rule_122_b200.inputs import WORKLOADS, make_inputs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    parts, t = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = make_inputs(WORKLOADS["small"].scaled(B=5, H=2, T=24, dk=16, dv=16))
    o_ref, s_ref = oracle.forward(x["q"], x["k"], x["v"], x["alpha"], x["beta"], s0=x["s0"],
                                  scale=x["scale"])
    o = np.concatenate([p[2] for p in parts], axis=0)
    S = np.concatenate([p[3] for p in parts], axis=0)
    assert [p[:2] for p in parts] == [(0, 3), (3, 5)]
    assert np.array_equal(o, o_ref) and np.array_equal(S, s_ref)
    assert t == [2.0, 10.0]
