"""Pins of the serving-side oracle functions: per-token states and whole-state copies.

"Module 03 -- KDA I: The Delta-Rule Recurrence", section 5 "State vs. checkpoint
weights": a state belongs to a sequence prefix, so the state after token t must be
the exact point from which the rest of the sequence continues, and a copied state
must continue exactly like the original.  Section 4 fixes the one-step values.
"""
import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(B, T, H, dk, dv, seed):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))
    a = np.exp(-np.log1p(np.exp(r.standard_normal((B, T, H, dk)))))
    beta = 1 / (1 + np.exp(-r.standard_normal((B, T, H))))
    s0 = 0.1 * r.standard_normal((B, H, dk, dv))
    return q, k, v, a, beta, s0


def test_token_states_first_token_is_the_worked_example():
    with open(os.path.join(GOLDEN, "module03_worked_example.json")) as f:
        g = json.load(f)
    sh = lambda x, *s: np.asarray(x, dtype=np.float64).reshape(*s)
    dk, dv = len(g["k"]), len(g["v"])
    ts = oracle.token_states(np.ones((1, 1, 1, dk)), sh(g["k"], 1, 1, 1, dk), sh(g["v"], 1, 1, 1, dv),
                             np.broadcast_to(sh(g["alpha"], -1), (dk,)).reshape(1, 1, 1, dk),
                             sh(g["beta"], 1, 1, 1), s0=sh(g["S_prev"], 1, 1, dk, dv), scale=1.0)
    assert np.array_equal(ts[0, 0, 0], sh(g["expected_S"], dk, dv))


def test_token_states_are_continuation_points():
    # continuing from the state after token t over tokens t+1.. gives the full run,
    # for every t: an off-by-one in the prefix cut fails this
    q, k, v, a, beta, s0 = _rand(2, 7, 2, 6, 5, 1)
    ts = oracle.token_states(q, k, v, a, beta, s0=s0)
    o_full, s_full = oracle.forward(q, k, v, a, beta, s0=s0)
    for t in range(6):
        sl = lambda x: x[:, t + 1:]
        o_rest, s_rest = oracle.forward(sl(q), sl(k), sl(v), sl(a), sl(beta), s0=ts[:, t])
        assert np.allclose(s_rest, s_full, rtol=0, atol=1e-12)
        assert np.allclose(o_rest, o_full[:, t + 1:], rtol=0, atol=1e-12)
    assert np.allclose(ts[:, -1], s_full, rtol=0, atol=1e-13)


def test_token_states_move_only_along_the_key():
    # between consecutive tokens the decayed state changes only along k_t (the locality
    # of the delta write, section 2): x orthogonal to k_t reads D_t S_{t-1} unchanged
    q, k, v, a, beta, s0 = _rand(1, 5, 1, 6, 4, 2)
    ts = oracle.token_states(q, k, v, a, beta, s0=s0)
    prev = s0[0, 0]
    r = np.random.default_rng(3)
    for t in range(5):
        kt = k[0, t, 0]
        x = r.standard_normal(6)
        x -= (x @ kt) * kt
        dec = a[0, t, 0][:, None] * prev
        assert np.allclose(ts[0, t, 0].T @ x, dec.T @ x, rtol=0, atol=1e-12)
        prev = ts[0, t, 0]


def test_state_copy_by_hand():
    src = np.arange(4 * 2, dtype=np.float64).reshape(4, 1, 1, 2)     # slot s holds [2s, 2s+1]
    dst = -np.ones((3, 1, 1, 2))
    new, bad = oracle.state_copy(src, dst, src_index=[3, -1, 0, 9], dst_index=[0, 1, 2, 1])
    assert not np.shares_memory(new, dst)
    assert new[:, 0, 0].tolist() == [[6, 7], [-1, -1], [0, 1]] and bad


def test_copied_state_continues_like_the_original():
    # a fork: the copy, fed the same tokens, reaches the same state as the original
    q, k, v, a, beta, s0 = _rand(1, 6, 2, 4, 4, 4)
    pool = np.zeros((3, 2, 4, 4))
    pool[2] = s0[0]
    pool, bad = oracle.state_copy(pool, pool, src_index=[2], dst_index=[0])
    assert not bad
    _, s_a = oracle.forward(q, k, v, a, beta, s0=pool[2:3])
    _, s_b = oracle.forward(q, k, v, a, beta, s0=pool[0:1])
    assert np.array_equal(s_a, s_b)
