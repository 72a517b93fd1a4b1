"""Pins of the GDN-2 oracle (decoupled erase and write gates) to facts the pages fix.

"From Fast Weight Programmers to KDA" (jonahsamost.bearblog.dev), section
"Gated DeltaNet-2": decay the state, retrieve through the gated key b_t * k_t,
write the residual w_t * v_t - vh at the original key k_t; b_t = beta_t 1 and
w_t = beta_t 1 collapse it back to KDA.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def _rand(B, T, H, dk, dv, seed):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))
    a = np.exp(-0.1 * np.log1p(np.exp(r.standard_normal((B, T, H, dk)))))
    s0 = 0.1 * r.standard_normal((B, H, dk, dv))
    return q, k, v, a, s0, r


def test_gdn2_single_step_by_hand():
    # S0 = [[2, 0], [0, 4]] (rows = key channels), k = [1, 0], alpha = 1,
    # b = [0.5, 0.9], w = [1, 0.5], v = [4, 2], q = [1, 1], scale 1:
    #   vh = S0^T (b * k) = S0^T [0.5, 0] = [1, 0]
    #   e  = w * v - vh = [4, 1] - [1, 0] = [3, 1]
    #   S  = S0 + k e^T = [[5, 1], [0, 4]];   o = S^T q = [5, 5]
    f = lambda *x: np.array(x, dtype=np.float64).reshape(1, 1, 1, -1)
    o, S = oracle.forward_gdn2(f(1, 1), f(1, 0), f(4, 2), f(1, 1), f(0.5, 0.9), f(1, 0.5),
                               s0=np.array([[2.0, 0.0], [0.0, 4.0]]).reshape(1, 1, 2, 2), scale=1.0)
    assert np.array_equal(o.ravel(), [5.0, 5.0])
    assert np.array_equal(S.reshape(2, 2), [[5.0, 1.0], [0.0, 4.0]])


def test_gdn2_collapses_to_kda():
    q, k, v, a, s0, r = _rand(2, 37, 3, 16, 8, 1)
    beta = r.uniform(0, 1, (2, 37, 3))
    b = np.repeat(beta[..., None], 16, axis=-1)
    w = np.repeat(beta[..., None], 8, axis=-1)
    o1, s1 = oracle.forward_gdn2(q, k, v, a, b, w, s0=s0)
    o2, s2 = oracle.forward(q, k, v, a, beta, s0=s0)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(s1, s2, rtol=0, atol=1e-12)


def test_gdn2_no_erase_is_additive_write():
    # b = 0: nothing is retrieved, S_t = Diag(alpha) S + k (w * v)^T, which is KDA's
    # correction-dropped mode with beta folded into v when w = beta 1
    q, k, v, a, s0, r = _rand(1, 29, 2, 8, 8, 2)
    beta = r.uniform(0, 1, (1, 29, 2))
    o1, s1 = oracle.forward_gdn2(q, k, v, a, np.zeros_like(k), np.repeat(beta[..., None], 8, axis=-1), s0=s0)
    o2, s2 = oracle.forward(q, k, v, a, beta, s0=s0, mode="drop_correction")
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(s1, s2, rtol=0, atol=1e-12)


def test_gdn2_write_is_local_to_the_key():
    # the update is stored at k_t: any x orthogonal to k_t reads the decayed state unchanged
    q, k, v, a, s0, r = _rand(1, 1, 1, 6, 5, 3)
    b, w = r.uniform(0, 1, (1, 1, 1, 6)), r.uniform(0, 1, (1, 1, 1, 5))
    _, S = oracle.forward_gdn2(q, k, v, a, b, w, s0=s0)
    x = r.standard_normal(6)
    x -= (x @ k[0, 0, 0]) * k[0, 0, 0]
    S_dec = a[0, 0, 0][:, None] * s0[0, 0]
    assert np.allclose(S[0, 0].T @ x, S_dec.T @ x, rtol=0, atol=1e-12)


def test_gdn2_full_erase_overwrites():
    # b = w = 1 and a unit key: the new state reads back exactly v at k
    q, k, v, a, s0, r = _rand(1, 1, 2, 8, 4, 4)
    _, S = oracle.forward_gdn2(q, k, v, a, np.ones_like(k), np.ones_like(v), s0=s0)
    for h in range(2):
        assert np.allclose(S[0, h].T @ k[0, 0, h], v[0, 0, h], rtol=0, atol=1e-12)


def test_gdn2_decoupled_gates_matter():
    # a strong erase with a weak write differs from the tied gate at the same beta
    q, k, v, a, s0, r = _rand(1, 16, 1, 8, 8, 5)
    o1, _ = oracle.forward_gdn2(q, k, v, a, np.full_like(k, 0.9), np.full_like(v, 0.1), s0=s0)
    o2, _ = oracle.forward_gdn2(q, k, v, a, np.full_like(k, 0.5), np.full_like(v, 0.5), s0=s0)
    assert np.abs(o1 - o2).max() > 1e-3


@pytest.mark.parametrize("T,chunk", [(37, 8), (64, 32), (5, 16)])
def test_gdn2_chunked_schedule_matches_sequential(T, chunk):
    # the chunked form the CUDA-core kernel follows reaches the sequential recurrence
    from oracle.chunked import forward_chunked_gdn2
    q, k, v, a, s0, r = _rand(2, T, 2, 8, 6, 6)
    b, w = r.uniform(0, 1, (2, T, 2, 8)), r.uniform(0, 1, (2, T, 2, 6))
    o1, s1 = oracle.forward_gdn2(q, k, v, a, b, w, s0=s0)
    o2, s2 = forward_chunked_gdn2(q, k, v, a, b, w, s0=s0, chunk=chunk)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(s1, s2, rtol=0, atol=1e-12)
