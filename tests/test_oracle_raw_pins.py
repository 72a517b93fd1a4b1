"""Pins of the oracle's input preprocessing (normalised q and k, gate and beta logits).

"Notes on Linear Attention" section 5.3: with a unit key the read-back after a
write interpolates exactly between the old prediction and the target, so the key
is L2-normalised (section 3: the query likewise).  "Kimi Delta Attention (KDA)":
the log-decay g = log alpha <= 0 is what is stored; the workloads' gate is
alpha = exp(-softplus(x)).  "From Fast Weight Programmers to KDA": beta = sigmoid
of a projection.
"""
import numpy as np

import oracle


def _rand(B, T, H, dk, dv, seed):
    r = np.random.default_rng(seed)
    return (3.0 * r.standard_normal((B, T, H, dk)), 0.5 * r.standard_normal((B, T, H, dk)),
            r.standard_normal((B, T, H, dv)), r.standard_normal((B, T, H, dk)), r.standard_normal((B, T, H)),
            0.1 * r.standard_normal((B, H, dk, dv)))


def test_logit_maps_at_known_points():
    # softplus(0) = log 2 -> alpha = 1/2; sigmoid(0) = 1/2; softplus(log 3) = log 4 -> alpha = 1/4;
    # sigmoid(log 3) = 3/4; large logits saturate without overflow
    x = np.array([0.0, np.log(3.0), -np.log(3.0), 800.0, -800.0]).reshape(1, 1, 1, 5)
    y = np.array([0.0, np.log(3.0), 800.0, -800.0]).reshape(1, 1, 4)
    _, _, alpha, beta = oracle.preprocess(np.ones((1, 1, 1, 5)), np.ones((1, 1, 1, 5)), x, y)
    assert np.allclose(alpha.ravel(), [0.5, 0.25, 0.75, 0.0, 1.0], rtol=1e-15, atol=0)
    assert np.allclose(beta.ravel(), [0.5, 0.75, 1.0, 0.0], rtol=1e-15, atol=0)


def test_rows_become_unit_and_zero_rows_stay_zero():
    q = np.array([[3.0, 4.0], [0.0, 0.0]]).reshape(1, 2, 1, 2)
    qn, kn, _, _ = oracle.preprocess(q, 2 * q, np.zeros((1, 2, 1, 2)), np.zeros((1, 2, 1)))
    assert np.array_equal(qn.reshape(2, 2), [[0.6, 0.8], [0.0, 0.0]])
    assert np.array_equal(kn, qn)


def test_raw_equals_forward_on_preprocessed_values():
    # with unit rows and the logits that invert the maps, forward_raw is forward
    q, k, v, _, _, s0 = _rand(1, 19, 2, 8, 4, 1)
    r = np.random.default_rng(2)
    alpha, beta = r.uniform(0.05, 0.95, (1, 19, 2, 8)), r.uniform(0.05, 0.95, (1, 19, 2))
    x, y = np.log((1 - alpha) / alpha), np.log(beta / (1 - beta))    # softplus^-1(-log alpha), logit(beta)
    qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
    kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
    o1, s1 = oracle.forward_raw(q, k, v, x, y, s0=s0)
    o2, s2 = oracle.forward(qn, kn, v, alpha, beta, s0=s0)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(s1, s2, rtol=0, atol=1e-12)


def test_raw_is_invariant_to_row_scaling():
    # positive per-token scalings of q and k do not change the result (normalisation
    # is applied); dropping it would change o by the scale factors
    q, k, v, x, y, s0 = _rand(2, 11, 1, 6, 5, 3)
    r = np.random.default_rng(4)
    cq, ck = r.uniform(0.1, 10, (2, 11, 1, 1)), r.uniform(0.1, 10, (2, 11, 1, 1))
    o1, s1 = oracle.forward_raw(q, k, v, x, y, s0=s0)
    o2, s2 = oracle.forward_raw(cq * q, ck * k, v, x, y, s0=s0)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(s1, s2, rtol=0, atol=1e-12)


def test_unit_key_full_write_reads_back_v():
    # beta -> 1 (large logit), a raw key of any length: reading S_t with k_t/||k_t|| gives v_t
    q, k, v, x, _, s0 = _rand(1, 1, 1, 6, 3, 5)
    _, S = oracle.forward_raw(q, k, v, x, np.full((1, 1, 1), 800.0), s0=s0)
    kn = k[0, 0, 0] / np.linalg.norm(k[0, 0, 0])
    assert np.allclose(S[0, 0].T @ kn, v[0, 0, 0], rtol=0, atol=1e-12)
