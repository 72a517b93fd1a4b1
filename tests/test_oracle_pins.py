"""Pins for the fp64 oracle: values and identities the pages fix.

Each test checks the oracle against something other than itself -- a printed
worked example, a closed form, an invariant, or an independent restatement of a
special case -- and the planted-mistake tests show that a plausible error in the
recurrence (wrong operator order, predicting before forgetting, a dropped
correction) fails those pins.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.chunked import forward_chunked

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_inputs(rng, B, T, H, dk, dv, unit=True, s0=True, alpha_lo=0.3):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(alpha_lo, 1.0, (B, T, H, dk))
    beta = rng.uniform(0.0, 1.0, (B, T, H))
    S0 = 0.3 * rng.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, alpha, beta, S0


def _one_step(S_prev, k, v, beta, alpha, q=None, scale=1.0, mode="exact"):
    dk, dv = S_prev.shape
    q = np.zeros(dk) if q is None else np.asarray(q, dtype=float)
    o, S = oracle.forward(q.reshape(1, 1, 1, dk), np.reshape(k, (1, 1, 1, dk)),
                          np.reshape(v, (1, 1, 1, dv)), np.reshape(alpha, (1, 1, 1, dk)),
                          np.full((1, 1, 1), beta), s0=np.reshape(S_prev, (1, 1, dk, dv)),
                          scale=scale, mode=mode)
    return o[0, 0, 0], S[0, 0]


# --- Module 03, section 4: the worked example, exactly --------------------------------
def test_module03_worked_example_exact():
    g = _load("module03_worked_example.json")
    q = np.array([1.0, 0.0])
    o, S = _one_step(np.array(g["S_prev"]), g["k"], g["v"], g["beta"], g["alpha"], q=q)
    assert np.array_equal(S, np.array(g["expected_S"]))
    # o = S_t^T q for q = e_0 is the first row of S_t
    assert np.array_equal(o, np.array(g["expected_S"])[0])
    # the internal prediction and error of the page: S_t = S + beta k e^T
    S_prev = np.array(g["S_prev"])
    k = np.array(g["k"])
    assert np.array_equal(S_prev.T @ k, np.array(g["expected_prediction"]))
    e = np.array(g["v"]) - S_prev.T @ k
    assert np.array_equal(e, np.array(g["expected_error"]))


# --- Notes on Linear Attention, section 11: two orthogonal keys ------------------------
def test_two_dim_orthogonal_example():
    g = _load("two_dim_orthogonal_keys.json")
    ka, kb = np.array(g["k_a"]), np.array(g["k_b"])
    v1, v2, vb = (np.array(g[x]) for x in ("v1", "v2", "vb"))
    Z = np.zeros((2, 3))
    one = np.ones(2)
    # additive memory (correction dropped, alpha = beta = 1): row a accumulates
    _, S = _one_step(Z, ka, v1, 1.0, one, mode="drop_correction")
    _, S = _one_step(S, ka, v2, 1.0, one, mode="drop_correction")
    assert np.allclose(S[0], g["expected_additive_row_a"], rtol=0, atol=1e-15)
    # delta rule, beta = 1: the second write replaces row a, row b is untouched
    _, S = _one_step(Z, ka, v1, 1.0, one)
    _, S = _one_step(S, kb, vb, 1.0, one)
    _, S = _one_step(S, ka, v2, 1.0, one)
    assert np.array_equal(S[0], np.array(g["expected_delta_row_a"]))
    assert np.array_equal(S[1], np.array(g["expected_delta_row_b"]))
    # KDA: rows decay independently by 0.2 and 0.99 (beta = 0: no write)
    _, S2 = _one_step(np.stack([v1, vb]), ka, np.zeros(3), 0.0, g["kda_decay"])
    assert np.array_equal(S2[0], np.array(g["expected_kda_row_a"]))
    assert np.array_equal(S2[1], np.array(g["expected_kda_row_b"]))


# --- brain.bigb.es, DeltaNet: read-back and locality ------------------------------------
@pytest.mark.parametrize("seed", range(5))
def test_read_back_invariant(seed):
    rng = np.random.default_rng(seed)
    dk, dv = 8, 5
    S_prev = rng.standard_normal((dk, dv))
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(dv)
    alpha = rng.uniform(0.2, 1.0, dk)
    beta = rng.uniform()
    _, S = _one_step(S_prev, k, v, beta, alpha)
    S_tilde = alpha[:, None] * S_prev
    assert np.allclose(S.T @ k, (1 - beta) * (S_tilde.T @ k) + beta * v, atol=1e-13)
    # beta = 1, alpha = 1: the memory returns exactly v for its key
    _, S1 = _one_step(S_prev, k, v, 1.0, np.ones(dk))
    assert np.allclose(S1.T @ k, v, atol=1e-13)


@pytest.mark.parametrize("seed", range(5))
def test_write_is_local(seed):
    rng = np.random.default_rng(100 + seed)
    dk, dv = 8, 6
    S_prev = rng.standard_normal((dk, dv))
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    alpha = rng.uniform(0.2, 1.0, dk)
    _, S = _one_step(S_prev, k, rng.standard_normal(dv), rng.uniform(), alpha)
    x = rng.standard_normal(dk)
    x -= (x @ k) * k                       # x orthogonal to k
    S_tilde = alpha[:, None] * S_prev
    assert np.allclose((S - S_tilde).T @ x, 0.0, atol=1e-13)


# --- reductions --------------------------------------------------------------------------
def _deltanet_value_key_layout(q, k, v, beta, M0, scale):
    """DeltaNet as stated on brain.bigb.es: M_t = M_{t-1}(I - b k k^T) + b v k^T, o = M_t q."""
    T, dk = q.shape
    M = M0.copy()
    out = []
    for t in range(T):
        M = M @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        out.append(M @ (scale * q[t]))
    return np.array(out), M


def test_reduces_to_deltanet_at_unit_alpha():
    rng = np.random.default_rng(7)
    q, k, v, _, beta, S0 = _rand_inputs(rng, 1, 40, 2, 6, 5)
    alpha = np.ones_like(q)
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0, scale=0.7)
    for h in range(2):
        o_ref, M = _deltanet_value_key_layout(q[0, :, h], k[0, :, h], v[0, :, h],
                                              beta[0, :, h], S0[0, h].T, 0.7)
        assert np.allclose(o[0, :, h], o_ref, atol=1e-12)
        assert np.allclose(S[0, h], M.T, atol=1e-12)


def test_reduces_to_additive_linear_attention():
    """Correction dropped, alpha = beta = 1: o_t = scale * (S0^T q_t + sum_{i<=t} (k_i . q_t) v_i)."""
    rng = np.random.default_rng(8)
    q, k, v, _, _, S0 = _rand_inputs(rng, 2, 30, 3, 7, 4)
    ones = np.ones_like(q)
    o, S = oracle.forward(q, k, v, ones, np.ones(q.shape[:3]), s0=S0, scale=0.5,
                          mode="drop_correction")
    scores = np.einsum("btho,bsho->bhts", q, k)             # (k_s . q_t)
    causal = np.tril(np.ones((30, 30)))
    o_ref = 0.5 * (np.einsum("bhts,bshv->bthv", scores * causal, v)
                   + np.einsum("btho,bhov->bthv", q, S0))
    assert np.allclose(o, o_ref, atol=1e-12)
    assert np.allclose(S, S0 + np.einsum("btho,bthv->bhov", k, v), atol=1e-12)


# --- Module 03 section 3 / Notes section 9: the closed form by brute force ---------------
def _closed_form(q, k, v, alpha, beta, S0, scale):
    """S_t = P_t ... P_1 S_0 + sum_i P_t ... P_{i+1} beta_i k_i v_i^T, P_t = (I - b k k^T) D_t."""
    T, dk = q.shape
    P = [(np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(alpha[t]) for t in range(T)]
    outs, S_t = [], None
    for t in range(T):
        prod = np.eye(dk)
        for s in range(t, -1, -1):
            prod = prod @ P[s]                 # P_t P_{t-1} ... P_s
        S_t = prod @ S0
        for i in range(t + 1):
            tail = np.eye(dk)
            for s in range(t, i, -1):
                tail = tail @ P[s]             # P_t ... P_{i+1}
            S_t = S_t + tail @ (beta[i] * np.outer(k[i], v[i]))
        outs.append(S_t.T @ (scale * q[t]))
    return np.array(outs), S_t


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_brute_force_closed_form(T):
    rng = np.random.default_rng(20 + T)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 1, T, 2, 5, 4, alpha_lo=0.1)
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0, scale=0.9)
    for h in range(2):
        o_ref, S_ref = _closed_form(q[0, :, h], k[0, :, h], v[0, :, h], alpha[0, :, h],
                                    beta[0, :, h], S0[0, h], 0.9)
        assert np.allclose(o[0, :, h], o_ref, atol=1e-12)
        assert np.allclose(S[0, h], S_ref, atol=1e-12)


# --- planted mistakes must fail the pins --------------------------------------------------
@pytest.mark.parametrize("mode", ["swap_order", "predict_first", "drop_correction"])
def test_planted_mistakes_fail_closed_form(mode):
    rng = np.random.default_rng(5)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 1, 6, 1, 5, 4, alpha_lo=0.1)
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0, scale=1.0, mode=mode)
    o_ref, S_ref = _closed_form(q[0, :, 0], k[0, :, 0], v[0, :, 0], alpha[0, :, 0],
                                beta[0, :, 0], S0[0, 0], 1.0)
    rel = np.linalg.norm(S[0, 0] - S_ref) / np.linalg.norm(S_ref)
    assert rel > 1e-3, f"{mode} mutant not detected (rel={rel})"


def test_swapped_order_differs_on_random_data():
    rng = np.random.default_rng(11)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 2, 64, 2, 16, 16)
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0)
    o2, S2 = oracle.forward(q, k, v, alpha, beta, s0=S0, mode="swap_order")
    assert np.abs(o - o2).max() / np.sqrt(np.mean(o ** 2)) > 1e-3
    assert np.linalg.norm(S - S2) / np.linalg.norm(S) > 1e-3


def test_swapped_order_agrees_when_decay_is_scalar():
    """With D = a I the two orders commute (Module 03, section 3): the mutant must agree."""
    rng = np.random.default_rng(12)
    q, k, v, _, beta, S0 = _rand_inputs(rng, 1, 20, 1, 6, 3)
    a = rng.uniform(0.5, 1.0, (1, 20, 1, 1)) * np.ones((1, 20, 1, 6))
    o, S = oracle.forward(q, k, v, a, beta, s0=S0)
    o2, S2 = oracle.forward(q, k, v, a, beta, s0=S0, mode="swap_order")
    assert np.allclose(o, o2, atol=1e-12) and np.allclose(S, S2, atol=1e-12)


# --- DPLR view: the transition is a contraction ------------------------------------------
def test_contraction_bound():
    rng = np.random.default_rng(13)
    dk, dv = 8, 8
    S = rng.standard_normal((dk, dv))
    for _ in range(50):
        k = rng.standard_normal(dk)
        k /= np.linalg.norm(k)
        v = rng.standard_normal(dv)
        beta = rng.uniform()
        _, S_new = _one_step(S, k, v, beta, rng.uniform(0.0, 1.0, dk))
        bound = np.linalg.norm(S, 2) + beta * np.linalg.norm(v) * np.linalg.norm(k)
        assert np.linalg.norm(S_new, 2) <= bound + 1e-12
        S = S_new


# --- the chunkwise schedule equals the sequential one -------------------------------------
@pytest.mark.parametrize("T,C", [(64, 64), (130, 64), (100, 16), (37, 8), (1, 64)])
def test_chunked_matches_sequential(T, C):
    rng = np.random.default_rng(T * 7 + C)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 1, T, 2, 16, 12, alpha_lo=0.05)
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0, scale=0.25)
    oc, Sc = forward_chunked(q, k, v, alpha, beta, s0=S0, scale=0.25, chunk=C)
    rms = np.sqrt(np.mean(o ** 2))
    assert np.abs(o - oc).max() / rms < 1e-12
    assert np.linalg.norm(S - Sc) / np.linalg.norm(S) < 1e-12


def test_chunked_handles_zero_retention():
    rng = np.random.default_rng(3)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 1, 70, 1, 8, 8)
    alpha[0, 10, 0, :4] = 0.0
    alpha[0, 40:45, 0, 2] = 0.0
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0)
    oc, Sc = forward_chunked(q, k, v, alpha, beta, s0=S0, chunk=32)
    assert np.abs(o - oc).max() < 1e-12 and np.abs(S - Sc).max() < 1e-12


def test_decode_step_is_one_token_forward():
    rng = np.random.default_rng(4)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 3, 1, 2, 8, 6)
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0)
    od, Sd = oracle.decode_step(q[:, 0], k[:, 0], v[:, 0], alpha[:, 0], beta[:, 0], S0)
    assert np.array_equal(od, o[:, 0]) and np.array_equal(Sd, S)


def test_split_sequence_continues_from_final_state():
    """The state is the resume point (Module 03, section 5): two calls equal one."""
    rng = np.random.default_rng(9)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 2, 50, 2, 8, 8)
    o, S = oracle.forward(q, k, v, alpha, beta, s0=S0)
    o1, S1 = oracle.forward(q[:, :20], k[:, :20], v[:, :20], alpha[:, :20], beta[:, :20], s0=S0)
    o2, S2 = oracle.forward(q[:, 20:], k[:, 20:], v[:, 20:], alpha[:, 20:], beta[:, 20:], s0=S1)
    assert np.array_equal(np.concatenate([o1, o2], axis=1), o) and np.array_equal(S2, S)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(10)
    q, k, v, alpha, beta, S0 = _rand_inputs(rng, 2, 33, 3, 8, 8)
    a = oracle.forward(q, k, v, alpha, beta, s0=S0, n_threads=1)
    b = oracle.forward(q, k, v, alpha, beta, s0=S0, n_threads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
