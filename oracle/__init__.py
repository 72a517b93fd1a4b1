"""KDA oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct fp64 CPU implementation of the KDA recurrence
that the CUDA library is checked against.  Only ``tests/``, the smoke check and
the benchmark's CPU-baseline leg may import it; the library itself never does,
and the two share no code.

``forward`` runs the sequential five-step update of "Module 03 -- KDA I: The
Delta-Rule Recurrence", section 2, in C (``kda_oracle.c``), in fp64, over all
(sequence, head) pairs.  ``decode_step`` is the same loop for one token.
``forward_gdn2`` is the same loop with the decoupled erase and write gates of
"From Fast Weight Programmers to KDA", section "Gated DeltaNet-2".
``forward_raw`` applies the input preprocessing in fp64 first (q and k divided by
their L2 norms, log alpha = -softplus(gate logit), beta = sigmoid(beta logit)) and
then runs ``forward``.  ``token_states`` gives the state after every token (the forward loop run on each
prefix) and ``state_copy`` the whole-state copy between slot pools, the two
serving operations of "Module 03 -- KDA I", section 5 "State vs. checkpoint
weights".  ``chunked.forward_chunked`` (numpy, fp64) is the second schedule of "Kimi Delta
Attention (KDA)", "Two schedules for the same recurrence"; the tests pin it to
the sequential loop; ``chunked.forward_chunked_gdn2`` is the same schedule for
GDN-2, pinned the same way.

Every function here is pinned by ``tests/test_oracle_pins.py`` against values
and identities the pages fix; no part is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libkda_oracle.so")

MODES = {"exact": 0, "drop_correction": 1, "swap_order": 2, "predict_first": 3}

_lib = None
_lib_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, -O2, no fast-math) into oracle/_build."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
               "-ffp-contract=off", "-pthread", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lib_lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            lib.kda_ref_forward.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                            ctypes.c_int, ctypes.c_int]
            lib.kda_ref_forward.restype = ctypes.c_int
            lib.kda_ref_forward_gdn2.argtypes = [dp] * 9 + [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int]
            lib.kda_ref_forward_gdn2.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Upcast a numpy array or CPU torch tensor (fp32 / bf16 / fp64) to fp64 exactly."""
    if hasattr(x, "detach"):  # torch tensor: bf16 -> fp64 is exact
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def threads_for(n_items: int, n_threads: int = 0) -> int:
    """Number of POSIX threads ``forward`` uses for n_items (sequence, head) pairs."""
    n = n_threads if n_threads > 0 else (os.cpu_count() or 1)
    return max(1, min(n, max(n_items, 1)))


def forward(q, k, v, alpha, beta, s0=None, scale=None, mode="exact", n_threads=0):
    """Sequential fp64 KDA over q,k,alpha [B,T,H,dk], v [B,T,H,dv], beta [B,T,H].

    s0: [B,H,dk,dv] or None (zeros).  scale defaults to dk**-0.5 and multiplies
    q at the read only.  Returns (o [B,T,H,dv], s_final [B,H,dk,dv]) in fp64.
    """
    q, k, v, alpha, beta = (_f64(x) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and alpha.shape == q.shape, "q, k, alpha shapes differ"
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H), "v/beta shape"
    s0a = None
    if s0 is not None:
        s0a = _f64(s0)
        assert s0a.shape == (B, H, dk, dv), "s0 shape"
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    s_final = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = _load().kda_ref_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                 _ptr(s0a), _ptr(o), _ptr(s_final), B, T, H, dk, dv,
                                 float(scale), MODES[mode], int(n_threads))
    if rc != 0:
        raise RuntimeError(f"kda_ref_forward failed with code {rc}")
    return o, s_final


def forward_gdn2(q, k, v, alpha, erase, write, s0=None, scale=None, n_threads=0):
    """Sequential fp64 GDN-2: per-key-channel erase gate [B,T,H,dk] and per-value-channel
    write gate [B,T,H,dv] in place of beta; otherwise as ``forward``."""
    q, k, v, alpha, erase, write = (_f64(x) for x in (q, k, v, alpha, erase, write))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and alpha.shape == q.shape and erase.shape == q.shape, "dk shapes"
    assert v.shape == (B, T, H, dv) and write.shape == v.shape, "dv shapes"
    s0a = None
    if s0 is not None:
        s0a = _f64(s0)
        assert s0a.shape == (B, H, dk, dv), "s0 shape"
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    s_final = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = _load().kda_ref_forward_gdn2(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(erase), _ptr(write),
                                      _ptr(s0a), _ptr(o), _ptr(s_final), B, T, H, dk, dv,
                                      float(scale), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"kda_ref_forward_gdn2 failed with code {rc}")
    return o, s_final


def decode_step(q, k, v, alpha, beta, state, scale=None, mode="exact"):
    """One token per sequence: q,k,alpha [N,H,dk], v [N,H,dv], beta [N,H], state [N,H,dk,dv].

    Returns (o [N,H,dv], new_state [N,H,dk,dv]) in fp64; the input is not modified.
    """
    q, k, v, alpha, beta = (_f64(x) for x in (q, k, v, alpha, beta))
    o, s = forward(q[:, None], k[:, None], v[:, None], alpha[:, None], beta[:, None],
                   s0=state, scale=scale, mode=mode)
    return o[:, 0], s


def token_states(q, k, v, alpha, beta, s0=None, scale=None):
    """State after each token, [B,T,H,dk,dv] fp64: entry t is the final state of ``forward``
    run on tokens 0..t.  A state is request-scoped and a speculative step is rolled back
    to the state after its last accepted token ("Module 03 -- KDA I", section 5)."""
    q = _f64(q)
    B, T, H, dk = q.shape
    dv = _f64(v).shape[-1]
    out = np.zeros((B, T, H, dk, dv))
    for t in range(T):
        sl = lambda x: _f64(x)[:, :t + 1]
        _, S = forward(sl(q), sl(k), sl(v), sl(alpha), sl(beta), s0=s0, scale=scale)
        out[:, t] = S
    return out


def state_copy(src, dst, src_index=None, dst_index=None, count=None):
    """Whole-state copy between slot pools, on copies of the arrays: entry i sets
    dst[dst_index[i]] = src[src_index[i]] (identity index when None); entries with a
    negative or out-of-range index are skipped.  Returns (new dst, any index out of range)."""
    src, dst = np.array(src, dtype=np.float64), np.array(dst, dtype=np.float64)
    if count is None:
        idx = src_index if src_index is not None else dst_index
        count = len(idx) if idx is not None else min(len(src), len(dst))
    bad = False
    for i in range(count):
        si = int(src_index[i]) if src_index is not None else i
        di = int(dst_index[i]) if dst_index is not None else i
        if si < 0 or di < 0:
            continue
        if si >= len(src) or di >= len(dst):
            bad = True
            continue
        dst[di] = src[si]
    return dst, bad


def preprocess(q, k, gate_logit, beta_logit):
    """The input preprocessing, in fp64: q_t / ||q_t|| and k_t / ||k_t|| (a zero row stays
    zero; "Notes on Linear Attention", section 5.3 "Why L2-normalize the key?"),
    alpha = exp(-softplus(x)) (the stored log-decay g = log alpha = -softplus(x) <= 0,
    "Kimi Delta Attention (KDA)"), beta = sigmoid(y) ("From Fast Weight Programmers to
    KDA", the delta rule's learned write strength).  Returns (q, k, alpha, beta)."""
    def unit(x):
        x = _f64(x)
        n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
        return np.divide(x, n, out=np.zeros_like(x), where=n > 0)

    x = _f64(gate_logit)
    softplus = np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))
    y = _f64(beta_logit)
    beta = np.where(y >= 0, 1.0 / (1.0 + np.exp(-np.abs(y))), np.exp(-np.abs(y)) / (1.0 + np.exp(-np.abs(y))))
    return unit(q), unit(k), np.exp(-softplus), beta


def forward_raw(q, k, v, gate_logit, beta_logit, s0=None, scale=None, n_threads=0):
    """``forward`` on preprocessed inputs: un-normalised q, k [B,T,H,dk], gate logits
    [B,T,H,dk] and beta logits [B,T,H] (see ``preprocess``)."""
    qn, kn, alpha, beta = preprocess(q, k, gate_logit, beta_logit)
    return forward(qn, kn, v, alpha, beta, s0=s0, scale=scale, n_threads=n_threads)
