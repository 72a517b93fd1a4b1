"""Chunkwise KDA in fp64 numpy -- TEST INFRASTRUCTURE ONLY.

The second schedule of the same recurrence, written from "Kimi Delta Attention
(KDA)" (brain.bigb.es), "Two schedules for the same recurrence", and the
chunked KDA of "From Fast Weight Programmers to KDA" (jonahsamost.bearblog.dev),
section "Kimi Delta Attention", in the d_k x d_v state layout.  For a chunk
holding tokens i = 0 .. L-1 and the incoming state S:

  decay from token j to token i (j <= i), per key channel:
      G[i, j] = prod_{t=j+1..i} alpha_t          (G[i, i] = 1)
  decay from the chunk start to token i:  g[i] = prod_{t=0..i} alpha_t
  provisional errors (no in-chunk writes):
      ebar_i = beta_i (v_i - S^T (g_i * k_i))
  correction coefficients, j < i:  rho_ij = beta_i sum_d k_jd G[i,j,d] k_id
  true errors:  (I + R) E = Ebar  (R strictly lower triangular; forward solve)
  outputs, j <= i (a token reads its own write):
      o_i = scale [ S^T (g_i * q_i) + sum_{j<=i} (sum_d q_id G[i,j,d] k_jd) e_j ]
  next state:   S' = Diag(g_{L-1}) S + sum_j (G[L-1, j] * k_j) e_j^T

Here e_j already carries beta_j (the brain.bigb.es convention e = beta (v - vh)).
The pairwise decays are formed as direct products, never as ratios, so
alpha = 0 is exact.  A ragged last chunk is just a shorter chunk.  The tests
pin this to the sequential loop to ~1e-12.
"""
from __future__ import annotations

import numpy as np


def _pairwise_decay(a: np.ndarray) -> np.ndarray:
    """a: [L, d] retention factors -> G [L, L, d] with G[i, j] = prod_{t=j+1..i} a_t (j <= i), 0 above."""
    L, d = a.shape
    G = np.zeros((L, L, d))
    for j in range(L):
        G[j, j] = 1.0
        if j + 1 < L:
            G[j + 1:, j] = np.cumprod(a[j + 1:], axis=0)
    return G


def _chunk_head(q, k, v, a, b, S, scale, C):
    T, dk = q.shape
    dv = v.shape[1]
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        qc, kc, vc, ac, bc = q[sl], k[sl], v[sl], a[sl], b[sl]
        L = qc.shape[0]
        g = np.cumprod(ac, axis=0)                      # [L, dk]
        G = _pairwise_decay(ac)                         # [L, L, dk]
        ebar = bc[:, None] * (vc - (g * kc) @ S)        # [L, dv]
        rho = bc[:, None] * np.einsum("jd,ijd,id->ij", kc, G, kc)
        R = np.tril(rho, -1)
        E = np.zeros((L, dv))
        for i in range(L):                              # forward substitution
            E[i] = ebar[i] - R[i, :i] @ E[:i]
        chi = np.tril(np.einsum("id,ijd,jd->ij", qc, G, kc))
        o[sl] = scale * ((g * qc) @ S + chi @ E)
        S = g[-1][:, None] * S + (G[L - 1] * kc).T @ E
    return o, S


def forward_chunked(q, k, v, alpha, beta, s0=None, scale=None, chunk=64):
    """Chunkwise fp64 KDA with the same arguments and layouts as ``oracle.forward``."""
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros((B, T, H, dv))
    s_final = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            o[b, :, h], s_final[b, h] = _chunk_head(q[b, :, h], k[b, :, h], v[b, :, h],
                                                    alpha[b, :, h], beta[b, :, h], S,
                                                    scale, chunk)
    return o, s_final


def _chunk_head_gdn2(q, k, v, a, er, wr, S, scale, C):
    """GDN-2 in the same chunked form: with the erase gate b and write gate w in place of
    beta, the in-chunk system is (I + R) E = w*V - ((g*b*K) S) with
    R_ij = sum_d b_id k_id G[i,j,d] k_jd (j < i), and the outputs and the next state are
    formed as for KDA ("From Fast Weight Programmers to KDA", section "Gated DeltaNet-2":
    retrieve through b*k, write w*v minus the retrieval at k)."""
    T = q.shape[0]
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        qc, kc, vc, ac, bc, wc = q[sl], k[sl], v[sl], a[sl], er[sl], wr[sl]
        L = qc.shape[0]
        g = np.cumprod(ac, axis=0)
        G = _pairwise_decay(ac)
        ebar = wc * vc - (g * bc * kc) @ S
        R = np.tril(np.einsum("id,ijd,jd->ij", bc * kc, G, kc), -1)
        E = np.zeros((L, vc.shape[1]))
        for i in range(L):
            E[i] = ebar[i] - R[i, :i] @ E[:i]
        chi = np.tril(np.einsum("id,ijd,jd->ij", qc, G, kc))
        o[sl] = scale * ((g * qc) @ S + chi @ E)
        S = g[-1][:, None] * S + (G[L - 1] * kc).T @ E
    return o, S


def forward_chunked_gdn2(q, k, v, alpha, erase, write, s0=None, scale=None, chunk=64):
    """Chunkwise fp64 GDN-2 with the arguments and layouts of ``oracle.forward_gdn2``."""
    q, k, v, alpha, erase, write = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, erase, write))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros((B, T, H, dv))
    s_final = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            o[b, :, h], s_final[b, h] = _chunk_head_gdn2(q[b, :, h], k[b, :, h], v[b, :, h], alpha[b, :, h],
                                                         erase[b, :, h], write[b, :, h], S, scale, chunk)
    return o, s_final
