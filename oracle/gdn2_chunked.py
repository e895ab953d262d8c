"""Chunk-parallel (WY/UT) form of the GDN-2 recurrence with decoupled gates, NumPy fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  A second algorithm for the same
real numbers as ``oracle.gdn2_forward``, used only to pin it.  Within a chunk, with
per-channel cumulative log decay G_t (G_0 = 0) and state H (= S^T, [dk, dv]) at its start:
    u_t + sum_{s<t} (e^{G_t - G_s} . b_t . k_t . k_s) u_s = w_t v_t - H^T (e^{G_t} b_t k_t)
solved as one unit-lower-triangular system; then
    o_t = q_t^T (e^{G'_t} H) + sum_{s<=t} (sum_d q_td k_sd e^{G'_td - G_sd}) u_s
    H  <- e^{G_C} H + sum_s (e^{G_C - G_s} . k_s) u_s^T
(G' = G_t for the post-write read, G_{t-1} for the pre-write read).  Derived from the
recurrence of Rondo-Exp ``tiny_gdn/fugue.py`` (BidirectionalGatedDeltaNet2 docstring) the
way Prizma ``seq/delta.py`` ``chunked_delta`` derives the scalar form.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def forward(q, k, v, g, b, w, S0=None, chunk: int = 16, read_mode: str = "post",
            scale: float = 1.0, qk_l2norm: bool = True):
    """q, k [B, T, H, dk]; v, w [B, T, H, dv]; g, b [B, T, H, dk] (Hk = Hv), fp64 arrays."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if qk_l2norm:
        q = q / np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), 1e-6)
        k = k / np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), 1e-6)
    o = np.zeros((B, T, H, dv))
    S = np.zeros((B, H, dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    for n in range(B):
        for h in range(H):
            Hs = S[n, h].copy()
            for c0 in range(0, T, chunk):
                c1 = min(c0 + chunk, T)
                K, Q, V = k[n, c0:c1, h], q[n, c0:c1, h], v[n, c0:c1, h]
                Bg, Wg = b[n, c0:c1, h], w[n, c0:c1, h]
                G = np.cumsum(g[n, c0:c1, h], axis=0)                  # [C, dk]
                Gp = G if read_mode == "post" else np.vstack([np.zeros((1, dk)), G[:-1]])
                C = c1 - c0
                A = np.zeros((C, C))
                for t in range(C):
                    for s in range(t):
                        A[t, s] = np.sum(np.exp(G[t] - G[s]) * Bg[t] * K[t] * K[s])
                rhs = Wg * V - (np.exp(G) * Bg * K) @ Hs
                U = solve_triangular(np.eye(C) + A, rhs, lower=True, unit_diagonal=True)
                P = np.zeros((C, C))
                for t in range(C):
                    for s in range(C):
                        if s < t or (s == t and read_mode == "post"):
                            P[t, s] = np.sum(Q[t] * K[s] * np.exp(Gp[t] - G[s]))
                o[n, c0:c1, h] = scale * ((Q * np.exp(Gp)) @ Hs + P @ U)
                Hs = np.exp(G[-1])[:, None] * Hs + (np.exp(G[-1] - G) * K).T @ U
            S[n, h] = Hs
    return o, S
