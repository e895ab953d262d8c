"""NumPy fp64 chunk-parallel WY/UT form of the gated delta rule.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Its one use is to pin the
per-token oracle: it reaches the same real numbers by a different algorithm.

It follows the gated branch of Prizma "seq/delta.py" ``chunked_delta`` (the
WY/UT chunk-parallel form whose docstring says it must agree with the per-token
reference), with the state held transposed, H = S^T [dk, dv].  Per chunk of
tokens i = 1..C with in-chunk log decay G_i = g_1 + ... + g_i:

  A_ij   = beta_i (k_i . k_j) exp(G_i - G_j)            for j < i   (strictly lower)
  (I + A) U = diag(beta) V - diag(beta exp(G)) K H       (unit-lower solve)
  post:  o_i = scale (exp(G_i) q_i H + sum_{j<=i} exp(G_i - G_j)(q_i . k_j) U_j)
  pre:   o_i = scale (exp(G_{i-1}) q_i H + sum_{j<i} exp(G_{i-1} - G_j)(q_i . k_j) U_j)
  H  <-  exp(G_C) H + sum_i exp(G_C - G_i) k_i U_i^T

Every decay ratio is formed as exp of a log difference on the triangle where it
is <= 1 (the page's comment on log-space cumulative decay), never as a quotient
of two cumulative products.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _normalise(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-6)


def _decay(Gr: np.ndarray, Gc: np.ndarray, strict: bool) -> np.ndarray:
    """exp(Gr_i - Gc_j) on the lower triangle (strict or inclusive), 0 elsewhere."""
    C = Gr.shape[0]
    mask = np.tril(np.ones((C, C), dtype=bool), -1 if strict else 0)
    diff = np.where(mask, Gr[:, None] - Gc[None, :], -np.inf)
    return np.exp(diff)


def chunked_scan(q, k, v, g, beta, H0, chunk, read_mode="post", scale=1.0):
    """One (sequence, head): q, k [L, dk]; v [L, dv]; g, beta [L]; H0 [dk, dv] (fp64).
    Returns o [L, dv] and the final state [dk, dv]."""
    L, dv = v.shape
    H = H0.copy()
    o = np.zeros((L, dv))
    for c0 in range(0, L, chunk):
        c1 = min(c0 + chunk, L)
        Q, K, V = q[c0:c1], k[c0:c1], v[c0:c1]
        b, gl = beta[c0:c1], g[c0:c1]
        G = np.cumsum(gl)
        Gprev = G - gl
        C = c1 - c0
        A = b[:, None] * (K @ K.T) * _decay(G, G, strict=True)
        rhs = b[:, None] * V - (b * np.exp(G))[:, None] * (K @ H)
        U = solve_triangular(np.eye(C) + A, rhs, lower=True, unit_diagonal=True)
        QK = Q @ K.T
        if read_mode == "post":
            O = np.exp(G)[:, None] * (Q @ H) + (QK * _decay(G, G, strict=False)) @ U
        else:
            O = np.exp(Gprev)[:, None] * (Q @ H) + (QK * _decay(Gprev, G, strict=True)) @ U
        o[c0:c1] = scale * O
        H = np.exp(G[-1]) * H + (np.exp(G[-1] - G)[:, None] * K).T @ U
    return o, H


def chunked_forward(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk=64, read_mode="post",
                    scale=1.0, qk_l2norm=True, reverse=False):
    """Same contract as ``oracle.forward`` (fp64 numpy in, fp64 numpy out)."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    grp = Hv // Hk
    if cu_seqlens is None:
        spans = [(b * T, (b + 1) * T) for b in range(B)]
    else:
        cu = [int(x) for x in cu_seqlens]
        spans = [(cu[s], cu[s + 1]) for s in range(len(cu) - 1)]
    qf, kf = q.reshape(B * T, Hk, dk), k.reshape(B * T, Hk, dk)
    vf, gf, bf = v.reshape(B * T, Hv, dv), g.reshape(B * T, Hv), beta.reshape(B * T, Hv)
    if qk_l2norm:
        qf, kf = _normalise(qf), _normalise(kf)
    o = np.zeros((B * T, Hv, dv))
    S_final = np.zeros((len(spans), Hv, dk, dv))
    for s, (t0, t1) in enumerate(spans):
        idx = np.arange(t0, t1)
        if reverse:
            idx = idx[::-1]
        for h in range(Hv):
            H0 = np.zeros((dk, dv)) if S0 is None else np.asarray(S0[s, h], dtype=np.float64)
            os_, H = chunked_scan(qf[idx, h // grp], kf[idx, h // grp], vf[idx, h], gf[idx, h],
                                  bf[idx, h], H0, chunk, read_mode, scale)
            o[idx, h] = os_
            S_final[s, h] = H
    return o.reshape(B, T, Hv, dv), S_final
