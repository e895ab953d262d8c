"""Exact rational evaluation of the gated delta rule on tiny inputs.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Used to pin the fp64
oracle and to write the exact fixtures under ``tests/golden``.

It does not step the recurrence.  With the state held transposed (H = S^T,
[dk, dv]) the update of Prizma "seq/delta.py" (module docstring,
``_delta_reference``),
    u_t = beta_t (v_t - alpha_t H^T k_t),   H_t = alpha_t H_{t-1} + k_t u_t^T,
rearranges to the affine map
    H_t = M_t H_{t-1} + beta_t k_t v_t^T,    M_t = alpha_t (I - beta_t k_t k_t^T),
so the state after token t is the closed product form
    H_t = (M_t ... M_1) H_0 + sum_{s<=t} (M_t ... M_{s+1}) beta_s k_s v_s^T.
Each H_t is built from that sum of products in ``fractions.Fraction``; reads are
o_t = scale H_t^T q_t (post-write) or scale H_{t-1}^T q_t (pre-write).

Inputs are nested lists of ints / Fractions; alpha is given directly (not its
log).  Optional L2 normalisation is exact only when every q and k has a rational
norm, which the caller guarantees (integer vectors with integer length).
"""
from __future__ import annotations

from fractions import Fraction
from math import isqrt


def _eye(n):
    return [[Fraction(int(i == j)) for j in range(n)] for i in range(n)]


def _matmul(A, B):
    n, m, p = len(A), len(B), len(B[0])
    return [[sum((A[i][r] * B[r][j] for r in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def _add(A, B):
    return [[a + b for a, b in zip(ra, rb)] for ra, rb in zip(A, B)]


def _outer(x, y, c=Fraction(1)):
    return [[c * xi * yj for yj in y] for xi in x]


def _exact_unit(x):
    """x / ||x|| for an integer vector whose squared norm is a perfect square."""
    ss = sum(Fraction(a) * a for a in x)
    if ss.denominator != 1 or isqrt(ss.numerator) ** 2 != ss.numerator:
        raise ValueError("vector norm is not rational; choose integer vectors with integer length")
    n = isqrt(ss.numerator)
    return [Fraction(a) / n for a in x]


def forward_exact(q, k, v, alpha, beta, H0, read_mode="post", scale=Fraction(1), qk_l2norm=False):
    """One (sequence, head): q, k [T][dk]; v [T][dv]; alpha, beta [T]; H0 [dk][dv].
    Returns (o [T][dv], H_T [dk][dv]) as Fractions."""
    T = len(v)
    dk, dv = len(k[0]), len(v[0])
    q = [_exact_unit(x) if qk_l2norm else [Fraction(a) for a in x] for x in q]
    k = [_exact_unit(x) if qk_l2norm else [Fraction(a) for a in x] for x in k]
    v = [[Fraction(a) for a in x] for x in v]
    alpha = [Fraction(a) for a in alpha]
    beta = [Fraction(b) for b in beta]
    H0 = [[Fraction(a) for a in row] for row in H0]
    scale = Fraction(scale)
    I = _eye(dk)
    M = []
    for t in range(T):
        kk = _outer(k[t], k[t], beta[t])
        M.append([[alpha[t] * (I[i][j] - kk[i][j]) for j in range(dk)] for i in range(dk)])

    def prod(hi, lo):
        """M_hi ... M_lo (1-based token indices); identity if hi < lo."""
        P = _eye(dk)
        for t in range(lo, hi + 1):
            P = _matmul(M[t - 1], P)
        return P

    def state(t):
        Ht = _matmul(prod(t, 1), H0)
        for s in range(1, t + 1):
            Ht = _add(Ht, _matmul(prod(t, s + 1), _outer(k[s - 1], v[s - 1], beta[s - 1])))
        return Ht

    def read(Ht, qt):
        return [scale * sum((Ht[d][j] * qt[d] for d in range(dk)), Fraction(0)) for j in range(dv)]

    o = []
    for t in range(1, T + 1):
        Ht = state(t - 1) if read_mode == "pre" else state(t)
        o.append(read(Ht, q[t - 1]))
    return o, state(T)
