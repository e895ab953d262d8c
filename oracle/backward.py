"""fp64 reverse-mode (backward pass) of the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the test suite, the smoke check
and the CPU-baseline leg of the benchmark may use it, and it shares no code with the CUDA
library.

What it computes.  Prizma "seq/delta.py" (module docstring) asks that its chunk-parallel
form agree with the per-token recurrence on the forward AND on the gradients; the gradient
is the one of the per-token recurrence.  For upstream gradients dO (of o) and dS_final (of
S_final) this returns the gradients of

    L = <dO, o> + <dS_final, S_final>

with respect to q, k, v, g, beta and S0, for the same recurrence, layouts and options as
``oracle.forward`` (H = S^T stored [dk, dv]; GQA by key-head sharing; varlen; the post- and
pre-write reads; reversal within each sequence; in-kernel L2 normalisation of q and k).

How.  Reverse-mode by hand, one token at a time, from the recurrence's own steps.  The
forward step of one (sequence, v-head) is

    k^ = k / max(|k|, eps),  q^ = q / max(|q|, eps)        (if qk_l2norm)
    a = exp(g),  s = H^T k^,  u = beta (v - a s),  H' = a H + k^ u^T
    o = scale H'^T q^   (post)      or      o = scale H^T q^   (pre)

and its adjoint, with dH' the gradient reaching H' from later tokens, is

    post: dH' += scale q^ do^T,  dq^ = scale H' do
    da  = <dH', H>,  dH = a dH',  dk^ = dH' u,  du = dH'^T k^
    dv  = beta du,  dbeta = du . (v - a s),  da -= beta du . s
    ds  = -a beta du,  dH += k^ ds^T,  dk^ += H ds
    pre:  dq^ = scale H do,  dH += scale q^ do^T
    dg  = a da
    x^ = x / |x| (|x| > eps):  dx = (dx^ - x^ (x^ . dx^)) / |x|;   |x| <= eps:  dx = dx^ / eps

The states are recomputed forward from checkpoints every ``ckpt`` tokens (the same fp64
operations in the same order, so the values equal those of one stored pass) to bound
memory on long sequences.
"""
from __future__ import annotations

import numpy as np

_EPS = 1e-6


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _normalise(x, on: bool):
    """(x^, |x|) per row of x [H, d]."""
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return (x / np.maximum(n, _EPS), n) if on else (x, n)


def _normalise_adjoint(dxh, xh, n, on: bool):
    if not on:
        return dxh
    big = n > _EPS
    proj = np.sum(xh * dxh, axis=-1, keepdims=True)
    return np.where(big, (dxh - xh * proj) / np.where(big, n, 1.0), dxh / _EPS)


def backward(q, k, v, g, beta, dO, S0=None, dS_final=None, cu_seqlens=None,
             read_mode: str = "post", scale: float = 1.0, qk_l2norm: bool = True,
             reverse: bool = False, ckpt: int = 64):
    """Gradients of <dO, o> + <dS_final, S_final>.

    q, k [B, T, Hk, dk]; v, dO [B, T, Hv, dv]; g, beta [B, T, Hv]; S0, dS_final
    [n_seqs, Hv, dk, dv] or None (zero).  Returns a dict of fp64 arrays: dq, dk
    [B, T, Hk, dk]; dv [B, T, Hv, dv]; dg, dbeta [B, T, Hv]; dS0 [n_seqs, Hv, dk, dv].
    """
    q, k, v, g, beta, dO, S0, dS_final = (_f64(x) for x in (q, k, v, g, beta, dO, S0,
                                                            dS_final))
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    group = Hv // Hk
    pre = read_mode == "pre"
    if cu_seqlens is None:
        segs = [(n, 0, T) for n in range(B)]
    else:
        cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                        dtype=np.int64)
        segs = [(0, int(cu[s]), int(cu[s + 1])) for s in range(len(cu) - 1)]
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dg": np.zeros_like(g), "dbeta": np.zeros_like(beta),
           "dS0": np.zeros((len(segs), Hv, dk, dv))}

    def token(row, t):
        """Normalised q, k of token t for every v-head, with their norms."""
        qr = np.repeat(q[row, t], group, axis=0)
        kr = np.repeat(k[row, t], group, axis=0)
        qh, qn = _normalise(qr, qk_l2norm)
        kh, kn = _normalise(kr, qk_l2norm)
        return qh, qn, kh, kn

    def step(H, row, t, kh):
        """One forward step from H: (a, s, u, H')."""
        a = np.exp(g[row, t])                                   # [Hv]
        s = np.einsum("hd,hde->he", kh, H)                      # [Hv, dv]
        u = beta[row, t][:, None] * (v[row, t] - a[:, None] * s)
        return a, s, u, a[:, None, None] * H + kh[:, :, None] * u[:, None, :]

    for si, (row, t0, t1) in enumerate(segs):
        order = list(range(t1 - 1, t0 - 1, -1)) if reverse else list(range(t0, t1))
        L = len(order)
        # forward: the state before every checkpointed position
        H = np.zeros((Hv, dk, dv)) if S0 is None else S0[si].copy()
        marks = {}
        for i, t in enumerate(order):
            if i % ckpt == 0:
                marks[i] = H.copy()
            H = step(H, row, t, token(row, t)[2])[3]
        # backward, block by block from the end
        dH = np.zeros((Hv, dk, dv)) if dS_final is None else dS_final[si].copy()
        for b0 in sorted(marks, reverse=True):
            states = [marks[b0]]
            for i in range(b0, min(b0 + ckpt, L) - 1):
                t = order[i]
                states.append(step(states[-1], row, t, token(row, t)[2])[3])
            for i in range(min(b0 + ckpt, L) - 1, b0 - 1, -1):
                t = order[i]
                H = states[i - b0]
                qh, qn, kh, kn = token(row, t)
                a, s, u, Hn = step(H, row, t, kh)
                do = dO[row, t]                                         # [Hv, dv]
                if not pre:
                    dH = dH + scale * qh[:, :, None] * do[:, None, :]
                    dqh = scale * np.einsum("hde,he->hd", Hn, do)
                da = np.einsum("hde,hde->h", dH, H)
                dkh = np.einsum("hde,he->hd", dH, u)
                du = np.einsum("hde,hd->he", dH, kh)
                dHp = a[:, None, None] * dH
                bt = beta[row, t]
                out["dv"][row, t] = bt[:, None] * du
                out["dbeta"][row, t] = np.sum(du * (v[row, t] - a[:, None] * s), axis=-1)
                da = da - bt * np.sum(du * s, axis=-1)
                ds = -(a * bt)[:, None] * du
                dHp = dHp + kh[:, :, None] * ds[:, None, :]
                dkh = dkh + np.einsum("hde,he->hd", H, ds)
                if pre:
                    dqh = scale * np.einsum("hde,he->hd", H, do)
                    dHp = dHp + scale * qh[:, :, None] * do[:, None, :]
                out["dg"][row, t] = a * da
                dq_h = _normalise_adjoint(dqh, qh, qn, qk_l2norm)
                dk_h = _normalise_adjoint(dkh, kh, kn, qk_l2norm)
                out["dq"][row, t] += dq_h.reshape(Hk, group, dk).sum(axis=1)
                out["dk"][row, t] += dk_h.reshape(Hk, group, dk).sum(axis=1)
                dH = dHp
        out["dS0"][si] = dH
    return out
