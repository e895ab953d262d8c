"""Pins of the backward oracle (``oracle.backward``), each independent of its hand-derived
adjoint: central finite differences of the forward oracle, autograd of a plain fp64 PyTorch
loop, a closed form, and checkpoint invariance."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bw

RNG = np.random.default_rng(23)


def problem(B, T, Hk, Hv, dk, dv, lengths=None, s0=True):
    cu = None
    if lengths is not None:
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        B, T = 1, int(cu[-1])
    n = B if cu is None else len(cu) - 1
    x = dict(q=RNG.normal(size=(B, T, Hk, dk)), k=RNG.normal(size=(B, T, Hk, dk)),
             v=RNG.normal(size=(B, T, Hv, dv)),
             g=-np.log1p(np.exp(RNG.normal(-2, 1, (B, T, Hv)))),
             beta=1 / (1 + np.exp(-RNG.normal(size=(B, T, Hv)))),
             S0=RNG.normal(size=(n, Hv, dk, dv)) * 0.5 if s0 else None)
    up = dict(dO=RNG.normal(size=(B, T, Hv, dv)), dS_final=RNG.normal(size=(n, Hv, dk, dv)))
    return x, up, cu


def loss(x, up, cu, **kw):
    o, S = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], cu, **kw)
    return float(np.sum(up["dO"] * o) + np.sum(up["dS_final"] * S))


def fd_grads(x, up, cu, h=1e-6, **kw):
    out = {}
    for name in ("q", "k", "v", "g", "beta", "S0"):
        base = x[name]
        if base is None:
            continue
        grad = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            keep = base[idx]
            base[idx] = keep + h
            lp = loss(x, up, cu, **kw)
            base[idx] = keep - h
            lm = loss(x, up, cu, **kw)
            base[idx] = keep
            grad[idx] = (lp - lm) / (2 * h)
        out["d" + name] = grad
    return out


def oracle_grads(x, up, cu, **kw):
    return bw.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], up["dO"], x["S0"],
                       up["dS_final"], cu, **kw)


CASES = [
    dict(read_mode="post", reverse=False, qk_l2norm=True),
    dict(read_mode="pre", reverse=False, qk_l2norm=True),
    dict(read_mode="post", reverse=True, qk_l2norm=False),
    dict(read_mode="pre", reverse=True, qk_l2norm=True),
]


@pytest.mark.parametrize("kw", CASES, ids=lambda c: f"{c['read_mode']}-rev{int(c['reverse'])}-l2{int(c['qk_l2norm'])}")
def test_finite_differences(kw):
    """Every gradient entry equals the central difference of the forward oracle's loss."""
    x, up, cu = problem(1, 0, 1, 2, 3, 2, lengths=[3, 1, 4])
    got = oracle_grads(x, up, cu, scale=0.7, **kw)
    want = fd_grads(x, up, cu, scale=0.7, **kw)
    for name, ref in want.items():
        np.testing.assert_allclose(got[name], ref, rtol=1e-6, atol=1e-7, err_msg=name)


def test_finite_differences_batched_gqa():
    x, up, cu = problem(2, 4, 1, 3, 2, 3)
    got = oracle_grads(x, up, None, scale=1.3, read_mode="post", qk_l2norm=True)
    want = fd_grads(x, up, None, scale=1.3, read_mode="post", qk_l2norm=True)
    for name, ref in want.items():
        np.testing.assert_allclose(got[name], ref, rtol=1e-6, atol=1e-7, err_msg=name)


def _torch_loss(x, up, read_mode, scale, group, cu):
    """The recurrence as a plain fp64 PyTorch loop (autograd takes its derivative)."""
    q, k, v, g, beta, S0 = (x[n] for n in ("q", "k", "v", "g", "beta", "S0"))
    total = 0.0
    B, T = q.shape[:2]
    segs = [(b, 0, T) for b in range(B)] if cu is None else [
        (0, int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1)]
    for si, (b, t0, t1) in enumerate(segs):
        H = S0[si].clone()
        for t in range(t0, t1):
            kh = torch.nn.functional.normalize(k[b, t], dim=-1, eps=1e-6).repeat_interleave(group, 0)
            qh = torch.nn.functional.normalize(q[b, t], dim=-1, eps=1e-6).repeat_interleave(group, 0)
            a = torch.exp(g[b, t])
            if read_mode == "pre":
                total = total + (up["dO"][b, t] * scale * torch.einsum("hd,hde->he", qh, H)).sum()
            u = beta[b, t][:, None] * (v[b, t] - a[:, None] * torch.einsum("hd,hde->he", kh, H))
            H = a[:, None, None] * H + kh[:, :, None] * u[:, None, :]
            if read_mode == "post":
                total = total + (up["dO"][b, t] * scale * torch.einsum("hd,hde->he", qh, H)).sum()
        total = total + (up["dS_final"][si] * H).sum()
    return total


@pytest.mark.parametrize("read_mode", ["post", "pre"])
def test_autograd_of_plain_loop(read_mode):
    """Against PyTorch autograd of the recurrence written as a plain loop, at a size with
    several checkpoint blocks."""
    x, up, cu = problem(1, 0, 2, 4, 8, 6, lengths=[13, 0, 21, 5])
    got = oracle_grads(x, up, cu, scale=0.4, read_mode=read_mode, qk_l2norm=True, ckpt=4)
    tx = {n: torch.tensor(a, requires_grad=True) for n, a in x.items()}
    tup = {n: torch.tensor(a) for n, a in up.items()}
    _torch_loss(tx, tup, read_mode, 0.4, 2, cu).backward()
    for n in ("q", "k", "v", "g", "beta", "S0"):
        np.testing.assert_allclose(got["d" + n], tx[n].grad.numpy(), rtol=1e-9, atol=1e-11,
                                   err_msg=n)


def test_decay_only_closed_form():
    """beta = 0: S_t = e^{G_t} S0 and o_t = scale e^{G_t} S0^T q^_t (post), so
    dS0 = sum_t scale e^{G_t} q^_t do_t^T + e^{G_T} dS_T,
    dg_j = sum_{t>=j} scale e^{G_t} do_t . (S0^T q^_t) + e^{G_T} <dS_T, S0>, dv = 0."""
    x, up, _ = problem(1, 7, 1, 1, 4, 3)
    x["beta"][:] = 0.0
    r = oracle_grads(x, up, None, scale=0.9, read_mode="post", qk_l2norm=True)
    q = x["q"][0, :, 0]
    qh = q / np.linalg.norm(q, axis=-1, keepdims=True)
    G = np.cumsum(x["g"][0, :, 0])
    S0, dST, do = x["S0"][0, 0], up["dS_final"][0, 0], up["dO"][0, :, 0]
    dS0 = sum(0.9 * np.exp(G[t]) * np.outer(qh[t], do[t]) for t in range(7)) + np.exp(G[-1]) * dST
    np.testing.assert_allclose(r["dS0"][0, 0], dS0, rtol=1e-12, atol=1e-13)
    per_t = np.array([0.9 * np.exp(G[t]) * do[t] @ (S0.T @ qh[t]) for t in range(7)])
    dg = np.cumsum(per_t[::-1])[::-1] + np.exp(G[-1]) * np.sum(dST * S0)
    np.testing.assert_allclose(r["dg"][0, :, 0], dg, rtol=1e-12, atol=1e-13)
    assert np.all(r["dv"] == 0)


def test_checkpoint_invariance():
    """Recomputing states from checkpoints gives the same numbers as one stored pass."""
    x, up, cu = problem(1, 0, 1, 2, 5, 4, lengths=[9, 17])
    a = oracle_grads(x, up, cu, scale=0.5, ckpt=1000)
    b = oracle_grads(x, up, cu, scale=0.5, ckpt=3)
    for n in a:
        np.testing.assert_array_equal(a[n], b[n])


def test_finite_differences_random_shapes():
    """Random small shapes and options (key/value head counts, head sizes, varlen or batched,
    both read modes, reversal, normalisation on or off, a state or none): every gradient
    entry against central differences of the forward oracle."""
    hyp = pytest.importorskip("hypothesis")
    st = hyp.strategies

    @hyp.settings(max_examples=12, deadline=None, derandomize=True)
    @hyp.given(hk=st.integers(1, 2), group=st.integers(1, 2), dk=st.integers(1, 3),
               dv=st.integers(1, 3), lens=st.lists(st.integers(0, 4), min_size=1, max_size=3),
               varlen=st.booleans(), pre=st.booleans(), rev=st.booleans(), l2=st.booleans(),
               s0=st.booleans(), scale=st.floats(0.25, 2.0))
    def check(hk, group, dk, dv, lens, varlen, pre, rev, l2, s0, scale):
        if varlen:
            x, up, cu = problem(1, 0, hk, hk * group, dk, dv, lengths=lens, s0=s0)
        else:
            x, up, cu = problem(len(lens), max(lens), hk, hk * group, dk, dv, s0=s0)
        kw = dict(read_mode="pre" if pre else "post", reverse=rev, qk_l2norm=l2, scale=scale)
        got = oracle_grads(x, up, cu, **kw)
        want = fd_grads(x, up, cu, **kw)
        for name, ref in want.items():
            np.testing.assert_allclose(got[name], ref, rtol=1e-5, atol=1e-6, err_msg=name)

    check()
