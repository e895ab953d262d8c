"""Pins of the fp64 GDN-2 oracle ``oracle.gdn2_forward`` (decoupled gates: per key channel
log decay g and erase gate b, per value channel write gate w; Rondo-Exp tiny_gdn/fugue.py
BidirectionalGatedDeltaNet2):
- an independent chunk-parallel (WY/UT) form, at several chunk sizes and both read modes;
- the scalar gated delta rule (the C oracle) when the gates are the same on every channel,
  with GQA, varlen, reversal and an initial state;
- closed forms: decay only (b = w = 0), decayed accumulation without erase (b = 0), and the
  product of transitions (I - k (b k)^T) Diag(e^g) when nothing is written (w = 0)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import gdn2_chunked

RNG = np.random.default_rng(7)


def gates(shape_k, shape_v):
    g = -np.log1p(np.exp(RNG.normal(-2, 1, shape_k)))
    b = 1 / (1 + np.exp(-RNG.normal(0, 1, shape_k)))
    w = 1 / (1 + np.exp(-RNG.normal(0, 1, shape_v)))
    return g, b, w


@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("chunk", [4, 16, 64])
def test_matches_chunked_form(read_mode, chunk):
    B, T, H, dk, dv = 2, 45, 2, 8, 6
    q, k = RNG.normal(size=(B, T, H, dk)), RNG.normal(size=(B, T, H, dk))
    v = RNG.normal(size=(B, T, H, dv))
    g, b, w = gates((B, T, H, dk), (B, T, H, dv))
    S0 = 0.3 * RNG.normal(size=(B, H, dk, dv))
    o1, S1 = oracle.gdn2_forward(q, k, v, g, b, w, S0, read_mode=read_mode, scale=0.7)
    o2, S2 = gdn2_chunked.forward(q, k, v, g, b, w, S0, chunk=chunk, read_mode=read_mode,
                                  scale=0.7)
    assert np.abs(o1 - o2).max() < 1e-12 and np.abs(S1 - S2).max() < 1e-12


@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("reverse", [False, True])
def test_scalar_gates_reduce_to_gated_delta_rule(read_mode, reverse):
    Hk, Hv, dk, dv = 2, 4, 8, 5
    lengths = [7, 0, 13, 20]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    T = int(cu[-1])
    q, k = RNG.normal(size=(1, T, Hk, dk)), RNG.normal(size=(1, T, Hk, dk))
    v = RNG.normal(size=(1, T, Hv, dv))
    alpha = RNG.uniform(0.5, 1.0, (1, T, Hv))
    beta = RNG.uniform(0.0, 1.5, (1, T, Hv))
    S0 = 0.2 * RNG.normal(size=(len(lengths), Hv, dk, dv))
    g = np.repeat(np.log(alpha)[..., None], dk, -1)
    b = np.repeat(beta[..., None], dk, -1)
    w = np.repeat(beta[..., None], dv, -1)
    o1, S1 = oracle.gdn2_forward(q, k, v, g, b, w, S0, cu, read_mode=read_mode, scale=0.5,
                                 reverse=reverse)
    o2, S2 = oracle.forward(q, k, v, np.log(alpha), beta, S0, cu, read_mode=read_mode,
                            scale=0.5, reverse=reverse)
    assert np.abs(o1 - o2).max() < 1e-12 and np.abs(S1 - S2).max() < 1e-12


def test_decay_only_and_accumulation_closed_forms():
    B, T, H, dk, dv = 1, 9, 1, 4, 3
    q, k = RNG.normal(size=(B, T, H, dk)), RNG.normal(size=(B, T, H, dk))
    v = RNG.normal(size=(B, T, H, dv))
    g, _, w = gates((B, T, H, dk), (B, T, H, dv))
    S0 = RNG.normal(size=(B, H, dk, dv))
    # b = w = 0: H_T = Diag(e^{sum g}) H_0
    _, S = oracle.gdn2_forward(q, k, v, g, np.zeros_like(g), np.zeros_like(w), S0,
                               qk_l2norm=False)
    assert np.allclose(S[0, 0], np.exp(g[0, :, 0].sum(0))[:, None] * S0[0, 0], rtol=1e-13)
    # b = 0: H_T = Diag(e^{G_T}) H_0 + sum_t Diag(e^{G_T - G_t}) k_t (w_t v_t)^T
    _, S = oracle.gdn2_forward(q, k, v, g, np.zeros_like(g), w, S0, qk_l2norm=False)
    G = np.cumsum(g[0, :, 0], 0)
    ref = np.exp(G[-1])[:, None] * S0[0, 0]
    for t in range(T):
        ref += np.outer(np.exp(G[-1] - G[t]) * k[0, t, 0], w[0, t, 0] * v[0, t, 0])
    assert np.allclose(S[0, 0], ref, rtol=1e-12, atol=1e-14)


def test_product_of_transitions_without_writes():
    """w = 0: S_T = prod_t (I - k_t (b_t k_t)^T) Diag(e^{g_t}) S_0, in S = H layout."""
    B, T, H, dk, dv = 1, 11, 1, 5, 4
    q, k = RNG.normal(size=(B, T, H, dk)), RNG.normal(size=(B, T, H, dk))
    v = RNG.normal(size=(B, T, H, dv))
    g, b, w = gates((B, T, H, dk), (B, T, H, dv))
    S0 = RNG.normal(size=(B, H, dk, dv))
    o, S = oracle.gdn2_forward(q, k, v, g, b, np.zeros_like(w), S0, read_mode="post",
                               scale=1.0, qk_l2norm=False)
    M = S0[0, 0].copy()
    for t in range(T):
        kt = k[0, t, 0]
        M = (np.eye(dk) - np.outer(kt, b[0, t, 0] * kt)) @ np.diag(np.exp(g[0, t, 0])) @ M
        assert np.allclose(o[0, t, 0], q[0, t, 0] @ M, rtol=1e-11, atol=1e-12)
    assert np.allclose(S[0, 0], M, rtol=1e-11, atol=1e-12)


def test_matches_chunked_form_random_shapes():
    """Random shapes, chunk sizes and read modes: the per-token GDN-2 oracle against the
    independent chunked form."""
    hyp = pytest.importorskip("hypothesis")
    st = hyp.strategies

    @hyp.settings(max_examples=20, deadline=None, derandomize=True)
    @hyp.given(B=st.integers(1, 2), T=st.integers(1, 40), H=st.integers(1, 2),
               dk=st.integers(1, 6), dv=st.integers(1, 5), chunk=st.sampled_from([1, 3, 8, 16]),
               pre=st.booleans(), s0=st.booleans(), seed=st.integers(0, 1000))
    def check(B, T, H, dk, dv, chunk, pre, s0, seed):
        r = np.random.default_rng(seed)
        q, k = r.normal(size=(B, T, H, dk)), r.normal(size=(B, T, H, dk))
        v = r.normal(size=(B, T, H, dv))
        g = -np.log1p(np.exp(r.normal(-2, 1, (B, T, H, dk))))
        b = 1 / (1 + np.exp(-r.normal(0, 1, (B, T, H, dk))))
        w = 1 / (1 + np.exp(-r.normal(0, 1, (B, T, H, dv))))
        S0 = 0.3 * r.normal(size=(B, H, dk, dv)) if s0 else None
        mode = "pre" if pre else "post"
        o1, S1 = oracle.gdn2_forward(q, k, v, g, b, w, S0, read_mode=mode, scale=0.7)
        o2, S2 = gdn2_chunked.forward(q, k, v, g, b, w, S0, chunk=chunk, read_mode=mode,
                                      scale=0.7)
        assert np.abs(o1 - o2).max() < 1e-11 and np.abs(S1 - S2).max() < 1e-11

    check()
