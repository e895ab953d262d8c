"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own loop: each compares it with an
independent route to the same number (exact rational product form, the
chunk-parallel WY/UT form, closed forms, invariants of the recurrence).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact, wy_reference

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "exact_small.json")
RNG = np.random.default_rng(1234)


def rand_problem(B=1, T=64, Hk=2, Hv=2, dk=16, dv=16, rng=None, s0=False, alpha=None,
                 beta_max=1.0):
    rng = rng or np.random.default_rng(0)
    q = rng.standard_normal((B, T, Hk, dk))
    k = rng.standard_normal((B, T, Hk, dk))
    v = rng.standard_normal((B, T, Hv, dv))
    if alpha is None:
        g = -np.log1p(np.exp(rng.standard_normal((B, T, Hv)) - 2.0))
    else:
        g = np.full((B, T, Hv), math.log(alpha))
    beta = beta_max / (1.0 + np.exp(-rng.standard_normal((B, T, Hv))))
    S0 = rng.standard_normal((B, Hv, dk, dv)) * 0.5 if s0 else None
    return q, k, v, g, beta, S0


# --------------------------------------------------------------------------- exact

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def _run_exact_case(c, lib=None):
    fr = lambda rows: np.array([[float(Fraction(x)) for x in r] for r in rows])
    q, k, v = fr(c["q"]), fr(c["k"]), fr(c["v"])
    alpha = np.array([float(Fraction(x)) for x in c["alpha"]])
    beta = np.array([float(Fraction(x)) for x in c["beta"]])
    H0 = fr(c["H0"])
    o, S = oracle.forward(q[None, :, None], k[None, :, None], v[None, :, None],
                          np.log(alpha)[None, :, None], beta[None, :, None], H0[None, None],
                          read_mode=c["read_mode"], scale=float(Fraction(c["scale"])),
                          qk_l2norm=c["qk_l2norm"], _lib=lib)
    return o[0, :, 0], S[0, 0]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_matches_exact_golden(case):
    """Stored exact values (tests/golden/exact_small.json) to 1e-13 relative."""
    o, S = _run_exact_case(case)
    o_ref = np.array([[float(Fraction(x)) for x in r] for r in case["o"]])
    S_ref = np.array([[float(Fraction(x)) for x in r] for r in case["H_final"]])
    tol = 1e-13 * max(1.0, np.abs(o_ref).max(), np.abs(S_ref).max())
    assert np.abs(o - o_ref).max() <= tol
    assert np.abs(S - S_ref).max() <= tol


PYTH = [(1, 2, 2), (2, 1, 2), (2, 2, 1), (2, 3, 6), (3, 6, 2), (6, 2, 3), (1, 4, 8), (4, 4, 7),
        (2, 6, 9), (0, 3, 4), (4, 0, 3), (-1, 2, -2), (2, -3, 6), (-6, 2, 3), (8, -4, 1)]


def _random_rational_case(seed, read_mode, l2norm, T=7):
    r = np.random.default_rng(seed)
    dk = 3
    dv = int(r.integers(1, 4))
    if l2norm:
        q = [list(PYTH[i]) for i in r.integers(0, len(PYTH), T)]
        k = [list(PYTH[i]) for i in r.integers(0, len(PYTH), T)]
    else:
        q = r.integers(-3, 4, (T, dk)).tolist()
        k = r.integers(-2, 3, (T, dk)).tolist()
    v = r.integers(-4, 5, (T, dv)).tolist()
    alpha = [Fraction(int(a), 16) for a in r.integers(4, 17, T)]
    beta = [Fraction(int(b), 8) for b in r.integers(0, 16, T)]
    H0 = [[Fraction(int(x), 8) for x in row] for row in r.integers(-8, 9, (dk, dv))]
    scale = Fraction(int(r.integers(1, 5)), 4)
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta, H0=H0, read_mode=read_mode,
                scale=scale, qk_l2norm=l2norm)


def _check_vs_exact(c, lib=None):
    o_ex, H_ex = exact.forward_exact(c["q"], c["k"], c["v"], c["alpha"], c["beta"], c["H0"],
                                     read_mode=c["read_mode"], scale=c["scale"],
                                     qk_l2norm=c["qk_l2norm"])
    cc = dict(c)
    cc["q"] = [[str(x) for x in r] for r in c["q"]]
    cc["k"] = [[str(x) for x in r] for r in c["k"]]
    cc["v"] = [[str(x) for x in r] for r in c["v"]]
    cc["alpha"] = [str(x) for x in c["alpha"]]
    cc["beta"] = [str(x) for x in c["beta"]]
    cc["H0"] = [[str(x) for x in r] for r in c["H0"]]
    cc["scale"] = str(c["scale"])
    o, S = _run_exact_case(cc, lib=lib)
    o_ref = np.array([[float(x) for x in r] for r in o_ex])
    S_ref = np.array([[float(x) for x in r] for r in H_ex])
    tol = 1e-13 * max(1.0, np.abs(o_ref).max(), np.abs(S_ref).max())
    return np.abs(o - o_ref).max() <= tol and np.abs(S - S_ref).max() <= tol


@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("l2norm", [False, True])
def test_brute_force_exact_small(read_mode, l2norm):
    """T<=8 against exact rational arithmetic (product of transitions), 12 random cases."""
    for seed in range(12):
        c = _random_rational_case(seed, read_mode, l2norm, T=1 + seed % 8)
        assert _check_vs_exact(c), f"seed {seed}"


# ------------------------------------------------------------------ WY/UT form

@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("read_mode", ["post", "pre"])
def test_matches_wy_form_all_chunks(chunk, read_mode):
    """Chunk-parallel WY/UT form (any chunk size) = per-token oracle to 1e-10 (fp64)."""
    q, k, v, g, beta, S0 = rand_problem(B=2, T=200, Hk=2, Hv=4, dk=32, dv=24, s0=True,
                                        rng=np.random.default_rng(chunk))
    o, S = oracle.forward(q, k, v, g, beta, S0, read_mode=read_mode, scale=0.7)
    o2, S2 = wy_reference.chunked_forward(q, k, v, g, beta, S0, chunk=chunk,
                                          read_mode=read_mode, scale=0.7)
    assert np.abs(o - o2).max() < 1e-10
    assert np.abs(S - S2).max() < 1e-10


def test_oracle_sized_workload_vs_wy():
    """The fp32 oracle-sized workload (T=256, d=64, two heads) at chunk 64."""
    import workloads
    w = workloads.WORKLOADS["fp32_b1_h2_t256_d64"]
    x = workloads.workload_inputs(w)
    o, S = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], None,
                          read_mode="post", scale=w.scale)
    f64 = lambda t: t.double().numpy()
    o2, S2 = wy_reference.chunked_forward(*(f64(x[n]) for n in ("q", "k", "v", "g", "beta")),
                                          chunk=64, read_mode="post", scale=w.scale)
    assert np.abs(o - o2).max() < 1e-10 and np.abs(S - S2).max() < 1e-10


@pytest.mark.parametrize("chunk", [64, 128])
def test_alpha_half_floor(chunk):
    """alpha == 0.5 for every token: gamma reaches 2^-128 inside a 128-chunk, which only
    survives in log space (the page's 'gated.5floor' case)."""
    q, k, v, g, beta, S0 = rand_problem(T=300, dk=16, dv=16, alpha=0.5, s0=True)
    o, S = oracle.forward(q, k, v, g, beta, S0)
    o2, S2 = wy_reference.chunked_forward(q, k, v, g, beta, S0, chunk=chunk)
    assert np.abs(o - o2).max() < 1e-10 and np.abs(S - S2).max() < 1e-10


def test_repeated_keys_and_rectangular():
    """All tokens share one key; and dk != dv (48 x 16), both against the WY form."""
    r = np.random.default_rng(99)
    q, k, v, g, beta, _ = rand_problem(T=64, dk=16, dv=16, rng=r)
    k[:] = k[:, :1]
    o, S = oracle.forward(q, k, v, g, beta, None, read_mode="pre")
    o2, S2 = wy_reference.chunked_forward(q, k, v, g, beta, None, chunk=32, read_mode="pre")
    assert np.abs(o - o2).max() < 1e-10 and np.abs(S - S2).max() < 1e-10
    q, k, v, g, beta, S0 = rand_problem(B=2, T=200, Hk=3, Hv=3, dk=48, dv=16, rng=r, s0=True)
    o, S = oracle.forward(q, k, v, g, beta, S0)
    o2, S2 = wy_reference.chunked_forward(q, k, v, g, beta, S0, chunk=64)
    assert np.abs(o - o2).max() < 1e-10 and np.abs(S - S2).max() < 1e-10


# -------------------------------------------------------------- closed forms

def test_exact_overwrite_orthonormal_keys():
    """alpha = beta = 1 with orthonormal keys: the state then maps every k_i to v_i
    (S k_i = v_i), and from S0 = 0 it is exactly sum_i k_i v_i^T."""
    r = np.random.default_rng(7)
    dk, dv, m = 32, 20, 24
    Qm, _ = np.linalg.qr(r.standard_normal((dk, dk)))
    keys = Qm[:, :m].T  # m orthonormal rows
    v = r.standard_normal((1, m, 1, dv))
    q = r.standard_normal((1, m, 1, dk))
    g = np.zeros((1, m, 1))
    beta = np.ones((1, m, 1))
    S0 = r.standard_normal((1, 1, dk, dv))
    _, S = oracle.forward(q, keys[None, :, None], v, g, beta, S0, qk_l2norm=False)
    H = S[0, 0]
    for i in range(m):
        assert np.abs(H.T @ keys[i] - v[0, i, 0]).max() < 1e-12
    _, S = oracle.forward(q, keys[None, :, None], v, g, beta, None, qk_l2norm=False)
    assert np.abs(S[0, 0] - keys.T @ v[0, :, 0]).max() < 1e-12


def test_decay_only_and_identity():
    """beta = 0: S_T = exp(sum g) S0 and o_t = scale exp(G_t) S0 q_t (post).
    beta = 0 and g = 0: the state passes through unchanged (tiny_gdn/fugue.py: a slot
    with zero key and decay leaves the state as it was)."""
    q, k, v, g, beta, S0 = rand_problem(T=40, dk=8, dv=6, s0=True)
    beta[:] = 0
    o, S = oracle.forward(q, k, v, g, beta, S0, scale=0.5, qk_l2norm=False)
    G = np.cumsum(g[0, :, 0])
    assert np.abs(S[0, 0] - np.exp(G[-1]) * S0[0, 0]).max() < 1e-13
    expect = 0.5 * np.exp(G)[:, None] * (q[0, :, 0] @ S0[0, 0])
    assert np.abs(o[0, :, 0] - expect).max() < 1e-12
    g[:] = 0
    o, S = oracle.forward(q, k, v, g, beta, S0, read_mode="pre", qk_l2norm=False)
    assert np.array_equal(S[0, 0], S0[0, 0])
    assert np.abs(o[0, :, 0] - q[0, :, 0] @ S0[0, 0]).max() < 1e-13


def test_one_token_both_reads():
    """T = 1: the post read sees the written state, the pre read sees S0 only."""
    q, k, v, g, beta, S0 = rand_problem(T=1, dk=8, dv=8, s0=True)
    o_pre, S1 = oracle.forward(q, k, v, g, beta, S0, read_mode="pre", qk_l2norm=False)
    o_post, S1b = oracle.forward(q, k, v, g, beta, S0, read_mode="post", qk_l2norm=False)
    assert np.array_equal(S1, S1b)
    assert np.abs(o_pre[0, 0, 0] - q[0, 0, 0] @ S0[0, 0]).max() < 1e-13
    assert np.abs(o_post[0, 0, 0] - q[0, 0, 0] @ S1[0, 0]).max() < 1e-13


def test_linear_in_values_from_zero_state():
    """With S0 = 0 both o and S_T are linear in V (u_t is linear in v and S)."""
    q, k, v, g, beta, _ = rand_problem(T=50, dk=8, dv=8)
    v2 = np.random.default_rng(5).standard_normal(v.shape)
    o1, S1 = oracle.forward(q, k, v, g, beta)
    o2, S2 = oracle.forward(q, k, v2, g, beta)
    o3, S3 = oracle.forward(q, k, v + 2 * v2, g, beta)
    assert np.abs(o3 - (o1 + 2 * o2)).max() < 1e-12
    assert np.abs(S3 - (S1 + 2 * S2)).max() < 1e-12


# --------------------------------------------------------------- structure

def test_varlen_equals_separate_calls():
    r = np.random.default_rng(3)
    lens = [5, 64, 1, 0, 77]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v, g, beta, _ = rand_problem(T=T, Hk=1, Hv=2, dk=8, dv=4, rng=r)
    S0 = r.standard_normal((len(lens), 2, 8, 4))
    o, S = oracle.forward(q, k, v, g, beta, S0, cu_seqlens=cu, read_mode="pre")
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        if b == a:
            assert np.array_equal(S[s], S0[s])
            continue
        o1, S1 = oracle.forward(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b],
                                S0[s:s + 1], read_mode="pre")
        assert np.array_equal(o[:, a:b], o1) and np.array_equal(S[s], S1[0])


def test_gqa_equals_repeated_heads():
    q, k, v, g, beta, S0 = rand_problem(T=30, Hk=2, Hv=6, dk=8, dv=4, s0=True)
    o, S = oracle.forward(q, k, v, g, beta, S0)
    qr, kr = np.repeat(q, 3, axis=2), np.repeat(k, 3, axis=2)
    o2, S2 = oracle.forward(qr, kr, v, g, beta, S0)
    assert np.array_equal(o, o2) and np.array_equal(S, S2)


def test_reverse_equals_flipped_segments():
    """reverse=True scans each segment back to front in place; the same as flipping every
    segment on the host, scanning forward, and flipping the output back.  Reversal applied
    twice is the identity (tiny_gdn/fugue.py segment_layout.reverse_index)."""
    lens = [7, 20, 13]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, g, beta, _ = rand_problem(T=int(cu[-1]), dk=8, dv=8)
    rev = np.concatenate([np.arange(cu[s + 1] - 1, cu[s] - 1, -1) for s in range(len(lens))])
    assert np.array_equal(rev[rev], np.arange(cu[-1]))
    o, S = oracle.forward(q, k, v, g, beta, None, cu_seqlens=cu, read_mode="pre", reverse=True)
    flip = lambda x: x[:, rev]
    o2, S2 = oracle.forward(flip(q), flip(k), flip(v), flip(g), flip(beta), None, cu_seqlens=cu,
                            read_mode="pre")
    assert np.array_equal(o, flip(o2)) and np.array_equal(S, S2)


@pytest.mark.parametrize("split", [1, 37, 64, 99])
def test_continuation(split):
    """S_final of a call fed as S0 of the next equals one call over the whole sequence."""
    q, k, v, g, beta, S0 = rand_problem(T=100, dk=8, dv=8, s0=True)
    o, S = oracle.forward(q, k, v, g, beta, S0)
    sl1, sl2 = slice(0, split), slice(split, 100)
    o1, S1 = oracle.forward(q[:, sl1], k[:, sl1], v[:, sl1], g[:, sl1], beta[:, sl1], S0)
    o2, S2 = oracle.forward(q[:, sl2], k[:, sl2], v[:, sl2], g[:, sl2], beta[:, sl2], S1)
    assert np.abs(np.concatenate([o1, o2], axis=1) - o).max() < 1e-13
    assert np.abs(S2 - S).max() < 1e-13


def test_decode_steps_equal_forward():
    """64 one-token decode steps from S0 equal one forward over the 64 tokens."""
    q, k, v, g, beta, S0 = rand_problem(B=3, T=64, Hk=1, Hv=2, dk=8, dv=8, s0=True)
    o, S = oracle.forward(q, k, v, g, beta, S0)
    St = S0
    for t in range(64):
        ot, St = oracle.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], St)
        assert np.abs(ot - o[:, t]).max() < 1e-13
    assert np.abs(St - S).max() < 1e-13


def test_matches_wy_form_random_shapes():
    """Random shapes, GQA groups, chunk sizes, varlen layouts, read modes and reversal: the
    per-token C oracle against the NumPy WY/UT chunk form."""
    hyp = pytest.importorskip("hypothesis")
    st = hyp.strategies

    @hyp.settings(max_examples=25, deadline=None, derandomize=True)
    @hyp.given(hk=st.integers(1, 3), group=st.integers(1, 3), dk=st.integers(1, 9),
               dv=st.integers(1, 7), lens=st.lists(st.integers(0, 50), min_size=1, max_size=4),
               varlen=st.booleans(), chunk=st.sampled_from([1, 2, 5, 16, 64]),
               pre=st.booleans(), rev=st.booleans(), l2=st.booleans(), seed=st.integers(0, 999))
    def check(hk, group, dk, dv, lens, varlen, chunk, pre, rev, l2, seed):
        r = np.random.default_rng(seed)
        Hv = hk * group
        if varlen:
            B, T = 1, sum(lens)
            cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
            n = len(lens)
        else:
            B, T, cu, n = len(lens), max(lens), None, len(lens)
        q, k = r.normal(size=(B, T, hk, dk)), r.normal(size=(B, T, hk, dk))
        v = r.normal(size=(B, T, Hv, dv))
        g = -np.log1p(np.exp(r.normal(-2, 1, (B, T, Hv))))
        beta = 1 / (1 + np.exp(-r.normal(size=(B, T, Hv))))
        S0 = 0.3 * r.normal(size=(n, Hv, dk, dv))
        kw = dict(read_mode="pre" if pre else "post", scale=0.7, qk_l2norm=l2, reverse=rev)
        o, S = oracle.forward(q, k, v, g, beta, S0, cu, **kw)
        o2, S2 = wy_reference.chunked_forward(q, k, v, g, beta, S0, cu, chunk=chunk, **kw)
        assert np.abs(o - o2).max(initial=0.0) < 1e-9 and np.abs(S - S2).max(initial=0.0) < 1e-9

    check()


@pytest.mark.parametrize("read_mode,read_mode_bwd,combine", [("pre", None, 1.0),
                                                             ("post", "pre", 0.5)])
def test_bidirectional_is_forward_plus_host_flipped_scan(read_mode, read_mode_bwd, combine):
    """oracle.bidirectional against an independent assembly of its two directions
    (Rondo-Exp tiny_gdn/fugue.py, BidirectionalGatedDeltaNet2.forward and scan): the
    forward direction is the NumPy WY/UT form with (g_fwd, beta_fwd); the backward
    direction flips every segment on the host, runs the same WY form FORWARD with
    (g_bwd, beta_bwd), and flips the output back; the two are summed and scaled by the
    combine factor.  Neither the C oracle nor its reversal flag is used on this side."""
    lens = [9, 1, 30, 17]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(77)
    q, k, v, g_f, b_f, _ = rand_problem(T=int(cu[-1]), Hk=1, Hv=2, dk=8, dv=6, rng=rng)
    g_b = -np.log1p(np.exp(rng.standard_normal(g_f.shape) - 1.0))
    b_b = 1.5 / (1.0 + np.exp(-rng.standard_normal(b_f.shape)))
    got = oracle.bidirectional(q, k, v, g_f, b_f, g_b, b_b, cu, read_mode=read_mode,
                               scale=0.6, read_mode_bwd=read_mode_bwd, combine=combine)
    rev = np.concatenate([np.arange(cu[s + 1] - 1, cu[s] - 1, -1) for s in range(len(lens))])
    flip = lambda x: x[:, rev]
    o_f, _ = wy_reference.chunked_forward(q, k, v, g_f, b_f, None, cu, chunk=8,
                                          read_mode=read_mode, scale=0.6)
    o_b, _ = wy_reference.chunked_forward(flip(q), flip(k), flip(v), flip(g_b), flip(b_b), None,
                                          cu, chunk=8, read_mode=read_mode_bwd or read_mode,
                                          scale=0.6)
    want = combine * (o_f + flip(o_b))
    assert np.abs(got - want).max() < 1e-10
    # the directions are not interchangeable: swapping the gate pairs changes the result,
    # and so does dropping either direction
    swapped = oracle.bidirectional(q, k, v, g_b, b_b, g_f, b_f, cu, read_mode=read_mode,
                                   scale=0.6, read_mode_bwd=read_mode_bwd, combine=combine)
    assert np.abs(swapped - want).max() > 1e-3
    assert np.abs(combine * o_f - want).max() > 1e-3
    assert np.abs(combine * flip(o_b) - want).max() > 1e-3
