"""The seeded input generator follows the recipe the workloads state: same seed, same
tensors; the stated distributions; valid packed layouts."""
import math

import numpy as np
import torch

import workloads


def test_same_seed_same_tensors_and_different_seed_differs():
    a = workloads.chunk_inputs(2, 70, 1, 2, 16, 8, "bf16", s0_std=0.02, seed=5)
    b = workloads.chunk_inputs(2, 70, 1, 2, 16, 8, "bf16", s0_std=0.02, seed=5)
    c = workloads.chunk_inputs(2, 70, 1, 2, 16, 8, "bf16", s0_std=0.02, seed=6)
    for n in ("q", "k", "v", "g", "beta", "S0"):
        assert torch.equal(a[n], b[n]), n
    assert not torch.equal(a["q"], c["q"])


def test_distributions():
    x = workloads.chunk_inputs(1, 20000, 1, 4, 8, 8, "f32", s0_std=0.02, seed=0)
    for n in ("q", "k", "v"):
        t = x[n].double()
        assert abs(t.mean().item()) < 0.02 and abs(t.std().item() - 1.0) < 0.02, n
    alpha = torch.exp(x["g"].double())
    assert (alpha > 0).all() and (alpha < 1).all()
    # g = -softplus(N(-2, 1)): median alpha = exp(-softplus(-2)) ~ 0.881
    assert abs(alpha.median().item() - math.exp(-math.log1p(math.exp(-2.0)))) < 0.01
    beta = x["beta"].double()
    assert (beta > 0).all() and (beta < 1).all() and abs(beta.median().item() - 0.5) < 0.01
    assert abs(x["S0"].std().item() - 0.02) < 0.002


def test_packed_layouts():
    w = workloads.WORKLOADS["bf16_varlen64_h16_d128"]
    gen = torch.Generator("cpu").manual_seed(0)
    lengths = torch.randint(w.len_lo, w.len_hi + 1, (w.n_varlen,), generator=gen)
    assert lengths.min() >= 256 and lengths.max() <= 8192
    x = workloads.chunk_inputs(1, 0, 1, 1, 4, 4, "bf16", lengths=[3, 0, 5], seed=1)
    cu = x["cu_seqlens"]
    assert cu.dtype == torch.int32 and cu.tolist() == [0, 3, 3, 8]
    assert x["q"].shape == (1, 8, 1, 4)
    y = workloads.chunk_inputs(1, 0, 2, 2, 4, 4, "bf16", lengths=[4, 4], bidirectional=True,
                               seed=2)
    assert y["g_bwd"].shape == y["g"].shape and not torch.equal(y["g_bwd"], y["g"])


def test_gdn2_and_raw_gate_inputs():
    g, b, w = workloads.gdn2_gate_inputs((2, 50, 3), 16, 8, "f32", seed=3)
    assert g.shape == (2, 50, 3, 16) and b.shape == g.shape and w.shape == (2, 50, 3, 8)
    assert (g < 0).all() and ((b > 0) & (b < 1)).all() and ((w > 0) & (w < 1)).all()
    a, bb, A, dt = workloads.raw_gate_inputs((1, 4000, 2), 2, "f32", seed=4)
    assert torch.equal(A, torch.full((2,), -1.0)) and torch.equal(dt, torch.zeros(2))
    # with A = -1, dt = 0 the formed gates follow the direct gates' distributions
    alpha = torch.exp(-torch.nn.functional.softplus(a.double()))
    assert abs(alpha.median().item() - 0.881) < 0.02
    assert abs(torch.sigmoid(bb.double()).median().item() - 0.5) < 0.02


def test_decode_inputs():
    x = workloads.decode_inputs(4, 2, 4, 16, 8, steps=3, seed=0)
    assert x["q"].shape == (3, 4, 2, 16) and x["v"].shape == (3, 4, 4, 8)
    assert x["g"].shape == (3, 4, 4) and x["S"].shape == (4, 4, 16, 8)
    assert x["S"].dtype == torch.float32
