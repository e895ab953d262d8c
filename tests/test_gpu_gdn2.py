"""GPU parity of GDN-2 (decoupled gates: per-key-channel decay and erase gate, per-value-
channel write gate; Rondo-Exp ``tiny_gdn/fugue.py``, ``BidirectionalGatedDeltaNet2``) on the
chunked CUDA-core path and the decode step, against the fp64 per-token oracle
``oracle.gdn2_forward``."""
import math

import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
from gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def run_chunk(x, g, b, w, **kw):
    o, S = gdr.chunk_fwd(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), to_dev(g), to_dev(b),
                         to_dev(x["S0"]) if x["S0"] is not None else None,
                         to_dev(x["cu_seqlens"]) if x["cu_seqlens"] is not None else None,
                         gdn2_w=to_dev(w), **kw)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("read_mode", ["post", "pre"])
def test_chunk(dtype, read_mode):
    x = workloads.chunk_inputs(2, 150, 2, 4, 128, 128, dtype, s0_std=0.05, seed=51)
    g, b, w = workloads.gdn2_gate_inputs(x["v"].shape[:3], 128, 128, dtype, seed=52)
    args = gdr.make_chunk_args(to_dev(x["q"]), to_dev(x["v"]), to_dev(g), gdn2_w=to_dev(w))
    # bf16 with d = 128 and chunk 64 takes the tensor-core GDN-2 kernels, fp32 the CUDA cores
    assert gdr.chunk_fwd_path(args) == ("tc" if dtype == "bf16" else "simt")
    scale = 1 / math.sqrt(128)
    o, S = run_chunk(x, g, b, w, read_mode=read_mode, scale=scale)
    o_r, S_r = oracle.gdn2_forward(x["q"], x["k"], x["v"], g, b, w, x["S0"],
                                   read_mode=read_mode, scale=scale)
    assert_close("o", o, o_r, workloads.DTYPES[dtype])
    assert_close("S", S, S_r, workloads.DTYPES[dtype], kind="state")


@pytest.mark.parametrize("reverse", [False, True])
def test_chunk_varlen_small_heads(reverse):
    lengths = [1, 0, 64, 65, 130, 7]
    x = workloads.chunk_inputs(1, 0, 1, 2, 64, 32, "f32", lengths=lengths, s0_std=0.1, seed=53)
    g, b, w = workloads.gdn2_gate_inputs(x["v"].shape[:3], 64, 32, "f32", seed=54)
    o, S = run_chunk(x, g, b, w, read_mode="pre", scale=0.3, reverse=reverse)
    o_r, S_r = oracle.gdn2_forward(x["q"], x["k"], x["v"], g, b, w, x["S0"], x["cu_seqlens"],
                                   read_mode="pre", scale=0.3, reverse=reverse)
    assert_close("o", o, o_r, torch.float32)
    assert_close("S", S, S_r, torch.float32, kind="state")


def test_chunk_scalar_gates_match_gated_delta_rule():
    """With every channel's gates equal to the token's (g, beta, beta), GDN-2 on the GPU
    gives the scalar rule's oracle result."""
    x = workloads.chunk_inputs(1, 90, 1, 2, 64, 64, "f32", s0_std=0.05, seed=55)
    g = x["g"][..., None].expand(*x["g"].shape, 64).contiguous()
    b = x["beta"][..., None].expand(*x["beta"].shape, 64).contiguous()
    o, S = run_chunk(x, g, b, b.clone(), scale=0.125)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], scale=0.125)
    assert_close("o", o, o_r, torch.float32)
    assert_close("S", S, S_r, torch.float32, kind="state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("fused_norm", [False, True])
def test_decode(dtype, read_mode, fused_norm):
    N, Hk, Hv, d, steps = 6, 2, 4, 128, 4
    x = workloads.decode_inputs(N, Hk, Hv, d, d, steps=steps, dtype=dtype, s_std=0.1, seed=57)
    g, b, w = workloads.gdn2_gate_inputs((steps, N, Hv), d, d, dtype, seed=58)
    gen = torch.Generator("cpu").manual_seed(59)
    z = torch.randn((N, Hv, d), generator=gen).to(workloads.DTYPES[dtype])
    weight = 1 + 0.1 * torch.randn(d, generator=gen)
    S = x["S"].clone().cuda()
    S_ref = x["S"].double().numpy()
    scale = 1 / math.sqrt(d)
    kw = dict(norm_z=to_dev(z), norm_weight=to_dev(weight), norm_eps=1e-6) if fused_norm else {}
    for t in range(steps):
        o = gdr.decode_step(*(to_dev(x[n][t]) for n in ("q", "k", "v")), to_dev(g[t]),
                            to_dev(b[t]), S, scale=scale, read_mode=read_mode,
                            gdn2_w=to_dev(w[t]), **kw)
        o_ref, S_ref = oracle.gdn2_forward(*(x[n][t][:, None] for n in ("q", "k", "v")),
                                           g[t][:, None], b[t][:, None], w[t][:, None], S_ref,
                                           read_mode=read_mode, scale=scale)
        o_ref = o_ref[:, 0]
        if fused_norm:
            o_ref = oracle.gated_rmsnorm(o_ref, z, weight, 1e-6)
        torch.cuda.synchronize()
        assert_close(f"o step {t}", o, o_ref, workloads.DTYPES[dtype])
    assert_close("S", S, S_ref, torch.float32 if dtype == "f32" else torch.bfloat16, kind="state")


@pytest.mark.parametrize("chunk", [16, 32])
def test_chunk_sizes(chunk):
    """Chunks of 32 (one factored block below the diagonal blocks) and 16 (diagonal only);
    GDN-2 takes chunks up to 64."""
    x = workloads.chunk_inputs(1, 150, 2, 2, 64, 64, "f32", s0_std=0.05, seed=73)
    g, b, w = workloads.gdn2_gate_inputs(x["v"].shape[:3], 64, 64, "f32", seed=74)
    o, S = run_chunk(x, g, b, w, chunk=chunk, scale=0.125)
    o_r, S_r = oracle.gdn2_forward(x["q"], x["k"], x["v"], g, b, w, x["S0"], scale=0.125)
    assert_close("o", o, o_r, torch.float32)
    assert_close("S", S, S_r, torch.float32, kind="state")


def test_growing_and_strong_decays():
    """Head 0: log decays of either sign (a chunk where the decay grows takes one exp per
    term everywhere); head 1: strong decays (g ~ -2 per token, factors that underflow)."""
    x = workloads.chunk_inputs(1, 130, 1, 2, 64, 64, "f32", s0_std=0.1, seed=75)
    gen = torch.Generator("cpu").manual_seed(76)
    shape = (1, 130, 2, 64)
    g = torch.empty(shape)
    g[:, :, 0] = torch.randn((1, 130, 64), generator=gen) * 0.05
    g[:, :, 1] = -torch.nn.functional.softplus(torch.randn((1, 130, 64), generator=gen) + 2.0)
    b = torch.sigmoid(torch.randn(shape, generator=gen))
    w = torch.sigmoid(torch.randn((1, 130, 2, 64), generator=gen))
    for mode in ("post", "pre"):
        o, S = run_chunk(x, g, b, w, read_mode=mode, scale=0.125)
        o_r, S_r = oracle.gdn2_forward(x["q"], x["k"], x["v"], g, b, w, x["S0"], read_mode=mode,
                                       scale=0.125)
        assert_close(f"o {mode}", o, o_r, torch.float32)
        assert_close(f"S {mode}", S, S_r, torch.float32, kind="state")
