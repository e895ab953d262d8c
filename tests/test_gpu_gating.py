"""GPU parity of the fused gating prologue: the kernels take the raw per-token projections
a, b with per-head A (= -exp(A_log)) and dt_bias and form g and beta themselves; the oracle
forms them in fp64 (``oracle.gating``) and runs the plain recurrence."""
import math

import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
from gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def raw_gates(shape, Hv, dtype, seed):
    """Raw projections a ~ N(-1, 1.5^2), b ~ N(0, 1.5^2) in the gate dtype, and per-head
    A = -exp(N(0, 0.5^2)), dt_bias ~ N(0, 1) in fp32 (seeded, CPU)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    a = (torch.randn(shape, generator=gen) * 1.5 - 1.0).to(dtype)
    b = (torch.randn(shape, generator=gen) * 1.5).to(dtype)
    A = -torch.exp(torch.randn(Hv, generator=gen) * 0.5)
    dt = torch.randn(Hv, generator=gen)
    return a, b, A, dt


def run_chunk(x, a, b, A, dt, beta_scale, **kw):
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    o, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], to_dev(a), to_dev(b), d.get("S0"),
                         d.get("cu_seqlens"), gate_A=to_dev(A), gate_dt_bias=to_dev(dt),
                         beta_scale=beta_scale, **kw)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("beta_scale", [1.0, 2.0])
@pytest.mark.parametrize("read_mode", ["post", "pre"])
def test_tensor_core_path(beta_scale, read_mode):
    x = workloads.chunk_inputs(2, 200, 2, 4, 128, 128, "bf16", s0_std=0.02, seed=31)
    a, b, A, dt = raw_gates(x["g"].shape, 4, torch.bfloat16, 32)
    scale = 1 / math.sqrt(128)
    args = gdr.make_chunk_args(to_dev(x["q"]), to_dev(x["v"]), to_dev(a), gate_A=to_dev(A),
                               gate_dt_bias=to_dev(dt))
    assert gdr.chunk_fwd_path(args) == "tc"
    o, S = run_chunk(x, a, b, A, dt, beta_scale, read_mode=read_mode, scale=scale)
    g, beta = oracle.gating(a, b, A, dt, beta_scale)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], g, beta, x["S0"], read_mode=read_mode,
                              scale=scale)
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_tensor_core_varlen_reverse_fp32_gates():
    lengths = [1, 0, 64, 65, 130, 7]
    x = workloads.chunk_inputs(1, 0, 2, 2, 128, 128, "bf16", lengths=lengths, s0_std=0.05,
                               seed=33)
    a, b, A, dt = raw_gates(x["v"].shape[:3], 2, torch.float32, 34)
    o, S = run_chunk(x, a, b, A, dt, 1.0, read_mode="pre", scale=0.3, reverse=True)
    g, beta = oracle.gating(a, b, A, dt, 1.0)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], g, beta, x["S0"], x["cu_seqlens"],
                              read_mode="pre", scale=0.3, reverse=True)
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_cuda_core_path():
    x = workloads.chunk_inputs(2, 100, 1, 2, 64, 64, "f32", s0_std=0.05, seed=35)
    a, b, A, dt = raw_gates(x["g"].shape, 2, torch.float32, 36)
    args = gdr.make_chunk_args(to_dev(x["q"]), to_dev(x["v"]), to_dev(a), gate_A=to_dev(A),
                               gate_dt_bias=to_dev(dt))
    assert gdr.chunk_fwd_path(args) == "simt"
    o, S = run_chunk(x, a, b, A, dt, 2.0, scale=0.125)
    g, beta = oracle.gating(a, b, A, dt, 2.0)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], g, beta, x["S0"], scale=0.125)
    assert_close("o", o, o_r, torch.float32)
    assert_close("S", S, S_r, torch.float32, kind="state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode(dtype):
    x = workloads.decode_inputs(6, 2, 4, 128, 128, steps=4, dtype=dtype, s_std=0.1, seed=37)
    S = x["S"].clone().cuda()
    S_ref = x["S"].double().numpy()
    gdt = torch.float32 if dtype == "f32" else torch.bfloat16
    for t in range(4):
        a, b, A, dt = raw_gates(x["g"][t].shape, 4, gdt, 40 + t)
        o = gdr.decode_step(*(to_dev(x[n][t]) for n in ("q", "k", "v")), to_dev(a), to_dev(b),
                            S, scale=1 / math.sqrt(128), gate_A=to_dev(A),
                            gate_dt_bias=to_dev(dt), beta_scale=1.0)
        g, beta = oracle.gating(a, b, A, dt, 1.0)
        o_ref, S_ref = oracle.decode_step(*(x[n][t] for n in ("q", "k", "v")), g, beta, S_ref,
                                          scale=1 / math.sqrt(128))
        torch.cuda.synchronize()
        assert_close(f"o step {t}", o, o_ref, workloads.DTYPES[dtype])
    assert_close("S", S, S_ref, torch.float32 if dtype == "f32" else torch.bfloat16, kind="state")
