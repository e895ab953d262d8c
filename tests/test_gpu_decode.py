"""GPU parity of gdr_decode_step against the fp64 oracle."""
import math

import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
from gpu_helpers import Accum, assert_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (32, 128), (128, 32)])
def test_decode_steps_small(dtype, read_mode, dk, dv):
    x = workloads.decode_inputs(5, 2, 4, dk, dv, steps=6, dtype=dtype, s_std=0.1, seed=dk + dv)
    S = x["S"].clone().cuda()
    S_ref = x["S"].double().numpy()
    scale = 1 / math.sqrt(dk)
    for t in range(6):
        o = gdr.decode_step(*(to_dev(x[n][t]) for n in ("q", "k", "v", "g", "beta")), S,
                            read_mode=read_mode, scale=scale)
        o_ref, S_ref = oracle.decode_step(*(x[n][t] for n in ("q", "k", "v", "g", "beta")),
                                          S_ref, read_mode=read_mode, scale=scale)
        torch.cuda.synchronize()
        assert_close(f"o step {t}", o, o_ref, workloads.DTYPES[dtype])
    assert_close("S", S, S_ref, torch.float32 if dtype == "f32" else torch.bfloat16, kind="state")


def test_decode_matches_chunk_forward():
    """64 decode steps from S0 give the same o and state as one chunk_fwd over the 64
    tokens (both on the GPU; K4 against K1-K3)."""
    N, Hk, Hv, d, T = 4, 2, 4, 128, 64
    x = workloads.chunk_inputs(N, T, Hk, Hv, d, d, "f32", s0_std=0.05, seed=21)
    dev = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    o_c, S_c = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"])
    S = dev["S0"].clone()
    outs = []
    for t in range(T):
        outs.append(gdr.decode_step(dev["q"][:, t].contiguous(), dev["k"][:, t].contiguous(),
                                    dev["v"][:, t].contiguous(), dev["g"][:, t].contiguous(),
                                    dev["beta"][:, t].contiguous(), S))
    torch.cuda.synchronize()
    o_d = torch.stack(outs, 1)
    assert (o_d - o_c).abs().max().item() < 1e-4
    assert (S - S_c).abs().max().item() < 1e-4


def test_decode_workload_whole():
    """256 sequences x 32 v-heads (16 k-heads), 64 steps of fresh bf16 inputs from an
    N(0, 0.02^2) fp32 state: every output of every step and the whole final state against
    the oracle, which follows groups of 32 sequences through all 64 steps."""
    w = workloads.DECODE_WORKLOADS["bf16_decode_n256_hk16_hv32_d128"]
    x = workloads.decode_workload_inputs(w)
    S = x["S"].clone().cuda()
    outs = []
    for t in range(w.steps):
        o = gdr.decode_step(*(to_dev(x[n][t]) for n in ("q", "k", "v", "g", "beta")), S,
                            read_mode=w.read_mode, scale=w.scale)
        outs.append(o.cpu())
    torch.cuda.synchronize()
    S_gpu = S.cpu()
    ao = Accum("o (every step)", torch.bfloat16, "out")
    aS = Accum("S final", torch.bfloat16, "state")
    for s0 in range(0, w.N, 32):
        sl = slice(s0, s0 + 32)
        S_ref = x["S"][sl].double().numpy()
        for t in range(w.steps):
            o_ref, S_ref = oracle.decode_step(*(x[n][t][sl] for n in ("q", "k", "v", "g", "beta")),
                                              S_ref, read_mode=w.read_mode, scale=w.scale)
            ao.add(outs[t][sl], o_ref, label=f" step {t} seqs {s0}+")
        aS.add(S_gpu[sl], S_ref, label=f" seqs {s0}+")
    ao.check()
    aS.check()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 32)])
def test_decode_fused_gated_rmsnorm(dtype, dk, dv):
    """o = gated RMSNorm of the recurrent output (the decode chain's epilogue), the state
    updated exactly as without it."""
    x = workloads.decode_inputs(5, 2, 4, dk, dv, steps=3, dtype=dtype, s_std=0.1, seed=50 + dv)
    S = x["S"].clone().cuda()
    S_ref = x["S"].double().numpy()
    gen = torch.Generator("cpu").manual_seed(dk + dv)
    w = 1.0 + 0.2 * torch.randn(dv, generator=gen)
    scale = 1 / math.sqrt(dk)
    for t in range(3):
        z = torch.randn((5, 4, dv), generator=gen).to(workloads.DTYPES[dtype])
        o = gdr.decode_step(*(to_dev(x[n][t]) for n in ("q", "k", "v", "g", "beta")), S,
                            scale=scale, norm_z=to_dev(z), norm_weight=to_dev(w), norm_eps=1e-6)
        o_core, S_ref = oracle.decode_step(*(x[n][t] for n in ("q", "k", "v", "g", "beta")),
                                           S_ref, scale=scale)
        ref = oracle.gated_rmsnorm(o_core, z, w, 1e-6)
        torch.cuda.synchronize()
        assert_close(f"o step {t}", o, ref, workloads.DTYPES[dtype])
    assert_close("S", S, S_ref, torch.float32 if dtype == "f32" else torch.bfloat16, kind="state")
