"""GPU parity of the tensor-core GDN-2 forward (per-key-channel decay and erase gate, per-
value-channel write gate; Rondo-Exp ``tiny_gdn/fugue.py``, ``BidirectionalGatedDeltaNet2``)
against the fp64 per-token oracle ``oracle.gdn2_forward``: several chunks, ragged tails,
varlen with empty and one-token sequences, GQA, both read modes, S0 and S_final."""
import math

import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
import numpy as np

from gpu_helpers import Accum, assert_close, oracle_gdn2_sequence, to_dev

pytestmark = pytest.mark.gpu


def run(x, g, b, w, **kw):
    o, S = gdr.chunk_fwd(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), to_dev(g), to_dev(b),
                         to_dev(x["S0"]) if x["S0"] is not None else None,
                         to_dev(x["cu_seqlens"]) if x["cu_seqlens"] is not None else None,
                         gdn2_w=to_dev(w), **kw)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("lengths", [None, [300, 0, 1, 64, 65, 129]])
def test_tensor_core_gdn2(read_mode, lengths):
    T = 0 if lengths else 200
    x = workloads.chunk_inputs(1 if lengths else 2, T, 2, 4, 128, 128, "bf16", lengths=lengths,
                               s0_std=0.05, seed=91)
    g, b, w = workloads.gdn2_gate_inputs(x["v"].shape[:3], 128, 128, "bf16", seed=92)
    args = gdr.make_chunk_args(to_dev(x["q"]), to_dev(x["v"]), to_dev(g), gdn2_w=to_dev(w))
    assert gdr.chunk_fwd_path(args) == "tc"
    scale = 1 / math.sqrt(128)
    o, S = run(x, g, b, w, read_mode=read_mode, scale=scale)
    o_r, S_r = oracle.gdn2_forward(x["q"], x["k"], x["v"], g, b, w, x["S0"], x["cu_seqlens"],
                                   read_mode=read_mode, scale=scale)
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_tensor_core_gdn2_strong_and_growing_decays():
    """Head 0: log decays of either sign; head 1: strong decays (g ~ -2 per token)."""
    x = workloads.chunk_inputs(1, 260, 1, 2, 128, 128, "bf16", s0_std=0.1, seed=93)
    gen = torch.Generator("cpu").manual_seed(94)
    shape = (1, 260, 2, 128)
    g = torch.empty(shape)
    g[:, :, 0] = torch.randn((1, 260, 128), generator=gen) * 0.05
    g[:, :, 1] = -torch.nn.functional.softplus(torch.randn((1, 260, 128), generator=gen) + 2.0)
    b = torch.sigmoid(torch.randn(shape, generator=gen))
    w = torch.sigmoid(torch.randn(shape, generator=gen))
    g, b, w = (t.to(torch.bfloat16) for t in (g, b, w))
    for mode in ("post", "pre"):
        o, S = run(x, g, b, w, read_mode=mode, scale=0.125)
        o_r, S_r = oracle.gdn2_forward(x["q"], x["k"], x["v"], g, b, w, x["S0"], read_mode=mode,
                                       scale=0.125)
        assert_close(f"o {mode}", o, o_r, torch.bfloat16)
        assert_close(f"S {mode}", S, S_r, torch.bfloat16, kind="state")


def test_tensor_core_gdn2_scalar_gates_match_gated_delta_rule():
    """Every channel's gates equal to the token's (g, beta, beta): the scalar rule's oracle."""
    x = workloads.chunk_inputs(1, 150, 2, 2, 128, 128, "bf16", s0_std=0.05, seed=95)
    g = x["g"].float()[..., None].expand(*x["g"].shape, 128).contiguous().to(torch.bfloat16)
    b = x["beta"].float()[..., None].expand(*x["beta"].shape, 128).contiguous().to(torch.bfloat16)
    o, S = run(x, g, b, b.clone(), scale=0.1)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], g[..., 0], b[..., 0], x["S0"], scale=0.1)
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_training_shape_workload_whole():
    """The GDN-2 forward at the training workload's full size (8 x 4096 tokens, 16 heads,
    d = 128, bf16, the bench's GDN-2 gates): every element of o and S_final against the
    oracle, one sequence per process of a spawned pool."""
    import multiprocessing as mp
    w = workloads.WORKLOADS["bf16_b8_h16_t4096_d128"]
    x = workloads.workload_inputs(w)
    g, b, wg = workloads.gdn2_gate_inputs(x["v"].shape[:3], w.dk, w.dv, w.gate_dtype, seed=0)
    o, S = run(x, g, b, wg, read_mode=w.read_mode, scale=w.scale)
    o, S = o.cpu(), S.cpu()
    f32 = lambda t: None if t is None else t.float().numpy()
    jobs = []
    for r in range(w.B):
        sl = lambda t: f32(t[r:r + 1])
        arrays = (sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(g), sl(b), sl(wg),
                  None if x["S0"] is None else f32(x["S0"][r:r + 1]))
        jobs.append((arrays, {"read_mode": w.read_mode, "scale": w.scale}))
    ao, aS = Accum("o", torch.bfloat16, "out"), Accum("S_final", torch.bfloat16, "state")
    with mp.get_context("spawn").Pool(min(w.B, max(1, mp.cpu_count()))) as pool:
        for r, (o_r, S_r) in enumerate(pool.imap(oracle_gdn2_sequence, jobs)):
            ao.add(o[r:r + 1], o_r.astype(np.float64), label=f" row {r}")
            aS.add(S[r:r + 1], S_r.astype(np.float64), label=f" row {r}")
    ao.check()
    aS.check()
