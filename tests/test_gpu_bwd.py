"""GPU parity of the backward pass (gdr_chunk_bwd) against the fp64 reverse-mode oracle
``oracle.backward``, on the same seeded inputs and upstream gradients.

Tolerance: bf16 as for the forward (2e-2 RMS(ref) + 2^-8 |ref| element-wise for a gradient
written in bf16, 2e-2 RMS(ref) for the fp32 dS0).  fp32: the pages ask the two forms to
agree to 1e-4 on the forward and on the gradients; gradients scale with dO, T and the
state, so the bound used is 1e-4 max(1, RMS(ref)).  Every comparison's margin is recorded
in the session's parity table."""
import math

import numpy as np
import pytest
import torch

import oracle.backward as obw
import workloads
import gated_delta_rule_146_b200 as gdr
from gpu_helpers import Accum, assert_close, oracle_backward_sequence, record, to_dev

pytestmark = pytest.mark.gpu


def grad_close(name, gpu, ref, dtype):
    if dtype == torch.bfloat16:
        return assert_close(name, gpu, ref, dtype,
                            kind="state" if name.startswith("dS0") else "out")
    g = gpu.detach().double().cpu().numpy()
    if not ref.size:
        return
    rms = float(np.sqrt(np.mean(ref * ref)))
    tol = 1e-4 * max(1.0, rms)
    err = np.abs(g - ref)
    record(name, float(err.max()), rms, float(err.max()) / tol)
    assert err.max() <= tol, f"{name}: max err {err.max():.3e} > {tol:.3e}"


def upstream(x, dtype, seed, with_dS=True):
    gen = torch.Generator("cpu").manual_seed(seed)
    dO = torch.randn(x["v"].shape, generator=gen).to(workloads.DTYPES[dtype])
    n = x["S0"].shape[0] if x["S0"] is not None else (
        x["v"].shape[0] if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1)
    Hv, dk, dv = x["v"].shape[2], x["q"].shape[3], x["v"].shape[3]
    dS = torch.randn((n, Hv, dk, dv), generator=gen) if with_dS else None
    return dO, dS


def run_and_check(x, dO, dS, dtype, *, read_mode="post", scale=0.1, reverse=False, chunk=64,
                  qk_l2norm=True):
    dev = {n: to_dev(t) if t is not None else None for n, t in x.items()}
    a = gdr.make_chunk_args(dev["q"], dev["v"], dev["g"], dev["cu_seqlens"], chunk, read_mode,
                            scale, qk_l2norm, reverse)
    tc = dtype == "bf16" and x["q"].shape[3] == 128 and x["v"].shape[3] == 128 and chunk == 64
    assert gdr.chunk_bwd_path(a) == ("tc" if tc else "simt")
    got = gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], to_dev(dO),
                        dev["S0"], dev["cu_seqlens"], to_dev(dS), chunk=chunk,
                        read_mode=read_mode, scale=scale, reverse=reverse, qk_l2norm=qk_l2norm)
    torch.cuda.synchronize()
    ref = obw.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dO, x["S0"], dS,
                       x["cu_seqlens"], read_mode=read_mode, scale=scale, reverse=reverse,
                       qk_l2norm=qk_l2norm)
    dt = workloads.DTYPES[dtype]
    for name, g in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), got):
        grad_close(name, g, ref[name], dt)


@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gqa_several_chunks_ragged_tail(dtype, read_mode):
    x = workloads.chunk_inputs(2, 150, 2, 4, 128, 128, dtype, s0_std=0.05, seed=61)
    dO, dS = upstream(x, dtype, 62)
    run_and_check(x, dO, dS, dtype, read_mode=read_mode, scale=1 / math.sqrt(128))


@pytest.mark.parametrize("reverse", [False, True])
def test_varlen_empty_and_one_token_sequences(reverse):
    lengths = [1, 0, 64, 65, 130, 7]
    x = workloads.chunk_inputs(1, 0, 1, 2, 64, 64, "f32", lengths=lengths, s0_std=0.1, seed=63)
    dO, dS = upstream(x, "f32", 64)
    run_and_check(x, dO, dS, "f32", read_mode="pre", scale=0.3, reverse=reverse)


@pytest.mark.parametrize("chunk", [16, 32])
def test_smaller_chunks_rectangular_heads(chunk):
    x = workloads.chunk_inputs(1, 100, 1, 1, 96, 64, "f32", s0_std=0.05, seed=65)
    dO, dS = upstream(x, "f32", 66)
    run_and_check(x, dO, dS, "f32", chunk=chunk, scale=0.2)


def test_no_state_gradients_and_no_norm():
    """S0 = None and dS_final = None (zero), without the in-kernel normalisation."""
    x = workloads.chunk_inputs(1, 80, 2, 2, 32, 32, "f32", seed=67)
    x["q"] = x["q"] * 0.2
    x["k"] = x["k"] * 0.2
    dO, _ = upstream(x, "f32", 68, with_dS=False)
    run_and_check(x, dO, None, "f32", scale=1.0, qk_l2norm=False)


def test_bidirectional_workload_rows():
    """Two sequences of the bidirectional workload's shape (2048 tokens, H=12, d=64,
    pre-write read, scale 1): the reverse direction's backward."""
    x = workloads.chunk_inputs(1, 0, 12, 12, 64, 64, "bf16", lengths=[2048, 2048], seed=69)
    dO, dS = upstream(x, "bf16", 70, with_dS=False)
    run_and_check(x, dO, None, "bf16", read_mode="pre", scale=1.0, reverse=True)


def test_training_shape_workload_whole():
    """The backward at the training workload's full size (8 x 4096 tokens, 16 heads, d=128,
    bf16): every element of dq, dk, dv, dg, dbeta and dS0 against the oracle, which runs one
    sequence per process of a spawned pool (about a minute on the host's cores)."""
    import multiprocessing as mp
    w = workloads.WORKLOADS["bf16_b8_h16_t4096_d128"]
    x = workloads.workload_inputs(w)
    gen = torch.Generator("cpu").manual_seed(71)
    dO = torch.randn(x["v"].shape, generator=gen).to(torch.bfloat16)
    dev = {n: to_dev(t) if t is not None else None for n, t in x.items()}
    a = gdr.make_chunk_args(dev["q"], dev["v"], dev["g"], None, w.chunk, w.read_mode, w.scale)
    assert gdr.chunk_bwd_path(a) == "tc"  # the tensor-core kernels
    got = gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], to_dev(dO),
                        dev["S0"], None, None, chunk=w.chunk, read_mode=w.read_mode,
                        scale=w.scale)
    torch.cuda.synchronize()
    got = [t.detach().cpu() for t in got]
    f32 = lambda t: None if t is None else t.float().numpy()
    jobs = []
    for b in range(w.B):
        sl = lambda t: f32(t[b:b + 1])
        arrays = (sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["beta"]), sl(dO),
                  None if x["S0"] is None else f32(x["S0"][b:b + 1]), None)
        jobs.append((arrays, {"read_mode": w.read_mode, "scale": w.scale}))
    acc = {n: Accum(n, torch.bfloat16, "state" if n == "dS0" else "out")
           for n in ("dq", "dk", "dv", "dg", "dbeta", "dS0")}
    with mp.get_context("spawn").Pool(min(w.B, max(1, mp.cpu_count()))) as pool:
        for b, ref in enumerate(pool.imap(oracle_backward_sequence, jobs)):
            for i, n in enumerate(("dq", "dk", "dv", "dg", "dbeta")):
                acc[n].add(got[i][b:b + 1], ref[n].astype(np.float64), label=f" row {b}")
            acc["dS0"].add(got[5][b:b + 1], ref["dS0"].astype(np.float64), label=f" row {b}")
    for a in acc.values():
        a.check()


@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("reverse", [False, True])
def test_tensor_core_varlen_reverse(reverse, read_mode):
    """The tensor-core backward (bf16, d = 128, chunk 64) over packed sequences with an empty
    one, a one-token one and ragged tails, GQA 2 -> 4, S0 and dS_final, both directions and
    both read modes."""
    lengths = [1, 0, 64, 65, 130, 200]
    x = workloads.chunk_inputs(1, 0, 2, 4, 128, 128, "bf16", lengths=lengths, s0_std=0.1, seed=81)
    dO, dS = upstream(x, "bf16", 82)
    run_and_check(x, dO, dS, "bf16", read_mode=read_mode, scale=1 / math.sqrt(128),
                  reverse=reverse)


def test_tensor_core_no_norm_no_state():
    """The tensor-core backward without the in-kernel normalisation, S0 = None and
    dS_final = None."""
    x = workloads.chunk_inputs(2, 150, 2, 2, 128, 128, "bf16", seed=83)
    x["q"] = (x["q"].float() * 0.08).to(torch.bfloat16)
    x["k"] = (x["k"].float() * 0.08).to(torch.bfloat16)
    dO, _ = upstream(x, "bf16", 84, with_dS=False)
    run_and_check(x, dO, None, "bf16", scale=1.0, qk_l2norm=False)


def test_tensor_core_deterministic():
    """Two tensor-core backward calls on the same inputs agree bit for bit (every sum has a
    fixed order; no atomics)."""
    x = workloads.chunk_inputs(2, 300, 2, 4, 128, 128, "bf16", s0_std=0.05, seed=85)
    dO, dS = upstream(x, "bf16", 86)
    dev = {n: to_dev(t) if t is not None else None for n, t in x.items()}
    outs = []
    for _ in range(2):
        got = gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], to_dev(dO),
                            dev["S0"], None, to_dev(dS), scale=0.1)
        torch.cuda.synchronize()
        outs.append([t.detach().cpu() for t in got])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_tensor_core_range_reported():
    """An upstream gradient beyond the fp16 range of the recurrences' operands is reported as
    GDR_ERR_RANGE through the workspace (the outputs are then not valid)."""
    x = workloads.chunk_inputs(1, 130, 2, 2, 128, 128, "bf16", seed=87)
    dO, _ = upstream(x, "bf16", 88, with_dS=False)
    dO = (dO.float() * 1e6).to(torch.bfloat16)
    dev = {n: to_dev(t) if t is not None else None for n, t in x.items()}
    a = gdr.make_chunk_args(dev["q"], dev["v"], dev["g"], None, 64, "post", 0.1, True, False)
    assert gdr.chunk_bwd_path(a) == "tc"
    ws = torch.empty(gdr.chunk_bwd_workspace_size(a), dtype=torch.uint8, device="cuda")
    gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], to_dev(dO), None, None,
                  None, scale=0.1, workspace=ws)
    assert gdr.read_device_error(a, ws) == gdr._abi.GDR_ERR_RANGE
    # the same call at a normal scale is clean
    gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                  to_dev((dO.float() * 1e-6).to(torch.bfloat16)), None, None, None, scale=0.1,
                  workspace=ws)
    assert gdr.read_device_error(a, ws) == 0
