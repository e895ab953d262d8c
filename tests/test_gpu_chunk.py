"""GPU parity of gdr_chunk_fwd against the fp64 oracle, element by element.

Small problems span several chunks and a ragged tail; the full-size workloads are compared
on every element of o and S_final, the oracle running over groups of whole sequences.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
from gpu_helpers import assert_close, compare_whole, to_dev

pytestmark = pytest.mark.gpu


def run_gpu(x, **kw):
    dev = {n: to_dev(x[n]) if x.get(n) is not None else None
           for n in ("q", "k", "v", "g", "beta", "S0", "cu_seqlens")}
    o, S = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                         dev["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return o, S


def run_oracle(x, read_mode, scale, reverse=False):
    return oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"],
                          read_mode=read_mode, scale=scale, reverse=reverse)


def check(x, dtype, read_mode="post", scale=None, chunk=64, reverse=False, path=None):
    dk = x["q"].shape[-1]
    scale = 1.0 / math.sqrt(dk) if scale is None else scale
    o, S = run_gpu(x, chunk=chunk, read_mode=read_mode, scale=scale, reverse=reverse)
    o_ref, S_ref = run_oracle(x, read_mode, scale, reverse)
    eo, _ = assert_close("o", o, o_ref, dtype)
    es, _ = assert_close("S_final", S, S_ref, dtype, kind="state")
    return eo, es


def test_oracle_sized_fp32_workload():
    """fp32, B=1, H=2, T=256, d=64, chunk 64: max-abs <= 1e-4."""
    w = workloads.WORKLOADS["fp32_b1_h2_t256_d64"]
    x = workloads.workload_inputs(w)
    check(x, torch.float32, "post", w.scale, 64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
def test_chunk_sizes_ragged(dtype, read_mode, chunk):
    """Every chunk size, a ragged tail (T=200), initial state, GQA 2 -> 4 heads."""
    x = workloads.chunk_inputs(2, 200, 2, 4, 64, 64, dtype, s0_std=0.3, seed=chunk)
    check(x, workloads.DTYPES[dtype], read_mode, None, chunk)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (32, 32)])
def test_head_dims(dtype, dk, dv):
    x = workloads.chunk_inputs(1, 300, 1, 2, dk, dv, dtype, s0_std=0.02, seed=dk + dv)
    check(x, workloads.DTYPES[dtype], "post", None, 64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_with_empty_and_short_sequences(dtype):
    lengths = [1, 0, 64, 65, 130, 0, 7, 300]
    x = workloads.chunk_inputs(1, 0, 2, 2, 128, 128, dtype, lengths=lengths, s0_std=0.02, seed=5)
    check(x, workloads.DTYPES[dtype], "post", None, 64)
    check(x, workloads.DTYPES[dtype], "pre", 1.0, 64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reverse_scan(dtype):
    x = workloads.chunk_inputs(1, 0, 3, 3, 64, 64, dtype, lengths=[100, 37, 128], seed=9)
    check(x, workloads.DTYPES[dtype], "pre", 1.0, 64, reverse=True)
    check(x, workloads.DTYPES[dtype], "post", 0.5, 64, reverse=True)


def test_bidirectional_sum_with_accumulate():
    """Both directions over shared q, k, v with their own gates, summed through
    o_accumulate (tiny_gdn/fugue.py BidirectionalGatedDeltaNet2.forward / scan)."""
    x = workloads.chunk_inputs(1, 0, 4, 4, 64, 64, "bf16", lengths=[256] * 3 + [100],
                               bidirectional=True, seed=3)
    dev = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    o, _ = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], None,
                         dev["cu_seqlens"], read_mode="pre", scale=1.0, output_final_state=False)
    gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g_bwd"], dev["beta_bwd"], None,
                  dev["cu_seqlens"], read_mode="pre", scale=1.0, reverse=True, o=o,
                  o_accumulate=True, output_final_state=False)
    torch.cuda.synchronize()
    o_f, _ = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                            read_mode="pre", scale=1.0)
    o_b, _ = oracle.forward(x["q"], x["k"], x["v"], x["g_bwd"], x["beta_bwd"], None,
                            x["cu_seqlens"], read_mode="pre", scale=1.0, reverse=True)
    # each call writes its direction in bf16 before the sum is rounded: two more roundings
    assert_close("o_bidir", o, o_f + o_b, torch.bfloat16, rounded_parts=(o_f, o_b))


def test_alpha_half_floor_long_chunk():
    """alpha = 0.5 everywhere, chunk 128: in-chunk decay reaches 2^-127 (log space)."""
    x = workloads.chunk_inputs(1, 384, 1, 1, 64, 64, "f32", s0_std=0.5, seed=1)
    x["g"] = torch.full_like(x["g"], math.log(0.5))
    check(x, torch.float32, "post", None, 128)
    check(x, torch.float32, "pre", None, 64)


def test_repeated_keys_and_large_beta():
    """All keys equal and beta up to 2 (negative eigenvalues, tiny_gdn/fugue.py project)."""
    x = workloads.chunk_inputs(1, 256, 1, 1, 64, 64, "f32", seed=2)
    x["k"] = x["k"][:, :1].expand_as(x["k"]).contiguous()
    x["beta"] = 2.0 * x["beta"]
    check(x, torch.float32, "post", None, 64)


def test_zero_decay_zero_beta_passes_state_through():
    x = workloads.chunk_inputs(1, 130, 1, 2, 64, 64, "f32", s0_std=0.5, seed=4)
    x["g"].zero_()
    x["beta"].zero_()
    o, S = run_gpu(x, read_mode="pre", scale=1.0)
    assert torch.equal(S.cpu(), x["S0"])


def test_continuation_equals_one_call():
    x = workloads.chunk_inputs(1, 300, 2, 2, 128, 128, "f32", s0_std=0.1, seed=6)
    o, S = run_gpu(x)
    y = {n: (t[:, :137] if t is not None and t.dim() >= 3 else t) for n, t in x.items()}
    z = {n: (t[:, 137:] if t is not None and t.dim() >= 3 else t) for n, t in x.items()}
    y["S0"] = x["S0"]
    o1, S1 = run_gpu(y)
    z["S0"] = S1.cpu()
    o2, S2 = run_gpu(z)
    assert torch.allclose(torch.cat([o1, o2], 1), o, atol=2e-5)
    assert torch.allclose(S2, S, atol=2e-5)


def test_deterministic():
    x = workloads.chunk_inputs(2, 500, 2, 2, 128, 128, "bf16", s0_std=0.02, seed=8)
    o1, S1 = run_gpu(x)
    o2, S2 = run_gpu(x)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_bad_cu_seqlens_sets_device_error():
    x = workloads.chunk_inputs(1, 0, 1, 1, 64, 64, "bf16", lengths=[10, 20], seed=0)
    cu = torch.tensor([0, 20, 10], dtype=torch.int32)  # decreasing, does not end at T=30
    dev = {n: to_dev(x[n]) for n in ("q", "k", "v", "g", "beta")}
    args = gdr.make_chunk_args(dev["q"], dev["v"], dev["g"], cu)
    ws = torch.empty(gdr.chunk_fwd_workspace_size(args), dtype=torch.uint8, device="cuda")
    gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], None, cu.cuda(),
                  workspace=ws)
    assert gdr.read_device_error(args, ws) == gdr._abi.GDR_ERR_DEVICE_CHECK
    # a good call on the same workspace clears the word
    gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], None,
                  to_dev(x["cu_seqlens"]), workspace=ws)
    assert gdr.read_device_error(args, ws) == gdr._abi.GDR_OK


def test_workspace_poisoned_with_nan():
    """Outputs do not depend on stale workspace contents."""
    x = workloads.chunk_inputs(1, 0, 2, 2, 128, 128, "bf16", lengths=[70, 200], seed=12)
    dev = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    args = gdr.make_chunk_args(dev["q"], dev["v"], dev["g"], dev["cu_seqlens"])
    ws = torch.full((gdr.chunk_fwd_workspace_size(args) // 4,), float("nan"), device="cuda")
    o = torch.full_like(dev["v"], float("nan"))
    o, S = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], None,
                         dev["cu_seqlens"], workspace=ws, o=o)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    o_ref, S_ref = run_oracle(x, "post", 1 / math.sqrt(128))
    assert_close("o", o, o_ref, torch.bfloat16)


# ----------------------------------------------------------------- full-size workloads

def test_training_shape_workload_whole():
    """B=8, T=4096, H=16, d=128, bf16: every element of o and S_final."""
    w = workloads.WORKLOADS["bf16_b8_h16_t4096_d128"]
    x = workloads.workload_inputs(w)
    o, S = run_gpu(x, chunk=w.chunk, read_mode=w.read_mode, scale=w.scale)
    compare_whole(x, o, S, w.read_mode, w.scale, torch.bfloat16)


def test_varlen_workload_whole():
    """64 packed sequences of 256-8192 tokens with per-sequence S0: every element."""
    w = workloads.WORKLOADS["bf16_varlen64_h16_d128"]
    x = workloads.workload_inputs(w)
    o, S = run_gpu(x, chunk=w.chunk, read_mode=w.read_mode, scale=w.scale)
    compare_whole(x, o, S, w.read_mode, w.scale, torch.bfloat16)


def test_bidirectional_workload_whole():
    """16 x 2048 tokens, H=12, d=64, both directions pre-write, summed in one call (fp32 sum,
    one rounding): every element."""
    w = workloads.WORKLOADS["bf16_bidir_16x2048_h12_d64"]
    x = workloads.workload_inputs(w)
    dev = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    o = gdr.chunk_fwd_bidir(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["g_bwd"],
                            dev["beta_bwd"], dev["cu_seqlens"], chunk=w.chunk, read_mode="pre",
                            scale=w.scale)
    torch.cuda.synchronize()
    o_f, _ = run_oracle(x, "pre", w.scale)
    xb = dict(x, g=x["g_bwd"], beta=x["beta_bwd"])
    o_b, _ = run_oracle(xb, "pre", w.scale, reverse=True)
    assert_close("o", o, o_f + o_b, torch.bfloat16)
