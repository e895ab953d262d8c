"""Parity of the tcgen05 tensor-core path (bf16, dk = dv = 128 or 64, chunk 64) against the
oracle, on shapes that exercise every branch of the fused kernel."""
import math

import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
from gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def run(x, **kw):
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    o, S = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d.get("S0"),
                         d.get("cu_seqlens"), **kw)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("d", [128, 64])
def test_path_is_tensor_core(d):
    x = workloads.chunk_inputs(1, 64, 1, 1, d, d, "bf16")
    a = gdr.make_chunk_args(to_dev(x["q"]), to_dev(x["v"]), to_dev(x["g"]))
    assert gdr.chunk_fwd_path(a) == "tc"


@pytest.mark.parametrize("read_mode", ["post", "pre"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000])
@pytest.mark.parametrize("d", [128, 64])
def test_lengths(read_mode, T, d):
    x = workloads.chunk_inputs(2, T, 2, 4, d, d, "bf16", s0_std=0.02, seed=T + d)
    scale = 1 / math.sqrt(d)
    o, S = run(x, read_mode=read_mode, scale=scale)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"],
                              read_mode=read_mode, scale=scale)
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("d", [128, 64])
def test_varlen_reverse(reverse, d):
    lengths = [1, 0, 64, 65, 130, 0, 7, 300, 129]
    x = workloads.chunk_inputs(1, 0, 2, 2, d, d, "bf16", lengths=lengths, s0_std=0.05,
                               seed=11 + d)
    o, S = run(x, read_mode="pre", scale=0.3, reverse=reverse)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"],
                              x["cu_seqlens"], read_mode="pre", scale=0.3, reverse=reverse)
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_accumulate_and_fp32_gates():
    x = workloads.chunk_inputs(1, 300, 1, 2, 128, 128, "bf16", gate_dtype="f32", seed=13)
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    base = (0.01 * torch.randn(d["v"].shape, device="cuda")).to(torch.bfloat16)
    o = base.clone()
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], o=o, o_accumulate=True)
    torch.cuda.synchronize()
    o_r, _ = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], scale=1 / math.sqrt(128))
    # o = bf16(base + bf16(result)): this call's result is written in bf16 before the sum
    assert_close("o", o, o_r + base.double().cpu().numpy(), torch.bfloat16, rounded_parts=(o_r,))


def test_no_l2norm_and_large_beta():
    x = workloads.chunk_inputs(1, 256, 1, 1, 128, 128, "bf16", seed=14)
    q = x["q"].float()
    x["q"] = (q / q.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    k = x["k"].float()
    x["k"] = (k / k.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    x["beta"] = (2 * x["beta"].float()).to(torch.bfloat16)
    o, S = run(x, qk_l2norm=False)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], None,
                              scale=1 / math.sqrt(128), qk_l2norm=False)
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_alpha_half_and_repeated_keys():
    x = workloads.chunk_inputs(1, 256, 1, 1, 128, 128, "bf16", s0_std=0.5, seed=15)
    x["g"] = torch.full_like(x["g"], math.log(0.5))
    x["k"] = x["k"][:, :1].expand_as(x["k"]).contiguous()
    o, S = run(x)
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"],
                              scale=1 / math.sqrt(128))
    assert_close("o", o, o_r, torch.bfloat16)
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_state_aliasing_in_place():
    """S_final may alias S0 (each CTA reads its whole slice before it writes)."""
    x = workloads.chunk_inputs(2, 130, 1, 2, 128, 128, "bf16", s0_std=0.1, seed=16)
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    S = d["S0"].clone()
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, S_final=S)
    torch.cuda.synchronize()
    _, S_r = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"],
                            scale=1 / math.sqrt(128))
    assert_close("S", S, S_r, torch.bfloat16, kind="state")


def test_fp16_range_is_reported():
    """Values far beyond the fp16 range of the internal operands raise GDR_ERR_RANGE
    instead of returning silently wrong results."""
    x = workloads.chunk_inputs(1, 100, 1, 1, 128, 128, "bf16", seed=17)
    x["v"] = (x["v"].float() * 1e6).to(torch.bfloat16)
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    args = gdr.make_chunk_args(d["q"], d["v"], d["g"])
    ws = torch.empty(gdr.chunk_fwd_workspace_size(args), dtype=torch.uint8, device="cuda")
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], workspace=ws)
    assert gdr.read_device_error(args, ws) == gdr._abi.GDR_ERR_RANGE
    # the same status without a synchronisation inside the library: through the caller's
    # status word, from gdr_chunk_fwd and from gdr_chunk_fwd_noalloc
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], workspace=ws, status=status[0:1])
    na = gdr.make_chunk_args(d["q"], d["v"], d["g"], status=status[1:2])
    o = torch.empty_like(d["v"])
    S = torch.empty((1, 1, 128, 128), device="cuda")
    assert gdr.chunk_fwd_noalloc(na, d["q"], d["k"], d["v"], d["g"], d["beta"], None, None, o,
                                 S) == gdr._abi.GDR_OK
    assert status.tolist() == [gdr._abi.GDR_ERR_RANGE, gdr._abi.GDR_ERR_RANGE]
    x["v"] = (x["v"].float() * 1e-6).to(torch.bfloat16)
    status.zero_()
    gdr.chunk_fwd(d["q"], d["k"], to_dev(x["v"]), d["g"], d["beta"], workspace=ws,
                  status=status[0:1])
    assert gdr.read_device_error(args, ws) == gdr._abi.GDR_OK
    assert status.tolist() == [0, 0]


def test_head_size_64_accumulate_and_aliasing():
    """64-wide heads: accumulation into o (plain stores) and S_final aliasing S0."""
    x = workloads.chunk_inputs(2, 150, 1, 3, 64, 64, "bf16", s0_std=0.1, seed=18)
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    base = (0.01 * torch.randn(d["v"].shape, device="cuda")).to(torch.bfloat16)
    o = base.clone()
    S = d["S0"].clone()
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, o=o, o_accumulate=True,
                  S_final=S, scale=0.125)
    torch.cuda.synchronize()
    o_r, S_r = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], scale=0.125)
    assert_close("o", o, o_r + base.double().cpu().numpy(), torch.bfloat16, rounded_parts=(o_r,))
    assert_close("S", S, S_r, torch.bfloat16, kind="state")
