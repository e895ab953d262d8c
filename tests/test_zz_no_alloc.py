"""gdr_chunk_fwd_noalloc, the forward for callers that cannot allocate device memory (its
scratch is a static device array inside the library), against gdr_chunk_fwd with a
torch-allocated workspace, and against the fp64 oracle.

Both entry points run the same deterministic kernels on the same inputs, so their outputs
must be identical bit for bit; the oracle comparison checks that result itself.

This file is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.
"""
import math

import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
from gated_delta_rule_146_b200 import _abi
from gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _inputs(dtype, seed, lengths):
    d = 128 if dtype == "bf16" else 64
    x = workloads.chunk_inputs(1, 0, 2, 4, d, d, dtype, lengths=lengths, s0_std=0.02, seed=seed)
    return x, {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    """Two calls in a row (different inputs, so the second cannot reuse the first's scratch
    contents by accident): each identical to the workspace entry point, bit for bit, and
    the first also within the parity bound of the oracle."""
    for i, (seed, lengths) in enumerate(((1, [100, 300, 64]), (2, [257, 1, 70]))):
        x, d = _inputs(dtype, seed, lengths)
        o_ref, S_ref = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"],
                                     d["cu_seqlens"])
        args = gdr.make_chunk_args(d["q"], d["v"], d["g"], d["cu_seqlens"])
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        st = gdr.chunk_fwd_noalloc(args, d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"],
                                   d["cu_seqlens"], o, S)
        assert st == _abi.GDR_OK, gdr._abi.status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), "o differs from gdr_chunk_fwd"
        assert torch.equal(S, S_ref), "S_final differs from gdr_chunk_fwd"
        assert gdr.noalloc_read_device_error() == _abi.GDR_OK
        if i == 0:
            scale = 1.0 / math.sqrt(x["q"].shape[-1])
            o_or, S_or = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"],
                                        x["cu_seqlens"], scale=scale)
            tdt = workloads.DTYPES[dtype]
            assert_close("o (noalloc)", o, o_or, tdt)
            assert_close("S_final (noalloc)", S, S_or, tdt, kind="state")


def test_noalloc_device_errors_are_readable():
    """A cu_seqlens that decreases (caught on the device) is reported through the accessor
    and through the caller's status word; the next good call clears the scratch's word."""
    x, d = _inputs("bf16", 4, [10, 20])
    bad = torch.tensor([0, 20, 10], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = gdr.make_chunk_args(d["q"], d["v"], d["g"], bad, status=status)
    o = torch.empty_like(d["v"])
    S = torch.empty((2, 4, 128, 128), device="cuda")
    assert gdr.chunk_fwd_noalloc(args, d["q"], d["k"], d["v"], d["g"], d["beta"], None, bad, o,
                                 S) == _abi.GDR_OK
    assert gdr.noalloc_read_device_error() == _abi.GDR_ERR_DEVICE_CHECK
    assert int(status.item()) == _abi.GDR_ERR_DEVICE_CHECK
    args = gdr.make_chunk_args(d["q"], d["v"], d["g"], d["cu_seqlens"])
    assert gdr.chunk_fwd_noalloc(args, d["q"], d["k"], d["v"], d["g"], d["beta"], None,
                                 d["cu_seqlens"], o, S) == _abi.GDR_OK
    assert gdr.noalloc_read_device_error() == _abi.GDR_OK


def test_noalloc_rejects_scratch_beyond_the_array():
    """The CUDA-core path's scratch grows with B*T*Hv*(dk+dv); past the array it is refused
    before anything is enqueued."""
    x = workloads.chunk_inputs(1, 8192, 4, 4, 64, 64, "f32", seed=3)
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    args = gdr.make_chunk_args(d["q"], d["v"], d["g"])
    assert gdr.chunk_fwd_workspace_size(args) > (4 << 20)
    o = torch.empty_like(d["v"])
    S = torch.empty((1, 4, 64, 64), device="cuda")
    assert gdr.chunk_fwd_noalloc(args, d["q"], d["k"], d["v"], d["g"], d["beta"], None, None,
                                 o, S) == _abi.GDR_ERR_WORKSPACE
