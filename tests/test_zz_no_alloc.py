"""gdr_chunk_fwd_noalloc (the forward with its scratch in a static device array, for callers
that cannot allocate device memory) against gdr_chunk_fwd with a torch-allocated workspace.

This file is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.
"""
import ctypes

import pytest
import torch

import workloads
import gated_delta_rule_146_b200 as gdr
from gated_delta_rule_146_b200 import _abi
from gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(args, d, o, S_final):
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return _abi.lib().gdr_chunk_fwd_noalloc(
        ctypes.byref(args), vp(d["q"]), vp(d["k"]), vp(d["v"]), vp(d["g"]), vp(d["beta"]),
        vp(d.get("S0")), vp(d.get("cu_seqlens")), vp(o), vp(S_final),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    """Two calls in a row (different inputs, so the second cannot reuse the first's scratch
    contents by accident), each compared with the workspace entry point."""
    for seed, lengths in ((1, [100, 300, 64]), (2, [257, 1, 70])):
        x = workloads.chunk_inputs(1, 0, 2, 4, 128 if dtype == "bf16" else 64,
                                   128 if dtype == "bf16" else 64, dtype, lengths=lengths,
                                   s0_std=0.02, seed=seed)
        d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
        o_ref, S_ref = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"],
                                     d["cu_seqlens"])
        args = gdr.make_chunk_args(d["q"], d["v"], d["g"], d["cu_seqlens"])
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        assert _noalloc(args, d, o, S) == _abi.GDR_OK
        torch.cuda.synchronize()
        tdt = workloads.DTYPES[dtype]
        assert_close("o", o, o_ref.double().cpu().numpy(), tdt)
        assert_close("S_final", S, S_ref.double().cpu().numpy(), tdt)


def test_noalloc_rejects_scratch_beyond_the_array():
    """The CUDA-core path's scratch grows with B*T*Hv*(dk+dv); past the array it is refused
    before anything is enqueued."""
    x = workloads.chunk_inputs(1, 8192, 4, 4, 64, 64, "f32", seed=3)
    d = {n: to_dev(x[n]) if x.get(n) is not None else None for n in x}
    args = gdr.make_chunk_args(d["q"], d["v"], d["g"])
    assert gdr.chunk_fwd_workspace_size(args) > (4 << 20)
    o = torch.empty_like(d["v"])
    S = torch.empty((1, 4, 64, 64), device="cuda")
    assert _noalloc(args, d, o, S) == _abi.GDR_ERR_WORKSPACE
