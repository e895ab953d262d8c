"""GPU parity of the one-call bidirectional forward (gdr_chunk_fwd_bidir) against the fp64
oracle's bidirectional scan (both directions from zero states, outputs summed), and of the
two-call form (forward, then the reverse scan accumulating into o).

On the tensor-core path the one call runs both scans of every (sequence, head) as a pair of
CTAs that sum the two directions in fp32 and round once; the two-call form rounds each
direction's output to bf16 before the sum."""
import pytest
import torch

import oracle
import workloads
import gated_delta_rule_146_b200 as gdr
from gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def both(x, **kw):
    d = {n: to_dev(t) if t is not None else None for n, t in x.items()}
    o1 = gdr.chunk_fwd_bidir(d["q"], d["k"], d["v"], d["g"], d["beta"], d["g_bwd"],
                             d["beta_bwd"], d["cu_seqlens"], **kw)
    o2, _ = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["cu_seqlens"],
                          output_final_state=False, **kw)
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g_bwd"], d["beta_bwd"], None, d["cu_seqlens"],
                  output_final_state=False, reverse=True, o=o2, o_accumulate=True, **kw)
    torch.cuda.synchronize()
    return o1, o2


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("read_mode", ["pre", "post"])
def test_tensor_core_path(d, read_mode):
    # lengths that are not multiples of the chunk (the reverse scan's chunks are aligned with
    # the forward scan's), an empty and a one-token sequence, and odd and even chunk counts
    lengths = [70, 0, 200, 1, 128, 150, 1000]
    x = workloads.chunk_inputs(1, 0, 2, 4, d, d, "bf16", lengths=lengths, bidirectional=True,
                               seed=81)
    args = gdr.make_chunk_args(to_dev(x["q"]), to_dev(x["v"]), to_dev(x["g"]))
    assert gdr.chunk_fwd_path(args) == "tc"
    o1, o2 = both(x, read_mode=read_mode, scale=1.0)
    o_f, _ = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                            read_mode=read_mode, scale=1.0)
    o_b, _ = oracle.forward(x["q"], x["k"], x["v"], x["g_bwd"], x["beta_bwd"], None,
                            x["cu_seqlens"], read_mode=read_mode, scale=1.0, reverse=True)
    # one call: the sum rounded once; two calls: each direction rounded, then the sum
    assert_close("o (one call)", o1, o_f + o_b, torch.bfloat16)
    assert_close("o (two calls)", o2, o_f + o_b, torch.bfloat16, rounded_parts=(o_f, o_b))


def test_swapped_directions_differ():
    """The pair gives each CTA its own direction's gates: swapping the two gate pairs changes
    the result (a pair that read one direction's gates twice would not notice)."""
    x = workloads.chunk_inputs(1, 0, 2, 2, 64, 64, "bf16", lengths=[300, 77], bidirectional=True,
                               seed=85)
    d = {n: to_dev(t) if t is not None else None for n, t in x.items()}
    o1 = gdr.chunk_fwd_bidir(d["q"], d["k"], d["v"], d["g"], d["beta"], d["g_bwd"],
                             d["beta_bwd"], d["cu_seqlens"], read_mode="pre", scale=1.0)
    o2 = gdr.chunk_fwd_bidir(d["q"], d["k"], d["v"], d["g_bwd"], d["beta_bwd"], d["g"],
                             d["beta"], d["cu_seqlens"], read_mode="pre", scale=1.0)
    torch.cuda.synchronize()
    assert not torch.equal(o1, o2)


def test_cuda_core_path_fp32():
    x = workloads.chunk_inputs(1, 0, 1, 2, 64, 32, "f32", lengths=[33, 100, 0, 7],
                               bidirectional=True, seed=83)
    o1, o2 = both(x, read_mode="pre", scale=0.5)
    ref = oracle.bidirectional(x["q"], x["k"], x["v"], x["g"], x["beta"], x["g_bwd"],
                               x["beta_bwd"], x["cu_seqlens"], read_mode="pre", scale=0.5)
    assert_close("o", o1, ref, torch.float32)
    assert_close("o (two calls)", o2, ref, torch.float32)


def test_one_call_is_deterministic():
    """The pair's hand-off is ordered by its counter, not by timing: two calls on the
    bidirectional workload give the same bits."""
    w = workloads.WORKLOADS["bf16_bidir_16x2048_h12_d64"]
    x = workloads.workload_inputs(w)
    d = {n: to_dev(t) if t is not None else None for n, t in x.items()}
    o = [gdr.chunk_fwd_bidir(d["q"], d["k"], d["v"], d["g"], d["beta"], d["g_bwd"],
                             d["beta_bwd"], d["cu_seqlens"], read_mode="pre", scale=w.scale)
         for _ in range(2)]
    torch.cuda.synchronize()
    assert torch.isfinite(o[0].float()).all()
    assert torch.equal(o[0], o[1])
