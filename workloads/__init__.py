"""Seeded synthetic inputs for the gated delta-rule workloads.

This module holds no arithmetic of the method: it only draws random tensors
with the shapes and value distributions the workloads call for, on the CPU,
from an explicit ``torch.Generator``.  Both the CUDA path (tests, benchmark)
and the fp64 oracle consume what it returns.

Distributions (shared by every workload):
  q, k   ~ N(0, 1); the L2 normalisation the workloads ask for is done by the
           path itself (``qk_l2norm=1``), on the GPU and in the oracle alike,
  v      ~ N(0, 1),
  g      = -softplus(x), x ~ N(-2, 1)   (log of the decay alpha, alpha in (0, 1)),
  beta   = sigmoid(N(0, 1)),
  S0     ~ N(0, 0.02^2) in fp32 where a workload has an initial state.
Draw order: (varlen lengths), q, k, v, g-logits, beta-logits, (second direction's
g-logits, beta-logits), S0.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class ChunkWorkload:
    name: str
    B: int
    T: int              # tokens per row (fixed length) -- ignored when n_varlen > 0
    Hk: int
    Hv: int
    dk: int
    dv: int
    chunk: int
    dtype: str          # io dtype of q, k, v, o ("f32" or "bf16")
    gate_dtype: str     # dtype of g and beta
    read_mode: str      # "post" or "pre"
    scale: float
    n_varlen: int = 0   # >0: that many packed sequences with random lengths
    len_lo: int = 0
    len_hi: int = 0
    fixed_seg: int = 0  # >0: B=1 packed segments of this length (bidirectional)
    n_seg: int = 0
    s0_std: float = 0.0  # >0: per-sequence initial state N(0, s0_std^2)
    bidirectional: bool = False


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    N: int
    Hk: int
    Hv: int
    dk: int
    dv: int
    steps: int
    dtype: str
    gate_dtype: str
    read_mode: str
    scale: float
    s_std: float = 0.02


WORKLOADS = {
    # oracle-sized forward, fp32 end to end
    "fp32_b1_h2_t256_d64": ChunkWorkload(
        "fp32_b1_h2_t256_d64", B=1, T=256, Hk=2, Hv=2, dk=64, dv=64, chunk=64, dtype="f32",
        gate_dtype="f32", read_mode="post", scale=1.0 / math.sqrt(64)),
    # training-shape chunked forward
    "bf16_b8_h16_t4096_d128": ChunkWorkload(
        "bf16_b8_h16_t4096_d128", B=8, T=4096, Hk=16, Hv=16, dk=128, dv=128, chunk=64,
        dtype="bf16", gate_dtype="bf16", read_mode="post", scale=1.0 / math.sqrt(128)),
    # 64 packed sequences, lengths uniform in [256, 8192], per-sequence initial state
    "bf16_varlen64_h16_d128": ChunkWorkload(
        "bf16_varlen64_h16_d128", B=1, T=0, Hk=16, Hv=16, dk=128, dv=128, chunk=64,
        dtype="bf16", gate_dtype="bf16", read_mode="post", scale=1.0 / math.sqrt(128),
        n_varlen=64, len_lo=256, len_hi=8192, s0_std=0.02),
    # 16 segments x 2048, both directions, strictly causal pre-write read, outputs summed
    "bf16_bidir_16x2048_h12_d64": ChunkWorkload(
        "bf16_bidir_16x2048_h12_d64", B=1, T=0, Hk=12, Hv=12, dk=64, dv=64, chunk=64,
        dtype="bf16", gate_dtype="bf16", read_mode="pre", scale=1.0, fixed_seg=2048, n_seg=16,
        bidirectional=True),
}

DECODE_WORKLOADS = {
    # 256 sequences, 16 k-heads broadcast to 32 v-heads, 64 consecutive steps
    "bf16_decode_n256_hk16_hv32_d128": DecodeWorkload(
        "bf16_decode_n256_hk16_hv32_d128", N=256, Hk=16, Hv=32, dk=128, dv=128, steps=64,
        dtype="bf16", gate_dtype="bf16", read_mode="post", scale=1.0 / math.sqrt(128)),
}


def _gen(seed: int) -> torch.Generator:
    return torch.Generator("cpu").manual_seed(seed)


def _gates(shape, gen, gate_dtype):
    x = torch.randn(shape, generator=gen) - 2.0
    g = -torch.nn.functional.softplus(x)
    b = torch.sigmoid(torch.randn(shape, generator=gen))
    return g.to(DTYPES[gate_dtype]), b.to(DTYPES[gate_dtype])


def chunk_inputs(B, T, Hk, Hv, dk, dv, dtype="bf16", gate_dtype=None, lengths=None,
                 s0_std=0.0, bidirectional=False, seed=0, gen=None):
    """Draw one forward problem.  With ``lengths`` the sequences are packed into one row
    (B must be 1, T is ignored) and ``cu_seqlens`` is returned.  Returns a dict of CPU
    tensors: q, k [B,T,Hk,dk]; v [B,T,Hv,dv]; g, beta [B,T,Hv]; S0 [n_seqs,Hv,dk,dv] or
    None; cu_seqlens int32 [n_seqs+1] or None; and g_bwd, beta_bwd when bidirectional."""
    gate_dtype = gate_dtype or dtype
    gen = gen or _gen(seed)
    cu = None
    if lengths is not None:
        lengths = torch.as_tensor(lengths, dtype=torch.int64)
        assert B == 1
        cu = torch.zeros(lengths.numel() + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(lengths, 0).to(torch.int32)
        T = int(cu[-1])
    n_seqs = B if cu is None else cu.numel() - 1
    dt = DTYPES[dtype]
    out = {
        "q": torch.randn((B, T, Hk, dk), generator=gen).to(dt),
        "k": torch.randn((B, T, Hk, dk), generator=gen).to(dt),
        "v": torch.randn((B, T, Hv, dv), generator=gen).to(dt),
    }
    out["g"], out["beta"] = _gates((B, T, Hv), gen, gate_dtype)
    if bidirectional:
        out["g_bwd"], out["beta_bwd"] = _gates((B, T, Hv), gen, gate_dtype)
    out["S0"] = (torch.randn((n_seqs, Hv, dk, dv), generator=gen) * s0_std
                 if s0_std > 0 else None)
    out["cu_seqlens"] = cu
    return out


def workload_inputs(w: ChunkWorkload, seed: int = 0):
    """Inputs of a named forward workload at its full size."""
    gen = _gen(seed)
    lengths = None
    if w.n_varlen:
        lengths = torch.randint(w.len_lo, w.len_hi + 1, (w.n_varlen,), generator=gen)
    elif w.fixed_seg:
        lengths = torch.full((w.n_seg,), w.fixed_seg, dtype=torch.int64)
    return chunk_inputs(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.dtype, w.gate_dtype, lengths,
                        w.s0_std, w.bidirectional, gen=gen)


def decode_inputs(N, Hk, Hv, dk, dv, steps, dtype="bf16", gate_dtype=None, s_std=0.02, seed=0):
    """Inputs of ``steps`` consecutive one-token decode steps: q, k [steps,N,Hk,dk];
    v [steps,N,Hv,dv]; g, beta [steps,N,Hv]; the initial state S [N,Hv,dk,dv] fp32."""
    gate_dtype = gate_dtype or dtype
    gen = _gen(seed)
    dt = DTYPES[dtype]
    out = {
        "q": torch.randn((steps, N, Hk, dk), generator=gen).to(dt),
        "k": torch.randn((steps, N, Hk, dk), generator=gen).to(dt),
        "v": torch.randn((steps, N, Hv, dv), generator=gen).to(dt),
    }
    out["g"], out["beta"] = _gates((steps, N, Hv), gen, gate_dtype)
    out["S"] = torch.randn((N, Hv, dk, dv), generator=gen) * s_std
    return out


def decode_workload_inputs(w: DecodeWorkload, seed: int = 0):
    return decode_inputs(w.N, w.Hk, w.Hv, w.dk, w.dv, w.steps, w.dtype, w.gate_dtype, w.s_std,
                         seed)


def raw_gate_inputs(shape, Hv, gate_dtype="bf16", seed=0):
    """Raw gate projections for the fused gating prologue: a ~ N(-2, 1) and b ~ N(0, 1) in
    the gate dtype, with per-head A = -1 and dt_bias = 0 (fp32), so that the gates the
    kernels form, g = A softplus(a + dt_bias) and beta = sigmoid(b), follow the same
    distributions as the workloads' direct gates."""
    gen = _gen(seed + 7919)
    dt = DTYPES[gate_dtype]
    a = (torch.randn(shape, generator=gen) - 2.0).to(dt)
    b = torch.randn(shape, generator=gen).to(dt)
    return a, b, torch.full((Hv,), -1.0), torch.zeros(Hv)


def gdn2_gate_inputs(shape, dk, dv, gate_dtype="bf16", seed=0):
    """Decoupled GDN-2 gates for tokens of ``shape`` (e.g. [B, T, Hv]): per key channel the
    log decay g = -softplus(N(-2, 1)) and erase gate b = sigmoid(N(0, 1)) [*shape, dk], per
    value channel the write gate w = sigmoid(N(0, 1)) [*shape, dv], in the gate dtype."""
    gen = _gen(seed + 104729)
    dt = DTYPES[gate_dtype]
    shape = tuple(shape)
    g = -torch.nn.functional.softplus(torch.randn(shape + (dk,), generator=gen) - 2.0)
    b = torch.sigmoid(torch.randn(shape + (dk,), generator=gen))
    w = torch.sigmoid(torch.randn(shape + (dv,), generator=gen))
    return g.to(dt), b.to(dt), w.to(dt)
