"""Helpers shared by the GPU parity tests: run the library and the oracle on the same
seeded inputs and compare with the tolerances the workloads state.

Tolerances (written here once, used by every parity test):
  fp32 inputs:  max |gpu - oracle| <= 1e-4 on o and on S_final.
  bf16 inputs, a result written in bf16 (o, and the backward's bf16 gradients):
                |gpu - oracle| <= 2e-2 RMS(oracle) + 2^-8 |oracle| element-wise.
                The first term is the stated budget (max-abs 2e-2 RMS(o)); the second is
                the one rounding of the exact result to bf16 (round to nearest: at most half
                an ulp, 2^-8 relative), which no bf16 output can avoid and which alone
                exceeds 2e-2 RMS on heavy-tailed outputs (max |o| ~ 10 RMS).
  bf16 inputs, an fp32 result (S_final, the decode state, dS0):
                max |gpu - oracle| <= 2e-2 RMS(oracle), nothing added: fp32 results are
                never rounded to bf16.
A result assembled from parts that were each rounded to bf16 first (the two-call
bidirectional form: each direction written in bf16, then their sum) adds 2^-8 |part| for
every such part: those roundings are what the call is defined to do.

Every comparison is recorded (max |err| / RMS and the fraction of the bound used) and the
session prints the table at the end (``conftest.py``), so the margins are on record.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
REL_BF16 = 2e-2
ROUND_BF16 = 2.0 ** -8

# (test id, name, max |err|, RMS(ref), fraction of the allowed bound used)
RECORDS: list[tuple] = []


def _test_id() -> str:
    t = os.environ.get("PYTEST_CURRENT_TEST", "")
    return t.split(" ")[0] if t else "?"


def record(name: str, max_err: float, rms: float, used: float) -> None:
    RECORDS.append((_test_id(), name, max_err, rms, used))


def to_dev(x):
    return None if x is None else x.cuda().contiguous()


def max_err(gpu: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu.detach().double().cpu().numpy()
    return float(np.abs(g - ref).max()) if ref.size else 0.0


def _np(x):
    if isinstance(x, np.ndarray):
        return x
    return x.detach().double().cpu().numpy()


class Accum:
    """Parity of one tensor accumulated over groups of a large workload: the RMS term of the
    bound is the RMS of the WHOLE tensor, so each group only keeps the part of its error the
    RMS term has to cover (err - 2^-8 |ref| for a bf16 output) and the sums of squares."""

    def __init__(self, name: str, dtype, kind: str = "out"):
        assert kind in ("out", "state")
        self.name, self.dtype, self.kind = name, dtype, kind
        self.excess = 0.0     # max over elements of err - rounding allowance
        self.err = 0.0        # max |err|
        self.ss = 0.0         # sum of ref^2
        self.n = 0
        self.where = ""

    def add(self, gpu, ref, rounded_parts=(), label: str = "") -> None:
        g, r = _np(gpu), _np(ref)
        if not r.size:
            return
        e = np.abs(g - r)
        if not np.all(np.isfinite(g)):
            raise AssertionError(f"{self.name}{label}: non-finite GPU values")
        allow = 0.0
        if self.dtype == torch.bfloat16 and self.kind == "out":
            allow = ROUND_BF16 * np.abs(r)
            for p in rounded_parts:
                allow = allow + ROUND_BF16 * np.abs(_np(p))
        ex = e - allow
        i = int(np.argmax(ex))
        if ex.flat[i] > self.excess or not self.where:
            self.where = (f"{label} flat index {i}: ref {r.flat[i]:.5e}, gpu {g.flat[i]:.5e}, "
                          f"err {e.flat[i]:.3e}")
        self.excess = max(self.excess, float(ex.flat[i]))
        self.err = max(self.err, float(e.max()))
        self.ss += float(np.sum(r * r))
        self.n += r.size

    def check(self) -> tuple[float, float]:
        """Assert the bound over everything added; returns (max |err|, allowed base)."""
        if self.n == 0:
            return 0.0, 0.0
        rms = float(np.sqrt(self.ss / self.n))
        base = TOL_F32 if self.dtype == torch.float32 else REL_BF16 * max(rms, 1e-30)
        used = self.excess / base
        record(self.name, self.err, rms, used)
        assert self.excess <= base, (
            f"{self.name}: error beyond the bound by {self.excess - base:.3e} "
            f"(base {base:.3e}, RMS {rms:.3e}; worst at {self.where}); max err {self.err:.3e}")
        return self.err, base


def assert_close(name, gpu, ref, dtype, kind: str = "out", rounded_parts=()):
    """Element-wise parity check of one tensor; returns (max error, base tolerance).
    kind "out": a result written in the io dtype; "state": an fp32 state (S_final, dS0)."""
    a = Accum(name, dtype, kind)
    a.add(gpu, ref, rounded_parts)
    return a.check()


def oracle_units(x, units, read_mode, scale, qk_l2norm=True, reverse=False, gkey="g",
                 bkey="beta"):
    """Oracle on selected (sequence, v-head) units of a (possibly packed) problem.
    Returns {(s, h): (o [L, dv], S_final [dk, dv])}."""
    q, k, v, g, b = x["q"], x["k"], x["v"], x[gkey], x[bkey]
    B, T, Hk, dk = q.shape
    Hv = v.shape[2]
    grp = Hv // Hk
    cu = x.get("cu_seqlens")
    out = {}
    for s, h in units:
        if cu is None:
            row, t0, t1 = s, 0, T
        else:
            row, t0, t1 = 0, int(cu[s]), int(cu[s + 1])
        sl = slice(t0, t1)
        S0 = None if x.get("S0") is None else x["S0"][s:s + 1, h:h + 1]
        o, S = oracle.forward(q[row:row + 1, sl, h // grp:h // grp + 1],
                              k[row:row + 1, sl, h // grp:h // grp + 1],
                              v[row:row + 1, sl, h:h + 1], g[row:row + 1, sl, h:h + 1],
                              b[row:row + 1, sl, h:h + 1], S0, read_mode=read_mode, scale=scale,
                              qk_l2norm=qk_l2norm, reverse=reverse)
        out[(s, h)] = (o[0, :, 0], S[0, 0])
    return out


def sequence_groups(x, max_tokens: int = 1 << 16):
    """Split a problem into groups of whole sequences for the oracle, each at most about
    ``max_tokens`` tokens (one sequence may exceed it): yields (row slice, token slice,
    sequence slice, cu_seqlens of the group or None)."""
    cu = x.get("cu_seqlens")
    B, T = x["q"].shape[:2]
    if cu is None:
        per = max(1, max_tokens // max(T, 1))
        for r0 in range(0, B, per):
            r1 = min(B, r0 + per)
            yield slice(r0, r1), slice(0, T), slice(r0, r1), None
        return
    c = [int(t) for t in cu]
    n = len(c) - 1
    s0 = 0
    while s0 < n:
        s1 = s0 + 1
        while s1 < n and c[s1 + 1] - c[s0] <= max_tokens:
            s1 += 1
        t0, t1 = c[s0], c[s1]
        sub = torch.tensor([t - t0 for t in c[s0:s1 + 1]], dtype=torch.int32)
        yield slice(0, 1), slice(t0, t1), slice(s0, s1), sub
        s0 = s1


def oracle_group(x, rows, toks, seqs, cu, read_mode, scale, reverse=False, gkey="g",
                 bkey="beta", with_s0=True):
    """The fp64 oracle over one group of whole sequences (from ``sequence_groups``)."""
    sl = lambda t: t[rows, toks]
    S0 = x.get("S0")
    S0 = None if (S0 is None or not with_s0) else S0[seqs]
    return oracle.forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x[gkey]), sl(x[bkey]), S0, cu,
                          read_mode=read_mode, scale=scale, reverse=reverse)


def compare_whole(x, o, S, read_mode, scale, dtype, name="", reverse=False, gkey="g",
                  bkey="beta"):
    """Every element of o (and S_final, unless None) of a whole workload against the oracle,
    computed group by group so the fp64 copies stay bounded."""
    ao = Accum(f"o{name}", dtype, "out")
    aS = Accum(f"S_final{name}", dtype, "state")
    o_c = o.detach().cpu()
    S_c = None if S is None else S.detach().cpu()
    for rows, toks, seqs, cu in sequence_groups(x):
        o_r, S_r = oracle_group(x, rows, toks, seqs, cu, read_mode, scale, reverse, gkey, bkey)
        ao.add(o_c[rows, toks], o_r, label=f" seqs {seqs.start}-{seqs.stop - 1}")
        if S_c is not None:
            aS.add(S_c[seqs], S_r, label=f" seqs {seqs.start}-{seqs.stop - 1}")
    ao.check()
    if S_c is not None:
        aS.check()


def oracle_backward_sequence(job):
    """One sequence of a fixed-length workload through the fp64 backward oracle (a process
    pool's task: the arrays arrive and leave as NumPy, the reference as float32, whose
    rounding is far below any bound it is compared with)."""
    import oracle.backward as obw
    arrays, kw = job
    ref = obw.backward(*arrays, **kw)
    return {n: a.astype(np.float32) for n, a in ref.items()}


def oracle_gdn2_sequence(job):
    """One sequence of a fixed-length workload through the fp64 GDN-2 oracle (a process
    pool's task; the reference returns as float32, far below any bound it meets)."""
    arrays, kw = job
    o, S = oracle.gdn2_forward(*arrays, **kw)
    return o.astype(np.float32), S.astype(np.float32)
