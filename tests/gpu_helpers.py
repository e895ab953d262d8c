"""Helpers shared by the GPU parity tests: run the library and the oracle on the same
seeded inputs and compare with the tolerances the workloads state.

Tolerances (written here once, used by every parity test):
  fp32 inputs:  max |gpu - oracle| <= 1e-4 on o and on S_final;
  bf16 inputs:  |gpu - oracle| <= 2e-2 * RMS(oracle) + 2^-7 |oracle| element-wise, on o
                and on the fp32 S_final alike.  The first term is the stated budget; the
                second is the relative error bf16 itself puts on each element: a bf16
                result is rounded once (<= 2^-8 relative, near a rounding boundary), and a
                product of two bf16 tensor-core operands (normalised k, V') carries two
                roundings of <= 2^-9 each; 2^-7 leaves a factor 2 over that.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
REL_BF16 = 2e-2
REL_ELEM_BF16 = 2.0 ** -7


def tol_for(dtype, ref: np.ndarray) -> float:
    if dtype == torch.float32:
        return TOL_F32
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return REL_BF16 * max(rms, 1e-30)


def to_dev(x):
    return None if x is None else x.cuda().contiguous()


def max_err(gpu: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu.detach().double().cpu().numpy()
    return float(np.abs(g - ref).max()) if ref.size else 0.0


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """One bf16 ulp of |x|: 2^(floor(log2 |x|) - 7) (8 significant bits)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 7), 0.0)


def assert_close(name, gpu, ref, dtype):
    """Element-wise parity check; returns (max error, max allowed) for the report."""
    tol = tol_for(dtype, ref)
    g = gpu.detach().double().cpu().numpy()
    if not ref.size:
        return 0.0, tol
    err = np.abs(g - ref)
    allowed = tol + (REL_ELEM_BF16 * np.abs(ref) if dtype == torch.bfloat16 else 0.0)
    worst = int(np.argmax(err - allowed))
    assert np.all(err <= allowed), (
        f"{name}: err {err.flat[worst]:.3e} > allowed {np.asarray(allowed).flat[worst] if np.ndim(allowed) else allowed:.3e} "
        f"at flat index {worst} (ref {ref.flat[worst]:.4e}, gpu {g.flat[worst]:.4e}); "
        f"max err {err.max():.3e}, base tol {tol:.3e}")
    return float(err.max()), tol


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
