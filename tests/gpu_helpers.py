"""Helpers shared by the GPU parity tests: run the library and the oracle on the same
seeded inputs and compare with the tolerances the workloads state.

Tolerances (written here once, used by every parity test):
  fp32 inputs:  max |gpu - oracle| <= 1e-4 on o and on S_final;
  bf16 inputs:  max |gpu - oracle| <= 2e-2 * RMS(oracle o) on o, and
                <= 2e-2 * RMS(oracle S_final) on S_final (fp32 state and accumulation).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
REL_BF16 = 2e-2


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


def assert_close(name, gpu, ref, dtype):
    tol = tol_for(dtype, ref)
    err = max_err(gpu, ref)
    assert err <= tol, f"{name}: max abs err {err:.3e} > tol {tol:.3e}"
    return err, tol


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
