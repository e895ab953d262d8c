"""fp64 CPU oracle of the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call, link
or execute anything in this package: only the test suite, the smoke check of
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` use it.  It shares
no code with the CUDA library under ``gated_delta_rule_146_b200``.

Three independent implementations live here:

* ``forward`` / ``decode_step`` -- the plain per-token recurrence in fp64 C
  (``gdr_oracle.c``), OpenMP over (sequence, v-head).  This is the oracle the
  GPU path is compared with.  It follows Prizma "seq/delta.py"
  ``_delta_reference`` (the per-token loop) and its module docstring.
* ``wy_reference.chunked_forward`` -- a NumPy fp64 transcription of the
  chunk-parallel WY/UT form of Prizma "seq/delta.py" ``chunked_delta``; used
  only to pin the oracle (different algorithm, same real numbers).
* ``exact.forward_exact`` -- exact rational arithmetic through the
  product-of-transitions form; used only to pin the oracle on tiny inputs.

``gating`` forms the gates from raw projections (the fused gating prologue)
in fp64; the recurrence oracles take its output like any other gates.
``gated_rmsnorm`` is the decode chain's output epilogue in fp64.

Every input arrives already rounded to the dtype the GPU sees (bf16 / fp32);
it is widened exactly to fp64 here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


class _Args(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("Hk", ctypes.c_int), ("Hv", ctypes.c_int),
        ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("n_seqs", ctypes.c_int),
        ("read_pre", ctypes.c_int), ("qk_l2norm", ctypes.c_int), ("reverse", ctypes.c_int),
        ("scale", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile ``gdr_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, strict IEEE)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """Open a compiled oracle library and declare its entry point."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gdr_oracle_forward.argtypes = [ctypes.POINTER(_Args), dp, dp, dp, dp, dp, dp,
                                       ctypes.POINTER(ctypes.c_int32), dp, dp]
    lib.gdr_oracle_forward.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _f64(x) -> np.ndarray:
    """Widen an input (numpy array or CPU torch tensor, any float dtype) to contiguous fp64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: bf16 has no numpy dtype, widen in torch first
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def forward(q, k, v, g, beta, S0=None, cu_seqlens=None, read_mode: str = "post",
            scale: float = 1.0, qk_l2norm: bool = True, reverse: bool = False, _lib=None):
    """Per-token fp64 recurrence over every sequence and v-head.

    q, k: [B, T, Hk, dk]; v: [B, T, Hv, dv]; g, beta: [B, T, Hv]; S0: [n_seqs, Hv, dk, dv]
    or None; cu_seqlens: int [n_seqs+1] or None (then n_seqs = B).  g is log(alpha).
    Returns (o [B, T, Hv, dv], S_final [n_seqs, Hv, dk, dv]) as fp64 numpy arrays.
    ``_lib`` substitutes another compiled copy of the oracle (used by the test that plants
    mistakes in the oracle to show the pins catch them).
    """
    q, k, v, g, beta, S0 = (_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))
        n_seqs = cu.shape[0] - 1
    else:
        cu, n_seqs = None, B
    args = _Args(B, T, Hk, Hv, dk, dv, n_seqs, 1 if read_mode == "pre" else 0,
                 1 if qk_l2norm else 0, 1 if reverse else 0, float(scale))
    o = np.zeros((B, T, Hv, dv), dtype=np.float64)
    S_final = np.zeros((n_seqs, Hv, dk, dv), dtype=np.float64)
    rc = (_lib or _load()).gdr_oracle_forward(
        ctypes.byref(args), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
        None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _ptr(o), _ptr(S_final))
    if rc != 0:
        raise ValueError(f"oracle refused the arguments (code {rc})")
    return o, S_final


def decode_step(q, k, v, g, beta, S, read_mode: str = "post", scale: float = 1.0,
                qk_l2norm: bool = True):
    """One recurrent token per sequence: q, k [N, Hk, dk]; v [N, Hv, dv]; g, beta [N, Hv];
    S [N, Hv, dk, dv].  Returns (o [N, Hv, dv], S_new) in fp64 (S is not modified)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    o, S_new = forward(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                       S0=_f64(S), read_mode=read_mode, scale=scale, qk_l2norm=qk_l2norm)
    return o[:, 0], S_new


def bidirectional(q, k, v, g_fwd, beta_fwd, g_bwd, beta_bwd, cu_seqlens, read_mode: str = "pre",
                  scale: float = 1.0, qk_l2norm: bool = True, read_mode_bwd: str | None = None,
                  combine: float = 1.0):
    """Both scan directions over shared q, k, v, each with its own gates, outputs summed and
    multiplied by ``combine`` (tiny_gdn/fugue.py ``BidirectionalGatedDeltaNet2.forward`` and
    ``scan``; the backward direction scans every segment reversed in place)."""
    o_f, _ = forward(q, k, v, g_fwd, beta_fwd, None, cu_seqlens, read_mode, scale, qk_l2norm)
    o_b, _ = forward(q, k, v, g_bwd, beta_bwd, None, cu_seqlens, read_mode_bwd or read_mode,
                     scale, qk_l2norm, reverse=True)
    return combine * (o_f + o_b)


def gating(a, b, A, dt_bias, beta_scale: float = 1.0):
    """Gates from the raw per-token projections (the fused gating prologue), fp64.

    sparse-delta-memory 2.0.0 ``sparse_delta_memory/layer.py``, ``compute_gates``:
    ``A = -exp(A_log)`` per head, ``g = A * softplus(a + dt_bias)``, ``beta = sigmoid(b)``;
    Rondo-Exp ``tiny_gdn/fugue.py``, ``project``: beta doubled to allow negative eigenvalues
    (``beta_scale = 2``).  ``a``, ``b`` are ``[..., Hv]`` (any dtype, widened exactly);
    ``A``, ``dt_bias`` are ``[Hv]``.  softplus and sigmoid are evaluated in closed form
    (``log(1 + e^x)`` and ``1 / (1 + e^-x)``) through their overflow-free rearrangements;
    torch's softplus returns ``x`` itself above 20, within 2e-9 relative of this.
    Returns ``(g, beta)`` as fp64 arrays of ``a``'s shape.
    """
    a, b = _f64(a), _f64(b)
    A, dt_bias = _f64(A), _f64(dt_bias)
    x = a + dt_bias
    softplus = np.logaddexp(0.0, x)            # log(1 + e^x)
    g = A * softplus
    beta = beta_scale * np.exp(-np.logaddexp(0.0, -b))  # 1 / (1 + e^-b)
    return g, beta


def gated_rmsnorm(o, z, weight, eps: float):
    """Output epilogue of the decode chain, fp64: per head (last axis, dv values)
    ``o / sqrt(mean(o^2) + eps) * weight * silu(z)``, ``silu(x) = x sigmoid(x)``
    (flashrt-structures 0.2.0 ``impls/gated_delta_core/fused_layer.py``, ``_decode_one``:
    ``rms_norm_gated_silu(core_out, z, norm.weight, eps)``; the normalisation is read as
    coming before the gate and the weight as one [dv] vector shared by the heads).
    ``o``, ``z`` are ``[..., dv]``; returns fp64 of that shape."""
    o, z, weight = _f64(o), _f64(z), _f64(weight)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    silu = z * np.exp(-np.logaddexp(0.0, -z))
    return o / rms * weight * silu


def _l2n(x):
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-6)


def gdn2_forward(q, k, v, g, b, w, S0=None, cu_seqlens=None, read_mode: str = "post",
                 scale: float = 1.0, qk_l2norm: bool = True, reverse: bool = False):
    """GDN-2 recurrence with decoupled gates, per-token loop in fp64 (Rondo-Exp
    ``tiny_gdn/fugue.py``, ``BidirectionalGatedDeltaNet2`` docstring:
    ``S_t = (I - k_t (b_t * k_t)^T) Diag(exp g_t) S_{t-1} + k_t (w_t * v_t)^T`` with S of
    shape [dk, dv], the forward read ``q_t^T S_t``).

    q, k [B, T, Hk, dk]; v [B, T, Hv, dv]; g, b [B, T, Hv, dk] (per key channel: log decay
    and erase gate); w [B, T, Hv, dv] (per value channel write gate); S0 [n_seqs, Hv, dk,
    dv] or None.  Same conventions as ``forward`` (H = S^T layout, GQA by repeating key
    heads, varlen, the read modes, reversal within each sequence).  With g = log(alpha),
    b = w = beta on every channel this is the scalar gated delta rule.
    Returns (o [B, T, Hv, dv], S_final [n_seqs, Hv, dk, dv]) in fp64.
    """
    q, k, v, g, b, w = (_f64(x) for x in (q, k, v, g, b, w))
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    group = Hv // Hk
    if cu_seqlens is None:
        segs = [(n, 0, T) for n in range(B)]
    else:
        cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                        dtype=np.int64)
        segs = [(0, int(cu[s]), int(cu[s + 1])) for s in range(len(cu) - 1)]
    o = np.zeros((B, T, Hv, dv))
    S_out = np.zeros((len(segs), Hv, dk, dv))
    S0 = _f64(S0)
    for si, (row, t0, t1) in enumerate(segs):
        H = np.zeros((Hv, dk, dv)) if S0 is None else S0[si].copy()
        order = range(t1 - 1, t0 - 1, -1) if reverse else range(t0, t1)
        for t in order:
            qt = np.repeat(q[row, t], group, axis=0)          # [Hv, dk]
            kt = np.repeat(k[row, t], group, axis=0)
            if qk_l2norm:
                qt, kt = _l2n(qt), _l2n(kt)
            if read_mode == "pre":
                o[row, t] = scale * np.einsum("hd,hde->he", qt, H)
            D = np.exp(g[row, t])                             # [Hv, dk]
            DH = D[:, :, None] * H
            u = w[row, t] * v[row, t] - np.einsum("hd,hde->he", b[row, t] * kt, DH)
            H = DH + kt[:, :, None] * u[:, None, :]
            if read_mode == "post":
                o[row, t] = scale * np.einsum("hd,hde->he", qt, H)
        S_out[si] = H
    return o, S_out
