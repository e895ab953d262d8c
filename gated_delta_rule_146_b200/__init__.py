"""B200 gated delta-rule library: thin Python binding over the C ABI of libgdr.so.

Every computation runs in the library's CUDA kernels (include/gdr.h).  This
module only marshals torch CUDA tensors into pointers, allocates the outputs and
the workspace with torch, and passes the current CUDA stream.  There is no CPU
fallback: if the compiled library is missing, importing the entry points raises.

Entry points (names follow the C ABI):
  chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, ...) -> (o, S_final)
  decode_step(q, k, v, g, beta, S, ...) -> o           (S updated in place)
  chunk_fwd_workspace_size(...), chunk_fwd_path(...), chunk_bwd_path(...),
  read_device_error(...)
"""
from __future__ import annotations

import ctypes
import math
import os

from . import _abi
from ._abi import GdrError, ChunkArgs, DecodeArgs, F32, BF16, READ_POST, READ_PRE  # noqa: F401

__all__ = ["chunk_fwd", "chunk_fwd_bidir", "chunk_bwd", "decode_step",
           "chunk_fwd_workspace_size", "chunk_fwd_bidir_workspace_size",
           "chunk_bwd_workspace_size", "chunk_fwd_path", "chunk_bwd_path",
           "read_device_error", "chunk_fwd_noalloc", "noalloc_read_device_error", "library",
           "GdrError"]


def library():
    """The loaded libgdr.so (raises if it has not been built)."""
    return _abi.lib()


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _check_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("gdr kernels take CUDA tensors only (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError("gdr kernels take contiguous tensors")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _gating_fields(gate_A, gate_dt_bias, beta_scale):
    """(gate_raw, A pointer, dt_bias pointer, beta_scale) of the fused gating prologue:
    with gate_A ([Hv] fp32, = -exp(A_log)) and gate_dt_bias ([Hv] fp32) given, g and beta
    are the raw projections a, b and the kernels form g = A softplus(a + dt_bias),
    beta = beta_scale sigmoid(b)."""
    if (gate_A is None) != (gate_dt_bias is None):
        raise ValueError("gate_A and gate_dt_bias come together")
    if gate_A is None:
        return 0, None, None, float(beta_scale)
    import torch
    for t in (gate_A, gate_dt_bias):
        if t.dtype != torch.float32 or t.dim() != 1 or not t.is_contiguous():
            raise TypeError("gate_A and gate_dt_bias are contiguous float32 [Hv] tensors")
    return 1, gate_A.data_ptr(), gate_dt_bias.data_ptr(), float(beta_scale)


def _gdn2_fields(g, v, gdn2_w):
    """(gdn2, write-gate pointer): with gdn2_w ([.., Hv, dv], gate dtype) given, g and beta
    are the per-key-channel log decay and erase gate of GDN-2 ([.., Hv, dk])."""
    if gdn2_w is None:
        return 0, None
    if gdn2_w.dtype != g.dtype or tuple(gdn2_w.shape) != tuple(v.shape):
        raise TypeError("gdn2_w has the shape of v and the dtype of g")
    if g.dim() != v.dim():
        raise TypeError("with gdn2_w, g and beta carry a key-channel axis")
    return 1, gdn2_w.data_ptr()


def make_chunk_args(q, v, g, cu_seqlens=None, chunk=64, read_mode="post", scale=None,
                    qk_l2norm=True, reverse=False, o_accumulate=False, gate_A=None,
                    gate_dt_bias=None, beta_scale=1.0, gdn2_w=None, status=None):
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    return ChunkArgs(B, T, Hk, Hv, dk, dv, n_seqs, chunk, _dtype_code(q), _dtype_code(g),
                     READ_PRE if read_mode == "pre" else READ_POST, float(scale),
                     int(bool(qk_l2norm)), int(bool(reverse)), int(bool(o_accumulate)),
                     *_gating_fields(gate_A, gate_dt_bias, beta_scale), *_gdn2_fields(g, v, gdn2_w),
                     _status_field(status))


def _status_field(status):
    """Device address of the caller's optional status word (an int32 CUDA tensor that the
    caller zeroes; a failed device-side check stores its gdr_status there), or None."""
    if status is None:
        return None
    import torch
    if status.dtype != torch.int32 or not status.is_cuda or status.numel() < 1:
        raise TypeError("status must be an int32 CUDA tensor")
    return status.data_ptr()


def chunk_fwd_workspace_size(args: ChunkArgs) -> int:
    return int(_abi.lib().gdr_chunk_fwd_workspace_size(ctypes.byref(args)))


def chunk_fwd_path(args: ChunkArgs):
    r = _abi.lib().gdr_chunk_fwd_path(ctypes.byref(args))
    return None if r is None else r.decode()


def chunk_bwd_path(args: ChunkArgs):
    """gdr_chunk_bwd_path: "tc", "simt" or None (unsupported)."""
    r = _abi.lib().gdr_chunk_bwd_path(ctypes.byref(args))
    return None if r is None else r.decode()


def chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, *, chunk=64, read_mode="post",
              scale=None, qk_l2norm=True, reverse=False, o=None, o_accumulate=False,
              output_final_state=True, S_final=None, workspace=None, stream=None,
              gate_A=None, gate_dt_bias=None, beta_scale=1.0, gdn2_w=None, status=None):
    """Chunk-parallel forward (gdr_chunk_fwd).  Shapes: q, k [B,T,Hk,dk]; v [B,T,Hv,dv];
    g, beta [B,T,Hv]; S0 [n_seqs,Hv,dk,dv] fp32 or None; cu_seqlens int32 [n_seqs+1] or
    None.  With gate_A and gate_dt_bias ([Hv] fp32) given, g and beta are the raw
    projections a and b of the fused gating prologue.  With gdn2_w ([B,T,Hv,dv]) given, the
    gates are GDN-2's: g the per-key-channel log decay and beta the erase gate, both
    [B,T,Hv,dk], gdn2_w the write gate.  ``status``: an optional int32 CUDA tensor the
    caller zeroes, where a failed device-side check stores its gdr_status without any
    synchronisation.  Returns (o [B,T,Hv,dv], S_final [n_seqs,Hv,dk,dv] fp32 or None)."""
    import torch
    _check_cuda(q, k, v, g, beta, S0, cu_seqlens, o, S_final, workspace, gate_A, gate_dt_bias,
                gdn2_w, status)
    args = make_chunk_args(q, v, g, cu_seqlens, chunk, read_mode, scale, qk_l2norm, reverse,
                           o_accumulate, gate_A, gate_dt_bias, beta_scale, gdn2_w, status)
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != g.dtype:
        raise TypeError("q, k, v share one dtype and g, beta another")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if S0 is not None and S0.dtype != torch.float32:
        raise TypeError("S0 must be float32")
    if o is None:
        if o_accumulate:
            raise ValueError("o_accumulate needs an existing o")
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if S_final is None and output_final_state:
        S_final = torch.empty((args.n_seqs, args.Hv, args.dk, args.dv), dtype=torch.float32,
                              device=q.device)
    need = chunk_fwd_workspace_size(args)
    if need == 0:
        raise GdrError(_abi.GDR_ERR_UNSUPPORTED, "no kernel path for these arguments")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = _abi.lib().gdr_chunk_fwd(
        ctypes.byref(args), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
        _ptr(cu_seqlens), _ptr(o), _ptr(S_final), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream))
    _abi.check(st)
    return o, S_final


def chunk_fwd_bidir(q, k, v, g_fwd, beta_fwd, g_bwd, beta_bwd, cu_seqlens=None, *, chunk=64,
                    read_mode="pre", scale=None, qk_l2norm=True, o=None, workspace=None,
                    stream=None, gate_A=None, gate_dt_bias=None, beta_scale=1.0, gdn2_w=None,
                    status=None):
    """Bidirectional forward (gdr_chunk_fwd_bidir): o = forward scan with (g_fwd, beta_fwd)
    + reverse scan within each sequence with (g_bwd, beta_bwd), from zero states, in one
    call.  Shapes as for ``chunk_fwd``; ``status`` as there.  Returns o."""
    import torch
    _check_cuda(q, k, v, g_fwd, beta_fwd, g_bwd, beta_bwd, cu_seqlens, o, workspace, gate_A,
                gate_dt_bias, gdn2_w, status)
    args = make_chunk_args(q, v, g_fwd, cu_seqlens, chunk, read_mode, scale, qk_l2norm, False,
                           False, gate_A, gate_dt_bias, beta_scale, gdn2_w, status)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v share one dtype")
    if len({t.dtype for t in (g_fwd, beta_fwd, g_bwd, beta_bwd)}) != 1:
        raise TypeError("the gates of both directions share one dtype")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    need = int(_abi.lib().gdr_chunk_fwd_bidir_workspace_size(ctypes.byref(args)))
    if need == 0:
        raise GdrError(_abi.GDR_ERR_UNSUPPORTED, "no kernel path for these arguments")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = _abi.lib().gdr_chunk_fwd_bidir(
        ctypes.byref(args), _ptr(q), _ptr(k), _ptr(v), _ptr(g_fwd), _ptr(beta_fwd), _ptr(g_bwd),
        _ptr(beta_bwd), _ptr(cu_seqlens), _ptr(o), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream))
    _abi.check(st)
    return o


def chunk_fwd_bidir_workspace_size(args: ChunkArgs) -> int:
    return int(_abi.lib().gdr_chunk_fwd_bidir_workspace_size(ctypes.byref(args)))


def chunk_bwd_workspace_size(args: ChunkArgs) -> int:
    return int(_abi.lib().gdr_chunk_bwd_workspace_size(ctypes.byref(args)))


def chunk_bwd(q, k, v, g, beta, dO, S0=None, cu_seqlens=None, dS_final=None, *, chunk=64,
              read_mode="post", scale=None, qk_l2norm=True, reverse=False, dS0=True,
              workspace=None, stream=None, status=None):
    """Backward pass of ``chunk_fwd`` (gdr_chunk_bwd): the gradients of
    <dO, o> + <dS_final, S_final> for the same inputs.  dO has the shape of v (io dtype);
    dS_final [n_seqs,Hv,dk,dv] fp32 or None.  Returns (dq, dk, dv, dg, dbeta, dS0) with the
    shapes and dtypes of q, k, v, g, beta and S0 (dS0 fp32, None when ``dS0=False``)."""
    import torch
    _check_cuda(q, k, v, g, beta, dO, S0, cu_seqlens, dS_final, workspace, status)
    args = make_chunk_args(q, v, g, cu_seqlens, chunk, read_mode, scale, qk_l2norm, reverse,
                           status=status)
    if k.dtype != q.dtype or v.dtype != q.dtype or dO.dtype != q.dtype or beta.dtype != g.dtype:
        raise TypeError("q, k, v, dO share one dtype and g, beta another")
    if tuple(dO.shape) != tuple(v.shape):
        raise TypeError("dO has the shape of v")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    for t in (S0, dS_final):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("S0 and dS_final must be float32")
    need = chunk_bwd_workspace_size(args)
    if need == 0:
        raise GdrError(_abi.GDR_ERR_UNSUPPORTED, "no backward kernel for these arguments")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg, dbeta = torch.empty_like(g), torch.empty_like(beta)
    dS0_t = (torch.empty((args.n_seqs, args.Hv, args.dk, args.dv), dtype=torch.float32,
                         device=q.device) if dS0 else None)
    st = _abi.lib().gdr_chunk_bwd(
        ctypes.byref(args), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
        _ptr(cu_seqlens), _ptr(dO), _ptr(dS_final), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
        _ptr(dbeta), _ptr(dS0_t), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream))
    _abi.check(st)
    return dq, dk, dv, dg, dbeta, dS0_t


def read_device_error(args: ChunkArgs, workspace, stream=None) -> int:
    """Synchronising diagnostic: the device-side status recorded in `workspace`."""
    return int(_abi.lib().gdr_read_device_error(ctypes.byref(args), _ptr(workspace),
                                                _stream(stream)))


def chunk_fwd_noalloc(args: ChunkArgs, q, k, v, g, beta, S0, cu_seqlens, o, S_final,
                      stream=None) -> int:
    """gdr_chunk_fwd_noalloc: the forward with its scratch in the library's static device
    array (no workspace).  ``args`` from ``make_chunk_args``; o and S_final are
    caller-allocated outputs (S_final may be None).  Returns the gdr_status (not raised)."""
    _check_cuda(q, k, v, g, beta, S0, cu_seqlens, o, S_final)
    return int(_abi.lib().gdr_chunk_fwd_noalloc(
        ctypes.byref(args), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
        _ptr(cu_seqlens), _ptr(o), _ptr(S_final), _stream(stream)))


def noalloc_read_device_error(stream=None) -> int:
    """Synchronising diagnostic: the device-side status the last gdr_chunk_fwd_noalloc call
    left in the static scratch array of the current device."""
    return int(_abi.lib().gdr_noalloc_read_device_error(_stream(stream)))


def _norm_fields(q, norm_z, norm_weight, norm_eps):
    """(out_norm, z pointer, weight pointer, eps) of the fused gated RMSNorm epilogue."""
    if (norm_z is None) != (norm_weight is None):
        raise ValueError("norm_z and norm_weight come together")
    if norm_z is None:
        return 0, None, None, float(norm_eps)
    import torch
    if norm_z.dtype != q.dtype:
        raise TypeError("norm_z has the dtype of q, k, v and o")
    if norm_weight.dtype != torch.float32 or norm_weight.dim() != 1:
        raise TypeError("norm_weight is a float32 [dv] tensor")
    return 1, norm_z.data_ptr(), norm_weight.data_ptr(), float(norm_eps)


def make_decode_args(q, v, g, read_mode="post", scale=None, qk_l2norm=True, gate_A=None,
                     gate_dt_bias=None, beta_scale=1.0, norm_z=None, norm_weight=None,
                     norm_eps=1e-6, gdn2_w=None):
    N, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    return DecodeArgs(N, Hk, Hv, dk, dv, _dtype_code(q), _dtype_code(g),
                      READ_PRE if read_mode == "pre" else READ_POST, float(scale),
                      int(bool(qk_l2norm)), *_gating_fields(gate_A, gate_dt_bias, beta_scale),
                      *_norm_fields(q, norm_z, norm_weight, norm_eps), *_gdn2_fields(g, v, gdn2_w))


def decode_step(q, k, v, g, beta, S, *, read_mode="post", scale=None, qk_l2norm=True, o=None,
                stream=None, gate_A=None, gate_dt_bias=None, beta_scale=1.0, norm_z=None,
                norm_weight=None, norm_eps=1e-6, gdn2_w=None):
    """One recurrent token per sequence (gdr_decode_step): q, k [N,Hk,dk]; v [N,Hv,dv];
    g, beta [N,Hv]; S [N,Hv,dk,dv] fp32, updated in place.  With gate_A and gate_dt_bias
    ([Hv] fp32) given, g and beta are the raw projections of the fused gating prologue;
    with norm_z ([N,Hv,dv]) and norm_weight ([dv] fp32) given, o is the gated RMSNorm of
    the recurrent output; with gdn2_w ([N,Hv,dv]) given, g and beta are GDN-2's
    per-key-channel log decay and erase gate ([N,Hv,dk]).  Returns o [N,Hv,dv]."""
    import torch
    _check_cuda(q, k, v, g, beta, S, o, gate_A, gate_dt_bias, norm_z, norm_weight, gdn2_w)
    if S.dtype != torch.float32:
        raise TypeError("the state must be float32")
    args = make_decode_args(q, v, g, read_mode, scale, qk_l2norm, gate_A, gate_dt_bias,
                            beta_scale, norm_z, norm_weight, norm_eps, gdn2_w)
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    st = _abi.lib().gdr_decode_step(ctypes.byref(args), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                    _ptr(beta), _ptr(S), _ptr(o), _stream(stream))
    _abi.check(st)
    return o
