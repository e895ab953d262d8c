"""The C-ABI library loads, exports what include/gdr.h declares, and validates its
arguments on the host (no GPU needed: every call here is refused before any launch)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_146_b200 import _abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "gdr.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdr_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(_abi.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
    assert b"sm_100a" in lib.gdr_version()


def test_status_strings(lib):
    for s in range(9):
        assert lib.gdr_status_string(s).startswith(b"GDR_")


def args(**kw):
    base = dict(B=2, T=100, Hk=2, Hv=4, dk=64, dv=64, n_seqs=2, chunk=64, io_dtype=_abi.BF16,
                gate_dtype=_abi.BF16, read_mode=_abi.READ_POST, scale=0.125, qk_l2norm=1,
                reverse=0, o_accumulate=0)
    base.update(kw)
    return _abi.ChunkArgs(**base)


def test_workspace_size(lib):
    a = args()
    n = lib.gdr_chunk_fwd_workspace_size(ctypes.byref(a))
    assert n > 0 and n % 256 == 0
    assert lib.gdr_chunk_fwd_workspace_size(ctypes.byref(args(Hv=3))) == 0
    assert lib.gdr_chunk_fwd_workspace_size(ctypes.byref(args(chunk=48))) == 0
    assert lib.gdr_chunk_fwd_path(ctypes.byref(args(dk=100))) in (b"simt", None)


FAKE = 0x10000  # a well-aligned address that is never dereferenced: every call below is
                # refused by host validation before anything is enqueued


def call(lib, a, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, cu=None, o=FAKE,
             S_final=FAKE, ws=FAKE)
    p.update(ptrs)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdr_chunk_fwd(ctypes.byref(a), vp(p["q"]), vp(p["k"]), vp(p["v"]), vp(p["g"]),
                             vp(p["beta"]), vp(p["S0"]), vp(p["cu"]), vp(p["o"]),
                             vp(p["S_final"]), vp(p["ws"]), ctypes.c_size_t(p.get("wsb", 0)),
                             None)


def test_host_validation(lib):
    a = args()
    need = lib.gdr_chunk_fwd_workspace_size(ctypes.byref(a))
    assert call(lib, args(Hv=3)) == _abi.GDR_ERR_INVALID_ARG
    assert call(lib, args(chunk=8)) == _abi.GDR_ERR_INVALID_ARG
    assert call(lib, args(io_dtype=7)) == _abi.GDR_ERR_INVALID_ARG
    assert call(lib, args(read_mode=2)) == _abi.GDR_ERR_INVALID_ARG
    assert call(lib, a, q=None, wsb=need) == _abi.GDR_ERR_INVALID_ARG
    assert call(lib, args(n_seqs=3), wsb=need) == _abi.GDR_ERR_INVALID_ARG  # n_seqs != B
    assert call(lib, a, cu=FAKE, wsb=need) == _abi.GDR_ERR_INVALID_ARG      # varlen needs B=1
    assert call(lib, a, k=FAKE + 4, wsb=need) == _abi.GDR_ERR_ALIGNMENT
    assert call(lib, a, ws=FAKE + 16, wsb=need) == _abi.GDR_ERR_ALIGNMENT   # workspace 256 B
    assert call(lib, a, ws=None, wsb=need) == _abi.GDR_ERR_WORKSPACE
    assert call(lib, a, wsb=need - 1) == _abi.GDR_ERR_WORKSPACE


def test_decode_host_validation(lib):
    d = _abi.DecodeArgs(N=4, Hk=2, Hv=4, dk=128, dv=128, io_dtype=_abi.BF16,
                        gate_dtype=_abi.BF16, read_mode=_abi.READ_POST, scale=0.1, qk_l2norm=1)
    vp = ctypes.c_void_p
    f = lambda a, **kw: lib.gdr_decode_step(ctypes.byref(a), *[vp(kw.get(n, FAKE)) for n in
                                                              ("q", "k", "v", "g", "b", "S", "o")],
                                            None)
    bad = _abi.DecodeArgs(**{**{n: getattr(d, n) for n, _ in d._fields_}, "Hv": 5})
    assert f(bad) == _abi.GDR_ERR_INVALID_ARG
    unsup = _abi.DecodeArgs(**{**{n: getattr(d, n) for n, _ in d._fields_}, "dk": 96})
    assert f(unsup) == _abi.GDR_ERR_UNSUPPORTED
    assert f(d, S=FAKE + 8) == _abi.GDR_ERR_ALIGNMENT
    empty = _abi.DecodeArgs(**{**{n: getattr(d, n) for n, _ in d._fields_}, "N": 0})
    assert f(empty) == _abi.GDR_OK  # nothing to do, nothing launched


def test_gating_host_validation(lib):
    """The fused gating fields: flags, scale and per-head arrays are checked on the host."""
    ok = args(gate_raw=1, gate_A=FAKE, gate_dt_bias=FAKE, beta_scale=2.0)
    need = lib.gdr_chunk_fwd_workspace_size(ctypes.byref(ok))
    assert need > 0
    assert lib.gdr_chunk_fwd_workspace_size(ctypes.byref(args(gate_raw=2))) == 0
    assert lib.gdr_chunk_fwd_workspace_size(
        ctypes.byref(args(gate_raw=1, beta_scale=float("inf")))) == 0
    assert call(lib, args(gate_raw=1, gate_dt_bias=FAKE, beta_scale=1.0),
                wsb=need) == _abi.GDR_ERR_INVALID_ARG                       # no gate_A
    assert call(lib, args(gate_raw=1, gate_A=FAKE + 2, gate_dt_bias=FAKE, beta_scale=1.0),
                wsb=need) == _abi.GDR_ERR_ALIGNMENT
    assert call(lib, ok, wsb=need - 1) == _abi.GDR_ERR_WORKSPACE            # gating accepted
    d = _abi.DecodeArgs(N=4, Hk=2, Hv=4, dk=128, dv=128, io_dtype=_abi.BF16,
                        gate_dtype=_abi.BF16, read_mode=_abi.READ_POST, scale=0.1, qk_l2norm=1,
                        gate_raw=1, gate_A=None, gate_dt_bias=FAKE, beta_scale=1.0)
    vp = ctypes.c_void_p
    assert lib.gdr_decode_step(ctypes.byref(d), *[vp(FAKE)] * 7, None) == _abi.GDR_ERR_INVALID_ARG


def test_struct_layout_matches_header(tmp_path):
    """ctypes mirrors of the argument structs have the C header's size and field offsets."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no host C compiler")
    fields = {"gdr_chunk_args": _abi.ChunkArgs, "gdr_decode_args": _abi.DecodeArgs}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "gdr.h"', "int main(void) {"]
    for cname, py in fields.items():
        lines.append(f'printf("%zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'printf("%zu\\n", offsetof({cname}, {fname}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    want = []
    for py in fields.values():
        want.append(ctypes.sizeof(py))
        want.extend(getattr(py, n).offset for n, _ in py._fields_)
    assert got == want


def test_decode_norm_host_validation(lib):
    """The fused output epilogue's flag, eps and arrays are checked on the host."""
    base = dict(N=4, Hk=2, Hv=4, dk=128, dv=128, io_dtype=_abi.BF16, gate_dtype=_abi.BF16,
                read_mode=_abi.READ_POST, scale=0.1, qk_l2norm=1)
    vp = ctypes.c_void_p
    f = lambda **kw: lib.gdr_decode_step(ctypes.byref(_abi.DecodeArgs(**{**base, **kw})),
                                         *[vp(FAKE)] * 7, None)
    assert f(out_norm=2) == _abi.GDR_ERR_INVALID_ARG
    assert f(out_norm=1, norm_z=FAKE, norm_weight=FAKE, norm_eps=-1.0) == _abi.GDR_ERR_INVALID_ARG
    assert f(out_norm=1, norm_weight=FAKE, norm_eps=1e-6) == _abi.GDR_ERR_INVALID_ARG
    assert f(out_norm=1, norm_z=FAKE + 8, norm_weight=FAKE, norm_eps=1e-6) == _abi.GDR_ERR_ALIGNMENT
    assert f(out_norm=1, norm_z=FAKE, norm_weight=FAKE + 2, norm_eps=1e-6) == _abi.GDR_ERR_ALIGNMENT


def test_gdn2_host_validation(lib):
    """GDN-2's flag and write-gate pointer are checked on the host; the decoupled gates take
    the CUDA-core chunk path and a workspace with per-key-channel cumulative decays."""
    scalar = args()
    g2 = args(gdn2=1, gdn2_w=FAKE)
    need = lib.gdr_chunk_fwd_workspace_size(ctypes.byref(g2))
    assert need > lib.gdr_chunk_fwd_workspace_size(ctypes.byref(scalar))
    assert lib.gdr_chunk_fwd_path(ctypes.byref(g2)) == b"simt"
    assert lib.gdr_chunk_fwd_workspace_size(ctypes.byref(args(gdn2=2))) == 0
    # GDN-2's local kernel tiles 64 rows: no path for chunks of 128
    assert lib.gdr_chunk_fwd_workspace_size(ctypes.byref(args(gdn2=1, gdn2_w=FAKE, chunk=128))) == 0
    assert lib.gdr_chunk_fwd_path(ctypes.byref(args(gdn2=1, gdn2_w=FAKE, chunk=128))) is None
    assert lib.gdr_chunk_fwd_path(ctypes.byref(args(chunk=128))) == b"simt"  # scalar gates do
    assert lib.gdr_chunk_fwd_workspace_size(
        ctypes.byref(args(gdn2=1, gate_raw=1, gate_A=FAKE, gate_dt_bias=FAKE))) == 0
    assert call(lib, args(gdn2=1), wsb=need) == _abi.GDR_ERR_INVALID_ARG     # no write gate
    assert call(lib, args(gdn2=1, gdn2_w=FAKE + 4), wsb=need) == _abi.GDR_ERR_ALIGNMENT
    assert call(lib, g2, wsb=need - 1) == _abi.GDR_ERR_WORKSPACE             # GDN-2 accepted
    base = dict(N=4, Hk=2, Hv=4, dk=128, dv=128, io_dtype=_abi.BF16, gate_dtype=_abi.BF16,
                read_mode=_abi.READ_POST, scale=0.1, qk_l2norm=1)
    vp = ctypes.c_void_p
    f = lambda **kw: lib.gdr_decode_step(ctypes.byref(_abi.DecodeArgs(**{**base, **kw})),
                                         *[vp(FAKE)] * 7, None)
    assert f(gdn2=3, gdn2_w=FAKE) == _abi.GDR_ERR_INVALID_ARG
    assert f(gdn2=1) == _abi.GDR_ERR_INVALID_ARG
    assert f(gdn2=1, gdn2_w=FAKE + 8) == _abi.GDR_ERR_ALIGNMENT
    assert f(gdn2=1, gdn2_w=FAKE, gate_raw=1, gate_A=FAKE, gate_dt_bias=FAKE) \
        == _abi.GDR_ERR_INVALID_ARG


def test_backward_host_validation(lib):
    """gdr_chunk_bwd: sizes, options and pointers are checked on the host."""
    a = args(dk=128, dv=128)
    need = lib.gdr_chunk_bwd_workspace_size(ctypes.byref(a))
    assert need > lib.gdr_chunk_fwd_workspace_size(ctypes.byref(a))
    assert lib.gdr_chunk_bwd_workspace_size(ctypes.byref(args(chunk=128))) == 0
    assert lib.gdr_chunk_bwd_workspace_size(ctypes.byref(args(dv=48))) == 0
    assert lib.gdr_chunk_bwd_workspace_size(ctypes.byref(args(gdn2=1, gdn2_w=FAKE))) == 0
    assert lib.gdr_chunk_bwd_workspace_size(
        ctypes.byref(args(gate_raw=1, gate_A=FAKE, gate_dt_bias=FAKE))) == 0
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def bwd(a, wsb=need, **kw):
        p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, cu=None, dO=FAKE,
                 dS=None, dq=FAKE, dk=FAKE, dv=FAKE, dg=FAKE, db=FAKE, dS0=FAKE, ws=FAKE)
        p.update(kw)
        return lib.gdr_chunk_bwd(ctypes.byref(a), *[vp(p[n]) for n in (
            "q", "k", "v", "g", "beta", "S0", "cu", "dO", "dS", "dq", "dk", "dv", "dg", "db",
            "dS0", "ws")], ctypes.c_size_t(wsb), None)

    assert bwd(args(dk=128, dv=128, Hv=3)) == _abi.GDR_ERR_INVALID_ARG
    assert bwd(a, dO=None) == _abi.GDR_ERR_INVALID_ARG
    assert bwd(a, dg=FAKE + 4) == _abi.GDR_ERR_ALIGNMENT
    assert bwd(a, ws=FAKE + 16) == _abi.GDR_ERR_ALIGNMENT
    assert bwd(args(dk=128, dv=128, o_accumulate=1)) == _abi.GDR_ERR_UNSUPPORTED
    assert bwd(args(dk=128, dv=128, chunk=128)) == _abi.GDR_ERR_UNSUPPORTED
    assert bwd(a, ws=None) == _abi.GDR_ERR_WORKSPACE
    assert bwd(a, wsb=need - 1) == _abi.GDR_ERR_WORKSPACE


def test_bidirectional_host_validation(lib):
    """gdr_chunk_fwd_bidir: the reverse and accumulate flags are its own; pointers checked."""
    a = args(dk=128, dv=128)
    need = lib.gdr_chunk_fwd_bidir_workspace_size(ctypes.byref(a))
    assert need > lib.gdr_chunk_fwd_workspace_size(ctypes.byref(a))  # scratch output (tc)
    assert lib.gdr_chunk_fwd_bidir_workspace_size(ctypes.byref(args(reverse=1))) == 0
    assert lib.gdr_chunk_fwd_bidir_workspace_size(ctypes.byref(args(o_accumulate=1))) == 0
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def bidir(a, wsb=need, **kw):
        p = dict(q=FAKE, k=FAKE, v=FAKE, gf=FAKE, bf=FAKE, gb=FAKE, bb=FAKE, cu=None, o=FAKE,
                 ws=FAKE)
        p.update(kw)
        return lib.gdr_chunk_fwd_bidir(ctypes.byref(a), *[vp(p[n]) for n in (
            "q", "k", "v", "gf", "bf", "gb", "bb", "cu", "o", "ws")], ctypes.c_size_t(wsb), None)

    assert bidir(args(dk=128, dv=128, reverse=1)) == _abi.GDR_ERR_INVALID_ARG
    assert bidir(a, gb=None) == _abi.GDR_ERR_INVALID_ARG
    assert bidir(a, bb=FAKE + 2) == _abi.GDR_ERR_ALIGNMENT
    assert bidir(a, wsb=need - 1) == _abi.GDR_ERR_WORKSPACE
    assert bidir(a, ws=None) == _abi.GDR_ERR_WORKSPACE


def test_binding_refuses_host_tensors(lib):
    """Every entry point of the binding refuses CPU tensors before reaching the library:
    there is no CPU path to fall back on."""
    import torch
    import gated_delta_rule_146_b200 as gdr
    q = torch.zeros((1, 8, 1, 64), dtype=torch.bfloat16)
    v = torch.zeros((1, 8, 1, 64), dtype=torch.bfloat16)
    g = torch.zeros((1, 8, 1), dtype=torch.bfloat16)
    calls = [
        lambda: gdr.chunk_fwd(q, q, v, g, g),
        lambda: gdr.chunk_fwd_bidir(q, q, v, g, g, g, g),
        lambda: gdr.chunk_bwd(q, q, v, g, g, v),
        lambda: gdr.decode_step(q[:, 0], q[:, 0], v[:, 0], g[:, 0], g[:, 0],
                                torch.zeros((1, 1, 64, 64))),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensors only"):
            call()


def test_binding_argument_counts_match_header(lib):
    """Each prototype in include/gdr.h has as many parameters as the binding declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = re.findall(r"\b(gdr_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S)
    assert protos
    for name, params in protos:
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None and len(argtypes) == n, (name, n, argtypes)


def test_noalloc_and_status_word_host_validation(lib):
    """gdr_chunk_fwd_noalloc names invalid arguments and valid ones without a kernel path
    (GDN-2 with chunks of 128) as such, before touching the device; a misaligned status
    word is refused by every entry point that takes the argument struct."""
    vp = ctypes.c_void_p
    na = lambda a: lib.gdr_chunk_fwd_noalloc(ctypes.byref(a), *[vp(FAKE)] * 9, None)
    assert na(args(Hv=3)) == _abi.GDR_ERR_INVALID_ARG
    g2 = args(dk=128, dv=128, chunk=128, gdn2=1, gdn2_w=FAKE)
    assert lib.gdr_chunk_fwd_path(ctypes.byref(g2)) is None
    assert na(g2) == _abi.GDR_ERR_UNSUPPORTED
    a = args(status=FAKE + 2)
    need = lib.gdr_chunk_fwd_workspace_size(ctypes.byref(a))
    assert call(lib, a, wsb=need) == _abi.GDR_ERR_ALIGNMENT
    assert lib.gdr_chunk_fwd_bidir(ctypes.byref(a), *[vp(FAKE)] * 7, None, vp(FAKE), vp(FAKE),
                                   ctypes.c_size_t(1 << 30), None) == _abi.GDR_ERR_ALIGNMENT


def test_backward_path(lib):
    """gdr_chunk_bwd_path: the tensor-core kernels for bf16, d = 128, chunk 64; the CUDA-core
    ones for fp32 inputs and for other sizes; none where the backward is not built."""
    path = lambda **kw: lib.gdr_chunk_bwd_path(ctypes.byref(args(**kw)))
    assert path(dk=128, dv=128) == b"tc"
    assert path(dk=128, dv=128, io_dtype=_abi.F32, gate_dtype=_abi.F32) == b"simt"
    assert path(dk=64, dv=64) == b"simt"
    assert path(dk=128, dv=128, chunk=32) == b"simt"
    assert path(dk=128, dv=128, gate_raw=1) is None
    assert path(dk=128, dv=128, o_accumulate=1) is None
