"""The C-ABI boundary on the host: the library loads, exports every call include/gdn.h declares,
and rejects bad arguments before anything is launched (no GPU needed).

Calls here pass null or fake device pointers only in combinations that the host-side checks must
reject; on a host with a GPU those fake-pointer cases are skipped, so nothing here can reach a
kernel with an invalid address.
"""
import ctypes
import os
import re

import pytest

from gated_deltanet_fwd_b200 import build as gbuild
from gated_deltanet_fwd_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gdn.load()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_five_calls():
    names = _declared_functions()
    for n in ["gdn_gates", "gdn_causal_conv1d_silu", "gdn_chunk_fwd", "gdn_recurrent_step",
              "gdn_gated_rmsnorm"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), f"libgdn.so does not export {name}"
    assert set(_declared_functions()) == set(gdn.SIGNATURES), \
        "binding signatures out of sync with include/gdn.h"


def test_library_is_built_for_sm100a(lib):
    """The build line targets sm_100a only (checked on the build recipe, not the binary)."""
    assert gbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "-lineinfo" in gbuild.FLAGS


def test_status_strings(lib):
    for code in range(6):
        s = gdn.status_string(code)
        assert s.startswith("GDN_")
    assert "unknown" in gdn.status_string(99)


def _no_gpu():
    import torch
    return not torch.cuda.is_available()


fake_ptr_only_without_gpu = pytest.mark.skipif(
    not _no_gpu(), reason="fake-pointer rejection cases run only on hosts without a GPU")

P = ctypes.c_void_p
A16 = P(0x7f0000000000)      # aligned fake address (never dereferenced: the call must reject)
MIS = P(0x7f0000000004)      # misaligned fake address
NUL = None
STREAM = None


@fake_ptr_only_without_gpu
def test_gates_rejections(lib):
    f = lib.gdn_gates
    assert f(A16, A16, 7, A16, A16, 4, 2, A16, A16, STREAM) == gdn.GDN_ERR_INVALID_ARG  # dtype
    assert f(A16, A16, 0, A16, A16, -1, 2, A16, A16, STREAM) == gdn.GDN_ERR_INVALID_ARG
    assert f(A16, A16, 0, A16, A16, 4, 0, A16, A16, STREAM) == gdn.GDN_ERR_INVALID_ARG
    assert f(NUL, A16, 0, A16, A16, 4, 2, A16, A16, STREAM) == gdn.GDN_ERR_INVALID_ARG
    assert f(NUL, NUL, 0, NUL, NUL, 0, 2, NUL, NUL, STREAM) == gdn.GDN_OK  # empty: no launch


@fake_ptr_only_without_gpu
def test_chunk_rejections(lib):
    f = lib.gdn_chunk_fwd

    def call(q=A16, k=A16, v=A16, g=A16, b=A16, dt=0, scale=0.1, s0=NUL, cu=NUL, N=1, B=1,
             T=64, Hk=16, Hv=32, dk=128, dv=128, chunk=64, out=A16, sT=A16, ws=A16, wsb=256):
        return f(q, k, v, g, b, dt, scale, s0, cu, N, B, T, Hk, Hv, dk, dv, chunk, out, sT, ws,
                 wsb, STREAM)

    E, U = gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED
    assert call(Hv=24, Hk=16) == E                     # Hv not a multiple of Hk
    assert call(dk=96 + 8) == U                        # dk not a multiple of 16
    assert call(dv=256) == U                           # dv > 128
    assert call(chunk=48) == U
    assert call(N=2, B=1) == E                         # without cu_seqlens N must equal B
    assert call(cu=A16, B=2, N=2) == E                 # with cu_seqlens B must be 1
    assert call(ws=NUL) == E
    assert call(wsb=8) == E                            # workspace too small
    assert call(ws=P(0x7f0000000010)) == E             # workspace not 256-byte aligned
    assert call(q=MIS) == E                            # misaligned activation
    assert call(out=NUL) == E
    assert call(g=NUL) == E
    assert call(s0=MIS) == E
    assert call(cu=P(0x7f0000000002)) == E             # cu_seqlens not 4-byte aligned
    assert call(s0=A16, sT=A16) == E                   # final_state overlaps initial_state
    assert call(scale=float("nan")) == E
    assert call(dt=5) == E
    assert call(N=0, B=0) == gdn.GDN_OK                # nothing to do: no launch


@fake_ptr_only_without_gpu
def test_chunk_strided_rejections(lib):
    f = lib.gdn_chunk_fwd_strided

    def call(qs=2048, ks=2048, vs=4096, Hk=16, Hv=32, dk=128, dv=128):
        return f(A16, qs, A16, ks, A16, vs, A16, A16, 0, 0.1, NUL, NUL, 1, 1, 64, Hk, Hv, dk, dv,
                 64, A16, A16, A16, 256, STREAM)

    E = gdn.GDN_ERR_INVALID_ARG
    assert call(qs=2040) == E       # smaller than one token's heads
    assert call(ks=2052) == E       # not a multiple of 8 elements
    assert call(vs=4092) == E
    assert call(vs=0) == E


@fake_ptr_only_without_gpu
def test_chunk_gated_norm_rejections(lib):
    f = lib.gdn_chunk_fwd_gated_norm
    full = 1024 + (1 + 1) * 32 * (16384 + 512)  # per-chunk operands of one 64-token sequence

    Y = P(0x7f0000100000)  # past z's 512 KB

    def call(q=A16, a=A16, b=A16, z=A16, w=A16, y=Y, eps=1e-6, dt=0, s0=NUL, sT=A16, cu=NUL,
             N=1, B=1, T=64, Hk=16, Hv=32, dk=128, dv=128, chunk=64, ws=A16, wsb=full,
             qs=2048):
        return f(q, qs, A16, 2048, A16, 4096, a, b, A16, A16, z, w, eps, dt, 0.1, s0, cu, N, B,
                 T, Hk, Hv, dk, dv, chunk, y, sT, ws, wsb, STREAM)

    E, U = gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED
    assert call(dt=1) == U               # fp32 activations: use the unfused calls
    assert call(dk=64) == U
    assert call(chunk=32) == U
    assert call(wsb=4096) == U           # no room for the per-chunk operands
    assert call(dt=7) == E
    assert call(Hv=24) == E
    assert call(eps=-1.0) == E
    assert call(eps=float("nan")) == E
    assert call(qs=2047) == E
    assert call(ws=NUL) == E
    assert call(a=NUL) == E
    assert call(b=NUL) == E
    assert call(z=MIS) == E
    assert call(w=MIS) == E
    assert call(y=NUL) == E
    assert call(z=A16, y=A16) == E       # y overlaps z
    assert call(s0=A16, sT=A16) == E
    assert call(N=2, B=1) == E
    assert call(N=0, B=0) == gdn.GDN_OK


@fake_ptr_only_without_gpu
def test_recurrent_rejections(lib):
    f = lib.gdn_recurrent_step

    def call(q=A16, k=A16, v=A16, g=A16, b=A16, dt=0, scale=0.1, st=A16, N=4, Hk=16, Hv=32,
             dk=128, dv=128, out=A16):
        return f(q, k, v, g, b, dt, scale, st, N, Hk, Hv, dk, dv, out, STREAM)

    E, U = gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED
    assert call(dk=64) == U
    assert call(dv=12) == U
    assert call(Hv=33) == E
    assert call(st=MIS) == E
    assert call(st=NUL) == E
    assert call(out=NUL) == E
    assert call(N=-1) == E
    assert call(N=0) == gdn.GDN_OK


@fake_ptr_only_without_gpu
def test_decode_layer_rejections(lib):
    f = lib.gdn_decode_layer_step
    A2 = ctypes.c_void_p(0x20000000)  # a second, distant fake conv-state buffer

    def call(mix=A16, a=A16, b=A16, z=A16, dt=0, w=A16, bias=NUL, K=4, csi=A16, cso=A2,
             al=A16, db=A16, nw=A16, l2=1e-6, ne=1e-6, scale=0.1, st=A16, N=4, Hk=16, Hv=32,
             dk=128, dv=128, y=A16):
        return f(mix, a, b, z, dt, w, bias, K, csi, cso, al, db, nw, l2, ne, scale, st, N, Hk,
                 Hv, dk, dv, y, STREAM)

    E, U = gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED
    assert call(dk=64) == U
    assert call(dv=64) == U
    assert call(K=9) == U
    assert call(K=0) == E
    assert call(Hv=33) == E
    assert call(dt=7) == E
    assert call(st=MIS) == E
    assert call(y=NUL) == E
    assert call(csi=NUL) == E
    assert call(cso=A16) == E       # the advanced history may not overlap the old one
    assert call(K=1, csi=NUL, cso=NUL, N=0) == gdn.GDN_OK
    assert call(l2=float("nan")) == E
    assert call(N=-1) == E
    assert call(N=0) == gdn.GDN_OK


@fake_ptr_only_without_gpu
def test_conv_rejections(lib):
    f = lib.gdn_causal_conv1d_silu

    def call(x=A16, dt=0, w=A16, bias=NUL, B=1, T=8, C=64, K=4, cu=NUL, N=1, nl2=0, grp=0,
             eps=1e-6, si=NUL, so=NUL, y=P(0x7f0000100000)):
        return f(x, dt, w, bias, B, T, C, K, cu, N, nl2, grp, eps, si, so, y, STREAM)

    E, U = gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED
    assert call(K=9) == U
    assert call(C=60) == U
    assert call(grp=48, nl2=48) == U
    assert call(grp=32, nl2=40) == E                   # n_l2norm_ch not a multiple of the group
    assert call(grp=0, nl2=32) == E
    assert call(y=A16) == E                            # y overlaps x
    assert call(x=MIS) == E
    assert call(w=NUL) == E
    assert call(N=2, B=1) == E
    assert call(si=A16, so=A16) == E                   # state in/out overlap
    assert call(eps=-1.0) == E


@fake_ptr_only_without_gpu
def test_rmsnorm_rejections(lib):
    f = lib.gdn_gated_rmsnorm
    E, U = gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED
    assert f(A16, A16, 0, A16, 1e-6, 10, 96, P(0x7f0000100000), STREAM) == U
    assert f(A16, A16, 0, A16, 1e-6, 10, 128, A16, STREAM) == E          # y overlaps z
    assert f(A16, MIS, 0, A16, 1e-6, 10, 128, P(0x7f0000100000), STREAM) == E
    assert f(A16, A16, 0, A16, -1.0, 10, 128, P(0x7f0000100000), STREAM) == E
    assert f(NUL, NUL, 0, NUL, 1e-6, 0, 128, NUL, STREAM) == gdn.GDN_OK


def test_binding_fails_loudly_without_library(tmp_path):
    """The binding never falls back: a missing library is an error, not a silent CPU path."""
    saved = gdn._lib
    gdn._lib = None
    try:
        with pytest.raises(RuntimeError, match="libgdn.so not found"):
            gdn.load(str(tmp_path / "libgdn.so"))
    finally:
        gdn._lib = saved
