"""The C ABI loads, exports every entry point include/poetx.h declares, and rejects bad
arguments on the host before touching a GPU.  CPU only: no call here launches a kernel."""
import ctypes
import glob
import os
import re

import pytest

from orthogonal_equivalence_build_b200 import poetx

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include")


def declared_symbols():
    syms = set()
    for h in glob.glob(os.path.join(INCLUDE, "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        syms |= set(re.findall(r"\b(poetx_[a-z_0-9]+)\s*\(", text))
    return sorted(syms)


def test_header_symbols_are_exported():
    syms = declared_symbols()
    assert len(syms) >= 17
    for s in syms:
        assert hasattr(poetx.lib, s), s
    assert set(syms) == set(poetx.EXPORTED)


def test_abi_version_and_strings():
    assert poetx.abi_version() == 2
    assert poetx.lib.poetx_status_string(0) == b"ok"
    assert poetx.lib.poetx_status_string(8) == b"workspace too small"


def _layer(**kw):
    base = dict(m=512, n=1024, b=64, dtype=poetx.BF16, flags=0, w0m=0x10000, perm_r=0x20000,
                perm_p=0x30000, q_r=0x40000, q_p=0x50000, g_r=0x60000, g_p=0x70000,
                g_r_lp=0x80000, g_p_lp=0x90000)
    base.update(kw)
    return poetx.Layer(**base)


def _fwd(L, x=0x100000, T=128, y=0x200000, ws=None, wsb=0):
    return poetx.lib.poetx_linear_fwd(ctypes.byref(L), x, T, y, None, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(b=48), 2),                           # b does not divide m
    (dict(b=1), 2),                             # b < 2
    (dict(m=0), 2),
    (dict(dtype=7), 4),
    (dict(flags=1), 1),
    (dict(w0m=None), 1),
    (dict(g_r_lp=None), 1),                     # bf16 layer needs the bf16 copies
    (dict(perm_r=0x20004), 3),                  # misaligned
    (dict(b=2048, m=4096, n=4096), 2),          # b too large
    (dict(flags=2), 1),                         # staged without the int8 flag
    (dict(flags=8), 1),                         # unknown flag
    (dict(flags=6), 1),                         # staged without the int8 flag, fused
    (dict(flags=1, w0m_scale=0xA0000, dtype=poetx.F32), 4),   # int8 W0' needs a bf16 layer
    (dict(flags=1, w0m_scale=0xA0004), 3),      # misaligned scales
    (dict(flags=1, w0m_scale=0xA0000, m=520, n=1040, b=8), 2),  # int8 W0' rows of 16 bytes
])
def test_layer_validation(kw, status):
    assert _fwd(_layer(**kw)) == status


def test_forward_argument_checks():
    L = _layer()
    assert _fwd(L, x=None) == 1
    assert _fwd(L, T=-1) == 2
    assert _fwd(L, T=0) == 0                    # nothing to do, no launch
    assert _fwd(L, y=0x200008) == 3
    need = poetx.lib.poetx_fwd_workspace_bytes(ctypes.byref(L), 128)
    assert need > 0
    assert _fwd(L, ws=0x400000, wsb=need - 1) == 8
    assert _fwd(L, ws=None, wsb=need) == 8
    # POETX_LAYER_FUSED_W0_P alone or with the 8-bit bits is a valid layer (the call then
    # stops at the missing workspace)
    for flags, scale in ((4, None), (5, 0xA0000), (7, 0xA0000)):
        Lf = _layer(flags=flags, w0m_scale=scale)
        assert _fwd(Lf, ws=None, wsb=need) == 8


def test_backward_argument_checks():
    L = _layer()
    bwd = poetx.lib.poetx_linear_bwd
    assert bwd(ctypes.byref(L), 0x100000, None, 0x300000, 128, None, None, None, None, 0, None) == 1
    assert bwd(ctypes.byref(L), None, 0x200000, None, 128, None, None, None, None, 0, None) == 1
    L2 = _layer(q_r=None)
    assert bwd(ctypes.byref(L2), 0x100000, 0x200000, 0x300000, 128, None, 0x500000, None,
               None, 0, None) == 1
    need = poetx.lib.poetx_bwd_workspace_bytes(ctypes.byref(L), 128)
    assert bwd(ctypes.byref(L), 0x100000, 0x200000, 0x300000, 128, None, None, None,
               0x400000, need - 1, None) == 8


def test_cnp_argument_checks():
    f = poetx.lib.poetx_cnp_build
    assert f(None, 2, 64, 0x1000, None, 1, None, 0, None) == 1
    assert f(0x1000, 2, 64, None, None, 1, None, 0, None) == 1
    assert f(0x1000, 2, 2048, 0x2000, None, 1, None, 0, None) == 2
    assert f(0x1000, 2, 64, 0x2000, 0x3000, 0, None, 0, None) == 4
    assert f(0x1000, 2, 64, 0x2004, None, 1, 0x8000, 1 << 30, None) == 3
    assert f(0x1000, 2, 64, 0x2000, None, 1, None, 0, None) == 8
    assert f(0x1000, 0, 64, 0x2000, None, 1, None, 0, None) == 0


def test_merge_argument_checks():
    f = poetx.lib.poetx_merge_permutations
    assert f(0x1000, 0x2000, 0x3000, 64, 64, 5, 0x9000, None) == 4
    assert f(None, 0x2000, 0x3000, 64, 64, 1, 0x9000, None) == 1
    # output overlapping the input
    assert f(0x10000, 0x2000, 0x3000, 64, 64, 1, 0x10000 + 64, None) == 1
    L = _layer(q_p=None)
    need = poetx.lib.poetx_merge_reinit_workspace_bytes(ctypes.byref(_layer()))
    assert need >= 2 * 512 * 1024 * 2
    assert poetx.lib.poetx_merge_reinit(ctypes.byref(L), 1, 0x100000, need, None) == 1
    assert poetx.lib.poetx_merge_reinit(ctypes.byref(_layer()), 1, 0x100000, need - 1, None) == 8


def test_workspace_queries_scale_with_tokens():
    L = _layer()
    f = poetx.lib.poetx_fwd_workspace_bytes
    assert f(ctypes.byref(L), 256) > f(ctypes.byref(L), 128) > 0
    assert poetx.lib.poetx_fwd_workspace_bytes(None, 128) == 0


def test_workspaces_never_hold_an_m_by_n_buffer():
    """R W0 P is never formed: the token-independent part of the forward/backward workspace
    grows linearly with m + n (b x b blocks), not with m * n."""
    def ws(fn, m, n, T):
        L = _layer(m=m, n=n, b=512)
        return fn(ctypes.byref(L), T)
    for fn in (poetx.lib.poetx_fwd_workspace_bytes, poetx.lib.poetx_bwd_workspace_bytes):
        base = ws(fn, 4096, 14336, 16)
        double = ws(fn, 8192, 28672, 16)
        assert double < 2.2 * base, (fn.__name__, base, double)
        assert ws(fn, 4096, 14336, 1) < 4096 * 14336 * 2 * 3   # below three copies of W0'
    # activations scale with T only
    f = poetx.lib.poetx_fwd_workspace_bytes
    L = _layer(m=4096, n=14336, b=512)
    assert f(ctypes.byref(L), 2048) - f(ctypes.byref(L), 1024) == \
        f(ctypes.byref(L), 4096) - f(ctypes.byref(L), 3072)


def test_int8_w0_workspace_only_where_the_product_is_not_fused():
    """8-bit W0' layers dequantise inside the tensor-core kernel when T >= 256 and m, n are
    multiples of 256; other shapes need one bf16 copy of W0' in the workspace."""
    L16 = _layer(m=4096, n=14336, b=512)
    L8 = _layer(m=4096, n=14336, b=512, flags=1, w0m_scale=0xA0000)
    for fn in (poetx.lib.poetx_fwd_workspace_bytes, poetx.lib.poetx_bwd_workspace_bytes):
        assert fn(ctypes.byref(L8), 4096) == fn(ctypes.byref(L16), 4096)
        extra = fn(ctypes.byref(L8), 128) - fn(ctypes.byref(L16), 128)
        assert 4096 * 14336 * 2 <= extra < 4096 * 14336 * 2 + 4096
    assert poetx.lib.poetx_merge_reinit_workspace_bytes(ctypes.byref(L8)) == \
        poetx.lib.poetx_merge_reinit_workspace_bytes(ctypes.byref(L16))
    # staged dequantisation always takes the bf16 copy of W0'
    L8s = _layer(m=4096, n=14336, b=512, flags=3, w0m_scale=0xA0000)
    for fn in (poetx.lib.poetx_fwd_workspace_bytes, poetx.lib.poetx_bwd_workspace_bytes):
        extra = fn(ctypes.byref(L8s), 4096) - fn(ctypes.byref(L16), 4096)
        assert 4096 * 14336 * 2 <= extra < 4096 * 14336 * 2 + 4096


def test_quantize_argument_checks():
    q = poetx.lib.poetx_quantize_w0
    assert q(0x1000, 64, 64, 5, 0x2000, 0x3000, None) == 4
    assert q(None, 64, 64, 1, 0x2000, 0x3000, None) == 1
    assert q(0x1000, -1, 64, 1, 0x2000, 0x3000, None) == 2
    assert q(0x1000, 64, 64, 1, 0x2000, 0x3004, None) == 3
    assert q(0x1000, 0, 64, 1, 0x2000, 0x3000, None) == 0
    d = poetx.lib.poetx_dequantize_w0
    assert d(None, 0x3000, 64, 64, 0x4000, None) == 1
    assert d(0x2000, 0x3000, 64, 64, 0x4008, None) == 3
    assert d(0x2000, 0x3000, 64, 0, 0x4000, None) == 0


def test_trace_select_is_host_only_and_accepts_lists():
    assert poetx.lib.poetx_trace_select(b"umma_dense_W0,umma_dense_W0T") == 0
    assert poetx.lib.poetx_trace_select(b",,x,") == 0
    assert poetx.lib.poetx_trace_select(None) == 0
    assert poetx.lib.poetx_trace_select(b"") == 0


def test_saved_a_entry_points_argument_checks():
    """poetx_linear_fwd_ex / poetx_linear_bwd_ex: x may be NULL in the backward only when
    saved_a is given; a misaligned saved_a is rejected before any launch."""
    L = _layer()
    f = poetx.lib.poetx_linear_fwd_ex
    assert f(ctypes.byref(L), 0x100000, 128, 0x200000, None, 0x300008, None, 0, None) == 3
    assert f(ctypes.byref(L), 0x100000, 0, 0x200000, None, 0x300000, None, 0, None) == 0
    bx = poetx.lib.poetx_linear_bwd_ex
    need = poetx.lib.poetx_bwd_workspace_bytes(ctypes.byref(L), 128)
    # neither x nor saved_a
    assert bx(ctypes.byref(L), None, 0x200000, 0x300000, None, 128, None, None, None,
              0x400000, need, None) == 1
    assert bx(ctypes.byref(L), None, 0x200000, 0x300000, 0x500008, 128, None, None, None,
              0x400000, need, None) == 3
    # x NULL with saved_a: passes the argument checks (then fails on the workspace size)
    assert bx(ctypes.byref(L), None, 0x200000, 0x300000, 0x500000, 128, None, None, None,
              0x400000, need - 1, None) == 8


def test_layers_cnp_build_argument_checks():
    """poetx_layers_cnp_build: nlayers = 0 is a no-op; a NULL array, a layer of another b or
    dtype, or a layer without q are rejected before any launch."""
    f = poetx.lib.poetx_layers_cnp_build
    arr = (ctypes.POINTER(poetx.Layer) * 2)()
    L0, L1 = _layer(), _layer(b=128)
    arr[0], arr[1] = ctypes.pointer(L0), ctypes.pointer(L1)
    assert f(arr, 0, None, 0, None) == 0
    assert f(None, 2, None, 0, None) == 1
    assert f(arr, -1, None, 0, None) == 1
    assert f(arr, 2, 0x400000, 1 << 30, None) == 2              # b differs
    L2 = _layer(dtype=poetx.F32, g_r_lp=None, g_p_lp=None)
    arr[1] = ctypes.pointer(L2)
    assert f(arr, 2, 0x400000, 1 << 30, None) == 4              # dtype differs
    L3 = _layer(q_p=None)
    arr[1] = ctypes.pointer(L3)
    assert f(arr, 2, 0x400000, 1 << 30, None) == 1              # no q
    arr[1] = ctypes.pointer(_layer(m=1024))
    need = poetx.lib.poetx_layers_cnp_workspace_bytes(arr, 2)
    assert need > poetx.lib.poetx_layer_cnp_workspace_bytes(ctypes.byref(L0))
    assert f(arr, 2, 0x400000, need - 1, None) == 8


def test_dg_backward_and_layers_dq_argument_checks():
    L = _layer()
    need = poetx.lib.poetx_bwd_workspace_bytes(ctypes.byref(L), 128)
    f = poetx.lib.poetx_linear_bwd_dg
    assert f(ctypes.byref(L), 0x100000, 0x200000, 0x300000, None, 128, None, None,
             0x400000, need, None) == 1                       # dG NULL
    assert f(ctypes.byref(L), 0x100000, 0x200000, 0x300000, None, 128, None, 0x500004,
             0x400000, need, None) == 3                       # dG misaligned
    g = poetx.lib.poetx_layers_dq_from_dg
    arr = (ctypes.POINTER(poetx.Layer) * 1)(ctypes.pointer(L))
    V1 = ctypes.c_void_p * 1
    assert g(arr, V1(0x500000), V1(0x600000), V1(0x700000), 0, None, 0, None) == 0
    assert g(arr, None, V1(0x600000), V1(0x700000), 1, None, 0, None) == 1
    assert g(arr, V1(None), V1(0x600000), V1(0x700000), 1, None, 0, None) == 1
    assert g(arr, V1(0x500008), V1(0x600000), V1(0x700000), 1, None, 0, None) == 3
    need = poetx.lib.poetx_layers_dq_workspace_bytes(arr, 1)
    assert need > 0
    assert g(arr, V1(0x500000), V1(0x600000), V1(None), 1, 0x800000, need - 1, None) == 8
