"""Host-side checks of the C ABI: the library loads, exports every symbol
that include/hyena.h declares, and rejects bad arguments on the host before
anything is enqueued.

Every call below that passes placeholder device addresses is built to fail
validation (a null, misaligned, aliased, oversized or unsupported argument),
so none of them can reach a kernel launch on any machine.
"""
import ctypes
import os
import re

import pytest

from subquadratic_sequence_b200 import build as hbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    from subquadratic_sequence_b200 import hyena
    return hyena.LIB


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"HYENA_API[^;(]*?\b(hyena_\w+)\s*\(", text))
    return names


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ("hyena_filter_gen", "hyena_filter_rfft", "hyena_fftconv_gate_forward",
                     "hyena_fftconv_workspace_size", "hyena_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(5):
        assert lib.hyena_status_string(s)
    assert b"unknown" in lib.hyena_status_string(99)


def test_workspace_size(lib):
    from subquadratic_sequence_b200 import hyena
    B, D, L, N = 8, 768, 2048, 2
    assert hyena.hyena_fftconv_workspace_size(B, D, L, N, BF16, True) == 0
    need = hyena.hyena_fftconv_workspace_size(B, D, L, N, BF16, False)
    assert need >= N * D * L * 8 and need % 256 == 0
    bad = ctypes.c_size_t(-1).value
    assert lib.hyena_fftconv_workspace_size(B, D, 1000, N, F32, 1) == bad
    assert lib.hyena_fftconv_workspace_size(B, D, L, 0, F32, 1) == bad
    assert lib.hyena_fftconv_workspace_size(B, D, L, N, 7, 1) == bad


# placeholder device addresses (never dereferenced: every call fails validation)
A = 0x7F0000000000          # 256-byte aligned
BIG = 1 << 30


def P(k):
    return ctypes.c_void_p(A + k * BIG)


def fwd(lib, v=P(0), xs=(P(1), P(2)), h=None, H=P(3), bias=P(4), B=2, D=3, L=64, N=None,
        io=F32, y=P(5), ws=None, wsb=0):
    N = len(xs) if N is None else N
    arr = (ctypes.c_void_p * max(len(xs), 1))(*[x.value if x is not None else None for x in xs])
    xp = None if xs is None else arr
    return lib.hyena_fftconv_gate_forward(v, xp, h, H, bias, B, D, L, N, io, y, ws, wsb, None)


def test_forward_rejects_bad_arguments(lib):
    assert fwd(lib, v=None) == INVALID
    assert fwd(lib, y=None) == INVALID
    assert fwd(lib, bias=None) == INVALID
    assert fwd(lib, H=None, h=None) == INVALID
    assert fwd(lib, xs=(P(1), None)) == INVALID
    assert fwd(lib, B=0) == INVALID
    assert fwd(lib, D=-1) == INVALID
    assert fwd(lib, L=0) == INVALID
    assert fwd(lib, N=0) == INVALID
    assert fwd(lib, io=5) == INVALID
    # valid but not implemented
    assert fwd(lib, L=1000) == UNSUPPORTED
    assert fwd(lib, L=8) == UNSUPPORTED
    assert fwd(lib, L=1 << 23) == UNSUPPORTED
    # long sequences need a workspace even with the spectrum given
    assert fwd(lib, L=1 << 16) == WORKSPACE
    xs17 = tuple(P(10 + i) for i in range(17))
    assert fwd(lib, xs=xs17) == UNSUPPORTED
    # misalignment
    assert fwd(lib, v=ctypes.c_void_p(A + 8)) == INVALID
    assert fwd(lib, y=ctypes.c_void_p(A + 5 * BIG + 4)) == INVALID
    assert fwd(lib, xs=(P(1), ctypes.c_void_p(A + 2 * BIG + 8))) == INVALID
    assert fwd(lib, H=ctypes.c_void_p(A + 3 * BIG + 8)) == INVALID
    assert fwd(lib, bias=ctypes.c_void_p(A + 4 * BIG + 2)) == INVALID
    # aliasing: y overlapping an input
    assert fwd(lib, y=P(0)) == INVALID
    assert fwd(lib, y=ctypes.c_void_p(A + 2 * BIG + 256)) == INVALID
    assert fwd(lib, y=P(3)) == INVALID
    # filters instead of spectra need a workspace
    assert fwd(lib, H=None, h=P(3)) == WORKSPACE
    assert fwd(lib, H=None, h=P(3), ws=P(6), wsb=16) == WORKSPACE
    assert fwd(lib, H=None, h=P(3), ws=ctypes.c_void_p(A + 6 * BIG + 16), wsb=1 << 20) == WORKSPACE
    # workspace overlapping y
    assert fwd(lib, H=None, h=P(3), ws=P(5), wsb=1 << 20) == INVALID


def bwd(lib, v=P(0), xs=(P(1), P(2)), H=P(3), bias=P(4), dy=P(5), B=2, D=3, L=64, N=None,
        io=F32, dv=P(6), dxs=(P(7), P(8)), dh=P(9), db=P(10), ws=P(11), wsb=1 << 24):
    N = len(xs) if N is None else N
    xa = (ctypes.c_void_p * max(len(xs), 1))(*[x.value if x is not None else None for x in xs])
    da = (ctypes.c_void_p * max(len(dxs), 1))(*[x.value if x is not None else None for x in dxs])
    return lib.hyena_fftconv_gate_backward(v, xa, H, bias, dy, B, D, L, N, io, dv, da, dh, db,
                                           ws, wsb, None)


def test_backward_rejects_bad_arguments(lib):
    lib.hyena_fftconv_backward_workspace_size.restype = ctypes.c_size_t
    lib.hyena_fftconv_backward_workspace_size.argtypes = [ctypes.c_int] * 4
    need = lib.hyena_fftconv_backward_workspace_size(2, 3, 64, 2)
    assert need >= 20 * 2 * 3 * 64 * 2                       # two batch slices
    # the slices stop at 8: a larger batch needs no more
    assert (lib.hyena_fftconv_backward_workspace_size(64, 3, 64, 2)
            == lib.hyena_fftconv_backward_workspace_size(8, 3, 64, 2)
            > lib.hyena_fftconv_backward_workspace_size(1, 3, 64, 2))
    # four-step lengths: the accumulated spectra plus the waves' saved spectra, c_n and scratch
    long_need = lib.hyena_fftconv_backward_workspace_size(2, 3, 1 << 15, 2)
    assert long_need >= 8 * 2 * 3 * (1 << 15) + (64 << 20) and long_need % 256 == 0
    assert lib.hyena_fftconv_backward_workspace_size(2, 3, 1 << 23, 2) == ctypes.c_size_t(-1).value
    assert lib.hyena_fftconv_backward_workspace_size(2, 0, 64, 2) == ctypes.c_size_t(-1).value
    assert lib.hyena_fftconv_backward_workspace_size(0, 3, 64, 2) == ctypes.c_size_t(-1).value
    for k in ("v", "H", "bias", "dy", "dv", "dh", "db"):
        assert bwd(lib, **{k: None}) == INVALID, k
    assert bwd(lib, xs=(P(1), None)) == INVALID
    assert bwd(lib, dxs=(P(7), None)) == INVALID
    assert bwd(lib, B=0) == INVALID
    assert bwd(lib, io=3) == INVALID
    # lengths up to 2^22 (the four-step path above 16384), powers of two
    assert bwd(lib, L=1 << 23) == UNSUPPORTED
    assert bwd(lib, L=100) == UNSUPPORTED
    assert bwd(lib, L=1 << 15, wsb=need) == WORKSPACE          # the four-step workspace is larger
    # workspace: missing, short, misaligned
    assert bwd(lib, ws=None) == WORKSPACE
    assert bwd(lib, wsb=need - 1) == WORKSPACE
    assert bwd(lib, ws=ctypes.c_void_p(A + 11 * BIG + 16)) == WORKSPACE
    # misalignment of an output
    assert bwd(lib, dh=ctypes.c_void_p(A + 9 * BIG + 4)) == INVALID
    assert bwd(lib, dxs=(P(7), ctypes.c_void_p(A + 8 * BIG + 8))) == INVALID
    # outputs overlapping inputs, each other, the workspace
    assert bwd(lib, dv=P(0)) == INVALID
    assert bwd(lib, dh=P(3)) == INVALID
    assert bwd(lib, db=ctypes.c_void_p(A + 6 * BIG + 64)) == INVALID
    assert bwd(lib, dxs=(P(7), P(7))) == INVALID
    assert bwd(lib, dxs=(P(11), P(8))) == INVALID


def test_circular_rejects_bad_arguments(lib):
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    f = lib.hyena_fftconv_gate_forward_circular
    assert f(P(0), xs, P(3), P(4), 2, 3, 16, 2, F32, P(5), None, 0, None) == UNSUPPORTED   # L < 32
    assert f(P(0), xs, P(3), P(4), 2, 3, 1 << 23, 2, F32, P(5), None, 0, None) == UNSUPPORTED
    assert f(P(0), xs, P(3), P(4), 2, 3, 96, 2, F32, P(5), None, 0, None) == UNSUPPORTED   # not a power of two
    assert f(None, xs, P(3), P(4), 2, 3, 64, 2, F32, P(5), None, 0, None) == INVALID
    assert f(P(0), xs, P(3), P(4), 2, 3, 64, 2, F32, P(0), None, 0, None) == INVALID       # y aliases v
    # above 16384 the four-step path needs a workspace
    assert f(P(0), xs, P(3), P(4), 2, 3, 1 << 15, 2, F32, P(5), None, 0, None) == WORKSPACE
    r = lib.hyena_filter_rfft_circular
    assert r(P(0), 2, 3, 16, P(1), None, 0, None) == UNSUPPORTED
    assert r(P(0), 2, 3, 64, ctypes.c_void_p(A + BIG + 8), None, 0, None) == INVALID
    assert r(P(0), 2, 3, 64, P(0), None, 0, None) == INVALID                               # H overlaps h
    assert r(P(0), 2, 3, 1 << 16, P(1), None, 0, None) == WORKSPACE


def test_circular_workspace_sizes(lib):
    ws = lib.hyena_fftconv_circular_workspace_size
    rs = lib.hyena_filter_rfft_circular_workspace_size
    ws.restype = rs.restype = ctypes.c_size_t
    assert ws(2, 3, 1 << 14, 2) == 0 and rs(2, 3, 1 << 14) == 0
    assert ws(2, 3, 1 << 16, 2) >= 6 * (1 << 15) * 8 and ws(2, 3, 1 << 16, 2) % 256 == 0
    assert rs(2, 3, 1 << 16) >= 6 * (1 << 15) * 8
    assert ws(2, 3, 16, 2) == ctypes.c_size_t(-1).value and rs(2, 3, 1 << 23) == ctypes.c_size_t(-1).value


def test_filter_rfft_rejects_bad_arguments(lib):
    r = lib.hyena_filter_rfft
    assert r(None, 2, 3, 64, P(1), None, 0, None) == INVALID
    assert r(P(0), 2, 3, 64, None, None, 0, None) == INVALID
    assert r(P(0), 0, 3, 64, P(1), None, 0, None) == INVALID
    assert r(P(0), 2, 3, 0, P(1), None, 0, None) == INVALID
    assert r(P(0), 2, 3, 48, P(1), None, 0, None) == UNSUPPORTED
    assert r(P(0), 2, 3, 1 << 23, P(1), None, 0, None) == UNSUPPORTED
    assert r(P(0), 2, 3, 64, ctypes.c_void_p(A + BIG + 8), None, 0, None) == INVALID
    assert r(P(0), 2, 3, 64, ctypes.c_void_p(A + 256), None, 0, None) == INVALID   # H overlaps h
    # long filters need a workspace
    assert r(P(0), 2, 3, 1 << 16, P(1), None, 0, None) == WORKSPACE
    assert r(P(0), 2, 3, 1 << 16, P(1), P(2), 1024, None) == WORKSPACE
    assert r(P(0), 2, 3, 1 << 16, P(1), P(1), 1 << 26, None) == INVALID        # workspace overlaps H


def test_rfft_workspace_size(lib):
    assert lib.hyena_filter_rfft_workspace_size(2, 3, 1 << 14) == 0
    n = lib.hyena_filter_rfft_workspace_size(2, 3, 1 << 16)
    assert n >= 6 * (1 << 16) * 8 and n % 256 == 0
    assert lib.hyena_filter_rfft_workspace_size(2, 3, 100) == ctypes.c_size_t(-1).value


def _ffn(lib, **kw):
    from subquadratic_sequence_b200.hyena import hyena_ffn_t
    f = dict(W1=A, W2=A + BIG, W3=A + 2 * BIG, Wout=A + 3 * BIG, alpha=A + 4 * BIG,
             n_bands=8, width=64, decay_div=64.0)
    f.update(kw)
    return hyena_ffn_t(**f)


def test_filter_gen_rejects_bad_arguments(lib):
    g = lib.hyena_filter_gen
    assert g(None, 2, 3, 64, P(5), None) == INVALID
    assert g(ctypes.byref(_ffn(lib, W2=None)), 2, 3, 64, P(5), None) == INVALID
    assert g(ctypes.byref(_ffn(lib, width=0)), 2, 3, 64, P(5), None) == INVALID
    assert g(ctypes.byref(_ffn(lib, width=65)), 2, 3, 64, P(5), None) == UNSUPPORTED
    assert g(ctypes.byref(_ffn(lib, n_bands=17)), 2, 3, 64, P(5), None) == UNSUPPORTED
    assert g(ctypes.byref(_ffn(lib, decay_div=0.0)), 2, 3, 64, P(5), None) == INVALID
    assert g(ctypes.byref(_ffn(lib)), 2, 3, 0, P(5), None) == INVALID
    assert g(ctypes.byref(_ffn(lib)), 2, 3, 64, None, None) == INVALID
    assert g(ctypes.byref(_ffn(lib, alpha=A + 4 * BIG + 2)), 2, 3, 64, P(5), None) == INVALID
    g2 = lib.hyena_filter_gen_2d
    assert g2(ctypes.byref(_ffn(lib)), 2, 3, 0, 8, P(5), None) == INVALID
    assert g2(ctypes.byref(_ffn(lib, width=100)), 2, 3, 8, 8, P(5), None) == UNSUPPORTED


def test_binding_refuses_cpu_tensors():
    import torch
    from subquadratic_sequence_b200 import hyena
    v = torch.zeros(1, 1, 16)
    with pytest.raises(TypeError):
        hyena.hyena_fftconv_gate_forward(v, [v], torch.zeros(1, 1), H=torch.zeros(1, 1, 16, dtype=torch.complex64))


def test_3d_rejects_bad_arguments(lib):
    from subquadratic_sequence_b200 import hyena
    ws = lib.hyena_fftconv3d_workspace_size
    n = ws(2, 3, 16, 32, 64, 2, F32, 1)
    assert n >= 2 * 3 * 16 * 64 * 64 * 8 and n % 256 == 0
    assert ws(2, 3, 16, 32, 64, 2, F32, 0) >= n + 2 * 3 * 32 * 64 * 64 * 8
    assert ws(2, 3, 8, 32, 64, 2, F32, 1) == ctypes.c_size_t(-1).value           # Z < 16
    assert ws(2, 3, 16, 512, 64, 2, F32, 1) == ctypes.c_size_t(-1).value         # H > 256
    assert ws(2, 3, 16, 32, 48, 2, F32, 1) == ctypes.c_size_t(-1).value          # W not a power of two
    with pytest.raises(hyena.HyenaError):
        hyena.hyena_fftconv3d_workspace_size(2, 3, 16, 16, 16, 17, F32, True)

    r = lib.hyena_filter_rfft3d
    assert r(None, 2, 3, 16, 16, 16, P(1), None) == INVALID
    assert r(P(0), 2, 3, 16, 16, 24, P(1), None) == UNSUPPORTED
    assert r(P(0), 2, 3, 512, 16, 16, P(1), None) == UNSUPPORTED
    assert r(P(0), 2, 3, 16, 16, 16, ctypes.c_void_p(A + BIG + 8), None) == INVALID
    assert r(P(0), 2, 3, 16, 16, 16, P(0), None) == INVALID                       # Hs overlaps h

    f = lib.hyena_fftconv3d_gate_forward
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    need = ws(2, 3, 16, 16, 16, 2, F32, 1)
    args = lambda **k: [k.get("v", P(0)), k.get("xs", xs), None, k.get("Hs", P(3)), P(4), 2, 3,
                        k.get("Z", 16), 16, 16, 2, k.get("io", F32), k.get("y", P(5)),
                        k.get("wsp", P(6)), k.get("nb", need), None]
    assert f(*args(v=None)) == INVALID
    assert f(*args(io=7)) == INVALID
    assert f(*args(Z=32 + 1)) == UNSUPPORTED
    assert f(*args(y=P(0))) == INVALID                                           # y aliases v
    assert f(*args(nb=need - 256)) == WORKSPACE
    assert f(*args(wsp=ctypes.c_void_p(A + BIG + 16))) == WORKSPACE              # misaligned
    assert f(*args(xs=(ctypes.c_void_p * 2)(P(1).value, None))) == INVALID


def test_circular_nd_rejects_bad_arguments(lib):
    ws2 = lib.hyena_fftconv2d_circular_workspace_size
    n = ws2(2, 3, 32, 64)
    assert n >= 2 * 3 * 32 * 32 * 8 and n % 256 == 0
    assert ws2(2, 3, 32, 16) == ctypes.c_size_t(-1).value           # W < 32
    assert ws2(2, 3, 8, 64) == ctypes.c_size_t(-1).value            # H < 16
    assert ws2(2, 3, 2048, 64) == ctypes.c_size_t(-1).value         # H > 1024
    r2 = lib.hyena_filter_rfft2d_circular
    assert r2(None, 2, 3, 32, 64, P(1), None) == INVALID
    assert r2(P(0), 2, 3, 32, 48, P(1), None) == UNSUPPORTED
    assert r2(P(0), 2, 3, 32, 64, P(0), None) == INVALID              # Hs overlaps h
    f2 = lib.hyena_fftconv2d_gate_forward_circular
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    need = ws2(2, 3, 32, 64)
    assert f2(P(0), xs, None, P(4), 2, 3, 32, 64, 2, F32, P(5), P(6), need, None) == INVALID   # no spectra
    assert f2(P(0), xs, P(3), P(4), 2, 3, 32, 64, 2, F32, P(0), P(6), need, None) == INVALID   # y aliases v
    assert f2(P(0), xs, P(3), P(4), 2, 3, 32, 64, 2, F32, P(5), P(6), need - 256, None) == WORKSPACE
    assert f2(P(0), xs, P(3), P(4), 2, 3, 32, 2048, 2, F32, P(5), P(6), need, None) == UNSUPPORTED

    ws3 = lib.hyena_fftconv3d_circular_workspace_size
    n = ws3(2, 3, 16, 32, 64)
    assert n >= 2 * 3 * 16 * 32 * 32 * 8 and n % 256 == 0
    assert ws3(2, 3, 16, 32, 512) == ctypes.c_size_t(-1).value      # W > 256
    r3 = lib.hyena_filter_rfft3d_circular
    assert r3(P(0), 2, 3, 16, 16, 16, P(1), None) == UNSUPPORTED       # W < 32
    assert r3(P(0), 2, 3, 16, 16, 32, P(0), None) == INVALID
    f3 = lib.hyena_fftconv3d_gate_forward_circular
    need = ws3(2, 3, 16, 16, 32)
    assert f3(P(0), xs, P(3), P(4), 2, 3, 16, 16, 32, 2, 7, P(5), P(6), need, None) == INVALID  # io
    assert f3(P(0), xs, P(3), P(4), 2, 3, 16, 16, 32, 2, F32, P(5), None, need, None) == WORKSPACE
    assert f3(P(0), xs, P(3), P(4), 2, 3, 16, 16, 32, 17, F32, P(5), P(6), need, None) == UNSUPPORTED


def test_backward_2d_rejects_bad_arguments(lib):
    ws = lib.hyena_fftconv2d_backward_workspace_size
    n = ws(2, 3, 32, 64, 2)
    # acc (N C 2H W) + saved spectra and c_n of one wave + scratch
    assert n >= (2 * 3 * 64 * 64 * 8) + (2 * 6 * 64 * 64 * 8) + (2 * 6 * 32 * 64 * 4) + (6 * 32 * 64 * 8)
    assert ws(2, 3, 8, 64, 2) == ctypes.c_size_t(-1).value
    assert ws(2, 3, 32, 64, 17) == ctypes.c_size_t(-1).value
    f = lib.hyena_fftconv2d_gate_backward
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    dxs = (ctypes.c_void_p * 2)(P(8).value, P(9).value)
    args = lambda **k: [k.get("v", P(0)), xs, k.get("Hs", P(3)), P(4), P(5), 2, 3, 32, 64, 2, k.get("io", F32),
                        k.get("dv", P(6)), k.get("dxs", dxs), k.get("dh", P(7)), P(10), k.get("wsp", P(11)),
                        k.get("nb", n), None]
    assert f(*args(v=None)) == INVALID
    assert f(*args(Hs=None)) == INVALID
    assert f(*args(io=9)) == INVALID
    assert f(*args(nb=n - 256)) == WORKSPACE
    assert f(*args(dv=P(0))) == INVALID                                    # dv aliases v
    assert f(*args(dh=P(6))) == INVALID                                    # dh aliases dv
    assert f(*args(dxs=(ctypes.c_void_p * 2)(P(8).value, P(8).value))) == INVALID   # dx_1 aliases dx_2


def test_filter_gen_3d_rejects_bad_arguments(lib):
    from subquadratic_sequence_b200 import hyena
    f = lib.hyena_filter_gen_3d
    ffn = hyena.hyena_ffn_t(P(0).value, P(1).value, P(2).value, P(3).value, P(4).value, 11, 64, 64.0)
    assert f(ctypes.byref(ffn), 2, 3, 4, 8, 16, P(5), None) == UNSUPPORTED        # n_bands > 10
    ffn.n_bands = 8
    assert f(ctypes.byref(ffn), 2, 3, 0, 8, 16, P(5), None) == INVALID           # Z < 1
    assert f(ctypes.byref(ffn), 2, 3, 4, 8, 16, None, None) == INVALID           # no output
    ffn.width = 65
    assert f(ctypes.byref(ffn), 2, 3, 4, 8, 16, P(5), None) == UNSUPPORTED        # width > 64


def test_backward_variants_reject_bad_arguments(lib):
    bad = ctypes.c_size_t(-1).value
    # per-sample: B dh spectra; any L up to 2^22
    ps = lib.hyena_fftconv_backward_per_sample_workspace_size
    assert ps(4, 3, 64, 2) >= 4 * 2 * 3 * 64 * 8 + 12 * 2 * 3 * 64
    assert ps(4, 3, 1 << 15, 2) > lib.hyena_fftconv_backward_workspace_size(4, 3, 1 << 15, 2)
    assert ps(4, 3, 1 << 23, 2) == bad and ps(0, 3, 64, 2) == bad
    # circular: 32 <= L <= 16384
    cs = lib.hyena_fftconv_backward_circular_workspace_size
    assert cs(2, 3, 64, 2) >= 12 * 2 * 3 * 64 * 2
    assert cs(2, 3, 16, 2) == bad and cs(2, 3, 1 << 23, 2) == bad and cs(2, 3, 96, 2) == bad
    assert cs(0, 3, 64, 2) == bad
    assert cs(2, 3, 1 << 15, 2) > (64 << 20)                 # the four-step layout above 16384
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    dxs = (ctypes.c_void_p * 2)(P(7).value, P(8).value)
    f = lib.hyena_fftconv_gate_backward_circular
    args = lambda **k: [k.get("v", P(0)), xs, P(3), P(4), P(5), 2, 3, k.get("L", 64), 2, F32, k.get("dv", P(6)),
                        dxs, k.get("dh", P(9)), P(10), k.get("ws", P(11)), k.get("nb", 1 << 24), None]
    assert f(*args(L=16)) == UNSUPPORTED
    assert f(*args(L=1 << 23)) == UNSUPPORTED
    assert f(*args(L=1 << 15)) == WORKSPACE                                      # four-step: more workspace
    assert f(*args(v=None)) == INVALID
    assert f(*args(ws=None)) == WORKSPACE
    assert f(*args(dv=P(0))) == INVALID                                          # dv aliases v
    g = lib.hyena_fftconv_gate_backward_per_sample
    # dh of B N D L floats: an output that starts inside it overlaps
    pa = lambda **k: [P(0), xs, P(3), P(4), P(5), 2, 3, 64, 2, F32, P(6), dxs, P(9),
                      k.get("db", P(10)), P(11), 1 << 24, None]
    assert g(*pa(db=ctypes.c_void_p(A + 9 * BIG + 4 * 2 * 2 * 3 * 64 - 64))) == INVALID
    # 2-D variants
    ws2 = lib.hyena_fftconv2d_backward_per_sample_workspace_size
    wc2 = lib.hyena_fftconv2d_backward_circular_workspace_size
    assert ws2(3, 2, 32, 64, 2) > lib.hyena_fftconv2d_backward_workspace_size(3, 2, 32, 64, 2)
    assert wc2(3, 2, 32, 64, 2) < lib.hyena_fftconv2d_backward_workspace_size(3, 2, 32, 64, 2)
    assert wc2(3, 2, 32, 16, 2) == bad and ws2(3, 2, 8, 64, 2) == bad
    h2 = lib.hyena_fftconv2d_gate_backward_circular
    a2 = lambda **k: [P(0), xs, k.get("Hs", P(3)), P(4), P(5), 2, 3, 32, k.get("W", 64), 2, F32, P(6), dxs, P(9),
                      P(10), P(11), 1 << 26, None]
    assert h2(*a2(W=16)) == UNSUPPORTED
    assert h2(*a2(Hs=None)) == INVALID


def test_3d_per_sample_entries_reject_bad_arguments(lib):
    from subquadratic_sequence_b200 import hyena
    f = lib.hyena_filter_gen_film_3d
    ffn = hyena.hyena_ffn_t(P(0).value, P(1).value, P(2).value, P(3).value, P(4).value, 8, 64, 64.0)
    film = hyena.hyena_film_t(None, None, None, None)
    assert f(ctypes.byref(ffn), None, 2, 2, 3, 4, 8, 16, P(5), None) == INVALID      # no film struct
    assert f(ctypes.byref(ffn), ctypes.byref(film), 0, 2, 3, 4, 8, 16, P(5), None) == INVALID   # B < 1
    film.gamma = ctypes.c_void_p(A + 6 * BIG + 2).value
    assert f(ctypes.byref(ffn), ctypes.byref(film), 2, 2, 3, 4, 8, 16, P(5), None) == INVALID  # misaligned
    film.gamma = None
    ffn.n_bands = 11
    assert f(ctypes.byref(ffn), ctypes.byref(film), 2, 2, 3, 4, 8, 16, P(5), None) == UNSUPPORTED
    g = lib.hyena_fftconv3d_gate_forward_per_sample
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    a = lambda **k: [P(0), xs, k.get("Hs", P(3)), P(4), 2, 3, 16, 16, k.get("W", 16), 2, F32, k.get("y", P(5)),
                     P(6), 1 << 28, None]
    assert g(*a(Hs=None)) == INVALID
    assert g(*a(W=8)) == UNSUPPORTED
    assert g(*a(y=P(0))) == INVALID                                              # y aliases v
    assert g(*a(Hs=ctypes.c_void_p(A + 3 * BIG + 8))) == INVALID


def fwd_noalloc(lib, v=P(0), xs=(P(1), P(2)), H=P(3), bias=P(4), B=2, D=3, L=64, N=None, io=F32,
                y=P(5)):
    N = len(xs) if N is None else N
    arr = (ctypes.c_void_p * max(len(xs), 1))(*[x.value if x is not None else None for x in xs])
    return lib.hyena_fftconv_gate_forward_noalloc(v, arr, H, bias, B, D, L, N, io, y, None)


def test_noalloc_rejects_bad_arguments(lib):
    assert fwd_noalloc(lib, v=None) == INVALID
    assert fwd_noalloc(lib, H=None) == INVALID
    assert fwd_noalloc(lib, y=None) == INVALID
    assert fwd_noalloc(lib, xs=(P(1), None)) == INVALID
    assert fwd_noalloc(lib, B=0) == INVALID
    assert fwd_noalloc(lib, io=3) == INVALID
    assert fwd_noalloc(lib, L=1000) == UNSUPPORTED
    assert fwd_noalloc(lib, L=1 << 23) == UNSUPPORTED
    # one sequence's four-step scratch (8 L bytes) must fit the built-in 16 MB
    assert fwd_noalloc(lib, L=1 << 22) == WORKSPACE
    assert fwd_noalloc(lib, v=ctypes.c_void_p(A + 8)) == INVALID
    assert fwd_noalloc(lib, H=ctypes.c_void_p(A + 3 * BIG + 8)) == INVALID
    # y overlapping v, an x_n, the spectra or the bias
    for L in (64, 1 << 16):
        assert fwd_noalloc(lib, y=P(0), L=L) == INVALID
        assert fwd_noalloc(lib, y=ctypes.c_void_p(A + 2 * BIG + 256), L=L) == INVALID
        assert fwd_noalloc(lib, y=ctypes.c_void_p(A + 1 * BIG - 256), L=L) == INVALID
        assert fwd_noalloc(lib, y=P(3), L=L) == INVALID
        assert fwd_noalloc(lib, y=ctypes.c_void_p(A + 4 * BIG - 16), L=L) == INVALID


def fwd_spill(lib, v=P(0), xs=(P(1), P(2)), H=P(3), bias=P(4), B=2, D=3, L=64, N=None, io=F32,
              y=P(5), ws=P(6), wsb=1 << 20):
    N = len(xs) if N is None else N
    arr = (ctypes.c_void_p * max(len(xs), 1))(*[x.value if x is not None else None for x in xs])
    return lib.hyena_fftconv_gate_forward_spill(v, arr, H, bias, B, D, L, N, io, y, ws, wsb, None)


def test_spill_rejects_bad_arguments(lib):
    bad = ctypes.c_size_t(-1).value
    assert lib.hyena_fftconv_spill_workspace_size(2, 3, 64, 2) == 2 * 3 * 64 * 4
    assert lib.hyena_fftconv_spill_workspace_size(2, 3, 64, 1) == 0
    assert lib.hyena_fftconv_spill_workspace_size(2, 3, 1 << 15, 2) == bad
    assert lib.hyena_fftconv_spill_workspace_size(2, 3, 100, 2) == bad
    assert fwd_spill(lib, v=None) == INVALID
    assert fwd_spill(lib, H=None) == INVALID
    assert fwd_spill(lib, xs=(P(1), None)) == INVALID
    assert fwd_spill(lib, io=2) == INVALID
    assert fwd_spill(lib, L=1 << 15) == UNSUPPORTED      # the spill variant covers the fused lengths
    assert fwd_spill(lib, L=48) == UNSUPPORTED
    assert fwd_spill(lib, ws=None) == WORKSPACE
    assert fwd_spill(lib, wsb=2 * 3 * 64 * 4 - 4) == WORKSPACE
    assert fwd_spill(lib, ws=ctypes.c_void_p(A + 6 * BIG + 16)) == INVALID   # 256-byte alignment
    assert fwd_spill(lib, y=P(0)) == INVALID
    assert fwd_spill(lib, ws=P(5)) == INVALID             # workspace overlapping y
    assert fwd_spill(lib, ws=P(2)) == INVALID             # workspace overlapping x_2
    assert fwd_spill(lib, ws=P(3)) == INVALID             # workspace overlapping H


def test_dft32_stage_rejects_bad_arguments(lib):
    f = lib.hyena_dft32_stage
    assert f(None, P(1), 4, 1, 0, None) == INVALID
    assert f(P(0), P(1), 0, 1, 0, None) == INVALID
    assert f(P(0), P(1), 4, 0, 0, None) == INVALID
    assert f(P(0), P(1), 4, 1, 2, None) == INVALID
    assert f(ctypes.c_void_p(A + 8), P(1), 4, 1, 0, None) == INVALID
    assert f(P(0), P(0), 4, 1, 1, None) == INVALID                  # y overlapping x
    assert f(P(0), P(1), (1 << 30) + 1, 1, 0, None) == UNSUPPORTED


def test_backward_2d_circular_per_sample_rejects_bad_arguments(lib):
    bad = ctypes.c_size_t(-1).value
    assert lib.hyena_fftconv2d_backward_circular_per_sample_workspace_size(2, 3, 32, 64, 2) != bad
    assert (lib.hyena_fftconv2d_backward_circular_per_sample_workspace_size(2, 3, 32, 64, 2)
            > lib.hyena_fftconv2d_backward_circular_workspace_size(2, 3, 32, 64, 2))
    assert lib.hyena_fftconv2d_backward_circular_per_sample_workspace_size(2, 3, 30, 64, 2) == bad
    assert lib.hyena_fftconv2d_backward_circular_per_sample_workspace_size(0, 3, 32, 64, 2) == bad
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    dxs = (ctypes.c_void_p * 2)(P(7).value, P(8).value)
    f = lib.hyena_fftconv2d_gate_backward_circular_per_sample
    assert f(None, xs, P(3), P(4), P(5), 2, 3, 32, 64, 2, F32, P(6), dxs, P(9), P(10), P(11), 1 << 30,
             None) == INVALID
    assert f(P(0), xs, P(3), P(4), P(5), 2, 3, 30, 64, 2, F32, P(6), dxs, P(9), P(10), P(11), 1 << 30,
             None) == UNSUPPORTED
    assert f(P(0), xs, P(3), P(4), P(5), 2, 3, 32, 64, 2, F32, P(6), dxs, P(9), P(10), P(11), 16,
             None) == WORKSPACE
    assert f(P(0), xs, P(3), P(4), P(5), 2, 3, 32, 64, 2, F32, P(0), dxs, P(9), P(10), P(11), 1 << 30,
             None) == INVALID                        # dv overlapping v


def test_backward_3d_rejects_bad_arguments(lib):
    bad = ctypes.c_size_t(-1).value
    shared = lib.hyena_fftconv3d_backward_workspace_size(2, 3, 16, 32, 64, 2)
    per_sample = lib.hyena_fftconv3d_backward_per_sample_workspace_size(2, 3, 16, 32, 64, 2)
    assert shared != bad and per_sample != bad and per_sample > shared
    # the accumulated dh spectra alone: N C 2Z 2H W complex64
    assert shared >= 2 * 3 * (2 * 16) * (2 * 32) * 64 * 8
    assert lib.hyena_fftconv3d_backward_workspace_size(2, 3, 16, 32, 512, 2) == bad     # W > 256
    assert lib.hyena_fftconv3d_backward_workspace_size(2, 3, 8, 32, 64, 2) == bad       # Z < 16
    assert lib.hyena_fftconv3d_backward_workspace_size(2, 3, 16, 32, 64, 17) == bad     # N > 16
    assert lib.hyena_fftconv3d_backward_per_sample_workspace_size(0, 3, 16, 32, 64, 2) == bad
    xs = (ctypes.c_void_p * 2)(P(1).value, P(2).value)
    dxs = (ctypes.c_void_p * 2)(P(7).value, P(8).value)
    circ = lib.hyena_fftconv3d_backward_circular_workspace_size(2, 3, 16, 32, 64, 2)
    circ_ps = lib.hyena_fftconv3d_backward_circular_per_sample_workspace_size(2, 3, 16, 32, 64, 2)
    assert bad not in (circ, circ_ps) and shared > circ and circ_ps > circ
    assert lib.hyena_fftconv3d_backward_circular_workspace_size(2, 3, 16, 32, 16, 2) == bad   # W < 32
    for f in (lib.hyena_fftconv3d_gate_backward, lib.hyena_fftconv3d_gate_backward_per_sample,
              lib.hyena_fftconv3d_gate_backward_circular, lib.hyena_fftconv3d_gate_backward_circular_per_sample):
        ok = (P(0), xs, P(3), P(4), P(5), 2, 3, 16, 32, 64, 2, F32, P(6), dxs, P(9), P(10), P(11), 1 << 30, None)

        def call(**kw):
            a = list(ok)
            for k, val in kw.items():
                a[int(k[1:])] = val
            return f(*a)

        assert call(a0=None) == INVALID                               # v missing
        assert call(a2=None) == INVALID                               # spectra missing
        assert call(a7=30) == UNSUPPORTED                             # H not a power of two
        assert call(a8=512) == UNSUPPORTED                            # W above 256
        assert call(a10=17) == UNSUPPORTED                            # order above 16
        assert call(a11=5) == INVALID                                 # no such storage type
        assert call(a17=16) == WORKSPACE                              # workspace too small
        assert call(a16=ctypes.c_void_p(A + 11 * BIG + 16)) == WORKSPACE   # workspace misaligned
        assert call(a12=P(0)) == INVALID                              # dv overlapping v
        assert call(a14=P(3)) == INVALID                              # dh overlapping the spectra
        assert call(a12=ctypes.c_void_p(A + 6 * BIG + 4)) == INVALID  # dv misaligned
