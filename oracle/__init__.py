"""Float64 CPU oracle for the Hyena long-convolution operator.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA product path never imports it, and the two share no code.

The arithmetic lives in ``hyena_oracle.c`` (plain C, float64, a textbook
radix-2 FFT and the direct O(L^2) sums); this module only compiles it with
gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyena_oracle.c")
_SO = os.path.join(_HERE, "_build", "libhyena_oracle.so")

ROUTE_DIRECT = 0
ROUTE_FFT = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libhyena_oracle.so``."""
    if (not force and os.path.exists(_SO)
            and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
        return _SO
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    tmp = _SO + f".tmp{os.getpid()}"
    # -ffp-contract=off: no fused multiply-adds, every product is rounded
    # to float64 exactly as written.
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    dp = ctypes.POINTER(ctypes.c_double)
    i, l, d = ctypes.c_int, ctypes.c_long, ctypes.c_double
    sigs = {
        "oracle_filter_gen": [dp, dp, dp, dp, dp, i, i, i, i, i, d, i, dp],
        "oracle_filter_gen_2d": [dp, dp, dp, dp, dp, i, i, i, i, i, i, d, i, dp],
        "oracle_fft": [dp, dp, l, i],
        "oracle_rfft_pad2": [dp, l, l, dp, dp],
        "oracle_rfft2_pad2": [dp, l, l, l, dp, dp],
        "oracle_conv": [dp, dp, l, i, dp],
        "oracle_conv2": [dp, dp, l, l, i, dp],
        "oracle_hyena_forward": [dp, dp, dp, dp, l, l, l, l, i, i, dp],
        "oracle_hyena_forward_2d": [dp, dp, dp, dp, l, l, l, l, l, i, i, dp],
        "oracle_hyena_backward": [dp, dp, dp, dp, dp, l, l, l, l, i, i, dp, dp, dp, dp],
        "oracle_filter_gen_film": [dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, i, d, i, dp],
        "oracle_cconv": [dp, dp, l, i, dp],
        "oracle_conv3": [dp, dp, l, l, l, i, dp],
        "oracle_hyena_forward_3d": [dp, dp, dp, dp, l, l, l, l, l, l, i, dp],
        "oracle_filter_gen_film_2d": [dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, i, i, d, i, dp],
        "oracle_rfft_circ": [dp, l, l, dp, dp],
        "oracle_hyena_forward_circular": [dp, dp, dp, dp, l, l, l, l, i, i, dp],
        "oracle_cconv3": [dp, dp, l, l, l, i, dp],
        "oracle_filter_gen_3d": [dp, dp, dp, dp, dp, i, i, i, i, i, i, i, d, i, dp],
        "oracle_hyena_backward_3d": [dp, dp, dp, dp, dp, l, l, l, l, l, l, i, dp, dp, dp, dp],
        "oracle_hyena_backward_circular_3d": [dp, dp, dp, dp, dp, l, l, l, l, l, l, i, dp, dp, dp, dp],
        "oracle_hyena_backward_circular_2d": [dp, dp, dp, dp, dp, l, l, l, l, l, i, i, dp, dp, dp, dp],
        "oracle_hyena_backward_circular": [dp, dp, dp, dp, dp, l, l, l, l, i, i, dp, dp, dp, dp],
        "oracle_filter_gen_film_3d": [dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, i, i, i, d, i, dp],
        "oracle_hyena_backward_2d": [dp, dp, dp, dp, dp, l, l, l, l, l, i, i, dp, dp, dp, dp],
        "oracle_hyena_forward_circular_nd": [dp, dp, dp, dp, l, l, l, l, l, l, i, dp],
    }
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    _lib = lib
    return lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc: int, name: str) -> None:
    if rc != 0:
        raise RuntimeError(f"{name} failed with status {rc}")


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _route(route) -> int:
    return {"direct": ROUTE_DIRECT, "fft": ROUTE_FFT}[route] if isinstance(route, str) else int(route)


def filter_gen(W1, W2, W3, Wout, alpha, N, D, L, n_bands=8, width=64,
               decay_div=64.0, threads=None) -> np.ndarray:
    """Implicit filters h[N][D][L] (float64)."""
    W1, W2, W3, Wout, alpha = map(_f64, (W1, W2, W3, Wout, alpha))
    assert W1.shape == (width, 1 + 2 * n_bands) and Wout.shape == (N * D, width)
    assert alpha.shape == (D,)
    h = np.empty((N, D, L), dtype=np.float64)
    rc = _load().oracle_filter_gen(_ptr(W1), _ptr(W2), _ptr(W3), _ptr(Wout),
                                   _ptr(alpha), N, D, L, n_bands, width,
                                   float(decay_div), threads or default_threads(),
                                   _ptr(h))
    _check(rc, "oracle_filter_gen")
    return h


def filter_gen_2d(W1, W2, W3, Wout, alpha, N, C, H, W, n_bands=8, width=64,
                  decay_div=64.0, threads=None) -> np.ndarray:
    """Implicit 2-D filters h[N][C][H][W] (float64)."""
    W1, W2, W3, Wout, alpha = map(_f64, (W1, W2, W3, Wout, alpha))
    assert W1.shape == (width, 2 + 4 * n_bands) and Wout.shape == (N * C, width)
    assert alpha.shape == (C,)
    h = np.empty((N, C, H, W), dtype=np.float64)
    rc = _load().oracle_filter_gen_2d(_ptr(W1), _ptr(W2), _ptr(W3), _ptr(Wout),
                                      _ptr(alpha), N, C, H, W, n_bands, width,
                                      float(decay_div),
                                      threads or default_threads(), _ptr(h))
    _check(rc, "oracle_filter_gen_2d")
    return h


def fft(x, sign: int = -1) -> np.ndarray:
    """Unnormalised DFT of a power-of-two length complex vector."""
    x = np.asarray(x, dtype=np.complex128)
    re, im = _f64(x.real).copy(), _f64(x.imag).copy()
    _check(_load().oracle_fft(_ptr(re), _ptr(im), re.size, sign), "oracle_fft")
    return re + 1j * im


def rfft_pad2(h) -> np.ndarray:
    """Bins 0..L of the DFT of each row of h[..., L] zero-padded to 2L."""
    h = _f64(h)
    L = h.shape[-1]
    rows = h.size // L
    re = np.empty(rows * (L + 1)); im = np.empty(rows * (L + 1))
    _check(_load().oracle_rfft_pad2(_ptr(h), rows, L, _ptr(re), _ptr(im)),
           "oracle_rfft_pad2")
    return (re + 1j * im).reshape(h.shape[:-1] + (L + 1,))


def rfft2_pad2(h) -> np.ndarray:
    """2-D DFT of each h[..., H, W] zero-padded to 2H x 2W, columns 0..W."""
    h = _f64(h)
    H, W = h.shape[-2:]
    rows = h.size // (H * W)
    n = rows * 2 * H * (W + 1)
    re = np.empty(n); im = np.empty(n)
    _check(_load().oracle_rfft2_pad2(_ptr(h), rows, H, W, _ptr(re), _ptr(im)),
           "oracle_rfft2_pad2")
    return (re + 1j * im).reshape(h.shape[:-2] + (2 * H, W + 1))


def conv(h, u, route="direct") -> np.ndarray:
    """Causal convolution of one sequence: y[t] = sum_{s<=t} h[s] u[t-s]."""
    h, u = _f64(h), _f64(u)
    assert h.shape == u.shape and h.ndim == 1
    y = np.empty_like(u)
    _check(_load().oracle_conv(_ptr(h), _ptr(u), u.size, _route(route), _ptr(y)),
           "oracle_conv")
    return y


def conv2(h, u, route="direct") -> np.ndarray:
    """Causal (first-quadrant) 2-D convolution of one image."""
    h, u = _f64(h), _f64(u)
    assert h.shape == u.shape and h.ndim == 2
    y = np.empty_like(u)
    _check(_load().oracle_conv2(_ptr(h), _ptr(u), u.shape[0], u.shape[1],
                                _route(route), _ptr(y)), "oracle_conv2")
    return y


def hyena_forward(v, x, h, bias, route="fft", threads=None) -> np.ndarray:
    """y = z_N of the order-N recurrence.

    v [B][D][L], x [N][B][D][L] (x_1..x_N stacked), h [N][D][L], bias [N][D].
    """
    v, x, h, bias = map(_f64, (v, x, h, bias))
    B, D, L = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, D, L) and h.shape == (N, D, L) and bias.shape == (N, D)
    y = np.empty_like(v)
    rc = _load().oracle_hyena_forward(_ptr(v), _ptr(x), _ptr(h), _ptr(bias),
                                      B, D, L, N, _route(route),
                                      threads or default_threads(), _ptr(y))
    _check(rc, "oracle_hyena_forward")
    return y


def hyena_forward_2d(v, x, h, bias, route="fft", threads=None) -> np.ndarray:
    """2-D recurrence: v [B][C][H][W], x [N][B][C][H][W], h [N][C][H][W],
    bias [N][C] -> y [B][C][H][W]."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    B, C, H, W = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, C, H, W) and h.shape == (N, C, H, W)
    assert bias.shape == (N, C)
    y = np.empty_like(v)
    rc = _load().oracle_hyena_forward_2d(_ptr(v), _ptr(x), _ptr(h), _ptr(bias),
                                         B, C, H, W, N, _route(route),
                                         threads or default_threads(), _ptr(y))
    _check(rc, "oracle_hyena_forward_2d")
    return y


def hyena_backward(v, x, h, bias, dy, route="fft", threads=None):
    """Gradients of a scalar loss with dL/dy = dy through the order-N
    recurrence: returns (dv [B][D][L], dx [N][B][D][L], dh [N][D][L],
    dbias [N][D]); dh and dbias are summed over the batch."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    B, D, L = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, D, L) and h.shape == (N, D, L) and bias.shape == (N, D)
    assert dy.shape == v.shape
    dv = np.empty_like(v)
    dx = np.empty_like(x)
    dh = np.empty_like(h)
    db = np.empty_like(bias)
    rc = _load().oracle_hyena_backward(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), _ptr(dy),
                                       B, D, L, N, _route(route), threads or default_threads(),
                                       _ptr(dv), _ptr(dx), _ptr(dh), _ptr(db))
    _check(rc, "oracle_hyena_backward")
    return dv, dx, dh, db


def hyena_backward_circular(v, x, h, bias, dy, route="fft", threads=None):
    """Gradients through :func:`hyena_forward_circular` (circular
    convolutions of length L): (dv, dx, dh [N][D][L], dbias [N][D]), dh and
    dbias summed over the batch."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    B, D, L = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, D, L) and h.shape == (N, D, L) and bias.shape == (N, D)
    assert dy.shape == v.shape
    dv, dx, dh, db = np.empty_like(v), np.empty_like(x), np.empty_like(h), np.empty_like(bias)
    rc = _load().oracle_hyena_backward_circular(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), _ptr(dy),
                                                B, D, L, N, _route(route), threads or default_threads(),
                                                _ptr(dv), _ptr(dx), _ptr(dh), _ptr(db))
    _check(rc, "oracle_hyena_backward_circular")
    return dv, dx, dh, db


def hyena_backward_per_sample(v, x, h, bias, dy, route="fft", threads=None):
    """The gradients through :func:`hyena_forward_per_sample` (a filter set
    per sample, h [B][N][D][L]): each sample's adjoint by
    :func:`hyena_backward` with its own filters.  Returns (dv, dx, dh
    [B][N][D][L] per sample, dbias [N][D] summed over the samples, as the
    bias is shared)."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    parts = [hyena_backward(v[b:b + 1], x[:, b:b + 1], h[b], bias, dy[b:b + 1], route, threads)
             for b in range(v.shape[0])]
    dv = np.concatenate([p[0] for p in parts])
    dx = np.concatenate([p[1] for p in parts], axis=1)
    dh = np.stack([p[2] for p in parts])
    db = np.sum([p[3] for p in parts], axis=0)
    return dv, dx, dh, db


def filter_gen_film(W1, W2, W3, Wout, omega, gamma, beta, window, gaussian, N, D, L, n_bands=8,
                    width=64, decay_div=64.0, threads=None) -> np.ndarray:
    """Per-sample (input-dependent) filters h [B][N][D][L]: the sine layers
    modulated by the sample's FiLM vectors, a_l = sin(omega_l (gamma_bl
    W_l a_(l-1) + beta_bl)); omega [3][width], gamma and beta [B][3][width];
    window [D] is alpha (exponential decay) or sigma (Gaussian)."""
    W1, W2, W3, Wout, omega, gamma, beta, window = map(
        _f64, (W1, W2, W3, Wout, omega, gamma, beta, window))
    B = gamma.shape[0]
    assert omega.shape == (3, width) and gamma.shape == (B, 3, width) and beta.shape == gamma.shape
    assert window.shape == (D,)
    h = np.empty((B, N, D, L))
    rc = _load().oracle_filter_gen_film(_ptr(W1), _ptr(W2), _ptr(W3), _ptr(Wout), _ptr(omega),
                                        _ptr(gamma), _ptr(beta), _ptr(window), int(bool(gaussian)),
                                        B, N, D, L, n_bands, width, float(decay_div),
                                        threads or default_threads(), _ptr(h))
    _check(rc, "oracle_filter_gen_film")
    return h


def hyena_forward_per_sample(v, x, h, bias, route="fft", threads=None) -> np.ndarray:
    """The forward with a filter set per sample, h [B][N][D][L]: the
    recurrence of :func:`hyena_forward` applied to each sample with its own
    filters."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    return np.concatenate([hyena_forward(v[b:b + 1], x[:, b:b + 1], h[b], bias, route, threads)
                           for b in range(v.shape[0])])


def cconv(h, u, route="direct") -> np.ndarray:
    """Circular convolution y[t] = sum_s h[s] u[(t - s) mod L]."""
    h, u = _f64(h), _f64(u)
    y = np.empty_like(u)
    _check(_load().oracle_cconv(_ptr(h), _ptr(u), u.shape[-1], _route(route), _ptr(y)), "oracle_cconv")
    return y


def rfft_circ(h) -> np.ndarray:
    """L-point spectrum (no padding) of each row of h [..., L]: bins 0..L/2."""
    h = _f64(h)
    L = h.shape[-1]
    rows = h.size // L
    re = np.empty(h.shape[:-1] + (L // 2 + 1,))
    im = np.empty_like(re)
    _check(_load().oracle_rfft_circ(_ptr(h), rows, L, _ptr(re), _ptr(im)), "oracle_rfft_circ")
    return re + 1j * im


def hyena_forward_circular(v, x, h, bias, route="fft", threads=None) -> np.ndarray:
    """The recurrence with circular convolutions of length L."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    B, D, L = v.shape
    N = h.shape[0]
    y = np.empty_like(v)
    rc = _load().oracle_hyena_forward_circular(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), B, D, L, N,
                                               _route(route), threads or default_threads(), _ptr(y))
    _check(rc, "oracle_hyena_forward_circular")
    return y


def filter_gen_film_2d(W1, W2, W3, Wout, omega, gamma, beta, window, gaussian, N, C, H, W, n_bands=8,
                       width=64, decay_div=64.0, threads=None) -> np.ndarray:
    """Per-sample 2-D filters h [B][N][C][H][W]: the FiLM-modulated sine
    layers on the 2-D features; window [C] is alpha (separable exponential
    decay) or sigma (Gaussian exp(-(ty^2 + tx^2) / (2 sigma^2)))."""
    W1, W2, W3, Wout, omega, gamma, beta, window = map(
        _f64, (W1, W2, W3, Wout, omega, gamma, beta, window))
    B = gamma.shape[0]
    h = np.empty((B, N, C, H, W))
    rc = _load().oracle_filter_gen_film_2d(_ptr(W1), _ptr(W2), _ptr(W3), _ptr(Wout), _ptr(omega),
                                           _ptr(gamma), _ptr(beta), _ptr(window), int(bool(gaussian)),
                                           B, N, C, H, W, n_bands, width, float(decay_div),
                                           threads or default_threads(), _ptr(h))
    _check(rc, "oracle_filter_gen_film_2d")
    return h


def hyena_forward_2d_per_sample(v, x, h, bias, route="fft", threads=None) -> np.ndarray:
    """The 2-D forward with a filter set per sample, h [B][N][C][H][W]."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    return np.concatenate([hyena_forward_2d(v[b:b + 1], x[:, b:b + 1], h[b], bias, route, threads)
                           for b in range(v.shape[0])])


def conv3(h, u, route="direct") -> np.ndarray:
    """3-D linear convolution on offsets 0..Z-1 x 0..H-1 x 0..W-1, cropped."""
    h, u = _f64(h), _f64(u)
    Z, H, W = u.shape
    y = np.empty_like(u)
    _check(_load().oracle_conv3(_ptr(h), _ptr(u), Z, H, W, _route(route), _ptr(y)), "oracle_conv3")
    return y


def hyena_forward_3d(v, x, h, bias, route="fft") -> np.ndarray:
    """The recurrence with 3-D convolutions: v [B][C][Z][H][W], x [N][B][C][Z][H][W],
    h [N][C][Z][H][W], bias [N][C] -> y [B][C][Z][H][W]."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    B, C, Z, H, W = v.shape
    N = h.shape[0]
    y = np.empty_like(v)
    _check(_load().oracle_hyena_forward_3d(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), B, C, Z, H, W, N,
                                           _route(route), _ptr(y)), "oracle_hyena_forward_3d")
    return y


def cconv3(h, u, route="direct") -> np.ndarray:
    """Circular convolution on a Z x H x W grid (a 2-D grid: Z = 1):
    y[p][q][r] = sum h[i][j][k] u[(p-i) mod Z][(q-j) mod H][(r-k) mod W]."""
    h, u = _f64(h), _f64(u)
    Z, H, W = u.shape
    y = np.empty_like(u)
    _check(_load().oracle_cconv3(_ptr(h), _ptr(u), Z, H, W, _route(route), _ptr(y)), "oracle_cconv3")
    return y


def hyena_forward_circular_nd(v, x, h, bias, route="fft") -> np.ndarray:
    """The recurrence with circular convolutions on 2-D grids or 3-D volumes:
    v [B][C][(Z)][H][W], x [N][B][C][(Z)][H][W], h [N][C][(Z)][H][W],
    bias [N][C] -> y of v's shape."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    shape = v.shape
    B, C = shape[:2]
    Z, H, W = (1,) + shape[2:] if v.ndim == 4 else shape[2:]
    N = h.shape[0]
    y = np.empty_like(v)
    _check(_load().oracle_hyena_forward_circular_nd(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), B, C, Z, H, W, N,
                                                    _route(route), _ptr(y)), "oracle_hyena_forward_circular_nd")
    return y


def hyena_backward_2d(v, x, h, bias, dy, route="fft", threads=None):
    """Gradients of a scalar loss with dL/dy = dy through the 2-D
    recurrence: returns (dv [B][C][H][W], dx [N][B][C][H][W], dh
    [N][C][H][W], dbias [N][C]); dh and dbias are summed over the batch."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    B, C, H, W = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, C, H, W) and h.shape == (N, C, H, W) and bias.shape == (N, C)
    assert dy.shape == v.shape
    dv, dx, dh, db = np.empty_like(v), np.empty_like(x), np.empty_like(h), np.empty_like(bias)
    rc = _load().oracle_hyena_backward_2d(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), _ptr(dy), B, C, H, W, N,
                                          _route(route), threads or default_threads(),
                                          _ptr(dv), _ptr(dx), _ptr(dh), _ptr(db))
    _check(rc, "oracle_hyena_backward_2d")
    return dv, dx, dh, db


def hyena_backward_circular_2d(v, x, h, bias, dy, route="fft", threads=None):
    """Gradients through the 2-D recurrence with circular convolutions on
    the H x W grid (:func:`hyena_forward_circular_nd` on 2-D grids): (dv,
    dx, dh [N][C][H][W], dbias [N][C]), dh and dbias summed over the batch."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    B, C, H, W = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, C, H, W) and h.shape == (N, C, H, W) and bias.shape == (N, C)
    assert dy.shape == v.shape
    dv, dx, dh, db = np.empty_like(v), np.empty_like(x), np.empty_like(h), np.empty_like(bias)
    rc = _load().oracle_hyena_backward_circular_2d(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), _ptr(dy), B, C, H, W,
                                                   N, _route(route), threads or default_threads(),
                                                   _ptr(dv), _ptr(dx), _ptr(dh), _ptr(db))
    _check(rc, "oracle_hyena_backward_circular_2d")
    return dv, dx, dh, db


def hyena_backward_3d(v, x, h, bias, dy, route="fft"):
    """Gradients of a scalar loss with dL/dy = dy through the 3-D
    recurrence: (dv [B][C][Z][H][W], dx [N][B][C][Z][H][W], dh
    [N][C][Z][H][W], dbias [N][C]); dh and dbias summed over the batch."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    B, C, Z, H, W = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, C, Z, H, W) and h.shape == (N, C, Z, H, W) and bias.shape == (N, C)
    assert dy.shape == v.shape
    dv, dx, dh, db = np.empty_like(v), np.empty_like(x), np.empty_like(h), np.empty_like(bias)
    rc = _load().oracle_hyena_backward_3d(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), _ptr(dy), B, C, Z, H, W, N,
                                          _route(route), _ptr(dv), _ptr(dx), _ptr(dh), _ptr(db))
    _check(rc, "oracle_hyena_backward_3d")
    return dv, dx, dh, db


def hyena_backward_circular_3d(v, x, h, bias, dy, route="fft"):
    """Gradients through the 3-D recurrence with circular convolutions on
    the Z x H x W grid (:func:`hyena_forward_circular_nd` on volumes): (dv,
    dx, dh [N][C][Z][H][W], dbias [N][C]), dh and dbias summed over the
    batch."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    B, C, Z, H, W = v.shape
    N = h.shape[0]
    assert x.shape == (N, B, C, Z, H, W) and h.shape == (N, C, Z, H, W) and bias.shape == (N, C)
    assert dy.shape == v.shape
    dv, dx, dh, db = np.empty_like(v), np.empty_like(x), np.empty_like(h), np.empty_like(bias)
    rc = _load().oracle_hyena_backward_circular_3d(_ptr(v), _ptr(x), _ptr(h), _ptr(bias), _ptr(dy), B, C, Z, H,
                                                   W, N, _route(route), _ptr(dv), _ptr(dx), _ptr(dh), _ptr(db))
    _check(rc, "oracle_hyena_backward_circular_3d")
    return dv, dx, dh, db


def hyena_backward_2d_per_sample(v, x, h, bias, dy, route="fft", threads=None):
    """The gradients through :func:`hyena_forward_2d_per_sample` (a filter
    set per sample, h [B][N][C][H][W]): each sample's 2-D adjoint with its
    own filters.  Returns (dv, dx, dh [B][N][C][H][W] per sample, dbias
    [N][C] summed over the samples)."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    parts = [hyena_backward_2d(v[b:b + 1], x[:, b:b + 1], h[b], bias, dy[b:b + 1], route, threads)
             for b in range(v.shape[0])]
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts], axis=1),
            np.stack([p[2] for p in parts]), np.sum([p[3] for p in parts], axis=0))


def filter_gen_3d(W1, W2, W3, Wout, alpha, N, C, Z, H, W, n_bands=8, width=64, decay_div=64.0,
                  threads=None) -> np.ndarray:
    """Implicit 3-D filters h[N][C][Z][H][W] (float64): the filter network
    on [tz, ty, tx, (sin, cos)(2 pi k t) per axis], window
    exp(-alpha_c (iz + iy + ix) / decay_div)."""
    W1, W2, W3, Wout, alpha = map(_f64, (W1, W2, W3, Wout, alpha))
    assert W1.shape == (width, 3 + 6 * n_bands) and Wout.shape == (N * C, width)
    assert alpha.shape == (C,)
    h = np.empty((N, C, Z, H, W), dtype=np.float64)
    rc = _load().oracle_filter_gen_3d(_ptr(W1), _ptr(W2), _ptr(W3), _ptr(Wout), _ptr(alpha), N, C, Z, H, W,
                                      n_bands, width, float(decay_div), threads or default_threads(), _ptr(h))
    _check(rc, "oracle_filter_gen_3d")
    return h


def filter_gen_film_3d(W1, W2, W3, Wout, omega, gamma, beta, window, gaussian, N, C, Z, H, W, n_bands=8,
                       width=64, decay_div=64.0, threads=None) -> np.ndarray:
    """Per-sample 3-D filters h [B][N][C][Z][H][W]: the FiLM-modulated sine
    layers on the 3-D features; window [C] is alpha (separable exponential
    decay) or sigma (Gaussian exp(-(tz^2 + ty^2 + tx^2) / (2 sigma^2)))."""
    W1, W2, W3, Wout, omega, gamma, beta, window = map(_f64, (W1, W2, W3, Wout, omega, gamma, beta, window))
    B = gamma.shape[0]
    h = np.empty((B, N, C, Z, H, W))
    rc = _load().oracle_filter_gen_film_3d(_ptr(W1), _ptr(W2), _ptr(W3), _ptr(Wout), _ptr(omega), _ptr(gamma),
                                           _ptr(beta), _ptr(window), int(bool(gaussian)), B, N, C, Z, H, W,
                                           n_bands, width, float(decay_div), threads or default_threads(),
                                           _ptr(h))
    _check(rc, "oracle_filter_gen_film_3d")
    return h


def hyena_forward_3d_per_sample(v, x, h, bias, route="fft") -> np.ndarray:
    """The 3-D forward with a filter set per sample, h [B][N][C][Z][H][W]."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    return np.concatenate([hyena_forward_3d(v[b:b + 1], x[:, b:b + 1], h[b], bias, route)
                           for b in range(v.shape[0])])


def hyena_forward_circular_per_sample(v, x, h, bias, route="fft", threads=None) -> np.ndarray:
    """The circular 1-D forward with a filter set per sample, h [B][N][D][L]:
    :func:`hyena_forward_circular` applied to each sample with its own filters."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    return np.concatenate([hyena_forward_circular(v[b:b + 1], x[:, b:b + 1], h[b], bias, route, threads)
                           for b in range(v.shape[0])])


def hyena_forward_circular_nd_per_sample(v, x, h, bias, route="fft") -> np.ndarray:
    """The circular 2-D / 3-D forward with a filter set per sample, h
    [B][N][C][(Z)][H][W]: :func:`hyena_forward_circular_nd` per sample."""
    v, x, h, bias = map(_f64, (v, x, h, bias))
    return np.concatenate([hyena_forward_circular_nd(v[b:b + 1], x[:, b:b + 1], h[b], bias, route)
                           for b in range(v.shape[0])])


def hyena_backward_circular_per_sample(v, x, h, bias, dy, route="fft", threads=None):
    """The gradients through :func:`hyena_forward_circular_per_sample` (a
    filter set per sample, h [B][N][D][L]): each sample's circular adjoint
    with its own filters; dh per sample, dbias summed over the samples."""
    v, x, h, bias, dy = map(_f64, (v, x, h, bias, dy))
    parts = [hyena_backward_circular(v[b:b + 1], x[:, b:b + 1], h[b], bias, dy[b:b + 1], route, threads)
             for b in range(v.shape[0])]
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts], axis=1),
            np.stack([p[2] for p in parts]), np.sum([p[3] for p in parts], axis=0))
