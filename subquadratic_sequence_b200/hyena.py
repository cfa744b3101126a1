"""Thin ctypes binding of ``libhyena_b200.so`` (the C ABI in include/hyena.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Tensors are torch CUDA tensors used as device memory; the work is
enqueued on the current torch stream unless a stream is given.  There is no
fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

HYENA_OK = 0
HYENA_ERR_INVALID_ARG = 1
HYENA_ERR_UNSUPPORTED = 2
HYENA_ERR_WORKSPACE = 3
HYENA_ERR_CUDA = 4
HYENA_F32 = 0
HYENA_BF16 = 1
HYENA_MAX_ORDER = 16


class HyenaError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn}: {message}")
        self.status = status


class hyena_ffn_t(ctypes.Structure):
    _fields_ = [("W1", ctypes.c_void_p), ("W2", ctypes.c_void_p), ("W3", ctypes.c_void_p),
                ("Wout", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("n_bands", ctypes.c_int), ("width", ctypes.c_int), ("decay_div", ctypes.c_float)]


class hyena_film_t(ctypes.Structure):
    _fields_ = [("omega", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("sigma", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(_build.LIB):
        raise ImportError(
            f"{_build.LIB} is missing: build the CUDA library first "
            "(python -m subquadratic_sequence_b200.build)")
    lib = ctypes.CDLL(_build.LIB)
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    ffn_p = ctypes.POINTER(hyena_ffn_t)
    sigs = {
        "hyena_status_string": ([i], ctypes.c_char_p),
        "hyena_last_cuda_error": ([], i),
        "hyena_filter_gen": ([ffn_p, i, i, i, vp, vp], i),
        "hyena_filter_gen_2d": ([ffn_p, i, i, i, i, vp, vp], i),
        "hyena_filter_gen_film": ([ffn_p, ctypes.POINTER(hyena_film_t), i, i, i, i, vp, vp], i),
        "hyena_fftconv_gate_forward_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, vp, vp,
                                                   sz, vp], i),
        "hyena_filter_rfft_workspace_size": ([i, i, i], sz),
        "hyena_filter_rfft": ([vp, i, i, i, vp, vp, sz, vp], i),
        "hyena_fftconv_workspace_size": ([i, i, i, i, i, i], sz),
        "hyena_fftconv_gate_forward": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, vp, vp,
                                        sz, vp], i),
        "hyena_fftconv_gate_forward_noalloc": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, vp,
                                                vp], i),
        "hyena_fftconv_spill_workspace_size": ([i, i, i, i], sz),
        "hyena_device_fault_count": ([], i),
        "hyena_fftconv2d_backward_circular_per_sample_workspace_size": ([i, i, i, i, i], sz),
        "hyena_fftconv2d_gate_backward_circular_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i,
                                                               i, vp, ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv3d_backward_workspace_size": ([i, i, i, i, i, i], sz),
        "hyena_fftconv3d_backward_per_sample_workspace_size": ([i, i, i, i, i, i], sz),
        "hyena_fftconv3d_gate_backward": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, i, vp,
                                           ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv3d_gate_backward_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, i,
                                                      vp, ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv3d_backward_circular_workspace_size": ([i, i, i, i, i, i], sz),
        "hyena_fftconv3d_backward_circular_per_sample_workspace_size": ([i, i, i, i, i, i], sz),
        "hyena_fftconv3d_gate_backward_circular": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, i, vp,
                                                    ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv3d_gate_backward_circular_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i,
                                                               i, i, vp, ctypes.POINTER(vp), vp, vp, vp, sz,
                                                               vp], i),
        "hyena_dft32_stage": ([vp, vp, ctypes.c_long, i, i, vp], i),
        "hyena_fftconv_gate_forward_spill": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, vp, vp, sz,
                                              vp], i),
        "hyena_fftconv_backward_workspace_size": ([i, i, i, i], sz),
        "hyena_fftconv_backward_per_sample_workspace_size": ([i, i, i, i], sz),
        "hyena_fftconv_backward_circular_workspace_size": ([i, i, i, i], sz),
        "hyena_fftconv_backward_circular_per_sample_workspace_size": ([i, i, i, i], sz),
        "hyena_fftconv_gate_backward_circular_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i,
                                                             vp, ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv_gate_backward_circular": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, vp,
                                                  ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv_gate_backward_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, vp,
                                                    ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv_gate_backward": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, vp,
                                         ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_filter_rfft_circular_workspace_size": ([i, i, i], sz),
        "hyena_filter_rfft_circular": ([vp, i, i, i, vp, vp, sz, vp], i),
        "hyena_fftconv_circular_workspace_size": ([i, i, i, i], sz),
        "hyena_fftconv_gate_forward_circular": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, vp, vp, sz,
                                                 vp], i),
        "hyena_fftconv_gate_forward_circular_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, vp, vp,
                                                            sz, vp], i),
        "hyena_filter_rfft2d": ([vp, i, i, i, i, vp, vp], i),
        "hyena_filter_gen_film_2d": ([ffn_p, ctypes.POINTER(hyena_film_t), i, i, i, i, i, vp, vp], i),
        "hyena_fftconv2d_gate_forward_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, i, vp, vp,
                                                     sz, vp], i),
        "hyena_fftconv2d_workspace_size": ([i, i, i, i, i, i, i], sz),
        "hyena_fftconv2d_gate_forward": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, vp,
                                          vp, sz, vp], i),
        "hyena_filter_rfft3d": ([vp, i, i, i, i, i, vp, vp], i),
        "hyena_filter_gen_3d": ([ffn_p, i, i, i, i, i, vp, vp], i),
        "hyena_filter_gen_film_3d": ([ffn_p, ctypes.POINTER(hyena_film_t), i, i, i, i, i, i, vp, vp], i),
        "hyena_fftconv3d_gate_forward_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, i, i, vp,
                                                     vp, sz, vp], i),
        "hyena_filter_rfft2d_circular": ([vp, i, i, i, i, vp, vp], i),
        "hyena_fftconv2d_backward_workspace_size": ([i, i, i, i, i], sz),
        "hyena_fftconv2d_backward_per_sample_workspace_size": ([i, i, i, i, i], sz),
        "hyena_fftconv2d_backward_circular_workspace_size": ([i, i, i, i, i], sz),
        "hyena_fftconv2d_gate_backward_circular": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, vp,
                                                    ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv2d_gate_backward_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, vp,
                                                      ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_fftconv2d_gate_backward": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, vp,
                                           ctypes.POINTER(vp), vp, vp, vp, sz, vp], i),
        "hyena_filter_rfft3d_circular": ([vp, i, i, i, i, i, vp, vp], i),
        "hyena_fftconv3d_circular_workspace_size": ([i, i, i, i, i], sz),
        "hyena_fftconv3d_gate_forward_circular": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, i, i, vp, vp,
                                                   sz, vp], i),
        "hyena_fftconv3d_gate_forward_circular_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, i, i,
                                                              vp, vp, sz, vp], i),
        "hyena_fftconv2d_circular_workspace_size": ([i, i, i, i], sz),
        "hyena_fftconv2d_gate_forward_circular": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, i, vp, vp,
                                                   sz, vp], i),
        "hyena_fftconv2d_gate_forward_circular_per_sample": ([vp, ctypes.POINTER(vp), vp, vp, i, i, i, i, i, i, vp,
                                                              vp, sz, vp], i),
        "hyena_fftconv3d_workspace_size": ([i, i, i, i, i, i, i, i], sz),
        "hyena_fftconv3d_gate_forward": ([vp, ctypes.POINTER(vp), vp, vp, vp, i, i, i, i, i, i, i,
                                          vp, vp, sz, vp], i),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


LIB = _load()


def status_string(status: int) -> str:
    return LIB.hyena_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != HYENA_OK:
        msg = status_string(status)
        if status == HYENA_ERR_CUDA:
            msg += f" (cudaError {LIB.hyena_last_cuda_error()})"
        raise HyenaError(fn, status, msg)


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return HYENA_F32
    if t.dtype == torch.bfloat16:
        return HYENA_BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def _ffn(W1, W2, W3, Wout, alpha, n_bands, width, decay_div) -> hyena_ffn_t:
    f32 = torch.float32
    return hyena_ffn_t(_dev(W1, f32, "W1"), _dev(W2, f32, "W2"), _dev(W3, f32, "W3"),
                       _dev(Wout, f32, "Wout"), _dev(alpha, f32, "alpha"),
                       n_bands, width, float(decay_div))


def hyena_filter_gen(W1, W2, W3, Wout, alpha, N: int, D: int, L: int, *, n_bands: int = 8,
                     width: int = 64, decay_div: float = 64.0, out=None, stream=None):
    """Implicit filters h [N][D][L] float32."""
    f = _ffn(W1, W2, W3, Wout, alpha, n_bands, width, decay_div)
    if out is None:
        out = torch.empty((N, D, L), device=W1.device, dtype=torch.float32)
    _check("hyena_filter_gen", LIB.hyena_filter_gen(
        ctypes.byref(f), N, D, L, ctypes.c_void_p(_dev(out, torch.float32, "h")), _stream(stream)))
    return out


def hyena_filter_gen_film(W1, W2, W3, Wout, alpha, N: int, D: int, L: int, *, B: int, omega=None,
                          gamma=None, beta=None, sigma=None, n_bands: int = 8, width: int = 64,
                          decay_div: float = 64.0, out=None, stream=None):
    """Per-sample (input-dependent) filters h [B][N][D][L] float32: the sine
    layers modulated by FiLM, a_l = sin(omega_l (gamma_bl W_l a_(l-1) +
    beta_bl)); omega [3][width], gamma / beta [B][3][width], sigma [D] (the
    Gaussian window; None keeps the exponential decay of alpha)."""
    f = _ffn(W1, W2, W3, Wout, alpha, n_bands, width, decay_div)
    opt = lambda t, name: ctypes.c_void_p(_dev(t, torch.float32, name)) if t is not None else None
    film = hyena_film_t(opt(omega, "omega"), opt(gamma, "gamma"), opt(beta, "beta"), opt(sigma, "sigma"))
    if out is None:
        out = torch.empty((B, N, D, L), device=W1.device, dtype=torch.float32)
    _check("hyena_filter_gen_film", LIB.hyena_filter_gen_film(
        ctypes.byref(f), ctypes.byref(film), B, N, D, L, ctypes.c_void_p(_dev(out, torch.float32, "h")),
        _stream(stream)))
    return out


def hyena_fftconv_gate_forward_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor, *,
                                          out=None, workspace=None, stream=None):
    """The forward with per-sample spectra H [B][N][D][L] complex64."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    need = hyena_fftconv_workspace_size(B, D, L, N, io, True)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=v.device, dtype=torch.uint8)
    _check("hyena_fftconv_gate_forward_per_sample", LIB.hyena_fftconv_gate_forward_per_sample(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, D, L, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def hyena_filter_gen_2d(W1, W2, W3, Wout, alpha, N: int, C: int, H: int, W: int, *,
                        n_bands: int = 8, width: int = 64, decay_div: float = 64.0, out=None,
                        stream=None):
    """Implicit 2-D filters h [N][C][H][W] float32."""
    f = _ffn(W1, W2, W3, Wout, alpha, n_bands, width, decay_div)
    if out is None:
        out = torch.empty((N, C, H, W), device=W1.device, dtype=torch.float32)
    _check("hyena_filter_gen_2d", LIB.hyena_filter_gen_2d(
        ctypes.byref(f), N, C, H, W, ctypes.c_void_p(_dev(out, torch.float32, "h")),
        _stream(stream)))
    return out


def hyena_filter_rfft_workspace_size(N: int, D: int, L: int) -> int:
    n = LIB.hyena_filter_rfft_workspace_size(N, D, L)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_filter_rfft_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_filter_rfft(h: torch.Tensor, *, out=None, workspace=None, stream=None):
    """Packed spectra [N][D][L] complex64 (slot 0 = (bin 0, bin L)) of the
    filters h [N][D][L] zero-padded to 2L."""
    N, D, L = h.shape
    if out is None:
        out = torch.empty((N, D, L), device=h.device, dtype=torch.complex64)
    need = hyena_filter_rfft_workspace_size(N, D, L)
    if need and workspace is None:
        workspace = torch.empty(need, device=h.device, dtype=torch.uint8)
    wp = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
    wn = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("hyena_filter_rfft", LIB.hyena_filter_rfft(
        ctypes.c_void_p(_dev(h, torch.float32, "h")), N, D, L,
        ctypes.c_void_p(_dev(out, torch.complex64, "H")), wp, wn, _stream(stream)))
    return out


def hyena_fftconv_workspace_size(B: int, D: int, L: int, N: int, io: int,
                                 spectrum_given: bool) -> int:
    n = LIB.hyena_fftconv_workspace_size(B, D, L, N, io, int(bool(spectrum_given)))
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv_gate_forward(v: torch.Tensor, xs, bias: torch.Tensor, *, H=None, h=None,
                               out=None, workspace=None, stream=None):
    """y = z_N of the order-N recurrence for v [B][D][L] (float32 or bf16),
    xs = [x_1 .. x_N] (same shape and dtype), bias [N][D] float32 and either
    the packed spectra H [N][D][L] complex64 or the filters h [N][D][L]."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    Hp = ctypes.c_void_p(_dev(H, torch.complex64, "H")) if H is not None else None
    hp = ctypes.c_void_p(_dev(h, torch.float32, "h")) if h is not None else None
    ws_need = hyena_fftconv_workspace_size(B, D, L, N, io, H is not None)
    if ws_need and workspace is None:
        workspace = torch.empty(ws_need, device=v.device, dtype=torch.uint8)
    wp = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
    wn = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("hyena_fftconv_gate_forward", LIB.hyena_fftconv_gate_forward(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, hp, Hp,
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, D, L, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), wp, wn, _stream(stream)))
    return out


def hyena_fftconv_spill_workspace_size(B: int, D: int, L: int, N: int) -> int:
    n = LIB.hyena_fftconv_spill_workspace_size(B, D, L, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv_spill_workspace_size", HYENA_ERR_UNSUPPORTED, "invalid sizes")
    return n


def hyena_fftconv_gate_forward_spill(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor, *,
                                     out=None, workspace=None, stream=None):
    """The order-N forward with z written to HBM (float32) between orders,
    one launch per order (L <= 16384): the counterpart of the fused forward,
    which chains the orders on chip."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    need = hyena_fftconv_spill_workspace_size(B, D, L, N)
    if need and workspace is None:
        workspace = torch.empty(need, device=v.device, dtype=torch.uint8)
    wp = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
    wn = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("hyena_fftconv_gate_forward_spill", LIB.hyena_fftconv_gate_forward_spill(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, D, L, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), wp, wn, _stream(stream)))
    return out


def hyena_dft32_stage(x: torch.Tensor, reps: int, method: int, *, out=None, stream=None):
    """x [count][32] complex64: each 32-point DFT (scaled by 1/sqrt(32))
    applied reps times; method 0 on the FP32 pipes, 1 on the tensor cores."""
    count = x.shape[0]
    if tuple(x.shape) != (count, 32):
        raise ValueError(f"x must be [count][32], got {tuple(x.shape)}")
    if out is None:
        out = torch.empty_like(x)
    _check("hyena_dft32_stage", LIB.hyena_dft32_stage(
        ctypes.c_void_p(_dev(x, torch.complex64, "x")), ctypes.c_void_p(_dev(out, torch.complex64, "y")),
        count, reps, method, _stream(stream)))
    return out


def hyena_fftconv_gate_forward_noalloc(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor, *,
                                       out=None, stream=None):
    """The forward without a workspace, for callers that cannot allocate
    device memory: long sequences use the library's built-in 16 MB scratch
    (shared by all calls on a device; order calls that could overlap)."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    # the C entry point trusts these extents: check them here, and that
    # every tensor lives on v's device, whose built-in scratch is used
    if tuple(H.shape) != (N, D, L):
        raise ValueError(f"H must be [N][D][L] = {(N, D, L)}, got {tuple(H.shape)}")
    if tuple(bias.shape) != (N, D):
        raise ValueError(f"bias must be [N][D] = {(N, D)}, got {tuple(bias.shape)}")
    for i, x in enumerate(xs):
        if tuple(x.shape) != (B, D, L):
            raise ValueError(f"x[{i}] must have v's shape {(B, D, L)}, got {tuple(x.shape)}")
    if out is not None and tuple(out.shape) != (B, D, L):
        raise ValueError(f"out must have v's shape {(B, D, L)}, got {tuple(out.shape)}")
    for name, t in [("H", H), ("bias", bias), ("out", out), *[(f"x[{i}]", x) for i, x in enumerate(xs)]]:
        if t is not None and t.device != v.device:
            raise ValueError(f"{name} is on {t.device}, v on {v.device}: all must be on one device")
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    with torch.cuda.device(v.device):
        _check("hyena_fftconv_gate_forward_noalloc", LIB.hyena_fftconv_gate_forward_noalloc(
            ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
            ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, D, L, N, io,
            ctypes.c_void_p(_dev(out, v.dtype, "y")), _stream(stream)))
    return out


# ------------------------------------------------------------------ 2-D

def hyena_fftconv_backward_workspace_size(B: int, D: int, L: int, N: int) -> int:
    n = LIB.hyena_fftconv_backward_workspace_size(B, D, L, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv_backward_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv_gate_backward(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor,
                                dy: torch.Tensor, *, workspace=None, stream=None):
    """Gradients of a loss with dL/dy = dy through the order-N forward:
    returns (dv [B][D][L], [dx_1..dx_N], dh [N][D][L] float32, dbias [N][D]
    float32); v, x_n, dy float32 or bf16, H the packed spectra, L <= 2^22."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((N, D, L), device=v.device, dtype=torch.float32)
    db = torch.empty((N, D), device=v.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(hyena_fftconv_backward_workspace_size(B, D, L, N), device=v.device,
                                dtype=torch.uint8)
    _check("hyena_fftconv_gate_backward", LIB.hyena_fftconv_gate_backward(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, D, L, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_fftconv_backward_per_sample_workspace_size(B: int, D: int, L: int, N: int) -> int:
    n = LIB.hyena_fftconv_backward_per_sample_workspace_size(B, D, L, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv_backward_per_sample_workspace_size", HYENA_ERR_UNSUPPORTED,
                         "invalid sizes")
    return n


def hyena_fftconv_gate_backward_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor,
                                           dy: torch.Tensor, *, workspace=None, stream=None):
    """The backward with a spectrum set per sample, H [B][N][D][L]: returns
    (dv, [dx_1..dx_N], dh [B][N][D][L] per sample, dbias [N][D] summed over
    the batch); L up to 2^22."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((B, N, D, L), device=v.device, dtype=torch.float32)
    db = torch.empty((N, D), device=v.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(hyena_fftconv_backward_per_sample_workspace_size(B, D, L, N), device=v.device,
                                dtype=torch.uint8)
    _check("hyena_fftconv_gate_backward_per_sample", LIB.hyena_fftconv_gate_backward_per_sample(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, D, L, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_fftconv_backward_circular_workspace_size(B: int, D: int, L: int, N: int) -> int:
    n = LIB.hyena_fftconv_backward_circular_workspace_size(B, D, L, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv_backward_circular_workspace_size", HYENA_ERR_UNSUPPORTED,
                         "invalid sizes (32 <= L <= 2^22)")
    return n


def hyena_fftconv_gate_backward_circular(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor,
                                         dy: torch.Tensor, *, workspace=None, stream=None):
    """The backward of the circular forward (H [N][D][L/2] from
    hyena_filter_rfft_circular): returns (dv, [dx_1..dx_N], dh [N][D][L],
    dbias [N][D]), dh and dbias summed over the batch."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((N, D, L), device=v.device, dtype=torch.float32)
    db = torch.empty((N, D), device=v.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(hyena_fftconv_backward_circular_workspace_size(B, D, L, N), device=v.device,
                                dtype=torch.uint8)
    _check("hyena_fftconv_gate_backward_circular", LIB.hyena_fftconv_gate_backward_circular(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, D, L, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_fftconv_gate_backward_circular_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor,
                                                    dy: torch.Tensor, *, workspace=None, stream=None):
    """The circular backward with per-sample spectra H [B][N][D][L/2]:
    returns (dv, [dx_1..dx_N], dh [B][N][D][L] per sample, dbias [N][D]
    summed over the batch)."""
    B, D, L = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((B, N, D, L), device=v.device, dtype=torch.float32)
    db = torch.empty((N, D), device=v.device, dtype=torch.float32)
    if workspace is None:
        n = LIB.hyena_fftconv_backward_circular_per_sample_workspace_size(B, D, L, N)
        if n == ctypes.c_size_t(-1).value:
            raise HyenaError("hyena_fftconv_backward_circular_per_sample_workspace_size", HYENA_ERR_UNSUPPORTED,
                             "invalid sizes")
        workspace = torch.empty(n, device=v.device, dtype=torch.uint8)
    _check("hyena_fftconv_gate_backward_circular_per_sample", LIB.hyena_fftconv_gate_backward_circular_per_sample(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, D, L, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def _circ_ws(fn, name, args, workspace, device):
    """The workspace of a circular-mode call: none up to L = 16384, else the
    caller's or a fresh one of the size the library asks for."""
    n = fn(*args)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError(name, HYENA_ERR_UNSUPPORTED, "invalid sizes")
    if n == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(n, device=device, dtype=torch.uint8)
    return ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()


def hyena_filter_rfft_circular(h: torch.Tensor, *, out=None, workspace=None, stream=None):
    """Circular-mode spectra H [N][D][L/2] complex64 of filters h [N][D][L]
    (the L-point DFT without padding, packed: slot 0 = (bin 0, bin L/2))."""
    N, D, L = h.shape
    if out is None:
        out = torch.empty((N, D, L // 2), device=h.device, dtype=torch.complex64)
    wp, wn = _circ_ws(LIB.hyena_filter_rfft_circular_workspace_size, "hyena_filter_rfft_circular_workspace_size",
                      (N, D, L), workspace, h.device)
    _check("hyena_filter_rfft_circular", LIB.hyena_filter_rfft_circular(
        ctypes.c_void_p(_dev(h, torch.float32, "h")), N, D, L,
        ctypes.c_void_p(_dev(out, torch.complex64, "H")), wp, wn, _stream(stream)))
    return out


def hyena_fftconv_gate_forward_circular(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor, *,
                                        out=None, workspace=None, stream=None,
                                        _name="hyena_fftconv_gate_forward_circular"):
    """The order-N forward with circular convolutions of length L."""
    B, D, L = v.shape
    N = len(xs)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    wp, wn = _circ_ws(LIB.hyena_fftconv_circular_workspace_size, "hyena_fftconv_circular_workspace_size",
                      (B, D, L, N), workspace, v.device)
    _check(_name, getattr(LIB, _name)(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(H, torch.complex64, "H")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, D, L, N, io_dtype(v),
        ctypes.c_void_p(_dev(out, v.dtype, "y")), wp, wn, _stream(stream)))
    return out


def hyena_fftconv_gate_forward_circular_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, H: torch.Tensor, *,
                                                   out=None, workspace=None, stream=None):
    """The circular forward with per-sample spectra H [B][N][D][L/2]."""
    return hyena_fftconv_gate_forward_circular(v, xs, bias, H, out=out, workspace=workspace, stream=stream,
                                               _name="hyena_fftconv_gate_forward_circular_per_sample")


def hyena_filter_rfft2d(h: torch.Tensor, *, out=None, stream=None):
    """Packed 2-D spectra [N][C][2H][W] complex64 of the filters h
    [N][C][H][W] zero-padded to 2H x 2W (slot [ky][0] holds the DFT over y
    of the bin-0 + i bin-W column)."""
    N, C, H, W = h.shape
    if out is None:
        out = torch.empty((N, C, 2 * H, W), device=h.device, dtype=torch.complex64)
    _check("hyena_filter_rfft2d", LIB.hyena_filter_rfft2d(
        ctypes.c_void_p(_dev(h, torch.float32, "h")), N, C, H, W,
        ctypes.c_void_p(_dev(out, torch.complex64, "Hs")), _stream(stream)))
    return out


def hyena_fftconv2d_workspace_size(B: int, C: int, H: int, W: int, N: int, io: int,
                                   spectrum_given: bool) -> int:
    n = LIB.hyena_fftconv2d_workspace_size(B, C, H, W, N, io, int(bool(spectrum_given)))
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv2d_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv2d_gate_forward(v: torch.Tensor, xs, bias: torch.Tensor, *, Hs=None, h=None,
                                 out=None, workspace=None, stream=None):
    """2-D order-N forward: v, x_n [B][C][H][W] (float32 or bf16), bias
    [N][C], and the packed spectra Hs [N][C][2H][W] or the filters h
    [N][C][H][W]."""
    B, C, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    need = hyena_fftconv2d_workspace_size(B, C, H, W, N, io, Hs is not None)
    if workspace is None:
        workspace = torch.empty(need, device=v.device, dtype=torch.uint8)
    Hp = ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")) if Hs is not None else None
    hp = ctypes.c_void_p(_dev(h, torch.float32, "h")) if h is not None else None
    _check("hyena_fftconv2d_gate_forward", LIB.hyena_fftconv2d_gate_forward(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, hp, Hp,
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, C, H, W, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def hyena_filter_gen_film_2d(W1, W2, W3, Wout, alpha, N: int, C: int, H: int, W: int, *, B: int,
                             omega=None, gamma=None, beta=None, sigma=None, n_bands: int = 8,
                             width: int = 64, decay_div: float = 64.0, out=None, stream=None):
    """Per-sample 2-D filters h [B][N][C][H][W] float32 (FiLM-modulated; the
    Gaussian window when sigma [C] is given)."""
    f = _ffn(W1, W2, W3, Wout, alpha, n_bands, width, decay_div)
    opt = lambda t, name: ctypes.c_void_p(_dev(t, torch.float32, name)) if t is not None else None
    film = hyena_film_t(opt(omega, "omega"), opt(gamma, "gamma"), opt(beta, "beta"), opt(sigma, "sigma"))
    if out is None:
        out = torch.empty((B, N, C, H, W), device=W1.device, dtype=torch.float32)
    _check("hyena_filter_gen_film_2d", LIB.hyena_filter_gen_film_2d(
        ctypes.byref(f), ctypes.byref(film), B, N, C, H, W, ctypes.c_void_p(_dev(out, torch.float32, "h")),
        _stream(stream)))
    return out


def hyena_fftconv2d_gate_forward_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor, *,
                                            out=None, workspace=None, stream=None):
    """The 2-D forward with per-sample spectra Hs [B][N][C][2H][W] complex64."""
    B, C, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    need = hyena_fftconv2d_workspace_size(B, C, H, W, N, io, True)
    if workspace is None:
        workspace = torch.empty(need, device=v.device, dtype=torch.uint8)
    _check("hyena_fftconv2d_gate_forward_per_sample", LIB.hyena_fftconv2d_gate_forward_per_sample(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, C, H, W, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def hyena_filter_rfft3d(h: torch.Tensor, *, out=None, stream=None):
    """Packed 3-D spectra [N][C][2Z][2H][W] complex64 of the filters h
    [N][C][Z][H][W] zero-padded to 2Z x 2H x 2W (slot [kz][ky][0] holds
    the bin-0 + i bin-W pair)."""
    N, C, Z, H, W = h.shape
    if out is None:
        out = torch.empty((N, C, 2 * Z, 2 * H, W), device=h.device, dtype=torch.complex64)
    _check("hyena_filter_rfft3d", LIB.hyena_filter_rfft3d(
        ctypes.c_void_p(_dev(h, torch.float32, "h")), N, C, Z, H, W,
        ctypes.c_void_p(_dev(out, torch.complex64, "Hs")), _stream(stream)))
    return out


def hyena_fftconv3d_workspace_size(B: int, C: int, Z: int, H: int, W: int, N: int, io: int,
                                   spectrum_given: bool) -> int:
    n = LIB.hyena_fftconv3d_workspace_size(B, C, Z, H, W, N, io, int(bool(spectrum_given)))
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv3d_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv3d_gate_forward(v: torch.Tensor, xs, bias: torch.Tensor, *, Hs=None, h=None,
                                 out=None, workspace=None, stream=None):
    """3-D order-N forward: v, x_n [B][C][Z][H][W] (float32 or bf16), bias
    [N][C], and the packed spectra Hs [N][C][2Z][2H][W] or the filters h
    [N][C][Z][H][W]."""
    B, C, Z, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    need = hyena_fftconv3d_workspace_size(B, C, Z, H, W, N, io, Hs is not None)
    if workspace is None:
        workspace = torch.empty(need, device=v.device, dtype=torch.uint8)
    Hp = ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")) if Hs is not None else None
    hp = ctypes.c_void_p(_dev(h, torch.float32, "h")) if h is not None else None
    _check("hyena_fftconv3d_gate_forward", LIB.hyena_fftconv3d_gate_forward(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, hp, Hp,
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, C, Z, H, W, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def hyena_filter_rfft2d_circular(h: torch.Tensor, *, out=None, stream=None):
    """Circular 2-D spectra [N][C][H][W/2] complex64 of the filters h
    [N][C][H][W] (no padding; slot [ky][0] holds the bin-0 + i bin-W/2
    column's DFT)."""
    N, C, H, W = h.shape
    if out is None:
        out = torch.empty((N, C, H, W // 2), device=h.device, dtype=torch.complex64)
    _check("hyena_filter_rfft2d_circular", LIB.hyena_filter_rfft2d_circular(
        ctypes.c_void_p(_dev(h, torch.float32, "h")), N, C, H, W,
        ctypes.c_void_p(_dev(out, torch.complex64, "Hs")), _stream(stream)))
    return out


def hyena_fftconv2d_circular_workspace_size(B: int, C: int, H: int, W: int) -> int:
    n = LIB.hyena_fftconv2d_circular_workspace_size(B, C, H, W)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv2d_circular_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv2d_gate_forward_circular(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor, *,
                                          out=None, workspace=None, stream=None,
                                          _name="hyena_fftconv2d_gate_forward_circular"):
    """The order-N recurrence with circular 2-D convolutions: v, x_n
    [B][C][H][W] (float32 or bf16), bias [N][C], Hs from
    hyena_filter_rfft2d_circular."""
    B, C, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(hyena_fftconv2d_circular_workspace_size(B, C, H, W), device=v.device,
                                dtype=torch.uint8)
    _check(_name, getattr(LIB, _name)(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, C, H, W, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def hyena_fftconv2d_gate_forward_circular_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                                     *, out=None, workspace=None, stream=None):
    """The circular 2-D forward with per-sample spectra Hs [B][N][C][H][W/2]."""
    return hyena_fftconv2d_gate_forward_circular(v, xs, bias, Hs, out=out, workspace=workspace, stream=stream,
                                                  _name="hyena_fftconv2d_gate_forward_circular_per_sample")


def hyena_filter_rfft3d_circular(h: torch.Tensor, *, out=None, stream=None):
    """Circular 3-D spectra [N][C][Z][H][W/2] complex64 of the filters h
    [N][C][Z][H][W] (no padding)."""
    N, C, Z, H, W = h.shape
    if out is None:
        out = torch.empty((N, C, Z, H, W // 2), device=h.device, dtype=torch.complex64)
    _check("hyena_filter_rfft3d_circular", LIB.hyena_filter_rfft3d_circular(
        ctypes.c_void_p(_dev(h, torch.float32, "h")), N, C, Z, H, W,
        ctypes.c_void_p(_dev(out, torch.complex64, "Hs")), _stream(stream)))
    return out


def hyena_fftconv3d_circular_workspace_size(B: int, C: int, Z: int, H: int, W: int) -> int:
    n = LIB.hyena_fftconv3d_circular_workspace_size(B, C, Z, H, W)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv3d_circular_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv3d_gate_forward_circular(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor, *,
                                          out=None, workspace=None, stream=None,
                                          _name="hyena_fftconv3d_gate_forward_circular"):
    """The order-N recurrence with circular 3-D convolutions: v, x_n
    [B][C][Z][H][W] (float32 or bf16), bias [N][C], Hs from
    hyena_filter_rfft3d_circular."""
    B, C, Z, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(hyena_fftconv3d_circular_workspace_size(B, C, Z, H, W), device=v.device,
                                dtype=torch.uint8)
    _check(_name, getattr(LIB, _name)(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, C, Z, H, W, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def hyena_fftconv3d_gate_forward_circular_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                                     *, out=None, workspace=None, stream=None):
    """The circular 3-D forward with per-sample spectra Hs [B][N][C][Z][H][W/2]."""
    return hyena_fftconv3d_gate_forward_circular(v, xs, bias, Hs, out=out, workspace=workspace, stream=stream,
                                                  _name="hyena_fftconv3d_gate_forward_circular_per_sample")


def hyena_fftconv2d_backward_workspace_size(B: int, C: int, H: int, W: int, N: int) -> int:
    n = LIB.hyena_fftconv2d_backward_workspace_size(B, C, H, W, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv2d_backward_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv2d_gate_backward(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                  dy: torch.Tensor, *, workspace=None, stream=None):
    """Gradients of a loss with dL/dy = dy through the 2-D forward: returns
    (dv [B][C][H][W], [dx_1..dx_N], dh [N][C][H][W] float32, dbias [N][C]
    float32); v, x_n, dy float32 or bf16, Hs the packed 2-D spectra."""
    B, C, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((N, C, H, W), device=v.device, dtype=torch.float32)
    db = torch.empty((N, C), device=v.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(hyena_fftconv2d_backward_workspace_size(B, C, H, W, N), device=v.device,
                                dtype=torch.uint8)
    _check("hyena_fftconv2d_gate_backward", LIB.hyena_fftconv2d_gate_backward(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, C, H, W, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_filter_gen_3d(W1, W2, W3, Wout, alpha, N: int, C: int, Z: int, H: int, W: int, *,
                        n_bands: int = 8, width: int = 64, decay_div: float = 64.0, out=None, stream=None):
    """Implicit 3-D filters h [N][C][Z][H][W] float32 (W1 [width][3 + 6 n_bands])."""
    f = _ffn(W1, W2, W3, Wout, alpha, n_bands, width, decay_div)
    if out is None:
        out = torch.empty((N, C, Z, H, W), device=W1.device, dtype=torch.float32)
    _check("hyena_filter_gen_3d", LIB.hyena_filter_gen_3d(
        ctypes.byref(f), N, C, Z, H, W, ctypes.c_void_p(_dev(out, torch.float32, "h")), _stream(stream)))
    return out


def hyena_filter_gen_film_3d(W1, W2, W3, Wout, alpha, N: int, C: int, Z: int, H: int, W: int, *, B: int,
                             omega=None, gamma=None, beta=None, sigma=None, n_bands: int = 8,
                             width: int = 64, decay_div: float = 64.0, out=None, stream=None):
    """Per-sample 3-D filters h [B][N][C][Z][H][W] float32 (FiLM-modulated;
    the Gaussian window when sigma [C] is given)."""
    f = _ffn(W1, W2, W3, Wout, alpha, n_bands, width, decay_div)
    opt = lambda t, name: ctypes.c_void_p(_dev(t, torch.float32, name)) if t is not None else None
    film = hyena_film_t(opt(omega, "omega"), opt(gamma, "gamma"), opt(beta, "beta"), opt(sigma, "sigma"))
    if out is None:
        out = torch.empty((B, N, C, Z, H, W), device=W1.device, dtype=torch.float32)
    _check("hyena_filter_gen_film_3d", LIB.hyena_filter_gen_film_3d(
        ctypes.byref(f), ctypes.byref(film), B, N, C, Z, H, W,
        ctypes.c_void_p(_dev(out, torch.float32, "h")), _stream(stream)))
    return out


def hyena_fftconv3d_gate_forward_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor, *,
                                            out=None, workspace=None, stream=None):
    """The 3-D forward with per-sample spectra Hs [B][N][C][2Z][2H][W] complex64."""
    B, C, Z, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    if out is None:
        out = torch.empty_like(v)
    need = hyena_fftconv3d_workspace_size(B, C, Z, H, W, N, io, True)
    if workspace is None:
        workspace = torch.empty(need, device=v.device, dtype=torch.uint8)
    _check("hyena_fftconv3d_gate_forward_per_sample", LIB.hyena_fftconv3d_gate_forward_per_sample(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), B, C, Z, H, W, N, io,
        ctypes.c_void_p(_dev(out, v.dtype, "y")), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def hyena_fftconv2d_gate_backward_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                             dy: torch.Tensor, *, workspace=None, stream=None):
    """The 2-D backward with per-sample spectra Hs [B][N][C][2H][W]: returns
    (dv, [dx_1..dx_N], dh [B][N][C][H][W] per sample, dbias [N][C] summed
    over the batch)."""
    B, C, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((B, N, C, H, W), device=v.device, dtype=torch.float32)
    db = torch.empty((N, C), device=v.device, dtype=torch.float32)
    if workspace is None:
        n = LIB.hyena_fftconv2d_backward_per_sample_workspace_size(B, C, H, W, N)
        if n == ctypes.c_size_t(-1).value:
            raise HyenaError("hyena_fftconv2d_backward_per_sample_workspace_size", HYENA_ERR_UNSUPPORTED,
                             "invalid sizes")
        workspace = torch.empty(n, device=v.device, dtype=torch.uint8)
    _check("hyena_fftconv2d_gate_backward_per_sample", LIB.hyena_fftconv2d_gate_backward_per_sample(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, C, H, W, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_fftconv2d_backward_circular_workspace_size(B: int, C: int, H: int, W: int, N: int) -> int:
    n = LIB.hyena_fftconv2d_backward_circular_workspace_size(B, C, H, W, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv2d_backward_circular_workspace_size", HYENA_ERR_UNSUPPORTED, "invalid sizes")
    return n


def hyena_fftconv2d_backward_per_sample_workspace_size(B: int, C: int, H: int, W: int, N: int) -> int:
    n = LIB.hyena_fftconv2d_backward_per_sample_workspace_size(B, C, H, W, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv2d_backward_per_sample_workspace_size", HYENA_ERR_UNSUPPORTED,
                         "invalid sizes")
    return n


def hyena_fftconv2d_gate_backward_circular(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                           dy: torch.Tensor, *, workspace=None, stream=None):
    """The backward of the circular 2-D forward (Hs [N][C][H][W/2] from
    hyena_filter_rfft2d_circular): returns (dv, [dx_1..dx_N], dh
    [N][C][H][W], dbias [N][C]), dh and dbias summed over the batch."""
    B, C, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((N, C, H, W), device=v.device, dtype=torch.float32)
    db = torch.empty((N, C), device=v.device, dtype=torch.float32)
    if workspace is None:
        n = LIB.hyena_fftconv2d_backward_circular_workspace_size(B, C, H, W, N)
        if n == ctypes.c_size_t(-1).value:
            raise HyenaError("hyena_fftconv2d_backward_circular_workspace_size", HYENA_ERR_UNSUPPORTED,
                             "invalid sizes")
        workspace = torch.empty(n, device=v.device, dtype=torch.uint8)
    _check("hyena_fftconv2d_gate_backward_circular", LIB.hyena_fftconv2d_gate_backward_circular(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, C, H, W, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_fftconv2d_gate_backward_circular_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                                      dy: torch.Tensor, *, workspace=None, stream=None):
    """The backward of the circular 2-D forward with a spectrum set per
    sample (Hs [B][N][C][H][W/2]): returns (dv, [dx_1..dx_N], dh
    [B][N][C][H][W] per sample, dbias [N][C] summed over the batch)."""
    B, C, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty((B, N, C, H, W), device=v.device, dtype=torch.float32)
    db = torch.empty((N, C), device=v.device, dtype=torch.float32)
    if workspace is None:
        n = LIB.hyena_fftconv2d_backward_circular_per_sample_workspace_size(B, C, H, W, N)
        if n == ctypes.c_size_t(-1).value:
            raise HyenaError("hyena_fftconv2d_backward_circular_per_sample_workspace_size", HYENA_ERR_UNSUPPORTED,
                             "invalid sizes")
        workspace = torch.empty(n, device=v.device, dtype=torch.uint8)
    _check("hyena_fftconv2d_gate_backward_circular_per_sample",
           LIB.hyena_fftconv2d_gate_backward_circular_per_sample(
               ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
               ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
               B, C, H, W, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
               ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
               workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_fftconv3d_backward_workspace_size(B: int, C: int, Z: int, H: int, W: int, N: int) -> int:
    n = LIB.hyena_fftconv3d_backward_workspace_size(B, C, Z, H, W, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv3d_backward_workspace_size", HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv3d_backward_per_sample_workspace_size(B: int, C: int, Z: int, H: int, W: int, N: int) -> int:
    n = LIB.hyena_fftconv3d_backward_per_sample_workspace_size(B, C, Z, H, W, N)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError("hyena_fftconv3d_backward_per_sample_workspace_size", HYENA_ERR_INVALID_ARG,
                         "invalid sizes")
    return n


def _ws3d(name: str, *dims) -> int:
    n = getattr(LIB, name)(*dims)
    if n == ctypes.c_size_t(-1).value:
        raise HyenaError(name, HYENA_ERR_INVALID_ARG, "invalid sizes")
    return n


def hyena_fftconv3d_backward_circular_workspace_size(B: int, C: int, Z: int, H: int, W: int, N: int) -> int:
    return _ws3d("hyena_fftconv3d_backward_circular_workspace_size", B, C, Z, H, W, N)


def hyena_fftconv3d_backward_circular_per_sample_workspace_size(B: int, C: int, Z: int, H: int, W: int,
                                                                N: int) -> int:
    return _ws3d("hyena_fftconv3d_backward_circular_per_sample_workspace_size", B, C, Z, H, W, N)


_BWD3D_WS = {
    "hyena_fftconv3d_gate_backward": hyena_fftconv3d_backward_workspace_size,
    "hyena_fftconv3d_gate_backward_per_sample": hyena_fftconv3d_backward_per_sample_workspace_size,
    "hyena_fftconv3d_gate_backward_circular": hyena_fftconv3d_backward_circular_workspace_size,
    "hyena_fftconv3d_gate_backward_circular_per_sample": hyena_fftconv3d_backward_circular_per_sample_workspace_size,
}


def _backward3d(name: str, per_sample: bool, v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                dy: torch.Tensor, workspace, stream):
    if v.dim() != 5 or dy.shape != v.shape:
        raise HyenaError(name, HYENA_ERR_INVALID_ARG, "v and dy must be [B][C][Z][H][W] of one shape")
    B, C, Z, H, W = v.shape
    N = len(xs)
    io = io_dtype(v)
    xp = (ctypes.c_void_p * max(N, 1))(*[_dev(x, v.dtype, f"x[{i}]") for i, x in enumerate(xs)])
    dv = torch.empty_like(v)
    dxs = [torch.empty_like(v) for _ in range(N)]
    dxp = (ctypes.c_void_p * max(N, 1))(*[d.data_ptr() for d in dxs])
    dh = torch.empty(((B,) if per_sample else ()) + (N, C, Z, H, W), device=v.device, dtype=torch.float32)
    db = torch.empty((N, C), device=v.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(_BWD3D_WS[name](B, C, Z, H, W, N), device=v.device, dtype=torch.uint8)
    _check(name, getattr(LIB, name)(
        ctypes.c_void_p(_dev(v, v.dtype, "v")), xp, ctypes.c_void_p(_dev(Hs, torch.complex64, "Hs")),
        ctypes.c_void_p(_dev(bias, torch.float32, "bias")), ctypes.c_void_p(_dev(dy, v.dtype, "dy")),
        B, C, Z, H, W, N, io, ctypes.c_void_p(dv.data_ptr()), dxp, ctypes.c_void_p(dh.data_ptr()),
        ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return dv, dxs, dh, db


def hyena_fftconv3d_gate_backward(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor, dy: torch.Tensor,
                                  *, workspace=None, stream=None):
    """Gradients of a loss with dL/dy = dy through the 3-D forward: returns
    (dv [B][C][Z][H][W], [dx_1..dx_N], dh [N][C][Z][H][W] float32, dbias
    [N][C] float32); Hs the packed 3-D spectra [N][C][2Z][2H][W]."""
    return _backward3d("hyena_fftconv3d_gate_backward", False, v, xs, bias, Hs, dy, workspace, stream)


def hyena_fftconv3d_gate_backward_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                             dy: torch.Tensor, *, workspace=None, stream=None):
    """The 3-D backward with a spectrum set per sample (Hs
    [B][N][C][2Z][2H][W]): returns (dv, [dx_1..dx_N], dh [B][N][C][Z][H][W]
    per sample, dbias [N][C] summed over the batch)."""
    return _backward3d("hyena_fftconv3d_gate_backward_per_sample", True, v, xs, bias, Hs, dy, workspace, stream)


def hyena_fftconv3d_gate_backward_circular(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                           dy: torch.Tensor, *, workspace=None, stream=None):
    """The backward of the circular 3-D forward (Hs [N][C][Z][H][W/2]):
    returns (dv, [dx_1..dx_N], dh [N][C][Z][H][W], dbias [N][C])."""
    return _backward3d("hyena_fftconv3d_gate_backward_circular", False, v, xs, bias, Hs, dy, workspace, stream)


def hyena_fftconv3d_gate_backward_circular_per_sample(v: torch.Tensor, xs, bias: torch.Tensor, Hs: torch.Tensor,
                                                      dy: torch.Tensor, *, workspace=None, stream=None):
    """The circular 3-D backward with a spectrum set per sample (Hs
    [B][N][C][Z][H][W/2]): dh [B][N][C][Z][H][W] per sample, dbias summed."""
    return _backward3d("hyena_fftconv3d_gate_backward_circular_per_sample", True, v, xs, bias, Hs, dy, workspace,
                       stream)
