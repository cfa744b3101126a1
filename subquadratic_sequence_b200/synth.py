"""Seeded synthetic inputs for the Hyena operator.

This module only draws random numbers and names the workloads.  It holds
none of the operator's arithmetic, and both the CUDA path and the float64
oracle consume exactly the arrays it returns (upcast exactly where the
oracle wants float64), so the random recipe cannot cause a parity
difference.

Recipe (every workload):

* one ``numpy.random.default_rng(seed)`` stream, drawn in this order:
  ``v``; ``x_1 .. x_N``; the bias ``b`` [N][D]; ``W1``, ``W2``, ``W3``,
  ``Wout``;
* activations ``v`` and ``x_n`` are float32 standard normals (``dtype=
  float32`` draws); for bf16 I/O they are then rounded to the nearest bf16
  (ties to even) and carried as float32 values that bf16 represents exactly;
* ``b`` and the FFN weights are float64 standard normals, the weights
  scaled by ``1/sqrt(fan_in)``, then rounded to float32;
* ``alpha`` is ``linspace(0.3, 1.5, D)`` rounded to float32.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

N_BANDS = 8
WIDTH = 64
DECAY_DIV = 64.0


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str        # "1d", "2d" or "3d"
    N: int           # order (number of long convolutions)
    B: int           # batch
    D: int           # channels (C for the 2-D operator)
    L: int = 0       # sequence length (1-D)
    H: int = 0       # grid height (2-D)
    W: int = 0       # grid width (2-D)
    Z: int = 0       # volume depth (3-D: volumes [Z][H][W])
    io: str = "f32"  # storage type of v, x_n, y: "f32" or "bf16"
    seed: int = 0
    film: bool = False  # input-dependent (per-sample, FiLM-modulated) filters
    circular: bool = False  # circular convolution on the grid itself (no padding)

    @property
    def per_channel(self) -> int:
        """Positions of one channel's sequence, grid or volume."""
        if self.kind == "1d":
            return self.L
        return self.H * self.W * (self.Z if self.kind == "3d" else 1)

    @property
    def shape(self) -> tuple:
        """Shape of the activations v, x_n, y."""
        if self.kind == "1d":
            return (self.B, self.D, self.L)
        if self.kind == "2d":
            return (self.B, self.D, self.H, self.W)
        return (self.B, self.D, self.Z, self.H, self.W)

    @property
    def positions(self) -> int:
        """Channel-positions per forward call: B*D*L (B*C*H*W, B*C*Z*H*W)."""
        return self.B * self.D * self.per_channel

    @property
    def io_bytes(self) -> int:
        return 2 if self.io == "bf16" else 4

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _seed(config: int, size_index: int = 0) -> int:
    return 1000 + 16 * config + size_index


WORKLOADS = {
    # order-2 operator at B=1, D=64, L=1024, fp32 (small parity case)
    "c0": Workload("c0", "1d", N=2, B=1, D=64, L=1024, io="f32", seed=_seed(0)),
    # order-2 operator at a GPT-small layer shape, bf16 storage
    "c1": Workload("c1", "1d", N=2, B=8, D=768, L=2048, io="bf16", seed=_seed(1)),
    # order-3 operator, B=2, D=768
    "c2_8k": Workload("c2_8k", "1d", N=3, B=2, D=768, L=8192, io="f32", seed=_seed(2, 0)),
    "c2_16k": Workload("c2_16k", "1d", N=3, B=2, D=768, L=16384, io="f32", seed=_seed(2, 1)),
    # order-2 long-context sweep, B=1, D=256
    "c3_64k": Workload("c3_64k", "1d", N=2, B=1, D=256, L=65536, io="f32", seed=_seed(3, 0)),
    "c3_256k": Workload("c3_256k", "1d", N=2, B=1, D=256, L=262144, io="f32", seed=_seed(3, 1)),
    "c3_1m": Workload("c3_1m", "1d", N=2, B=1, D=256, L=1048576, io="f32", seed=_seed(3, 2)),
    # order-2 2-D operator on a 256x256 grid, B=2, C=128
    "c4": Workload("c4", "2d", N=2, B=2, D=128, H=256, W=256, io="f32", seed=_seed(4)),
    # c1 with input-dependent filters: a filter set per sample (FiLM-modulated
    # sine layers, multi-frequency first layer, Gaussian window)
    "c1_film": Workload("c1_film", "1d", N=2, B=8, D=768, L=2048, io="bf16", seed=_seed(1), film=True),
    # c4 with input-dependent (per-sample, FiLM-modulated) 2-D filters
    "c4_film": Workload("c4_film", "2d", N=2, B=2, D=128, H=256, W=256, io="f32", seed=_seed(4), film=True),
    # order-2 3-D operator on 64^3 volumes, B=2, C=32, bf16 storage
    "c5_3d": Workload("c5_3d", "3d", N=2, B=2, D=32, Z=64, H=64, W=64, io="bf16", seed=_seed(5)),
    # c5_3d with input-dependent (per-sample, FiLM-modulated) 3-D filters
    "c5_3d_film": Workload("c5_3d_film", "3d", N=2, B=2, D=32, Z=64, H=64, W=64, io="bf16", seed=_seed(5),
                           film=True),
    # circular mode (periodic boundaries) at the shapes of c1, c4 and c5_3d
    "c1_circ": Workload("c1_circ", "1d", N=2, B=8, D=768, L=2048, io="bf16", seed=_seed(1), circular=True),
    "c3_64k_circ": Workload("c3_64k_circ", "1d", N=2, B=1, D=256, L=65536, io="f32", seed=_seed(3, 0),
                            circular=True),
    "c4_circ": Workload("c4_circ", "2d", N=2, B=2, D=128, H=256, W=256, io="f32", seed=_seed(4), circular=True),
    "c5_3d_circ": Workload("c5_3d_circ", "3d", N=2, B=2, D=32, Z=64, H=64, W=64, io="bf16", seed=_seed(5),
                           circular=True),
}


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); the result is
    float32 holding bf16-representable values."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of float32 values that bf16 represents
    exactly (as returned by :func:`bf16_round`)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def _activation(rng: np.random.Generator, shape, io: str) -> np.ndarray:
    a = np.empty(shape, dtype=np.float32)
    rng.standard_normal(out=a, dtype=np.float32)
    return bf16_round(a) if io == "bf16" else a


def _weights(rng: np.random.Generator, n_in: int, width: int, n_out: int):
    W1 = rng.standard_normal((width, n_in)) / np.sqrt(n_in)
    W2 = rng.standard_normal((width, width)) / np.sqrt(width)
    W3 = rng.standard_normal((width, width)) / np.sqrt(width)
    Wout = rng.standard_normal((n_out, width)) / np.sqrt(width)
    return [w.astype(np.float32) for w in (W1, W2, W3, Wout)]


def make_inputs(wl: Workload) -> dict:
    """All inputs of one workload as float32 numpy arrays.

    Keys: ``v``, ``x`` (list of N arrays), ``b`` [N][D], ``W1``, ``W2``,
    ``W3``, ``Wout``, ``alpha`` [D].
    """
    rng = np.random.default_rng(wl.seed)
    shape = wl.shape
    v = _activation(rng, shape, wl.io)
    x = [_activation(rng, shape, wl.io) for _ in range(wl.N)]
    b = rng.standard_normal((wl.N, wl.D)).astype(np.float32)
    n_in = {"1d": 1 + 2 * N_BANDS, "2d": 2 + 4 * N_BANDS, "3d": 3 + 6 * N_BANDS}[wl.kind]
    W1, W2, W3, Wout = _weights(rng, n_in, WIDTH, wl.N * wl.D)
    alpha = np.linspace(0.3, 1.5, wl.D).astype(np.float32)
    out = dict(v=v, x=x, b=b, W1=W1, W2=W2, W3=W3, Wout=Wout, alpha=alpha)
    if wl.film:
        out.update(make_film(wl))
    return out


def make_film(wl: Workload) -> dict:
    """FiLM inputs of an input-dependent workload, from their own stream
    (seed + 2): per-sample scales gamma = 1 + 0.1 N(0, 1) and shifts
    beta = 0.1 N(0, 1) [B][3][64]; per-unit frequencies omega [3][64] with
    the first layer in four blocks of 16 units at 1, 2, 4, 8 and the other
    layers at 1; Gaussian window widths sigma = linspace(0.05, 0.5, D)."""
    rng = np.random.default_rng(wl.seed + 2)
    gamma = (1.0 + 0.1 * rng.standard_normal((wl.B, 3, WIDTH))).astype(np.float32)
    beta = (0.1 * rng.standard_normal((wl.B, 3, WIDTH))).astype(np.float32)
    omega = np.ones((3, WIDTH), np.float32)
    omega[0] = np.repeat(np.array([1.0, 2.0, 4.0, 8.0], np.float32), WIDTH // 4)
    sigma = np.linspace(0.05, 0.5, wl.D).astype(np.float32)
    return dict(gamma=gamma, beta=beta, omega=omega, sigma=sigma)


def make_output_grad(wl: Workload) -> np.ndarray:
    """The upstream gradient dL/dy for the backward pass: i.i.d. N(0, 1) of
    the activation shape (bf16-rounded for bf16 storage), from its own
    stream (seed + 1) so the forward inputs are unchanged."""
    rng = np.random.default_rng(wl.seed + 1)
    return _activation(rng, wl.shape, wl.io)
