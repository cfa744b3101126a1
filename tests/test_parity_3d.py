"""GPU parity of the 3-D path against the float64 oracle (run with -m gpu).

Tolerances as for 1-D and 2-D: 1e-4 (float32 activations) and 2e-2 (bf16)
of the oracle's maximum |y|; spectra at 2e-5 of their maximum.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def unpack_spectrum_3d(P: np.ndarray) -> np.ndarray:
    """Packed [..., 2Z, 2H, W] -> natural bins [..., 2Z, 2H, W+1]."""
    W = P.shape[-1]
    out = np.empty(P.shape[:-1] + (W + 1,), dtype=np.complex128)
    out[..., 1:W] = P[..., 1:]
    A = P[..., 0]
    Ar = np.conj(np.roll(A[..., ::-1, ::-1], (1, 1), axis=(-2, -1)))      # conj A[-kz][-ky]
    out[..., 0] = 0.5 * (A + Ar)
    out[..., W] = (A - Ar) / 2j
    return out


def filters_3d(rng, N, C, Z, H, W):
    """Seeded decaying random filters [N][C][Z][H][W]."""
    h = rng.standard_normal((N, C, Z, H, W))
    h *= np.exp(-np.arange(Z) / (Z / 4))[:, None, None]
    h *= np.exp(-np.arange(H) / (H / 4))[:, None]
    h *= np.exp(-np.arange(W) / (W / 4))
    return (h / np.sqrt(Z * H * W) * 8).astype(np.float32)


def problem_3d(B, C, Z, H, W, N, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((B, C, Z, H, W)).astype(np.float32)
    x = [rng.standard_normal((B, C, Z, H, W)).astype(np.float32) for _ in range(N)]
    b = rng.standard_normal((N, C)).astype(np.float32)
    return v, x, b, filters_3d(rng, N, C, Z, H, W)


def gpu_forward_3d(hy, v, x, b, h, io, use_h=False):
    vd, xs, bd = dev(v, io), [dev(xx, io) for xx in x], dev(b)
    if use_h:
        y = hy.hyena_fftconv3d_gate_forward(vd, xs, bd, h=dev(h))
    else:
        y = hy.hyena_fftconv3d_gate_forward(vd, xs, bd, Hs=hy.hyena_filter_rfft3d(dev(h)))
    torch.cuda.synchronize()
    return host(y)


def as_io(a, io):
    """The values the device sees: bf16 inputs rounded through torch."""
    if io == "f32":
        return a.astype(np.float64)
    return torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("Z,H,W", [(16, 16, 16), (32, 16, 64), (16, 64, 32), (64, 32, 16)])
def test_rfft3d_matches_oracle_fft(hy, Z, H, W):
    rng = np.random.default_rng(Z + 3 * H + 7 * W)
    h = filters_3d(rng, 2, 2, Z, H, W)
    got = unpack_spectrum_3d(hy.hyena_filter_rfft3d(dev(h)).cpu().numpy().astype(np.complex128))
    # the 2-D padded DFT of every plane (the oracle's), then the 2Z-point
    # DFT along z of the planes zero-padded to 2Z (the oracle's complex DFT)
    planes = oracle.rfft2_pad2(h.astype(np.float64))               # [2][2][Z][2H][W+1]
    pad = np.zeros((2, 2, 2 * Z) + planes.shape[-2:], np.complex128)
    pad[:, :, :Z] = planes
    ref = np.apply_along_axis(lambda r: oracle.fft(r, -1), 2, pad)
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) <= 2e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("B,C,Z,H,W,N,io", [
    (1, 2, 16, 16, 16, 2, "f32"), (2, 1, 16, 32, 64, 2, "f32"), (1, 2, 32, 16, 16, 3, "f32"),
    (2, 2, 16, 16, 32, 1, "bf16"), (1, 1, 64, 16, 16, 2, "f32"), (1, 1, 16, 64, 16, 2, "bf16"),
])
def test_forward_3d_matches_oracle(hy, B, C, Z, H, W, N, io):
    v, x, b, h = problem_3d(B, C, Z, H, W, N, seed=Z + H + W + N)
    got = gpu_forward_3d(hy, v, x, b, h, io)
    ref = oracle.hyena_forward_3d(as_io(v, io), np.stack([as_io(xx, io) for xx in x]), h.astype(np.float64),
                                  b.astype(np.float64))
    assert_close(got, ref, io, f"3-D B{B} C{C} {Z}x{H}x{W} N{N} {io}")


def test_forward_3d_shift_filters(hy):
    # h_1 = delta at (0, 0, 0), h_2 = delta at (1, 2, 3): closed form
    B, C, Z, H, W, N = 2, 2, 16, 16, 32, 2
    v, x, b, _ = problem_3d(B, C, Z, H, W, N, seed=5)
    h = np.zeros((N, C, Z, H, W), np.float32)
    h[0, :, 0, 0, 0] = 1.0
    h[1, :, 1, 2, 3] = 1.0
    got = gpu_forward_3d(hy, v, x, b, h, "f32")
    v64, x64, b64 = v.astype(np.float64), [xx.astype(np.float64) for xx in x], b.astype(np.float64)
    z1 = x64[0] * v64 * (1 + b64[0])[None, :, None, None, None]
    sh = np.zeros_like(z1)
    sh[..., 1:, 2:, 3:] = z1[..., :-1, :-2, :-3]
    ref = x64[1] * (sh + b64[1][None, :, None, None, None] * z1)
    assert_close(got, ref, "f32", "3-D shift filters")


def test_forward_3d_from_filters_equals_from_spectrum(hy):
    v, x, b, h = problem_3d(1, 2, 16, 32, 16, 2, seed=6)
    assert np.array_equal(gpu_forward_3d(hy, v, x, b, h, "f32", use_h=False),
                          gpu_forward_3d(hy, v, x, b, h, "f32", use_h=True))


def test_forward_3d_separable_matches_2d_path(hy):
    # a filter that is a delta along z makes each plane an independent 2-D
    # problem: the 3-D forward equals the 2-D forward of the planes
    B, C, Z, H, W, N = 1, 2, 16, 32, 32, 2
    v, x, b, h = problem_3d(B, C, Z, H, W, N, seed=7)
    h[:, :, 1:] = 0.0
    y3 = gpu_forward_3d(hy, v, x, b, h, "f32")
    # planes as 2-D images: [B][C][Z][H][W] -> [B][C*Z][H][W], filters repeated over z
    h2 = np.repeat(h[:, :, 0], Z, axis=1)
    b2 = np.repeat(b, Z, axis=1)
    y2 = host(hy.hyena_fftconv2d_gate_forward(dev(v.reshape(B, C * Z, H, W)),
                                              [dev(xx.reshape(B, C * Z, H, W)) for xx in x], dev(b2),
                                              h=dev(h2)))
    assert_close(y3.reshape(B, C * Z, H, W), y2.astype(np.float64), "f32", "3-D separable vs 2-D")


@pytest.mark.parametrize("Z,H,W", [(256, 16, 16), (16, 256, 16), (16, 16, 256)])
def test_forward_3d_longest_axes(hy, Z, H, W):
    # each axis at its largest supported length against the oracle
    v, x, b, h = problem_3d(1, 1, Z, H, W, 2, seed=Z + 2 * H + 3 * W)
    got = gpu_forward_3d(hy, v, x, b, h, "f32")
    ref = oracle.hyena_forward_3d(v.astype(np.float64), np.stack(x).astype(np.float64), h.astype(np.float64),
                                  b.astype(np.float64))
    assert_close(got, ref, "f32", f"3-D {Z}x{H}x{W}")


def test_forward_3d_largest_volume_shift_filters(hy):
    """256^3 volumes (the largest supported: one volume per wave), bf16,
    shift filters: the closed form holds at any size."""
    B, C, Z, H, W, N = 1, 2, 256, 256, 256, 2
    rng = np.random.default_rng(8)
    v = rng.standard_normal((B, C, Z, H, W), dtype=np.float32)
    x = [rng.standard_normal((B, C, Z, H, W), dtype=np.float32) for _ in range(N)]
    b = rng.standard_normal((N, C)).astype(np.float32)
    h = np.zeros((N, C, Z, H, W), np.float32)
    h[0, :, 0, 0, 0] = 1.0
    h[1, :, 3, 5, 7] = 1.0
    got = gpu_forward_3d(hy, v, x, b, h, "bf16")
    v64, x64 = as_io(v, "bf16"), [as_io(xx, "bf16") for xx in x]
    # z_1 is rounded to bf16 nowhere on the device: it stays in the float32 scratch
    z1 = x64[0] * v64 * (1 + b[0].astype(np.float64))[None, :, None, None, None]
    sh = np.zeros_like(z1)
    sh[..., 3:, 5:, 7:] = z1[..., :-3, :-5, :-7]
    ref = x64[1] * (sh + b[1].astype(np.float64)[None, :, None, None, None] * z1)
    assert_close(got, ref, "bf16", "3-D 256^3 shift filters")


# ------------------------------------------------- implicit 3-D filters

def ffn_3d(rng, N, C, K, width=64):
    n_in = 3 + 6 * K
    W1 = rng.standard_normal((width, n_in)) / np.sqrt(n_in)
    W2 = rng.standard_normal((width, width)) / np.sqrt(width)
    W3 = rng.standard_normal((width, width)) / np.sqrt(width)
    Wout = rng.standard_normal((N * C, width)) / np.sqrt(width)
    alpha = np.linspace(0.3, 1.5, C)
    return [w.astype(np.float32) for w in (W1, W2, W3, Wout, alpha)]


@pytest.mark.parametrize("N,C,Z,H,W,K", [
    (2, 3, 4, 8, 16, 8), (1, 2, 16, 16, 16, 10), (2, 40, 8, 8, 8, 8), (2, 8, 64, 64, 64, 8),
    (1, 3, 3, 5, 7, 2), (3, 30, 16, 32, 16, 0),
])
def test_filter_gen_3d_matches_oracle(hy, N, C, Z, H, W, K):
    rng = np.random.default_rng(Z * 7 + H * 3 + W + K)
    w = ffn_3d(rng, N, C, K)
    got = host(hy.hyena_filter_gen_3d(*[dev(a) for a in w], N, C, Z, H, W, n_bands=K))
    ref = oracle.filter_gen_3d(*w, N, C, Z, H, W, n_bands=K)
    assert np.max(np.abs(got - ref)) <= 2e-5 * np.max(np.abs(ref))


def test_forward_3d_with_generated_filters(hy):
    # the 3-D step: filters from the network, their spectra, the forward
    B, C, Z, H, W, N = 2, 3, 16, 16, 32, 2
    rng = np.random.default_rng(12)
    w = ffn_3d(rng, N, C, 8)
    v, x, b, _ = problem_3d(B, C, Z, H, W, N, seed=13)
    h = hy.hyena_filter_gen_3d(*[dev(a) for a in w], N, C, Z, H, W)
    y = host(hy.hyena_fftconv3d_gate_forward(dev(v), [dev(xx) for xx in x], dev(b), Hs=hy.hyena_filter_rfft3d(h)))
    href = oracle.filter_gen_3d(*w, N, C, Z, H, W)
    ref = oracle.hyena_forward_3d(v.astype(np.float64), np.stack(x).astype(np.float64), href, b.astype(np.float64))
    assert_close(y, ref, "f32", "3-D generated filters")
