"""GPU parity of circular mode on 2-D grids (and 3-D volumes) against the
float64 oracle (run with -m gpu): convolution without padding ("Native
Multi-Dimensional Subquadratic Operators via Input Dependent Long
Convolutions", Handling Boundaries: circular convolution for periodic
systems).  Tolerances as everywhere: 1e-4 (float32 activations), 2e-2
(bf16) of the oracle's maximum |y|; spectra at 2e-5 of their maximum.
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


def as_io(a, io):
    if io == "f32":
        return a.astype(np.float64)
    return torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()


def decaying(rng, shape):
    """Seeded random filters with an exponential envelope along every grid axis."""
    h = rng.standard_normal(shape)
    for ax, n in enumerate(shape[2:]):
        env = np.exp(-np.arange(n) / (n / 4)).reshape([-1] + [1] * (len(shape) - 3 - ax))
        h = h * env
    return (h / np.sqrt(np.prod(shape[2:])) * 8).astype(np.float32)


def problem(B, C, grid, N, seed):
    rng = np.random.default_rng(seed)
    shape = (B, C) + tuple(grid)
    v = rng.standard_normal(shape).astype(np.float32)
    x = [rng.standard_normal(shape).astype(np.float32) for _ in range(N)]
    b = rng.standard_normal((N, C)).astype(np.float32)
    return v, x, b, decaying(rng, (N, C) + tuple(grid))


def dft_axis(a, axis):
    """The oracle's complex DFT (sign -1) along one axis."""
    return np.apply_along_axis(lambda r: oracle.fft(r, -1), axis, a.astype(np.complex128))


def unpack_circ_2d(P):
    """Packed [..., H, M] -> bins [..., H, M + 1] (M = W/2)."""
    M = P.shape[-1]
    out = np.empty(P.shape[:-1] + (M + 1,), np.complex128)
    out[..., 1:M] = P[..., 1:]
    A = P[..., 0]
    Ar = np.conj(np.roll(A[..., ::-1], 1, axis=-1))
    out[..., 0] = 0.5 * (A + Ar)
    out[..., M] = (A - Ar) / 2j
    return out


# ------------------------------------------------------------------ 2-D

@pytest.mark.parametrize("H,W", [(16, 32), (32, 64), (64, 16 * 2), (128, 256), (1024, 32), (16, 1024)])
def test_rfft2d_circular_matches_oracle_dft(hy, H, W):
    rng = np.random.default_rng(H + 3 * W)
    h = decaying(rng, (2, 3, H, W))
    got = unpack_circ_2d(hy.hyena_filter_rfft2d_circular(dev(h)).cpu().numpy().astype(np.complex128))
    ref = dft_axis(dft_axis(h.astype(np.float64), -1)[..., :W // 2 + 1], -2)
    assert np.max(np.abs(got - ref)) <= 2e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("B,C,H,W,N,io", [
    (1, 2, 16, 32, 2, "f32"), (2, 3, 32, 64, 2, "f32"), (1, 2, 64, 32, 3, "f32"), (2, 2, 16, 128, 1, "bf16"),
    (1, 1, 128, 32, 2, "f32"), (3, 1, 32, 32, 2, "bf16"), (1, 2, 256, 256, 2, "f32"),
    (1, 1, 1024, 32, 1, "f32"), (1, 1, 16, 1024, 2, "f32"), (1, 1, 512, 512, 1, "bf16"),
])
def test_forward_2d_circular_matches_oracle(hy, B, C, H, W, N, io):
    v, x, b, h = problem(B, C, (H, W), N, seed=H + W + N)
    Hs = hy.hyena_filter_rfft2d_circular(dev(h))
    y = host(hy.hyena_fftconv2d_gate_forward_circular(dev(v, io), [dev(xx, io) for xx in x], dev(b), Hs))
    ref = oracle.hyena_forward_circular_nd(as_io(v, io), np.stack([as_io(xx, io) for xx in x]),
                                           h.astype(np.float64), b.astype(np.float64))
    assert_close(y, ref, io, f"circular 2-D B{B} C{C} {H}x{W} N{N} {io}")


def test_forward_2d_circular_shift_filters_rotate(hy):
    # h_1 = delta at (0, 0), h_2 = delta at (5, 30): z_1 = x_1 v (1 + b_1),
    # y = x_2 (roll(z_1, (5, 30)) + b_2 z_1) -- with wrap-around
    B, C, H, W, N = 2, 2, 32, 64, 2
    v, x, b, _ = problem(B, C, (H, W), N, seed=3)
    h = np.zeros((N, C, H, W), np.float32)
    h[0, :, 0, 0] = 1.0
    h[1, :, 5, 30] = 1.0
    y = host(hy.hyena_fftconv2d_gate_forward_circular(dev(v), [dev(xx) for xx in x], dev(b),
                                                      hy.hyena_filter_rfft2d_circular(dev(h))))
    v64, x64, b64 = v.astype(np.float64), [xx.astype(np.float64) for xx in x], b.astype(np.float64)
    z1 = x64[0] * v64 * (1 + b64[0])[None, :, None, None]
    ref = x64[1] * (np.roll(z1, (5, 30), axis=(2, 3)) + b64[1][None, :, None, None] * z1)
    assert_close(y, ref, "f32", "circular 2-D shift filters")


def test_forward_2d_circular_on_padded_grids_is_the_linear_forward(hy):
    # grids zero-padded to 2H x 2W with x zero outside: the circular result
    # there is the padded (linear) 2-D forward of the GPU's other path
    B, C, H, W, N = 1, 2, 32, 32, 2
    v, x, b, h = problem(B, C, (H, W), N, seed=4)
    pad = lambda a: np.pad(a, [(0, 0)] * (a.ndim - 2) + [(0, H), (0, W)])
    yc = host(hy.hyena_fftconv2d_gate_forward_circular(dev(pad(v)), [dev(pad(xx)) for xx in x], dev(b),
                                                       hy.hyena_filter_rfft2d_circular(dev(pad(h)))))
    yl = host(hy.hyena_fftconv2d_gate_forward(dev(v), [dev(xx) for xx in x], dev(b), h=dev(h)))
    assert_close(yc[..., :H, :W], yl, "f32", "circular on padded grids")
    assert np.max(np.abs(yc[..., H:, :])) == 0.0 and np.max(np.abs(yc[..., :, W:])) == 0.0


# ------------------------------------------------------------------ 3-D

def check_backward(got, ref, io, name):
    dv, dx, dh, db = got
    rdv, rdx, rdh, rdb = ref
    assert_close(dv, rdv, io, f"{name} dv")
    assert_close(dx, rdx, io, f"{name} dx")
    err_h = np.max(np.abs(dh - rdh)) / np.max(np.abs(rdh))
    err_b = np.max(np.abs(db - rdb)) / np.max(np.abs(rdb))
    assert err_h <= 1e-4, f"{name} dh {err_h:.3e}"
    assert err_b <= 1e-4, f"{name} db {err_b:.3e}"


@pytest.mark.parametrize("B,C,H,W,N,io", [
    (1, 2, 16, 32, 1, "f32"), (2, 3, 32, 64, 2, "f32"), (2, 2, 16, 128, 2, "bf16"), (1, 1, 128, 32, 3, "f32"),
    (1, 1, 1024, 32, 1, "f32"), (1, 1, 16, 1024, 2, "f32"), (2, 2, 256, 256, 2, "f32"),
    (3, 22, 512, 512, 1, "f32"),     # 66 images, 64 a wave: channel 21 spans two waves
])
def test_backward_2d_circular_matches_oracle(hy, B, C, H, W, N, io):
    v, x, b, h = problem(B, C, (H, W), N, seed=2 * H + W + N)
    dy = np.random.default_rng(H * W).standard_normal((B, C, H, W)).astype(np.float32)
    Hs = hy.hyena_filter_rfft2d_circular(dev(h))
    dv, dxs, dh, db = hy.hyena_fftconv2d_gate_backward_circular(dev(v, io), [dev(xx, io) for xx in x], dev(b),
                                                                Hs, dev(dy, io))
    torch.cuda.synchronize()
    got = host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)
    ref = oracle.hyena_backward_circular_2d(as_io(v, io), np.stack([as_io(xx, io) for xx in x]),
                                            h.astype(np.float64), b.astype(np.float64), as_io(dy, io))
    check_backward(got, ref, io, f"circular 2-D backward B{B} C{C} {H}x{W} N{N} {io}")


@pytest.mark.parametrize("B,C,H,W,N,io", [
    (2, 2, 16, 32, 2, "f32"), (3, 3, 32, 64, 1, "f32"), (2, 2, 64, 128, 2, "bf16"), (2, 1, 256, 256, 3, "f32"),
    (3, 22, 512, 512, 1, "f32"),     # 66 images, 64 a wave
])
def test_backward_2d_circular_per_sample_matches_oracle(hy, B, C, H, W, N, io):
    """A spectrum set per sample: per sample b, the circular 2-D backward of
    the oracle with sample b's filters gives dv, dx and dh_b; db is the sum
    of the samples' db."""
    v, x, b, _ = problem(B, C, (H, W), N, seed=3 * H + W + N)
    rng = np.random.default_rng(H + 7 * W)
    h = np.stack([decaying(rng, (N, C, H, W)) for _ in range(B)])           # [B][N][C][H][W]
    dy = rng.standard_normal((B, C, H, W)).astype(np.float32)
    Hs = hy.hyena_filter_rfft2d_circular(dev(h.reshape(B * N, C, H, W))).view(B, N, C, H, W // 2)
    dv, dxs, dh, db = hy.hyena_fftconv2d_gate_backward_circular_per_sample(
        dev(v, io), [dev(xx, io) for xx in x], dev(b), Hs, dev(dy, io))
    torch.cuda.synchronize()
    got = host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)
    parts = [oracle.hyena_backward_circular_2d(as_io(v[i:i + 1], io), np.stack([as_io(xx[i:i + 1], io) for xx in x]),
                                               h[i].astype(np.float64), b.astype(np.float64), as_io(dy[i:i + 1], io))
             for i in range(B)]
    ref = (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts], axis=1),
           np.stack([p[2] for p in parts]), np.sum([p[3] for p in parts], axis=0))
    check_backward(got, ref, io, f"circular 2-D per-sample backward B{B} C{C} {H}x{W} N{N} {io}")


def test_backward_2d_circular_per_sample_with_equal_sets_is_the_shared_backward(hy):
    B, C, H, W, N = 3, 2, 32, 64, 2
    v, x, b, h = problem(B, C, (H, W), N, seed=31)
    dy = np.random.default_rng(5).standard_normal((B, C, H, W)).astype(np.float32)
    H1 = hy.hyena_filter_rfft2d_circular(dev(h))
    Hb = H1.unsqueeze(0).expand(B, -1, -1, -1, -1).contiguous()
    args = (dev(v), [dev(xx) for xx in x], dev(b))
    sdv, sdx, sdh, sdb = hy.hyena_fftconv2d_gate_backward_circular(*args, H1, dev(dy))
    pdv, pdx, pdh, pdb = hy.hyena_fftconv2d_gate_backward_circular_per_sample(*args, Hb, dev(dy))
    torch.cuda.synchronize()
    assert np.array_equal(host(pdv), host(sdv))
    for a_, b_ in zip(pdx, sdx):
        assert np.array_equal(host(a_), host(b_))
    assert np.max(np.abs(host(pdh).sum(axis=0) - host(sdh))) <= 1e-5 * np.max(np.abs(host(sdh)))
    assert np.max(np.abs(host(pdb) - host(sdb))) <= 1e-5 * np.max(np.abs(host(sdb)))


def test_backward_2d_circular_shift_filter_closed_form(hy):
    # N = 1, h = delta at (k, l), b = 0: y = x roll(v, (k, l)), so
    # dv = roll(dy x, (-k, -l)), dx = dy roll(v, (k, l)),
    # db = sum dy x v, dh[a][b] = sum dy x roll(v, (a, b))
    B, C, H, W, k, l = 2, 2, 32, 64, 5, 30
    rng = np.random.default_rng(9)
    v, x, dy = (rng.standard_normal((B, C, H, W)).astype(np.float32) for _ in range(3))
    h = np.zeros((1, C, H, W), np.float32)
    h[0, :, k, l] = 1.0
    dv, dxs, dh, db = hy.hyena_fftconv2d_gate_backward_circular(
        dev(v), [dev(x)], dev(np.zeros((1, C), np.float32)), hy.hyena_filter_rfft2d_circular(dev(h)), dev(dy))
    torch.cuda.synchronize()
    e = dy.astype(np.float64) * x
    assert_close(host(dv), np.roll(e, (-k, -l), axis=(2, 3)), "f32", "dv")
    assert_close(host(dxs[0]), dy.astype(np.float64) * np.roll(v, (k, l), axis=(2, 3)), "f32", "dx")
    for a_, b_ in [(0, 0), (1, 0), (0, 1), (k, l), (H - 1, W - 1), (7, 33)]:
        ref = np.sum(e * np.roll(v, (a_, b_), axis=(2, 3)), axis=(0, 2, 3))
        got = host(dh)[0, :, a_, b_]
        assert np.max(np.abs(got - ref)) <= 1e-4 * np.max(np.abs(host(dh))), (a_, b_)
    assert np.max(np.abs(host(db)[0] - np.sum(e * v, axis=(0, 2, 3)))) <= 1e-4 * np.max(np.abs(host(dh)))


def unpack_circ_3d(P):
    """Packed [..., Z, H, M] -> bins [..., Z, H, M + 1] (M = W/2)."""
    M = P.shape[-1]
    out = np.empty(P.shape[:-1] + (M + 1,), np.complex128)
    out[..., 1:M] = P[..., 1:]
    A = P[..., 0]
    Ar = np.conj(np.roll(A[..., ::-1, ::-1], (1, 1), axis=(-2, -1)))     # conj A[-kz][-ky]
    out[..., 0] = 0.5 * (A + Ar)
    out[..., M] = (A - Ar) / 2j
    return out


@pytest.mark.parametrize("Z,H,W", [(16, 16, 32), (32, 16, 64), (16, 64, 32), (64, 32, 32)])
def test_rfft3d_circular_matches_oracle_dft(hy, Z, H, W):
    rng = np.random.default_rng(Z + 5 * H + 7 * W)
    h = decaying(rng, (2, 2, Z, H, W))
    got = unpack_circ_3d(hy.hyena_filter_rfft3d_circular(dev(h)).cpu().numpy().astype(np.complex128))
    ref = dft_axis(dft_axis(dft_axis(h.astype(np.float64), -1)[..., :W // 2 + 1], -2), -3)
    assert np.max(np.abs(got - ref)) <= 2e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("B,C,Z,H,W,N,io", [
    (1, 2, 16, 16, 32, 2, "f32"), (2, 1, 16, 32, 64, 2, "f32"), (1, 2, 32, 16, 32, 3, "f32"),
    (2, 2, 16, 16, 32, 1, "bf16"), (1, 1, 64, 16, 32, 2, "f32"), (1, 1, 16, 64, 32, 2, "bf16"),
    (1, 1, 256, 16, 32, 1, "f32"), (1, 1, 16, 256, 32, 1, "f32"), (1, 1, 16, 16, 256, 2, "f32"),
])
def test_forward_3d_circular_matches_oracle(hy, B, C, Z, H, W, N, io):
    v, x, b, h = problem(B, C, (Z, H, W), N, seed=Z + H + W + N)
    Hs = hy.hyena_filter_rfft3d_circular(dev(h))
    y = host(hy.hyena_fftconv3d_gate_forward_circular(dev(v, io), [dev(xx, io) for xx in x], dev(b), Hs))
    ref = oracle.hyena_forward_circular_nd(as_io(v, io), np.stack([as_io(xx, io) for xx in x]),
                                           h.astype(np.float64), b.astype(np.float64))
    assert_close(y, ref, io, f"circular 3-D B{B} C{C} {Z}x{H}x{W} N{N} {io}")


def test_forward_3d_circular_largest_volume_shift_filters(hy):
    """256^3 volumes, bf16, shift filters with wrap-around: the closed form
    (np.roll) holds at any size."""
    B, C, Z, H, W, N = 1, 2, 256, 256, 256, 2
    rng = np.random.default_rng(8)
    v = rng.standard_normal((B, C, Z, H, W), dtype=np.float32)
    x = [rng.standard_normal((B, C, Z, H, W), dtype=np.float32) for _ in range(N)]
    b = rng.standard_normal((N, C)).astype(np.float32)
    h = np.zeros((N, C, Z, H, W), np.float32)
    h[0, :, 0, 0, 0] = 1.0
    h[1, :, 200, 5, 251] = 1.0
    y = host(hy.hyena_fftconv3d_gate_forward_circular(dev(v, "bf16"), [dev(xx, "bf16") for xx in x], dev(b),
                                                      hy.hyena_filter_rfft3d_circular(dev(h))))
    v64, x64, b64 = as_io(v, "bf16"), [as_io(xx, "bf16") for xx in x], b.astype(np.float64)
    z1 = x64[0] * v64 * (1 + b64[0])[None, :, None, None, None]
    ref = x64[1] * (np.roll(z1, (200, 5, 251), axis=(2, 3, 4)) + b64[1][None, :, None, None, None] * z1)
    assert_close(y, ref, "bf16", "circular 3-D 256^3 shift filters")


def test_forward_3d_circular_on_padded_volumes_is_the_linear_forward(hy):
    B, C, Z, H, W, N = 1, 2, 16, 16, 16, 2
    v, x, b, h = problem(B, C, (Z, H, W), N, seed=9)
    pad = lambda a: np.pad(a, [(0, 0)] * (a.ndim - 3) + [(0, Z), (0, H), (0, W)])
    yc = host(hy.hyena_fftconv3d_gate_forward_circular(dev(pad(v)), [dev(pad(xx)) for xx in x], dev(b),
                                                       hy.hyena_filter_rfft3d_circular(dev(pad(h)))))
    yl = host(hy.hyena_fftconv3d_gate_forward(dev(v), [dev(xx) for xx in x], dev(b), h=dev(h)))
    assert_close(yc[..., :Z, :H, :W], yl, "f32", "circular on padded volumes")
    outside = yc.copy()
    outside[..., :Z, :H, :W] = 0.0
    assert np.max(np.abs(outside)) == 0.0


# ------------------------------------- per-sample spectra (input-dependent)

@pytest.mark.parametrize("B,C,H,W,N,io", [(2, 3, 32, 64, 2, "f32"), (3, 2, 16, 128, 1, "bf16")])
def test_forward_2d_circular_per_sample_matches_oracle(hy, B, C, H, W, N, io):
    v, x, b, _ = problem(B, C, (H, W), N, seed=300 + H)
    rng = np.random.default_rng(301 + W)
    h = np.stack([decaying(rng, (N, C, H, W)) for _ in range(B)])                # [B][N][C][H][W]
    Hs = hy.hyena_filter_rfft2d_circular(dev(h.reshape(B * N, C, H, W))).reshape(B, N, C, H, W // 2)
    y = host(hy.hyena_fftconv2d_gate_forward_circular_per_sample(dev(v, io), [dev(xx, io) for xx in x], dev(b),
                                                                 Hs))
    ref = oracle.hyena_forward_circular_nd_per_sample(as_io(v, io), np.stack([as_io(xx, io) for xx in x]),
                                                      h.astype(np.float64), b.astype(np.float64))
    assert_close(y, ref, io, f"circular 2-D per-sample B{B} C{C} {H}x{W} N{N} {io}")


@pytest.mark.parametrize("B,C,Z,H,W,N,io", [(2, 2, 16, 16, 32, 2, "f32"), (2, 1, 16, 32, 64, 1, "bf16")])
def test_forward_3d_circular_per_sample_matches_oracle(hy, B, C, Z, H, W, N, io):
    v, x, b, _ = problem(B, C, (Z, H, W), N, seed=400 + Z + W)
    rng = np.random.default_rng(401 + H)
    h = np.stack([decaying(rng, (N, C, Z, H, W)) for _ in range(B)])             # [B][N][C][Z][H][W]
    Hs = hy.hyena_filter_rfft3d_circular(dev(h.reshape(B * N, C, Z, H, W))).reshape(B, N, C, Z, H, W // 2)
    y = host(hy.hyena_fftconv3d_gate_forward_circular_per_sample(dev(v, io), [dev(xx, io) for xx in x], dev(b),
                                                                 Hs))
    ref = oracle.hyena_forward_circular_nd_per_sample(as_io(v, io), np.stack([as_io(xx, io) for xx in x]),
                                                      h.astype(np.float64), b.astype(np.float64))
    assert_close(y, ref, io, f"circular 3-D per-sample B{B} C{C} {Z}x{H}x{W} N{N} {io}")


# ------------------------------------------------- circular 3-D backward

def gpu_backward_3d_circular(hy, v, x, b, h, dy, io, per_sample=False):
    if per_sample:
        B, N, C = h.shape[:3]
        Hs = hy.hyena_filter_rfft3d_circular(dev(h.reshape((B * N,) + h.shape[2:])))
        Hs = Hs.view((B, N) + tuple(Hs.shape[1:]))
        fn = hy.hyena_fftconv3d_gate_backward_circular_per_sample
    else:
        Hs = hy.hyena_filter_rfft3d_circular(dev(h))
        fn = hy.hyena_fftconv3d_gate_backward_circular
    dv, dxs, dh, db = fn(dev(v, io), [dev(xx, io) for xx in x], dev(b), Hs, dev(dy, io))
    torch.cuda.synchronize()
    return host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)


@pytest.mark.parametrize("B,C,Z,H,W,N,io", [
    (1, 2, 16, 16, 32, 2, "f32"), (2, 1, 32, 16, 64, 1, "f32"), (2, 2, 16, 32, 32, 2, "bf16"),
    (1, 1, 64, 16, 32, 3, "f32"), (2, 2, 16, 256, 64, 1, "f32"), (1, 1, 256, 16, 32, 1, "f32"),
    (1, 1, 16, 16, 256, 2, "bf16"), (1, 1, 256, 256, 32, 1, "f32"),
])
def test_backward_3d_circular_matches_oracle(hy, B, C, Z, H, W, N, io):
    v, x, b, h = problem(B, C, (Z, H, W), N, seed=Z + 2 * H + 5 * W + N)
    dy = np.random.default_rng(Z * W).standard_normal(v.shape).astype(np.float32)
    got = gpu_backward_3d_circular(hy, v, x, b, h, dy, io)
    ref = oracle.hyena_backward_circular_3d(as_io(v, io), np.stack([as_io(xx, io) for xx in x]),
                                            h.astype(np.float64), b.astype(np.float64), as_io(dy, io))
    check_backward(got, ref, io, f"circular 3-D backward B{B} C{C} {Z}x{H}x{W} N{N} {io}")


def test_backward_3d_circular_channel_across_two_waves(hy):
    """64 x 64 x 256 volumes (4 MB of scratch each, 16 a wave): 18 volumes
    of 6 channels put channel 5 across the two waves; the oracle on it."""
    B, C, Z, H, W, N = 3, 6, 64, 64, 256, 1
    v, x, b, h = problem(B, C, (Z, H, W), N, seed=66)
    dy = np.random.default_rng(67).standard_normal(v.shape).astype(np.float32)
    dv, dx, dh, db = gpu_backward_3d_circular(hy, v, x, b, h, dy, "f32")
    c = 5
    sl = slice(c, c + 1)
    ref = oracle.hyena_backward_circular_3d(v[:, sl], np.stack([xx[:, sl] for xx in x]), h[:, sl], b[:, sl],
                                            dy[:, sl])
    check_backward((dv[:, sl], dx[:, :, sl], dh[:, sl], db[:, sl]), ref, "f32", "circular 3-D split channel")


@pytest.mark.parametrize("B,C,Z,H,W,N,io", [(2, 2, 16, 16, 32, 2, "f32"), (3, 1, 16, 32, 32, 1, "bf16")])
def test_backward_3d_circular_per_sample_matches_oracle(hy, B, C, Z, H, W, N, io):
    v, x, b, _ = problem(B, C, (Z, H, W), N, seed=40 + Z + W)
    rng = np.random.default_rng(Z + H + W)
    h = np.stack([decaying(rng, (N, C, Z, H, W)) for _ in range(B)])        # [B][N][C][Z][H][W]
    dy = rng.standard_normal(v.shape).astype(np.float32)
    got = gpu_backward_3d_circular(hy, v, x, b, h, dy, io, per_sample=True)
    parts = [oracle.hyena_backward_circular_3d(as_io(v[i:i + 1], io), np.stack([as_io(xx[i:i + 1], io) for xx in x]),
                                               h[i].astype(np.float64), b.astype(np.float64), as_io(dy[i:i + 1], io))
             for i in range(B)]
    ref = (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts], axis=1),
           np.stack([p[2] for p in parts]), np.sum([p[3] for p in parts], axis=0))
    check_backward(got, ref, io, f"circular 3-D per-sample backward B{B} C{C} {Z}x{H}x{W} N{N} {io}")


def test_backward_3d_circular_shift_filter_closed_form(hy):
    # N = 1, h = delta at (k, l, m), b = 0: y = x roll(v, (k, l, m)), so
    # dv = roll(dy x, -(k, l, m)), dx = dy roll(v, (k, l, m)) and
    # dh[s] = sum over the batch of dy x roll(v, s)
    B, C, Z, H, W = 2, 2, 16, 16, 32
    v, x, _, _ = problem(B, C, (Z, H, W), 1, seed=88)
    k = (3, 5, 7)
    h = np.zeros((1, C, Z, H, W), np.float32)
    h[0, :, k[0], k[1], k[2]] = 1.0
    b = np.zeros((1, C), np.float32)
    dy = np.random.default_rng(89).standard_normal(v.shape).astype(np.float32)
    dv, dx, dh, db = gpu_backward_3d_circular(hy, v, x, b, h, dy, "f32")
    e = dy.astype(np.float64) * x[0]
    axes = (2, 3, 4)
    assert_close(dv, np.roll(e, tuple(-s for s in k), axis=axes), "f32", "shift dv")
    assert_close(dx[0], dy * np.roll(v.astype(np.float64), k, axis=axes), "f32", "shift dx")
    for s in [(0, 0, 0), k, (15, 1, 31), (8, 8, 16)]:
        want = np.sum(e * np.roll(v.astype(np.float64), s, axis=axes), axis=(0, 2, 3, 4))
        got = dh[0][:, s[0], s[1], s[2]]
        assert np.max(np.abs(got - want)) <= 1e-4 * np.max(np.abs(dh)), s
    assert np.max(np.abs(db[0] - dh[0][:, 0, 0, 0])) <= 1e-5 * np.max(np.abs(dh))
