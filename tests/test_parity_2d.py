"""GPU parity of the 2-D path against the float64 oracle (run with -m gpu).

Tolerances as for 1-D: 1e-4 (float32 activations) and 2e-2 (bf16) of the
oracle's maximum |y|; spectra at 2e-5 of their maximum.
"""
import numpy as np
import pytest
import torch

import oracle
from subquadratic_sequence_b200 import synth
from tests.gpu_helpers import assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def unpack_spectrum_2d(P: np.ndarray) -> np.ndarray:
    """Packed [..., 2H, W] -> natural bins [..., 2H, W+1]."""
    H2, W = P.shape[-2:]
    out = np.empty(P.shape[:-1] + (W + 1,), dtype=np.complex128)
    out[..., 1:W] = P[..., 1:]
    F = P[..., 0]
    Fr = np.conj(np.roll(F[..., ::-1], 1, axis=-1))        # conj F[-ky]
    out[..., 0] = 0.5 * (F + Fr)
    out[..., W] = (F - Fr) / 2j
    return out


def problem_2d(B, C, H, W, N, seed, io="f32"):
    wl = synth.Workload("case2d", "2d", N=N, B=B, D=C, H=H, W=W, io=io, seed=seed)
    inp = synth.make_inputs(wl)
    h = oracle.filter_gen_2d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"], inp["alpha"], N, C, H, W)
    return wl, inp, h.astype(np.float32)


def gpu_forward_2d(hy, inp, h32, io, use_h=False):
    v = dev(inp["v"], io)
    xs = [dev(x, io) for x in inp["x"]]
    b = dev(inp["b"])
    if use_h:
        y = hy.hyena_fftconv2d_gate_forward(v, xs, b, h=dev(h32))
    else:
        y = hy.hyena_fftconv2d_gate_forward(v, xs, b, Hs=hy.hyena_filter_rfft2d(dev(h32)))
    torch.cuda.synchronize()
    return host(y)


def oracle_forward_2d(inp, h, imgs=None):
    v = inp["v"].astype(np.float64)
    x = np.stack(inp["x"]).astype(np.float64)
    b = inp["b"].astype(np.float64)
    if imgs is None:
        return oracle.hyena_forward_2d(v, x, h, b, route="fft")
    return np.stack([oracle.hyena_forward_2d(v[bi:bi + 1, ci:ci + 1], x[:, bi:bi + 1, ci:ci + 1],
                                             h[:, ci:ci + 1], b[:, ci:ci + 1], route="fft")[0, 0]
                     for (bi, ci) in imgs])


@pytest.mark.parametrize("H,W", [(16, 16), (16, 64), (32, 16), (64, 128), (256, 256), (1024, 32)])
def test_rfft2d_matches_oracle(hy, H, W):
    rng = np.random.default_rng(H * 7 + W)
    h = (rng.standard_normal((2, 3, H, W)) * np.exp(-np.arange(W) / (W / 3))
         * np.exp(-np.arange(H) / (H / 5))[:, None]).astype(np.float32)
    got = unpack_spectrum_2d(hy.hyena_filter_rfft2d(dev(h)).cpu().numpy().astype(np.complex128))
    ref = oracle.rfft2_pad2(h.astype(np.float64))
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) <= 2e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("B,C,H,W,N,io", [
    (1, 2, 16, 16, 2, "f32"), (2, 3, 32, 64, 2, "f32"), (1, 2, 64, 32, 3, "f32"),
    (2, 2, 16, 128, 1, "bf16"), (1, 1, 128, 16, 2, "f32"), (3, 1, 32, 32, 2, "bf16"),
    (1, 2, 256, 256, 2, "f32"),
])
def test_forward_2d_matches_oracle(hy, B, C, H, W, N, io):
    wl, inp, h32 = problem_2d(B, C, H, W, N, seed=H + W + N, io=io)
    got = gpu_forward_2d(hy, inp, h32, io)
    ref = oracle_forward_2d(inp, h32.astype(np.float64))
    assert_close(got, ref, io, f"2-D B{B} C{C} {H}x{W} N{N} {io}")


def test_forward_2d_shift_filters(hy):
    # h_1 = delta at (0, 0), h_2 = delta at (1, 2): closed form
    B, C, H, W, N = 2, 2, 16, 32, 2
    wl, inp, _ = problem_2d(B, C, H, W, N, seed=3)
    h = np.zeros((N, C, H, W), np.float32); h[0, :, 0, 0] = 1.0; h[1, :, 1, 2] = 1.0
    got = gpu_forward_2d(hy, inp, h, "f32")
    v, x, b = inp["v"].astype(np.float64), [xx.astype(np.float64) for xx in inp["x"]], inp["b"]
    z1 = x[0] * v * (1 + b[0])[None, :, None, None]
    sh = np.zeros_like(z1); sh[..., 1:, 2:] = z1[..., :-1, :-2]
    ref = x[1] * (sh + b[1][None, :, None, None] * z1)
    assert_close(got, ref, "f32", "2-D shift filters")


def test_forward_2d_from_filters_equals_from_spectrum(hy):
    wl, inp, h32 = problem_2d(1, 3, 32, 64, 2, seed=4)
    assert np.array_equal(gpu_forward_2d(hy, inp, h32, "f32", use_h=False),
                          gpu_forward_2d(hy, inp, h32, "f32", use_h=True))


def test_c4_full_size_sampled(hy):
    """Order-2, B=2, C=128, 256x256, fp32: the whole workload on the GPU
    (2-D filter generation, packed spectra, forward); the oracle on 4
    sampled images, their filters generated for just those channels."""
    wl = synth.WORKLOADS["c4"]
    inp = synth.make_inputs(wl)
    h = hy.hyena_filter_gen_2d(dev(inp["W1"]), dev(inp["W2"]), dev(inp["W3"]), dev(inp["Wout"]),
                               dev(inp["alpha"]), wl.N, wl.D, wl.H, wl.W)
    Hs = hy.hyena_filter_rfft2d(h)
    y = hy.hyena_fftconv2d_gate_forward(dev(inp["v"]), [dev(x) for x in inp["x"]], dev(inp["b"]), Hs=Hs)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    imgs = [(int(rng.integers(wl.B)), int(rng.integers(wl.D))) for _ in range(2)] + [(0, 0), (1, 127)]
    got = np.stack([y[bi, ci].cpu().numpy() for (bi, ci) in imgs]).astype(np.float64)
    refs = []
    for (bi, ci) in imgs:
        rows = [n * wl.D + ci for n in range(wl.N)]
        hc = oracle.filter_gen_2d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["alpha"][[ci]],
                                  wl.N, 1, wl.H, wl.W)
        v = inp["v"][bi:bi + 1, ci:ci + 1].astype(np.float64)
        x = np.stack([xx[bi:bi + 1, ci:ci + 1] for xx in inp["x"]]).astype(np.float64)
        refs.append(oracle.hyena_forward_2d(v, x, hc, inp["b"][:, ci:ci + 1].astype(np.float64))[0, 0])
    assert_close(got, np.stack(refs), "f32", "c4")
