"""GPU parity of the 2-D backward pass against the float64 oracle (-m gpu).

The oracle's 2-D backward is pinned to finite differences of its 2-D
forward, to the 1-D adjoint on one-row grids and to transposition
(tests/test_oracle_backward_pins.py).  Tolerances as for 1-D: dv and dx_n
1e-4 of the maximum for float32 storage, 2e-2 for bf16; dh and dbias,
accumulated in float32 from float32 intermediates, 1e-4 of their maximum.
"""
import numpy as np
import pytest
import torch

import oracle
from subquadratic_sequence_b200 import synth
from tests.gpu_helpers import assert_close, dev, host, rel_max_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def problem(B, C, H, W, N, seed, io):
    wl = synth.Workload("bwd2d", "2d", N=N, B=B, D=C, H=H, W=W, io=io, seed=seed)
    inp = synth.make_inputs(wl)
    r = np.random.default_rng(seed + 7)
    decay = np.exp(-np.arange(H) / (H / 4))[:, None] * np.exp(-np.arange(W) / (W / 4))
    h = (r.standard_normal((N, C, H, W)) * decay * 8 / np.sqrt(H * W)).astype(np.float32)
    return wl, inp, h, synth.make_output_grad(wl)


def run(hy, wl, inp, h, dy):
    io = wl.io
    Hs = hy.hyena_filter_rfft2d(dev(h))
    dv, dxs, dh, db = hy.hyena_fftconv2d_gate_backward(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), Hs, dev(dy, io))
    torch.cuda.synchronize()
    return host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)


def check(got, ref, io, name):
    dv, dx, dh, db = got
    rdv, rdx, rdh, rdb = ref
    assert_close(dv, rdv, io, f"{name} dv")
    assert_close(dx, rdx, io, f"{name} dx")
    assert rel_max_err(dh, rdh) <= 1e-4, f"{name} dh {rel_max_err(dh, rdh):.3e}"
    assert rel_max_err(db, rdb) <= 1e-4, f"{name} db {rel_max_err(db, rdb):.3e}"


CASES = [
    (1, 2, 16, 16, 1, "f32"), (2, 3, 32, 64, 2, "f32"), (2, 2, 64, 32, 3, "f32"), (3, 2, 16, 128, 2, "bf16"),
    (1, 1, 256, 256, 2, "f32"), (2, 1, 1024, 16, 2, "f32"), (1, 2, 16, 1024, 1, "f32"),
    (2, 2, 32, 32, 16, "f32"),
    (3, 12, 512, 512, 1, "f32"),     # 36 images, 32 a wave: channel 10 spans two waves
]


@pytest.mark.parametrize("B,C,H,W,N,io", CASES)
def test_backward_2d_matches_oracle(hy, B, C, H, W, N, io):
    wl, inp, h, dy = problem(B, C, H, W, N, seed=500 + H + W + N, io=io)
    got = run(hy, wl, inp, h, dy)
    ref = oracle.hyena_backward_2d(inp["v"], np.stack(inp["x"]), h, inp["b"], dy)
    check(got, ref, io, f"B{B} C{C} {H}x{W} N{N} {io}")


def test_backward_2d_c4_full_size_sampled(hy):
    """Order-2, B=2, C=128, 256x256, fp32: the whole backward on the GPU;
    the oracle on 3 sampled channels (both batch elements each)."""
    wl, inp, h, dy = problem(2, 128, 256, 256, 2, seed=4, io="f32")
    dv, dx, dh, db = run(hy, wl, inp, h, dy)
    for c in (0, 77, 127):
        sl = slice(c, c + 1)
        ref = oracle.hyena_backward_2d(inp["v"][:, sl], np.stack([x[:, sl] for x in inp["x"]]), h[:, sl],
                                       inp["b"][:, sl], dy[:, sl])
        check((dv[:, sl], dx[:, :, sl], dh[:, sl], db[:, sl]), ref, "f32", f"c4 channel {c}")


def test_backward_2d_is_deterministic(hy):
    wl, inp, h, dy = problem(2, 3, 64, 64, 2, seed=9, io="f32")
    a, b = run(hy, wl, inp, h, dy), run(hy, wl, inp, h, dy)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_2d_delta_filter_closed_form(hy):
    # N = 1, h = delta at (0, 0): y = x (1 + b) v, so dv = dy x (1 + b),
    # dx = dy (1 + b) v, db = sum dy x v, dh[a][c] = sum_b sum dy x v(shifted)
    wl, inp, _, dy = problem(2, 2, 16, 32, 1, seed=10, io="f32")
    h = np.zeros((1, 2, 16, 32), np.float32)
    h[0, :, 0, 0] = 1.0
    dv, dx, dh, db = run(hy, wl, inp, h, dy)
    v, x, b = inp["v"].astype(np.float64), inp["x"][0].astype(np.float64), inp["b"].astype(np.float64)
    assert_close(dv, dy * x * (1 + b[0])[None, :, None, None], "f32", "delta dv")
    assert_close(dx[0], dy * (1 + b[0])[None, :, None, None] * v, "f32", "delta dx")
    e = dy * x
    want_db = np.sum(e * v, axis=(0, 2, 3))
    assert rel_max_err(db[0], want_db) <= 1e-4
    want_dh = np.zeros((2, 16, 32))
    for a in range(16):
        for c in range(32):
            want_dh[:, a, c] = np.sum(e[:, :, a:, c:] * v[:, :, :16 - a, :32 - c], axis=(0, 2, 3))
    assert rel_max_err(dh[0], want_dh) <= 1e-4


# ------------------------------------------------- per-sample filters

@pytest.mark.parametrize("B,C,H,W,N,io", [(2, 3, 32, 64, 2, "f32"), (3, 2, 16, 128, 2, "bf16"),
                                          (1, 2, 16, 16, 1, "f32"),
                                          (3, 12, 512, 512, 1, "f32")])   # a channel across two waves
def test_backward_2d_per_sample_matches_oracle(hy, B, C, H, W, N, io):
    wl, inp, _, dy = problem(B, C, H, W, N, seed=60 + H, io=io)
    r = np.random.default_rng(H + W)
    decay = np.exp(-np.arange(H) / (H / 4))[:, None] * np.exp(-np.arange(W) / (W / 4))
    h = (r.standard_normal((B, N, C, H, W)) * decay * 8 / np.sqrt(H * W)).astype(np.float32)
    Hs = hy.hyena_filter_rfft2d(dev(h.reshape(B * N, C, H, W))).reshape(B, N, C, 2 * H, W)
    dv, dxs, dh, db = hy.hyena_fftconv2d_gate_backward_per_sample(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), Hs, dev(dy, io))
    torch.cuda.synchronize()
    got = host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)
    ref = oracle.hyena_backward_2d_per_sample(inp["v"], np.stack(inp["x"]), h, inp["b"], dy)
    check(got, ref, io, f"2-D per-sample B{B} C{C} {H}x{W} N{N} {io}")


def test_backward_2d_per_sample_with_equal_sets_is_the_shared_backward(hy):
    B, C, H, W, N = 3, 4, 64, 64, 2
    wl, inp, h, dy = problem(B, C, H, W, N, seed=77, io="f32")
    Hs = hy.hyena_filter_rfft2d(dev(h))
    v, xs, b, g = dev(inp["v"]), [dev(x) for x in inp["x"]], dev(inp["b"]), dev(dy)
    dv, dxs, dh, db = hy.hyena_fftconv2d_gate_backward(v, xs, b, Hs, g)
    pv, pxs, ph, pb = hy.hyena_fftconv2d_gate_backward_per_sample(
        v, xs, b, Hs.unsqueeze(0).expand(B, -1, -1, -1, -1).contiguous(), g)
    torch.cuda.synchronize()
    assert torch.equal(dv, pv) and all(torch.equal(a, c) for a, c in zip(dxs, pxs))
    assert rel_max_err(host(ph).sum(axis=0), host(dh)) <= 1e-5
    assert rel_max_err(host(pb), host(db)) <= 1e-5
