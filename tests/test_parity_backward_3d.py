"""GPU parity of the 3-D backward pass against the float64 oracle (-m gpu).

The oracle's 3-D backward (oracle_hyena_backward_3d) is pinned to finite
differences of its 3-D forward, to agreement of its direct and FFT routes,
to the 2-D backward on one-plane volumes and to an axis permutation
(tests/test_oracle_backward_pins.py).  Tolerances as for 1-D and 2-D: dv and
dx_n 1e-4 of the maximum for float32 storage, 2e-2 for bf16; dh and dbias,
accumulated in float32, 1e-4 of their maximum.
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


def decaying(rng, shape):
    """Seeded random filters [..., Z, H, W] decaying along every axis."""
    Z, H, W = shape[-3:]
    h = rng.standard_normal(shape)
    h *= np.exp(-np.arange(Z) / (Z / 4))[:, None, None]
    h *= np.exp(-np.arange(H) / (H / 4))[:, None]
    h *= np.exp(-np.arange(W) / (W / 4))
    return (h * 8 / np.sqrt(Z * H * W)).astype(np.float32)


def problem(B, C, Z, H, W, N, seed, io):
    wl = synth.Workload("bwd3d", "3d", N=N, B=B, D=C, Z=Z, H=H, W=W, io=io, seed=seed)
    inp = synth.make_inputs(wl)
    h = decaying(np.random.default_rng(seed + 7), (N, C, Z, H, W))
    return inp, h, synth.make_output_grad(wl)


def run(hy, inp, h, dy, io):
    Hs = hy.hyena_filter_rfft3d(dev(h))
    dv, dxs, dh, db = hy.hyena_fftconv3d_gate_backward(
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


def channel_ref(inp, h, dy, c):
    """The oracle's backward of channel c alone (the channels are independent)."""
    sl = slice(c, c + 1)
    return oracle.hyena_backward_3d(inp["v"][:, sl], np.stack([x[:, sl] for x in inp["x"]]), h[:, sl],
                                    inp["b"][:, sl], dy[:, sl])


CASES = [
    (1, 2, 16, 16, 16, 2, "f32"), (2, 1, 16, 32, 64, 2, "f32"), (1, 2, 32, 16, 16, 3, "f32"),
    (2, 2, 16, 16, 32, 1, "bf16"), (1, 1, 64, 16, 16, 2, "f32"), (1, 1, 16, 64, 16, 2, "bf16"),
    (2, 1, 16, 16, 128, 1, "f32"), (1, 1, 16, 16, 16, 16, "f32"),
    # the longest axes (256: 512-point z, column and row transforms)
    (1, 1, 256, 16, 16, 1, "f32"), (1, 1, 16, 256, 16, 1, "f32"), (1, 1, 16, 16, 256, 2, "bf16"),
]


@pytest.mark.parametrize("B,C,Z,H,W,N,io", CASES)
def test_backward_3d_matches_oracle(hy, B, C, Z, H, W, N, io):
    inp, h, dy = problem(B, C, Z, H, W, N, seed=900 + Z + 3 * H + 7 * W + N, io=io)
    got = run(hy, inp, h, dy, io)
    ref = oracle.hyena_backward_3d(inp["v"], np.stack(inp["x"]), h, inp["b"], dy)
    check(got, ref, io, f"3-D B{B} C{C} {Z}x{H}x{W} N{N} {io}")


def test_backward_3d_channel_across_two_waves(hy):
    """16 x 256 x 64 volumes, 16 a wave: the 18 volumes of 6 channels put
    channel 5 (volumes 15, 16, 17) across the two waves, so its dh spectrum
    is accumulated by two launches; the oracle on that channel."""
    B, C, Z, H, W, N = 3, 6, 16, 256, 64, 1
    inp, h, dy = problem(B, C, Z, H, W, N, seed=41, io="f32")
    dv, dx, dh, db = run(hy, inp, h, dy, "f32")
    c = 5
    sl = slice(c, c + 1)
    check((dv[:, sl], dx[:, :, sl], dh[:, sl], db[:, sl]), channel_ref(inp, h, dy, c), "f32", "split channel")


def test_backward_3d_c5_3d_full_size_sampled(hy):
    """The c5_3d shape (B 2, C 32, 64^3, order 2, bf16): the whole backward
    on the GPU, the oracle on two channels (both samples each)."""
    wl = synth.WORKLOADS["c5_3d"]
    inp, h, dy = problem(wl.B, wl.D, wl.Z, wl.H, wl.W, wl.N, seed=wl.seed, io=wl.io)
    dv, dx, dh, db = run(hy, inp, h, dy, wl.io)
    for c in (0, 31):
        sl = slice(c, c + 1)
        check((dv[:, sl], dx[:, :, sl], dh[:, sl], db[:, sl]), channel_ref(inp, h, dy, c), wl.io,
              f"c5_3d channel {c}")


def test_backward_3d_is_deterministic(hy):
    inp, h, dy = problem(2, 2, 16, 32, 32, 2, seed=9, io="f32")
    a, b = run(hy, inp, h, dy, "f32"), run(hy, inp, h, dy, "f32")
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_3d_delta_filter_closed_form(hy):
    # N = 1, h = delta at the origin: y = x (1 + b) v, so dv = dy x (1 + b),
    # dx = dy (1 + b) v, db = sum dy x v and dh[a][p][q] = sum e[t][s][u]
    # v[t-a][s-p][u-q] over the batch (e = dy x)
    B, C, Z, H, W = 2, 2, 16, 16, 32
    inp, _, dy = problem(B, C, Z, H, W, 1, seed=10, io="f32")
    h = np.zeros((1, C, Z, H, W), np.float32)
    h[0, :, 0, 0, 0] = 1.0
    dv, dx, dh, db = run(hy, inp, h, dy, "f32")
    v, x, b = inp["v"].astype(np.float64), inp["x"][0].astype(np.float64), inp["b"].astype(np.float64)
    g = (1 + b[0])[None, :, None, None, None]
    assert_close(dv, dy * x * g, "f32", "delta dv")
    assert_close(dx[0], dy * g * v, "f32", "delta dx")
    e = dy * x
    assert rel_max_err(db[0], np.sum(e * v, axis=(0, 2, 3, 4))) <= 1e-4
    want = np.zeros((C, Z, H, W))
    for a in range(Z):
        for p in range(H):
            for q in range(W):
                want[:, a, p, q] = np.sum(e[:, :, a:, p:, q:] * v[:, :, :Z - a, :H - p, :W - q], axis=(0, 2, 3, 4))
    assert rel_max_err(dh[0], want) <= 1e-4


# ------------------------------------------------- per-sample filters

def run_per_sample(hy, inp, h, dy, io):
    B, N, C, Z, H, W = h.shape
    Hs = hy.hyena_filter_rfft3d(dev(h.reshape(B * N, C, Z, H, W))).reshape(B, N, C, 2 * Z, 2 * H, W)
    dv, dxs, dh, db = hy.hyena_fftconv3d_gate_backward_per_sample(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), Hs, dev(dy, io))
    torch.cuda.synchronize()
    return host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)


@pytest.mark.parametrize("B,C,Z,H,W,N,io", [(2, 2, 16, 16, 16, 2, "f32"), (3, 1, 16, 32, 16, 1, "bf16"),
                                            (2, 1, 32, 16, 32, 3, "f32")])
def test_backward_3d_per_sample_matches_oracle(hy, B, C, Z, H, W, N, io):
    inp, _, dy = problem(B, C, Z, H, W, N, seed=70 + Z + H, io=io)
    h = decaying(np.random.default_rng(Z + W), (B, N, C, Z, H, W))
    got = run_per_sample(hy, inp, h, dy, io)
    v, x = inp["v"], np.stack(inp["x"])
    parts = [oracle.hyena_backward_3d(v[i:i + 1], x[:, i:i + 1], h[i], inp["b"], dy[i:i + 1]) for i in range(B)]
    ref = (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts], axis=1),
           np.stack([p[2] for p in parts]), np.sum([p[3] for p in parts], axis=0))
    check(got, ref, io, f"3-D per-sample B{B} C{C} {Z}x{H}x{W} N{N} {io}")


def test_backward_3d_per_sample_with_equal_sets_is_the_shared_backward(hy):
    B, C, Z, H, W, N = 3, 2, 16, 32, 16, 2
    inp, h, dy = problem(B, C, Z, H, W, N, seed=77, io="f32")
    Hs = hy.hyena_filter_rfft3d(dev(h))
    v, xs, b, g = dev(inp["v"]), [dev(x) for x in inp["x"]], dev(inp["b"]), dev(dy)
    dv, dxs, dh, db = hy.hyena_fftconv3d_gate_backward(v, xs, b, Hs, g)
    pv, pxs, ph, pb = hy.hyena_fftconv3d_gate_backward_per_sample(
        v, xs, b, Hs.unsqueeze(0).expand(B, *Hs.shape).contiguous(), g)
    torch.cuda.synchronize()
    assert torch.equal(dv, pv) and all(torch.equal(a, c) for a, c in zip(dxs, pxs))
    assert rel_max_err(host(ph).sum(axis=0), host(dh)) <= 1e-5
    assert rel_max_err(host(pb), host(db)) <= 1e-5
