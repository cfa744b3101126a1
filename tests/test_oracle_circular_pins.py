"""Pins of the oracle's circular mode (convolution of length L without
padding; "Native Multi-Dimensional Subquadratic Operators via Input
Dependent Long Convolutions", Handling Boundaries).

Against numpy's FFT (a library routine), np.roll (the closed form of a
shift filter), and the separately pinned causal oracle: the circular
recurrence on sequences zero-padded to 2L is the causal recurrence.
"""
import numpy as np
import pytest

import oracle


def rel_err(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(np.max(np.abs(b)), 1e-300))


@pytest.mark.parametrize("L", [1, 2, 5, 16, 64])
def test_cconv_direct_is_numpy(L):
    r = np.random.default_rng(L)
    h, u = r.standard_normal(L), r.standard_normal(L)
    ref = np.real(np.fft.ifft(np.fft.fft(h) * np.fft.fft(u)))
    assert rel_err(oracle.cconv(h, u, "direct"), ref) < 1e-12


@pytest.mark.parametrize("L", [2, 16, 1024])
def test_cconv_fft_equals_direct(L):
    r = np.random.default_rng(L + 1)
    h, u = r.standard_normal(L), r.standard_normal(L)
    assert rel_err(oracle.cconv(h, u, "fft"), oracle.cconv(h, u, "direct")) < 1e-12


@pytest.mark.parametrize("k", [0, 1, 7, 15])
def test_cconv_shift_filter_is_a_rotation(k):
    L = 16
    u = np.random.default_rng(k).standard_normal(L)
    h = np.zeros(L)
    h[k] = 1.0
    assert np.array_equal(oracle.cconv(h, u, "direct"), np.roll(u, k))


def test_rfft_circ_is_numpy():
    h = np.random.default_rng(3).standard_normal((3, 64))
    assert rel_err(oracle.rfft_circ(h), np.fft.rfft(h)) < 1e-13


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_circular_on_padded_sequences_is_the_causal_recurrence(route):
    # zero-padded to 2L (filters and inputs), the circular recurrence's first
    # L outputs are the causal recurrence's
    r = np.random.default_rng(4)
    B, D, L, N = 2, 3, 32, 3
    v, x = r.standard_normal((B, D, L)), r.standard_normal((N, B, D, L))
    h, b = r.standard_normal((N, D, L)), r.standard_normal((N, D))
    pad = lambda a: np.concatenate([a, np.zeros_like(a)], axis=-1)
    yc = oracle.hyena_forward_circular(pad(v), pad(x), pad(h), b, route=route)
    assert rel_err(yc[..., :L], oracle.hyena_forward(v, x, h, b, route="direct")) < 1e-12
    assert np.max(np.abs(yc[..., L:])) == 0.0


def test_circular_forward_routes_agree_and_wrap():
    r = np.random.default_rng(5)
    B, D, L, N = 2, 2, 64, 2
    v, x = r.standard_normal((B, D, L)), r.standard_normal((N, B, D, L))
    h, b = r.standard_normal((N, D, L)), r.standard_normal((N, D))
    yd = oracle.hyena_forward_circular(v, x, h, b, route="direct")
    yf = oracle.hyena_forward_circular(v, x, h, b, route="fft")
    assert rel_err(yf, yd) < 1e-12
    # and it differs from the causal one (the wrap-around terms)
    assert rel_err(yd, oracle.hyena_forward(v, x, h, b, route="direct")) > 1e-3


# ------------------------------------------------------- 2-D grids and 3-D volumes

@pytest.mark.parametrize("shape", [(1, 1, 5), (1, 6, 4), (3, 4, 5), (4, 8, 8)])
def test_cconv3_direct_is_numpy(shape):
    r = np.random.default_rng(sum(shape))
    h, u = r.standard_normal(shape), r.standard_normal(shape)
    ref = np.real(np.fft.ifftn(np.fft.fftn(h) * np.fft.fftn(u)))
    assert rel_err(oracle.cconv3(h, u, "direct"), ref) < 1e-12


@pytest.mark.parametrize("shape", [(1, 16, 32), (8, 4, 16), (16, 16, 16)])
def test_cconv3_fft_equals_direct(shape):
    r = np.random.default_rng(sum(shape) + 1)
    h, u = r.standard_normal(shape), r.standard_normal(shape)
    assert rel_err(oracle.cconv3(h, u, "fft"), oracle.cconv3(h, u, "direct")) < 1e-12


@pytest.mark.parametrize("k", [(0, 0, 0), (0, 3, 5), (2, 0, 7), (3, 7, 1)])
def test_cconv3_shift_filter_is_a_rotation(k):
    shape = (4, 8, 8)
    u = np.random.default_rng(sum(k)).standard_normal(shape)
    h = np.zeros(shape)
    h[k] = 1.0
    assert np.array_equal(oracle.cconv3(h, u, "direct"), np.roll(u, k, axis=(0, 1, 2)))


def test_cconv3_of_a_line_is_the_1d_circular_convolution():
    r = np.random.default_rng(9)
    h, u = r.standard_normal(32), r.standard_normal(32)
    got = oracle.cconv3(h.reshape(1, 1, 32), u.reshape(1, 1, 32), "fft")[0, 0]
    assert rel_err(got, oracle.cconv(h, u, "direct")) < 1e-12


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_circular_nd_on_padded_volumes_is_the_linear_recurrence(route):
    # inputs in the low octant of a grid of twice the size and x zero
    # outside it: the circular recurrence there is the linear 3-D one
    # (pinned to scipy), and zero elsewhere
    B, C, Z, H, W, N = 1, 2, 4, 4, 8, 2
    r = np.random.default_rng(10)
    v, x = r.standard_normal((B, C, Z, H, W)), r.standard_normal((N, B, C, Z, H, W))
    h, b = r.standard_normal((N, C, Z, H, W)), r.standard_normal((N, C))
    pad = lambda a: np.pad(a, [(0, 0)] * (a.ndim - 3) + [(0, Z), (0, H), (0, W)])
    got = oracle.hyena_forward_circular_nd(pad(v), pad(x), pad(h), b, route=route)
    want = oracle.hyena_forward_3d(v, x, h, b, route="direct")
    assert rel_err(got[..., :Z, :H, :W], want) < 1e-12
    outside = got.copy()
    outside[..., :Z, :H, :W] = 0.0
    assert np.max(np.abs(outside)) == 0.0


def test_circular_nd_2d_grid_of_one_row_is_the_1d_circular_recurrence():
    B, C, W, N = 2, 3, 32, 3
    r = np.random.default_rng(11)
    v, x = r.standard_normal((B, C, W)), r.standard_normal((N, B, C, W))
    h, b = r.standard_normal((N, C, W)), r.standard_normal((N, C))
    got = oracle.hyena_forward_circular_nd(v[:, :, None], x[:, :, :, None], h[:, :, None], b)[:, :, 0]
    assert rel_err(got, oracle.hyena_forward_circular(v, x, h, b, route="direct")) < 1e-12


def test_circular_nd_routes_agree_and_differ_from_linear():
    B, C, H, W, N = 1, 2, 16, 16, 2
    r = np.random.default_rng(12)
    v, x = r.standard_normal((B, C, H, W)), r.standard_normal((N, B, C, H, W))
    h, b = r.standard_normal((N, C, H, W)), r.standard_normal((N, C))
    a = oracle.hyena_forward_circular_nd(v, x, h, b, route="fft")
    d = oracle.hyena_forward_circular_nd(v, x, h, b, route="direct")
    assert rel_err(a, d) < 1e-12
    assert rel_err(a, oracle.hyena_forward_2d(v, x, h, b, route="direct")) > 1e-2


def test_circular_per_sample_forward_is_each_sample_with_its_filters():
    # equal sets give the shared circular forward; each sample's output is
    # that sample alone through its own filters (1-D, 2-D and 3-D)
    r = np.random.default_rng(70)
    B, N, D, L = 3, 2, 2, 16
    v, x = r.standard_normal((B, D, L)), r.standard_normal((N, B, D, L))
    h, bias = r.standard_normal((B, N, D, L)) * 0.3, r.standard_normal((N, D))
    shared = oracle.hyena_forward_circular(v, x, h[0], bias)
    assert np.array_equal(oracle.hyena_forward_circular_per_sample(v, x, np.broadcast_to(h[0], h.shape), bias),
                          shared)
    ps = oracle.hyena_forward_circular_per_sample(v, x, h, bias)
    for b in range(B):
        assert np.array_equal(ps[b], oracle.hyena_forward_circular(v[b:b + 1], x[:, b:b + 1], h[b], bias)[0])
    for grid in ((4, 8), (2, 4, 8)):
        v, x = r.standard_normal((B, D) + grid), r.standard_normal((N, B, D) + grid)
        h = r.standard_normal((B, N, D) + grid) * 0.3
        ps = oracle.hyena_forward_circular_nd_per_sample(v, x, h, bias)
        for b in range(B):
            assert np.array_equal(ps[b], oracle.hyena_forward_circular_nd(v[b:b + 1], x[:, b:b + 1], h[b], bias)[0])
