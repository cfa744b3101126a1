"""Pins of the oracle's input-dependent filters (FiLM-modulated sine layers,
per-unit frequencies, Gaussian window) and of its per-sample forward.

Each test ties the oracle to something outside the routine under test: the
separately pinned shared-filter generator and forward, or an identity of the
sine (sin(x + pi) = -sin(x), sin(c * x / c) = sin(x)) that fails if FiLM
modulates the wrong layer, the wrong side of the product, or a sample's
filters leak into another sample's.
"""
import numpy as np
import pytest

import oracle

W, N, D, L = 64, 2, 3, 48


def net(seed=0):
    r = np.random.default_rng(seed)
    return dict(W1=r.standard_normal((W, 17)) / np.sqrt(17), W2=r.standard_normal((W, W)) / 8,
                W3=r.standard_normal((W, W)) / 8, Wout=r.standard_normal((N * D, W)) / 8)


def film(n, omega, gamma, beta, window, gaussian=False):
    return oracle.filter_gen_film(n["W1"], n["W2"], n["W3"], n["Wout"], omega, gamma, beta, window,
                                  gaussian, N, D, L)


ALPHA = np.linspace(0.3, 1.5, D)


def test_identity_modulation_is_the_shared_filter():
    n = net()
    B = 3
    h = film(n, np.ones((3, W)), np.ones((B, 3, W)), np.zeros((B, 3, W)), ALPHA)
    ref = oracle.filter_gen(n["W1"], n["W2"], n["W3"], n["Wout"], ALPHA, N, D, L)
    for b in range(B):
        assert np.array_equal(h[b], ref)


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_gamma_scales_the_pre_activation_of_its_layer(layer):
    # gamma_l = c is the same as W_l scaled by c
    n = net(1)
    c = 1.7
    g = np.ones((1, 3, W))
    g[0, layer] = c
    a = film(n, np.ones((3, W)), g, np.zeros((1, 3, W)), ALPHA)
    n2 = dict(n)
    key = ("W1", "W2", "W3")[layer]
    n2[key] = n[key] * c
    b = film(n2, np.ones((3, W)), np.ones((1, 3, W)), np.zeros((1, 3, W)), ALPHA)
    assert np.max(np.abs(a - b)) < 1e-12 * np.max(np.abs(b))


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_beta_pi_flips_the_sign_of_the_filter(layer):
    # sin(x + pi) = -sin(x), and every later layer is odd in its input
    n = net(2)
    be = np.zeros((1, 3, W))
    be[0, layer] = np.pi
    a = film(n, np.ones((3, W)), np.ones((1, 3, W)), be, ALPHA)
    b = film(n, np.ones((3, W)), np.ones((1, 3, W)), np.zeros((1, 3, W)), ALPHA)
    assert np.max(np.abs(a + b)) < 1e-12 * np.max(np.abs(b))


def test_omega_and_gamma_cancel():
    # sin(c * (x / c)) = sin(x), per unit
    n = net(3)
    om = np.random.default_rng(4).uniform(0.5, 3.0, (3, W))
    a = film(n, om, 1.0 / om[None], np.zeros((1, 3, W)), ALPHA)
    b = film(n, np.ones((3, W)), np.ones((1, 3, W)), np.zeros((1, 3, W)), ALPHA)
    assert np.max(np.abs(a - b)) < 1e-12 * np.max(np.abs(b))


def test_gaussian_window_ratio():
    # the two windows differ only in the window: the ratio of the filters is
    # exp(-t^2 / (2 sigma^2)) / exp(-alpha t L / 64) at every position
    n = net(5)
    sigma = np.array([0.1, 0.25, 0.6])
    r = np.random.default_rng(6)
    g, be = r.uniform(0.5, 1.5, (1, 3, W)), r.normal(0, 0.3, (1, 3, W))
    hg = film(n, np.ones((3, W)), g, be, sigma, gaussian=True)
    he = film(n, np.ones((3, W)), g, be, ALPHA)
    t = np.arange(L) / L
    want = np.exp(-t[None, :] ** 2 / (2 * sigma[:, None] ** 2)) / np.exp(-ALPHA[:, None] * t[None, :] * L / 64.0)
    np.testing.assert_allclose(hg[0], he[0] * want[None], rtol=1e-12, atol=1e-300)


def test_samples_do_not_mix():
    n = net(7)
    r = np.random.default_rng(8)
    g, be = r.uniform(0.5, 1.5, (3, 3, W)), r.normal(0, 0.3, (3, 3, W))
    h = film(n, np.ones((3, W)), g, be, ALPHA)
    perm = [2, 0, 1]
    hp = film(n, np.ones((3, W)), g[perm], be[perm], ALPHA)
    assert np.array_equal(hp, h[perm])
    assert np.max(np.abs(h[0] - h[1])) > 1e-3


def test_per_sample_forward_with_shared_filters_is_the_forward():
    r = np.random.default_rng(9)
    B = 3
    v, x = r.standard_normal((B, D, L)), r.standard_normal((N, B, D, L))
    h, bias = r.standard_normal((N, D, L)) * 0.3, r.standard_normal((N, D))
    hp = np.broadcast_to(h, (B, N, D, L))
    assert np.array_equal(oracle.hyena_forward_per_sample(v, x, hp, bias), oracle.hyena_forward(v, x, h, bias))


# ------------------------------------------------------------------ 2-D

H2, W2 = 12, 10


def film2(n, omega, gamma, beta, window, gaussian=False):
    return oracle.filter_gen_film_2d(n["W1"], n["W2"], n["W3"], n["Wout"], omega, gamma, beta, window,
                                     gaussian, N, D, H2, W2)


def net2(seed=0):
    r = np.random.default_rng(seed)
    return dict(W1=r.standard_normal((W, 34)) / np.sqrt(34), W2=r.standard_normal((W, W)) / 8,
                W3=r.standard_normal((W, W)) / 8, Wout=r.standard_normal((N * D, W)) / 8)


def test_2d_identity_modulation_is_the_shared_filter():
    n = net2()
    B = 2
    h = film2(n, np.ones((3, W)), np.ones((B, 3, W)), np.zeros((B, 3, W)), ALPHA)
    ref = oracle.filter_gen_2d(n["W1"], n["W2"], n["W3"], n["Wout"], ALPHA, N, D, H2, W2)
    for b in range(B):
        assert np.array_equal(h[b], ref)


@pytest.mark.parametrize("layer", [0, 2])
def test_2d_beta_pi_flips_the_sign(layer):
    n = net2(1)
    be = np.zeros((1, 3, W))
    be[0, layer] = np.pi
    a = film2(n, np.ones((3, W)), np.ones((1, 3, W)), be, ALPHA)
    b = film2(n, np.ones((3, W)), np.ones((1, 3, W)), np.zeros((1, 3, W)), ALPHA)
    assert np.max(np.abs(a + b)) < 1e-12 * np.max(np.abs(b))


def test_2d_gaussian_window_ratio():
    n = net2(2)
    sigma = np.array([0.1, 0.3, 0.7])
    r = np.random.default_rng(3)
    g, be = r.uniform(0.5, 1.5, (1, 3, W)), r.normal(0, 0.3, (1, 3, W))
    hg = film2(n, np.ones((3, W)), g, be, sigma, gaussian=True)
    he = film2(n, np.ones((3, W)), g, be, ALPHA)
    ty = (np.arange(H2) / H2)[:, None]
    tx = (np.arange(W2) / W2)[None, :]
    gauss = np.exp(-(ty ** 2 + tx ** 2)[None] / (2 * sigma[:, None, None] ** 2))
    expo = np.exp(-ALPHA[:, None, None] * (np.arange(H2)[:, None] + np.arange(W2)[None, :])[None] / 64.0)
    np.testing.assert_allclose(hg[0], he[0] * (gauss / expo)[None], rtol=1e-12, atol=1e-300)


def test_2d_per_sample_forward_with_shared_filters_is_the_forward():
    r = np.random.default_rng(9)
    B = 2
    v, x = r.standard_normal((B, D, 8, 8)), r.standard_normal((N, B, D, 8, 8))
    h, bias = r.standard_normal((N, D, 8, 8)) * 0.3, r.standard_normal((N, D))
    hp = np.broadcast_to(h, (B, N, D, 8, 8))
    assert np.array_equal(oracle.hyena_forward_2d_per_sample(v, x, hp, bias), oracle.hyena_forward_2d(v, x, h, bias))


# ------------------------------------------------------------------ 3-D

Z3, H3, W3_ = 4, 6, 8


def film3(n, omega, gamma, beta, window, gaussian=False):
    return oracle.filter_gen_film_3d(n["W1"], n["W2"], n["W3"], n["Wout"], omega, gamma, beta, window,
                                     gaussian, N, D, Z3, H3, W3_, n_bands=4)


def net3(seed=0):
    r = np.random.default_rng(seed)
    n_in = 3 + 6 * 4
    return dict(W1=r.standard_normal((W, n_in)) / np.sqrt(n_in), W2=r.standard_normal((W, W)) / 8,
                W3=r.standard_normal((W, W)) / 8, Wout=r.standard_normal((N * D, W)) / 8)


def test_3d_identity_modulation_is_the_shared_filter():
    n = net3()
    B = 2
    h = film3(n, np.ones((3, W)), np.ones((B, 3, W)), np.zeros((B, 3, W)), ALPHA)
    ref = oracle.filter_gen_3d(n["W1"], n["W2"], n["W3"], n["Wout"], ALPHA, N, D, Z3, H3, W3_, n_bands=4)
    for b in range(B):
        assert np.array_equal(h[b], ref)


@pytest.mark.parametrize("layer", [0, 1])
def test_3d_beta_pi_flips_the_sign(layer):
    n = net3(1)
    be = np.zeros((1, 3, W))
    be[0, layer] = np.pi
    a = film3(n, np.ones((3, W)), np.ones((1, 3, W)), be, ALPHA)
    b = film3(n, np.ones((3, W)), np.ones((1, 3, W)), np.zeros((1, 3, W)), ALPHA)
    assert np.max(np.abs(a + b)) < 1e-12 * np.max(np.abs(b))


def test_3d_gaussian_window_ratio():
    n = net3(2)
    sigma = np.array([0.1, 0.3, 0.7])
    r = np.random.default_rng(4)
    g, be = r.uniform(0.5, 1.5, (1, 3, W)), r.normal(0, 0.3, (1, 3, W))
    hg = film3(n, np.ones((3, W)), g, be, sigma, gaussian=True)
    he = film3(n, np.ones((3, W)), g, be, ALPHA)
    iz, iy, ix = np.meshgrid(np.arange(Z3), np.arange(H3), np.arange(W3_), indexing="ij")
    t2 = (iz / Z3) ** 2 + (iy / H3) ** 2 + (ix / W3_) ** 2
    gauss = np.exp(-t2[None] / (2 * sigma[:, None, None, None] ** 2))
    expo = np.exp(-ALPHA[:, None, None, None] * (iz + iy + ix)[None] / 64.0)
    np.testing.assert_allclose(hg[0], he[0] * (gauss / expo)[None], rtol=1e-12, atol=1e-300)


def test_3d_samples_do_not_mix():
    n = net3(3)
    r = np.random.default_rng(5)
    g, be = r.uniform(0.5, 1.5, (3, 3, W)), r.normal(0, 0.3, (3, 3, W))
    om = r.uniform(0.5, 2.0, (3, W))
    h = film3(n, om, g, be, ALPHA)
    for b in range(3):
        assert np.array_equal(h[b], film3(n, om, g[b:b + 1], be[b:b + 1], ALPHA)[0])


def test_3d_per_sample_forward_with_shared_filters_is_the_forward():
    r = np.random.default_rng(10)
    B = 2
    v, x = r.standard_normal((B, D, 4, 4, 8)), r.standard_normal((N, B, D, 4, 4, 8))
    h, bias = r.standard_normal((N, D, 4, 4, 8)) * 0.3, r.standard_normal((N, D))
    hp = np.broadcast_to(h, (B, N, D, 4, 4, 8))
    assert np.array_equal(oracle.hyena_forward_3d_per_sample(v, x, hp, bias), oracle.hyena_forward_3d(v, x, h, bias))
