"""Pins of the oracle's backward pass (the exact adjoint of the recurrence).

The pages give no training formulas; the gradient of the forward is fixed by
calculus.  Each test checks ``oracle.hyena_backward`` against something it
does not share code with: central finite differences of the (separately
pinned) oracle forward, a closed form for a delta filter written out with
numpy, and identities of the definitions.  A wrong sign, a transposed lag
(t - s vs s - t) or a dropped bias term fails at least one of them.
"""
import numpy as np
import pytest

import oracle


def problem(B, D, L, N, seed):
    r = np.random.default_rng(seed)
    v = r.standard_normal((B, D, L))
    x = r.standard_normal((N, B, D, L))
    h = r.standard_normal((N, D, L)) * np.exp(-np.arange(L) / 4.0)
    b = r.standard_normal((N, D))
    dy = r.standard_normal((B, D, L))
    return v, x, h, b, dy


def rel_err(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(np.max(np.abs(b)), 1e-300))


@pytest.mark.parametrize("N", [1, 2, 3])
def test_backward_matches_finite_differences(N):
    # loss = sum(dy * y); every gradient against a central difference of the
    # oracle forward (direct route), step 1e-6: truncation ~1e-12, rounding ~1e-10
    v, x, h, b, dy = problem(2, 2, 7, N, seed=N)
    dv, dx, dh, db = oracle.hyena_backward(v, x, h, b, dy, route="direct")

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_backward_delta_filter_closed_form(route):
    # N = 1, h = delta_0: y = x (1 + b) v, so
    # dv = dy x (1+b), dx = dy (1+b) v, db = sum_b sum_t dy x v,
    # dh[s] = sum_b sum_t dy[t] x[t] v[t - s]
    B, D, L = 3, 2, 12
    v, x, _, b, dy = problem(B, D, L, 1, seed=11)
    h = np.zeros((1, D, L))
    h[:, :, 0] = 1.0
    dv, dx, dh, db = oracle.hyena_backward(v, x, h, b, dy, route=route)
    gain = (1.0 + b[0])[None, :, None]
    assert rel_err(dv, dy * x[0] * gain) < 1e-13
    assert rel_err(dx[0], dy * gain * v) < 1e-13
    assert rel_err(db[0], np.sum(dy * x[0] * v, axis=(0, 2))) < 1e-13
    want = np.zeros((D, L))
    e = dy * x[0]
    for s in range(L):
        want[:, s] = np.sum(e[:, :, s:] * v[:, :, :L - s], axis=(0, 2))
    assert rel_err(dh[0], want) < 1e-13


def test_backward_routes_agree():
    v, x, h, b, dy = problem(2, 3, 100, 3, seed=5)
    a = oracle.hyena_backward(v, x, h, b, dy, route="direct")
    f = oracle.hyena_backward(v, x, h, b, dy, route="fft")
    for ga, gf in zip(a, f):
        assert rel_err(gf, ga) < 1e-12


def test_backward_bias_gradient_is_the_lag0_filter_gradient():
    # db_n[d] and dh_n[d][0] are the same sum over (b, t) of dL/dc_n z_{n-1}
    v, x, h, b, dy = problem(2, 4, 64, 2, seed=6)
    _, _, dh, db = oracle.hyena_backward(v, x, h, b, dy)
    assert rel_err(db, dh[:, :, 0]) < 1e-13


def test_backward_linear_in_dy_and_threads_agree():
    v, x, h, b, dy = problem(2, 3, 32, 2, seed=7)
    g1 = oracle.hyena_backward(v, x, h, b, dy, threads=1)
    g2 = oracle.hyena_backward(v, x, h, b, 2.5 * dy, threads=3)
    for a, c in zip(g1, g2):
        assert rel_err(c, 2.5 * a) < 1e-13


# ------------------------------------------------------------------ 2-D

def problem_2d(B, C, H, W, N, seed):
    r = np.random.default_rng(seed)
    v = r.standard_normal((B, C, H, W))
    x = r.standard_normal((N, B, C, H, W))
    h = r.standard_normal((N, C, H, W)) * np.exp(-np.arange(H) / 3.0)[:, None] * np.exp(-np.arange(W) / 3.0)
    b = r.standard_normal((N, C))
    dy = r.standard_normal((B, C, H, W))
    return v, x, h, b, dy


@pytest.mark.parametrize("N", [1, 2])
def test_backward_2d_matches_finite_differences(N):
    # loss = sum(dy * y) through the separately pinned 2-D oracle forward
    v, x, h, b, dy = problem_2d(2, 2, 3, 4, N, seed=20 + N)
    dv, dx, dh, db = oracle.hyena_backward_2d(v, x, h, b, dy, route="direct")

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward_2d(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


def test_backward_2d_of_one_row_is_the_1d_backward():
    # a 1 x W grid is a sequence: every gradient equals the pinned 1-D adjoint
    B, C, W, N = 2, 3, 16, 3
    v, x, h, b, dy = problem(B, C, W, N, seed=30)
    got = oracle.hyena_backward_2d(v[:, :, None], x[:, :, :, None], h[:, :, None], b, dy[:, :, None], route="fft")
    want = oracle.hyena_backward(v, x, h, b, dy, route="direct")
    for g_, w_, name in zip(got, want, ("dv", "dx", "dh", "db")):
        assert rel_err(np.squeeze(g_, axis=-2) if g_.ndim > 2 else g_, w_) < 1e-12, name


def test_backward_2d_transposed_grid_transposes_every_gradient():
    # the 2-D convolution commutes with transposing both operands: the
    # gradients of the transposed problem are the transposed gradients
    v, x, h, b, dy = problem_2d(1, 2, 4, 8, 2, seed=31)
    t = lambda a: np.swapaxes(a, -1, -2).copy()
    got = oracle.hyena_backward_2d(t(v), t(x), t(h), b, t(dy), route="fft")
    want = oracle.hyena_backward_2d(v, x, h, b, dy, route="direct")
    for g_, w_, name in zip(got, want, ("dv", "dx", "dh")):
        assert rel_err(g_, t(w_)) < 1e-12, name
    assert rel_err(got[3], want[3]) < 1e-12


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_backward_2d_routes_agree_and_db_is_dh_origin(route):
    v, x, h, b, dy = problem_2d(2, 3, 8, 16, 2, seed=32)
    got = oracle.hyena_backward_2d(v, x, h, b, dy, route=route)
    ref = oracle.hyena_backward_2d(v, x, h, b, dy, route="direct")
    for g_, w_ in zip(got, ref):
        assert rel_err(g_, w_) < 1e-12
    assert rel_err(got[3], got[2][:, :, 0, 0]) < 1e-12


# ------------------------------------------------- per-sample filters

def test_backward_per_sample_matches_finite_differences():
    # a filter set per sample: every gradient against a central difference
    # of the per-sample oracle forward; dh must be per sample (a sum over
    # the batch, or another sample's filters, fails), dbias summed
    B, D, L, N = 3, 2, 6, 2
    r = np.random.default_rng(21)
    v, x = r.standard_normal((B, D, L)), r.standard_normal((N, B, D, L))
    h = r.standard_normal((B, N, D, L)) * np.exp(-np.arange(L) / 4.0)
    b, dy = r.standard_normal((N, D)), r.standard_normal((B, D, L))
    dv, dx, dh, db = oracle.hyena_backward_per_sample(v, x, h, b, dy, route="direct")
    assert dh.shape == h.shape and db.shape == b.shape

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward_per_sample(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


def test_backward_per_sample_with_equal_sets_sums_to_the_shared_backward():
    B, D, L, N = 3, 4, 32, 2
    v, x, h, b, dy = problem(B, D, L, N, seed=22)
    dv, dx, dh, db = oracle.hyena_backward(v, x, h, b, dy)
    pv, px, ph, pb = oracle.hyena_backward_per_sample(v, x, np.broadcast_to(h, (B,) + h.shape), b, dy)
    assert rel_err(pv, dv) < 1e-13 and rel_err(px, dx) < 1e-13
    assert rel_err(ph.sum(axis=0), dh) < 1e-12 and rel_err(pb, db) < 1e-12
    # and each sample's dh is that sample's own shared-filter backward
    for s in range(B):
        one = oracle.hyena_backward(v[s:s + 1], x[:, s:s + 1], h, b, dy[s:s + 1])
        assert rel_err(ph[s], one[2]) < 1e-13


# ------------------------------------------------- circular convolution

@pytest.mark.parametrize("N", [1, 2])
def test_backward_circular_matches_finite_differences(N):
    v, x, h, b, dy = problem(2, 2, 8, N, seed=30 + N)
    dv, dx, dh, db = oracle.hyena_backward_circular(v, x, h, b, dy, route="direct")

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward_circular(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


def test_backward_circular_routes_agree_and_db_is_dh_lag0():
    v, x, h, b, dy = problem(3, 4, 64, 3, seed=33)
    d = oracle.hyena_backward_circular(v, x, h, b, dy, route="direct")
    f = oracle.hyena_backward_circular(v, x, h, b, dy, route="fft")
    for a, c in zip(d, f):
        assert rel_err(c, a) < 1e-12
    assert rel_err(d[3], d[2][:, :, 0]) < 1e-13


def test_backward_circular_on_zero_padded_sequences_is_the_causal_backward():
    # length 2L with v, x_n, dy and h_n zero beyond L: no product wraps
    # around, so every gradient's first L entries are the causal ones
    B, D, L, N = 2, 3, 16, 2
    v, x, h, b, dy = problem(B, D, L, N, seed=34)
    pad = lambda a: np.concatenate([a, np.zeros_like(a)], axis=-1)
    dv, dx, dh, db = oracle.hyena_backward_circular(pad(v), pad(x), pad(h), b, pad(dy))
    rv, rx, rh, rb = oracle.hyena_backward(v, x, h, b, dy)
    assert rel_err(dv[..., :L], rv) < 1e-12 and rel_err(dx[..., :L], rx) < 1e-12
    assert rel_err(dh[..., :L], rh) < 1e-12 and rel_err(db, rb) < 1e-12


def test_backward_2d_per_sample_matches_finite_differences():
    B, C, H, W, N = 2, 2, 3, 4, 2
    r = np.random.default_rng(40)
    v, x = r.standard_normal((B, C, H, W)), r.standard_normal((N, B, C, H, W))
    h = r.standard_normal((B, N, C, H, W)) * 0.5
    b, dy = r.standard_normal((N, C)), r.standard_normal((B, C, H, W))
    dv, dx, dh, db = oracle.hyena_backward_2d_per_sample(v, x, h, b, dy, route="direct")
    assert dh.shape == h.shape and db.shape == b.shape

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward_2d_per_sample(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


def test_backward_2d_per_sample_with_equal_sets_sums_to_the_shared_backward():
    B, C, H, W, N = 3, 2, 8, 16, 2
    r = np.random.default_rng(41)
    v, x = r.standard_normal((B, C, H, W)), r.standard_normal((N, B, C, H, W))
    h, b, dy = r.standard_normal((N, C, H, W)) * 0.3, r.standard_normal((N, C)), r.standard_normal((B, C, H, W))
    dv, dx, dh, db = oracle.hyena_backward_2d(v, x, h, b, dy)
    pv, px, ph, pb = oracle.hyena_backward_2d_per_sample(v, x, np.broadcast_to(h, (B,) + h.shape), b, dy)
    assert rel_err(pv, dv) < 1e-13 and rel_err(px, dx) < 1e-13
    assert rel_err(ph.sum(axis=0), dh) < 1e-12 and rel_err(pb, db) < 1e-12


# ------------------------------------------------- circular 2-D

@pytest.mark.parametrize("N", [1, 2])
def test_backward_circular_2d_matches_finite_differences(N):
    v, x, h, b, dy = problem_2d(2, 2, 4, 4, N, seed=50 + N)
    dv, dx, dh, db = oracle.hyena_backward_circular_2d(v, x, h, b, dy, route="direct")

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward_circular_nd(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


def test_backward_circular_2d_routes_agree_and_db_is_dh_origin():
    v, x, h, b, dy = problem_2d(2, 3, 16, 8, 2, seed=53)
    d = oracle.hyena_backward_circular_2d(v, x, h, b, dy, route="direct")
    f = oracle.hyena_backward_circular_2d(v, x, h, b, dy, route="fft")
    for a, c in zip(d, f):
        assert rel_err(c, a) < 1e-12
    assert rel_err(d[3], d[2][:, :, 0, 0]) < 1e-13


def test_backward_circular_2d_on_zero_padded_grids_is_the_linear_backward():
    # 2H x 2W grids with v, x_n, dy and h_n zero outside [0, H) x [0, W):
    # nothing wraps, so the gradients there are the linear 2-D backward's
    B, C, H, W, N = 2, 2, 4, 8, 2
    v, x, h, b, dy = problem_2d(B, C, H, W, N, seed=54)

    def pad(a):
        out = np.zeros(a.shape[:-2] + (2 * H, 2 * W))
        out[..., :H, :W] = a
        return out
    dv, dx, dh, db = oracle.hyena_backward_circular_2d(pad(v), pad(x), pad(h), b, pad(dy))
    rv, rx, rh, rb = oracle.hyena_backward_2d(v, x, h, b, dy)
    assert rel_err(dv[..., :H, :W], rv) < 1e-12 and rel_err(dx[..., :H, :W], rx) < 1e-12
    assert rel_err(dh[..., :H, :W], rh) < 1e-12 and rel_err(db, rb) < 1e-12


def test_backward_circular_2d_of_one_row_is_the_circular_1d_backward():
    # H = 1: the 2-D circular recurrence is the 1-D one along the row
    B, C, W, N = 2, 3, 16, 2
    v, x, h, b, dy = problem(B, C, W, N, seed=55)
    g2 = oracle.hyena_backward_circular_2d(v[:, :, None], x[:, :, :, None], h[:, :, None], b, dy[:, :, None])
    g1 = oracle.hyena_backward_circular(v, x, h, b, dy)
    for a, c in zip(g2[:3], g1[:3]):
        assert rel_err(a[..., 0, :], c) < 1e-12
    assert rel_err(g2[3], g1[3]) < 1e-12


# ------------------------------------------------- 3-D

def problem_3d(B, C, Z, H, W, N, seed):
    r = np.random.default_rng(seed)
    env = (np.exp(-np.arange(Z) / 3.0)[:, None, None] * np.exp(-np.arange(H) / 3.0)[:, None]
           * np.exp(-np.arange(W) / 3.0))
    return (r.standard_normal((B, C, Z, H, W)), r.standard_normal((N, B, C, Z, H, W)),
            r.standard_normal((N, C, Z, H, W)) * env, r.standard_normal((N, C)),
            r.standard_normal((B, C, Z, H, W)))


@pytest.mark.parametrize("N", [1, 2])
def test_backward_3d_matches_finite_differences(N):
    v, x, h, b, dy = problem_3d(2, 2, 2, 3, 3, N, seed=60 + N)
    dv, dx, dh, db = oracle.hyena_backward_3d(v, x, h, b, dy, route="direct")

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward_3d(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


def test_backward_3d_routes_agree_and_db_is_dh_origin():
    v, x, h, b, dy = problem_3d(2, 2, 4, 4, 8, 2, seed=63)
    d = oracle.hyena_backward_3d(v, x, h, b, dy, route="direct")
    f = oracle.hyena_backward_3d(v, x, h, b, dy, route="fft")
    for a, c in zip(d, f):
        assert rel_err(c, a) < 1e-12
    assert rel_err(d[3], d[2][:, :, 0, 0, 0]) < 1e-13


def test_backward_3d_of_one_plane_is_the_2d_backward():
    v, x, h, b, dy = problem_3d(2, 3, 1, 8, 4, 2, seed=64)
    g3 = oracle.hyena_backward_3d(v, x, h, b, dy)
    g2 = oracle.hyena_backward_2d(v[:, :, 0], x[:, :, :, 0], h[:, :, 0], b, dy[:, :, 0])
    for a, c in zip(g3[:3], g2[:3]):
        assert rel_err(a[..., 0, :, :], c) < 1e-12
    assert rel_err(g3[3], g2[3]) < 1e-12


def test_backward_3d_axis_permutation_permutes_every_gradient():
    v, x, h, b, dy = problem_3d(1, 2, 2, 4, 8, 2, seed=65)
    perm = lambda a: np.swapaxes(a, -1, -3)                 # z <-> x
    g = oracle.hyena_backward_3d(v, x, h, b, dy)
    gp = oracle.hyena_backward_3d(perm(v), perm(x), perm(h), b, perm(dy))
    for a, c in zip(g[:3], gp[:3]):
        assert rel_err(perm(c), a) < 1e-12
    assert rel_err(gp[3], g[3]) < 1e-12


# ------------------------------------------------- circular 3-D

@pytest.mark.parametrize("N", [1, 2])
def test_backward_circular_3d_matches_finite_differences(N):
    v, x, h, b, dy = problem_3d(2, 2, 2, 3, 3, N, seed=90 + N)
    dv, dx, dh, db = oracle.hyena_backward_circular_3d(v, x, h, b, dy, route="direct")

    def loss(v_, x_, h_, b_):
        return float(np.sum(dy * oracle.hyena_forward_circular_nd(v_, x_, h_, b_, route="direct")))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name


def test_backward_circular_3d_routes_agree_and_db_is_dh_origin():
    v, x, h, b, dy = problem_3d(2, 2, 4, 4, 8, 2, seed=93)
    d = oracle.hyena_backward_circular_3d(v, x, h, b, dy, route="direct")
    f = oracle.hyena_backward_circular_3d(v, x, h, b, dy, route="fft")
    for a, c in zip(d, f):
        assert rel_err(c, a) < 1e-12
    assert rel_err(d[3], d[2][:, :, 0, 0, 0]) < 1e-13


def test_backward_circular_3d_on_zero_padded_volumes_is_the_linear_backward():
    # 2Z x 2H x 2W volumes with v, x_n, dy and h_n zero outside the Z x H x W
    # corner: nothing wraps, so the gradients there are the linear 3-D backward's
    B, C, Z, H, W, N = 2, 2, 2, 4, 4, 2
    v, x, h, b, dy = problem_3d(B, C, Z, H, W, N, seed=94)

    def pad(a):
        out = np.zeros(a.shape[:-3] + (2 * Z, 2 * H, 2 * W))
        out[..., :Z, :H, :W] = a
        return out
    dv, dx, dh, db = oracle.hyena_backward_circular_3d(pad(v), pad(x), pad(h), b, pad(dy))
    rv, rx, rh, rb = oracle.hyena_backward_3d(v, x, h, b, dy)
    assert rel_err(dv[..., :Z, :H, :W], rv) < 1e-12 and rel_err(dx[..., :Z, :H, :W], rx) < 1e-12
    assert rel_err(dh[..., :Z, :H, :W], rh) < 1e-12 and rel_err(db, rb) < 1e-12


def test_backward_circular_3d_of_one_plane_is_the_circular_2d_backward():
    v, x, h, b, dy = problem_3d(2, 3, 1, 8, 4, 2, seed=95)
    g3 = oracle.hyena_backward_circular_3d(v, x, h, b, dy)
    g2 = oracle.hyena_backward_circular_2d(v[:, :, 0], x[:, :, :, 0], h[:, :, 0], b, dy[:, :, 0])
    for a, c in zip(g3[:3], g2[:3]):
        assert rel_err(a[..., 0, :, :], c) < 1e-12
    assert rel_err(g3[3], g2[3]) < 1e-12


def test_backward_circular_per_sample_matches_finite_differences():
    B, D, L, N = 2, 2, 8, 2
    r = np.random.default_rng(80)
    v, x = r.standard_normal((B, D, L)), r.standard_normal((N, B, D, L))
    h = r.standard_normal((B, N, D, L)) * np.exp(-np.arange(L) / 4.0)
    b, dy = r.standard_normal((N, D)), r.standard_normal((B, D, L))
    dv, dx, dh, db = oracle.hyena_backward_circular_per_sample(v, x, h, b, dy, route="direct")

    def loss(v_, x_, h_, b_):
        y = np.concatenate([oracle.hyena_forward_circular(v_[s:s + 1], x_[:, s:s + 1], h_[s], b_, route="direct")
                            for s in range(B)])
        return float(np.sum(dy * y))

    eps = 1e-6
    for arr, grad, name in ((v, dv, "v"), (x, dx, "x"), (h, dh, "h"), (b, db, "bias")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss(v, x, h, b)
            arr[idx] = orig - eps
            lm = loss(v, x, h, b)
            arr[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        assert rel_err(grad, fd) < 1e-7, name
