"""Pins of the float64 oracle to facts outside itself.

Each test checks the oracle against something it does not share code with:
numpy/scipy library routines (``numpy.fft``, ``numpy.convolve``,
``scipy.signal.convolve2d``), closed forms (DFT of a delta, a constant, a
geometric sequence; the IIR form of a geometric filter; shift filters),
invariants (Parseval, linearity, causality) and hand-worked values in
``tests/golden``.  They are chosen so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""
import os

import numpy as np
import pytest
import scipy.signal

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


def rel_err(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# --------------------------------------------------------------------- FFT

@pytest.mark.parametrize("n", [1, 2, 4, 8, 32, 256, 4096])
def test_fft_matches_numpy(n):
    r = rng(n)
    x = r.standard_normal(n) + 1j * r.standard_normal(n)
    assert rel_err(oracle.fft(x, -1), np.fft.fft(x)) < 1e-13
    assert rel_err(oracle.fft(x, +1), np.fft.ifft(x) * n) < 1e-13


@pytest.mark.parametrize("P", [8, 64, 1024])
def test_fft_closed_forms(P):
    j = np.arange(P)
    # delta at k: X[j] = exp(-2 pi i j k / P)
    for k in (0, 1, 3, P // 2, P - 1):
        x = np.zeros(P, complex); x[k] = 1.0
        # the angle is reduced exactly (j k mod P) so the reference itself is exact
        assert np.max(np.abs(oracle.fft(x) - np.exp(-2j * np.pi * ((j * k) % P) / P))) < 1e-13
    # constant: P * delta_0
    X = oracle.fft(np.ones(P))
    assert abs(X[0] - P) < 1e-12 * P and np.max(np.abs(X[1:])) < 1e-12 * P
    # zero-padded geometric a^i, i < L = P/2:
    #   X[j] = (1 - (a w^j)^L) / (1 - a w^j),  w = exp(-2 pi i / P)
    L, a = P // 2, 0.9
    x = np.zeros(P); x[:L] = a ** np.arange(L)
    q = a * np.exp(-2j * np.pi * j / P)
    assert rel_err(oracle.fft(x), (1 - q ** L) / (1 - q)) < 1e-12


def test_fft_parseval_and_roundtrip():
    r = rng(7)
    x = r.standard_normal(2048) + 1j * r.standard_normal(2048)
    X = oracle.fft(x)
    assert abs(np.sum(np.abs(x) ** 2) - np.sum(np.abs(X) ** 2) / x.size) < 1e-10 * np.sum(np.abs(x) ** 2)
    assert rel_err(oracle.fft(X, +1) / x.size, x) < 1e-13


@pytest.mark.parametrize("L", [1, 2, 16, 512, 1024])
def test_rfft_pad2_matches_numpy(L):
    h = rng(L).standard_normal((3, L))
    got = oracle.rfft_pad2(h)
    assert got.shape == (3, L + 1)
    assert rel_err(got, np.fft.rfft(h, n=2 * L, axis=-1)) < 1e-12


@pytest.mark.parametrize("H,W", [(1, 1), (2, 4), (8, 8), (16, 32)])
def test_rfft2_pad2_matches_numpy(H, W):
    h = rng(H * W).standard_normal((2, H, W))
    got = oracle.rfft2_pad2(h)
    assert got.shape == (2, 2 * H, W + 1)
    assert rel_err(got, np.fft.rfft2(h, s=(2 * H, 2 * W))) < 1e-12


# ------------------------------------------------------------ convolution

def _golden(kind):
    rows = []
    with open(os.path.join(GOLDEN, "conv_small.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.strip() for p in line.split("|")]
            if parts[0] == kind:
                rows.append([np.array([float(t) for t in p.split()]) for p in parts[1:]])
    assert rows
    return rows


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_conv_golden(route):
    for h, u, y in _golden("conv"):
        assert np.max(np.abs(oracle.conv(h, u, route) - y)) < 1e-13


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_gate_golden(route):
    for h, b, v, x, y in _golden("gate"):
        got = oracle.hyena_forward(v[None, None], x[None, None, None], h[None, None],
                                   b.reshape(1, 1), route=route)
        assert np.max(np.abs(got[0, 0] - y)) < 1e-13


@pytest.mark.parametrize("L", list(range(1, 17)) + [31, 64])
def test_conv_direct_is_numpy_convolve(L):
    r = rng(100 + L)
    h, u = r.standard_normal(L), r.standard_normal(L)
    ref = np.convolve(h, u)[:L]
    assert np.max(np.abs(oracle.conv(h, u, "direct") - ref)) < 1e-12
    assert np.max(np.abs(oracle.conv(h, u, "fft") - ref)) < 1e-12


@pytest.mark.parametrize("L", [3, 100, 1024, 4096])
def test_conv_fft_equals_direct(L):
    r = rng(200 + L)
    h, u = r.standard_normal(L), r.standard_normal(L)
    assert rel_err(oracle.conv(h, u, "fft"), oracle.conv(h, u, "direct")) < 1e-12


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_conv_geometric_filter_is_iir(route):
    # h[i] = c a^i turns the convolution into y[t] = a y[t-1] + c u[t]
    L, a, c = 4096, 0.999, 0.7
    u = rng(3).standard_normal(L)
    h = c * a ** np.arange(L)
    ref = np.empty(L); acc = 0.0
    for t in range(L):
        acc = a * acc + c * u[t]
        ref[t] = acc
    assert rel_err(oracle.conv(h, u, route), ref) < 1e-11


@pytest.mark.parametrize("route", ["direct", "fft"])
@pytest.mark.parametrize("k", [0, 1, 5, 63])
def test_conv_shift_filter(route, k):
    L = 64
    u = rng(k).standard_normal(L)
    h = np.zeros(L); h[k] = 1.0
    ref = np.zeros(L); ref[k:] = u[:L - k]
    assert np.max(np.abs(oracle.conv(h, u, route) - ref)) < 1e-13


# ------------------------------------------------------- the recurrence

def _rand_problem(B, D, L, N, seed):
    r = rng(seed)
    v = r.standard_normal((B, D, L))
    x = r.standard_normal((N, B, D, L))
    h = r.standard_normal((N, D, L)) * np.exp(-np.arange(L) / 50.0)
    b = r.standard_normal((N, D))
    return v, x, h, b


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_forward_delta_filter_identity(route):
    # h_n = delta_0 makes every convolution the identity:
    #   y = v * prod_n x_n (1 + b_n)
    B, D, L, N = 2, 3, 64, 3
    v, x, _, b = _rand_problem(B, D, L, N, 1)
    h = np.zeros((N, D, L)); h[:, :, 0] = 1.0
    ref = v.copy()
    for n in range(N):
        ref = ref * x[n] * (1.0 + b[n])[None, :, None]
    assert rel_err(oracle.hyena_forward(v, x, h, b, route=route), ref) < 1e-13


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_forward_shift_filters_fix_the_order_of_operations(route):
    # h_1 = delta_1, h_2 = delta_2:
    #   z_1[t] = x_1[t] (v[t-1] + b_1 v[t])
    #   y[t]   = x_2[t] (z_1[t-2] + b_2 z_1[t])
    # A gate applied before the convolution, a bias added after the gate,
    # a swapped x_n or a swapped h_n all break this.
    B, D, L, N = 2, 2, 32, 2
    v, x, _, b = _rand_problem(B, D, L, N, 2)
    h = np.zeros((N, D, L)); h[0, :, 1] = 1.0; h[1, :, 2] = 1.0

    def shift(a, k):
        out = np.zeros_like(a); out[..., k:] = a[..., :a.shape[-1] - k]
        return out

    z1 = x[0] * (shift(v, 1) + b[0][None, :, None] * v)
    ref = x[1] * (shift(z1, 2) + b[1][None, :, None] * z1)
    assert rel_err(oracle.hyena_forward(v, x, h, b, route=route), ref) < 1e-13


def test_forward_routes_agree():
    v, x, h, b = _rand_problem(2, 4, 1024, 2, 3)
    yd = oracle.hyena_forward(v, x, h, b, route="direct")
    yf = oracle.hyena_forward(v, x, h, b, route="fft")
    assert rel_err(yf, yd) < 1e-12


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_forward_linear_in_v(route):
    v, x, h, b = _rand_problem(1, 3, 256, 2, 4)
    v2 = rng(5).standard_normal(v.shape)
    lhs = oracle.hyena_forward(2.0 * v - 3.0 * v2, x, h, b, route=route)
    rhs = 2.0 * oracle.hyena_forward(v, x, h, b, route=route) - 3.0 * oracle.hyena_forward(v2, x, h, b, route=route)
    assert rel_err(lhs, rhs) < 1e-12


def test_forward_causality():
    # perturbing v[t0] and x_n[t0] leaves y[:t0] unchanged: bit-identical on
    # the direct route, at rounding level on the FFT route
    v, x, h, b = _rand_problem(1, 2, 512, 2, 6)
    t0 = 300
    v2, x2 = v.copy(), x.copy()
    v2[..., t0] += 10.0
    x2[..., t0] -= 5.0
    ya = oracle.hyena_forward(v, x, h, b, route="direct")
    yb = oracle.hyena_forward(v2, x2, h, b, route="direct")
    assert np.array_equal(ya[..., :t0], yb[..., :t0])
    assert not np.allclose(ya[..., t0:], yb[..., t0:])
    fa = oracle.hyena_forward(v, x, h, b, route="fft")
    fb = oracle.hyena_forward(v2, x2, h, b, route="fft")
    assert np.max(np.abs(fa[..., :t0] - fb[..., :t0])) < 1e-12 * np.max(np.abs(fa))


def test_forward_threads_do_not_change_results():
    v, x, h, b = _rand_problem(3, 5, 128, 2, 8)
    y1 = oracle.hyena_forward(v, x, h, b, route="fft", threads=1)
    y4 = oracle.hyena_forward(v, x, h, b, route="fft", threads=4)
    assert np.array_equal(y1, y4)


# ------------------------------------------------------------------ 2-D

@pytest.mark.parametrize("H,W", [(1, 1), (3, 5), (8, 8), (7, 16)])
def test_conv2_is_scipy_convolve2d(H, W):
    r = rng(H * 100 + W)
    h, u = r.standard_normal((H, W)), r.standard_normal((H, W))
    ref = scipy.signal.convolve2d(h, u, mode="full")[:H, :W]
    assert np.max(np.abs(oracle.conv2(h, u, "direct") - ref)) < 1e-12
    assert np.max(np.abs(oracle.conv2(h, u, "fft") - ref)) < 1e-12


def test_conv2_separable_reduces_to_1d():
    # (f (x) g) (*) (p (x) q) = (f (*) p) (x) (g (*) q)
    r = rng(11)
    H, W = 32, 16
    f, p = r.standard_normal(H), r.standard_normal(H)
    g, q = r.standard_normal(W), r.standard_normal(W)
    ref = np.outer(np.convolve(f, p)[:H], np.convolve(g, q)[:W])
    got = oracle.conv2(np.outer(f, g), np.outer(p, q), "fft")
    assert rel_err(got, ref) < 1e-12


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_forward_2d_delta_and_shift(route):
    r = rng(12)
    B, C, H, W, N = 2, 2, 8, 8, 2
    v = r.standard_normal((B, C, H, W))
    x = r.standard_normal((N, B, C, H, W))
    b = r.standard_normal((N, C))
    # h_1 = delta at (0, 0), h_2 = delta at (1, 2):
    #   z_1 = x_1 v (1 + b_1);  y[p, q] = x_2 (z_1[p-1, q-2] + b_2 z_1[p, q])
    h = np.zeros((N, C, H, W)); h[0, :, 0, 0] = 1.0; h[1, :, 1, 2] = 1.0
    z1 = x[0] * v * (1 + b[0])[None, :, None, None]
    sh = np.zeros_like(z1); sh[..., 1:, 2:] = z1[..., :-1, :-2]
    ref = x[1] * (sh + b[1][None, :, None, None] * z1)
    assert rel_err(oracle.hyena_forward_2d(v, x, h, b, route=route), ref) < 1e-13


def test_forward_2d_routes_agree():
    r = rng(13)
    B, C, H, W, N = 1, 3, 16, 32, 2
    v = r.standard_normal((B, C, H, W))
    x = r.standard_normal((N, B, C, H, W))
    h = r.standard_normal((N, C, H, W))
    b = r.standard_normal((N, C))
    yd = oracle.hyena_forward_2d(v, x, h, b, route="direct")
    yf = oracle.hyena_forward_2d(v, x, h, b, route="fft")
    assert rel_err(yf, yd) < 1e-12


# ----------------------------------------------------- filter generation

def _selector_ffn(n_in, width, rows, sel, coef, perm2, perm3, head):
    """Weights for which the FFN has a closed form:
    a1[j] = sin(coef[j] phi[sel[j]]), a2[j] = sin(a1[perm2[j]]),
    a3[j] = sin(a2[perm3[j]]), o[r] = a3[head[r]]."""
    W1 = np.zeros((width, n_in)); W1[np.arange(width), sel] = coef
    W2 = np.zeros((width, width)); W2[np.arange(width), perm2] = 1.0
    W3 = np.zeros((width, width)); W3[np.arange(width), perm3] = 1.0
    Wout = np.zeros((rows, width)); Wout[np.arange(rows), head] = 1.0
    return W1, W2, W3, Wout


def test_filter_gen_closed_form():
    # K = 3 bands -> features [t, s1, c1, s2, c2, s3, c3]
    K, width, N, D, L = 3, 5, 2, 3, 64
    n_in = 1 + 2 * K
    sel = np.array([0, 1, 4, 6, 3])           # t, sin1, cos2, cos3, sin2
    coef = np.array([1.3, -0.7, 2.1, 0.9, 1.7])
    perm2 = np.array([2, 0, 4, 1, 3])
    perm3 = np.array([1, 3, 0, 4, 2])
    head = np.array([4, 0, 2, 1, 3, 0])       # row n*D + d
    W1, W2, W3, Wout = _selector_ffn(n_in, width, N * D, sel, coef, perm2, perm3, head)
    alpha = np.array([0.3, 0.9, 1.5])
    h = oracle.filter_gen(W1, W2, W3, Wout, alpha, N, D, L, n_bands=K, width=width)

    i = np.arange(L); t = i / L
    feats = [t, np.sin(2 * np.pi * t), np.cos(2 * np.pi * t), np.sin(4 * np.pi * t),
             np.cos(4 * np.pi * t), np.sin(6 * np.pi * t), np.cos(6 * np.pi * t)]
    a1 = [np.sin(coef[j] * feats[sel[j]]) for j in range(width)]
    a2 = [np.sin(a1[perm2[j]]) for j in range(width)]
    a3 = [np.sin(a2[perm3[j]]) for j in range(width)]
    for n in range(N):
        for d in range(D):
            ref = a3[head[n * D + d]] * np.exp(-alpha[d] * i / 64.0)
            assert np.max(np.abs(h[n, d] - ref)) < 1e-14


def test_filter_gen_special_values():
    r = rng(21)
    N, D, L, width, K = 2, 4, 128, 16, 8
    W1 = r.standard_normal((width, 1 + 2 * K))
    W2, W3 = r.standard_normal((width, width)), r.standard_normal((width, width))
    Wout = r.standard_normal((N * D, width))
    alpha = np.linspace(0.3, 1.5, D)
    # zero first layer -> every activation is sin(0) = 0 -> h = 0
    assert np.all(oracle.filter_gen(0 * W1, W2, W3, Wout, alpha, N, D, L, width=width) == 0.0)
    # alpha = 0: no window; the decay of channel d is exp(-alpha_d i / 64)
    h0 = oracle.filter_gen(W1, W2, W3, Wout, 0 * alpha, N, D, L, width=width)
    h = oracle.filter_gen(W1, W2, W3, Wout, alpha, N, D, L, width=width)
    win = np.exp(-alpha[None, :, None] * np.arange(L)[None, None, :] / 64.0)
    assert rel_err(h, h0 * win) < 1e-14
    # at i = 0 the features are [0, 0, 1, 0, 1, ...] and the window is 1
    phi0 = np.zeros(1 + 2 * K); phi0[2::2] = 1.0
    o = Wout @ np.sin(W3 @ np.sin(W2 @ np.sin(W1 @ phi0)))
    assert np.max(np.abs(h[:, :, 0].reshape(-1) - o)) < 1e-13


def test_filter_gen_2d_closed_form():
    # K = 2 bands -> features [ty, tx, s1y, c1y, s2y, c2y, s1x, c1x, s2x, c2x]
    K, width, N, C, H, W = 2, 4, 2, 2, 8, 16
    n_in = 2 + 4 * K
    sel = np.array([0, 1, 5, 8])              # ty, tx, c2y, s2x
    coef = np.array([1.1, -0.6, 1.9, 0.8])
    perm2 = np.array([3, 2, 0, 1])
    perm3 = np.array([1, 0, 3, 2])
    head = np.array([0, 3, 2, 1])
    W1, W2, W3, Wout = _selector_ffn(n_in, width, N * C, sel, coef, perm2, perm3, head)
    alpha = np.array([0.3, 1.5])
    h = oracle.filter_gen_2d(W1, W2, W3, Wout, alpha, N, C, H, W, n_bands=K, width=width)
    iy, ix = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    ty, tx = iy / H, ix / W
    feats = [ty, tx,
             np.sin(2 * np.pi * ty), np.cos(2 * np.pi * ty), np.sin(4 * np.pi * ty), np.cos(4 * np.pi * ty),
             np.sin(2 * np.pi * tx), np.cos(2 * np.pi * tx), np.sin(4 * np.pi * tx), np.cos(4 * np.pi * tx)]
    a1 = [np.sin(coef[j] * feats[sel[j]]) for j in range(width)]
    a2 = [np.sin(a1[perm2[j]]) for j in range(width)]
    a3 = [np.sin(a2[perm3[j]]) for j in range(width)]
    for n in range(N):
        for c in range(C):
            ref = a3[head[n * C + c]] * np.exp(-alpha[c] * iy / 64.0) * np.exp(-alpha[c] * ix / 64.0)
            assert np.max(np.abs(h[n, c] - ref)) < 1e-14


def test_filter_gen_threads_do_not_change_results():
    r = rng(22)
    N, D, L, width = 2, 3, 97, 8
    W1 = r.standard_normal((width, 17)); W2 = r.standard_normal((width, width))
    W3 = r.standard_normal((width, width)); Wout = r.standard_normal((N * D, width))
    alpha = np.linspace(0.3, 1.5, D)
    a = oracle.filter_gen(W1, W2, W3, Wout, alpha, N, D, L, width=width, threads=1)
    b = oracle.filter_gen(W1, W2, W3, Wout, alpha, N, D, L, width=width, threads=5)
    assert np.array_equal(a, b)


# --------------------------------------------------------------------- 3-D

@pytest.mark.parametrize("Z,H,W", [(1, 1, 1), (2, 3, 4), (4, 8, 4)])
def test_conv3_direct_is_scipy(Z, H, W):
    r = rng(Z * 100 + H * 10 + W)
    h, u = r.standard_normal((Z, H, W)), r.standard_normal((Z, H, W))
    ref = scipy.signal.convolve(h, u, method="direct")[:Z, :H, :W]
    assert rel_err(oracle.conv3(h, u, "direct"), ref) < 1e-12


@pytest.mark.parametrize("Z,H,W", [(2, 2, 2), (4, 8, 4), (8, 4, 16)])
def test_conv3_fft_equals_direct(Z, H, W):
    r = rng(Z + H + W)
    h, u = r.standard_normal((Z, H, W)), r.standard_normal((Z, H, W))
    assert rel_err(oracle.conv3(h, u, "fft"), oracle.conv3(h, u, "direct")) < 1e-12


def test_conv3_separable_reduces_to_2d_and_1d():
    # h[i][j][k] = f[i] g[j][k]: conv3 = (1-D along z) of (2-D in each plane)
    r = rng(7)
    Z, H, W = 4, 8, 8
    f, g, u = r.standard_normal(Z), r.standard_normal((H, W)), r.standard_normal((Z, H, W))
    h = f[:, None, None] * g[None]
    planes = np.stack([oracle.conv2(g, u[z], "direct") for z in range(Z)])
    ref = np.stack([[[oracle.conv(f, planes[:, q, rr], "direct")[p] for rr in range(W)]
                     for q in range(H)] for p in range(Z)])
    assert rel_err(oracle.conv3(h, u, "direct"), ref) < 1e-12


@pytest.mark.parametrize("route", ["direct", "fft"])
def test_forward_3d_delta_filter_and_routes(route):
    r = rng(8)
    B, C, Z, H, W, N = 2, 2, 4, 4, 8, 2
    v, x = r.standard_normal((B, C, Z, H, W)), r.standard_normal((N, B, C, Z, H, W))
    b = r.standard_normal((N, C))
    h = np.zeros((N, C, Z, H, W))
    h[:, :, 0, 0, 0] = 1.0
    want = v * np.prod(x * (1.0 + b)[:, None, :, None, None, None], axis=0)
    assert rel_err(oracle.hyena_forward_3d(v, x, h, b, route=route), want) < 1e-12
    h = r.standard_normal((N, C, Z, H, W))
    assert rel_err(oracle.hyena_forward_3d(v, x, h, b, route="fft"),
                   oracle.hyena_forward_3d(v, x, h, b, route="direct")) < 1e-12


# --------------------------------------------------------- 3-D filters

def test_filter_gen_3d_closed_form():
    # K = 2 bands -> features [tz, ty, tx, s1z, c1z, s2z, c2z, s1y, c1y, s2y, c2y, s1x, c1x, s2x, c2x]
    K, width, N, C, Z, H, W = 2, 6, 2, 2, 4, 8, 16
    n_in = 3 + 6 * K
    sel = np.array([0, 1, 2, 6, 8, 13])          # tz, ty, tx, c2z, c1y, s2x
    coef = np.array([1.1, -0.6, 0.7, 1.9, 0.8, -1.3])
    perm2 = np.array([3, 2, 0, 1, 5, 4])
    perm3 = np.array([1, 0, 3, 2, 4, 5])
    head = np.array([0, 3, 5, 1])
    W1, W2, W3, Wout = _selector_ffn(n_in, width, N * C, sel, coef, perm2, perm3, head)
    alpha = np.array([0.3, 1.5])
    h = oracle.filter_gen_3d(W1, W2, W3, Wout, alpha, N, C, Z, H, W, n_bands=K, width=width)
    iz, iy, ix = np.meshgrid(np.arange(Z), np.arange(H), np.arange(W), indexing="ij")
    tz, ty, tx = iz / Z, iy / H, ix / W
    feats = [tz, ty, tx]
    for t in (tz, ty, tx):
        feats += [np.sin(2 * np.pi * t), np.cos(2 * np.pi * t), np.sin(4 * np.pi * t), np.cos(4 * np.pi * t)]
    a1 = [np.sin(coef[j] * feats[sel[j]]) for j in range(width)]
    a2 = [np.sin(a1[perm2[j]]) for j in range(width)]
    a3 = [np.sin(a2[perm3[j]]) for j in range(width)]
    for n in range(N):
        for c in range(C):
            ref = a3[head[n * C + c]] * np.exp(-alpha[c] * (iz + iy + ix) / 64.0)
            assert np.max(np.abs(h[n, c] - ref)) < 1e-14


def test_filter_gen_3d_without_z_features_is_the_2d_filter_times_the_z_window():
    # W1 columns of the z features zeroed: every plane is the 2-D filter
    # (the pinned 2-D oracle, same y/x columns) times exp(-alpha iz / 64)
    r = rng(40)
    K, width, N, C, Z, H, W = 3, 8, 2, 3, 4, 8, 16
    W1 = r.standard_normal((width, 3 + 6 * K))
    W2, W3 = r.standard_normal((width, width)), r.standard_normal((width, width))
    Wout, alpha = r.standard_normal((N * C, width)), np.linspace(0.3, 1.5, C)
    zcols = [0] + list(range(3, 3 + 2 * K))
    W1[:, zcols] = 0.0
    # the 2-D oracle's columns: [ty, tx, y bands, x bands]
    W1_2d = W1[:, [1, 2] + list(range(3 + 2 * K, 3 + 6 * K))]
    h3 = oracle.filter_gen_3d(W1, W2, W3, Wout, alpha, N, C, Z, H, W, n_bands=K, width=width)
    # cos(0) = 1 in the zeroed z columns contributes nothing, so each plane differs only by the window
    h2 = oracle.filter_gen_2d(W1_2d, W2, W3, Wout, alpha, N, C, H, W, n_bands=K, width=width)
    win_z = np.exp(-alpha[None, :, None, None, None] * np.arange(Z)[None, None, :, None, None] / 64.0)
    assert rel_err(h3, h2[:, :, None] * win_z) < 1e-13


def test_filter_gen_3d_axis_permutation():
    # swapping the roles of y and x (volume transposed, W1 columns swapped)
    # transposes the filter
    r = rng(41)
    K, width, N, C, Z, H, W = 2, 8, 1, 2, 4, 8, 16
    W1 = r.standard_normal((width, 3 + 6 * K))
    W2, W3 = r.standard_normal((width, width)), r.standard_normal((width, width))
    Wout, alpha = r.standard_normal((N * C, width)), np.array([0.4, 1.2])
    ycols = [1] + list(range(3 + 2 * K, 3 + 4 * K))
    xcols = [2] + list(range(3 + 4 * K, 3 + 6 * K))
    W1s = W1.copy()
    W1s[:, ycols], W1s[:, xcols] = W1[:, xcols], W1[:, ycols]
    a = oracle.filter_gen_3d(W1, W2, W3, Wout, alpha, N, C, Z, H, W, n_bands=K, width=width)
    b = oracle.filter_gen_3d(W1s, W2, W3, Wout, alpha, N, C, Z, W, H, n_bands=K, width=width)
    assert rel_err(b, np.swapaxes(a, -1, -2)) < 1e-13
