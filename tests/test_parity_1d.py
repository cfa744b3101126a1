"""GPU parity of the 1-D path against the float64 oracle (run with -m gpu).

Every expected value comes from ``oracle/``; the GPU side is called through
the C ABI binding.  Tolerances: max|y_gpu - y_oracle| <= 1e-4 max|y_oracle|
for float32 activations and <= 2e-2 max|y_oracle| for bf16 activations;
filters and spectra (float32 throughout) at 2e-5 of their maximum.
"""
import numpy as np
import pytest
import torch

import oracle
from subquadratic_sequence_b200 import synth
from tests.gpu_helpers import (assert_close, dev, gpu_filters, host, oracle_filters,
                               random_problem, rel_max_err, unpack_spectrum)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def run_forward(hy, inp, wl, h32, io=None, use_h=False):
    """GPU forward with the float32 filters h32 [N][D][L]."""
    io = io or wl.io
    hd = dev(h32)
    v = dev(inp["v"], io)
    xs = [dev(x, io) for x in inp["x"]]
    b = dev(inp["b"])
    if use_h:
        y = hy.hyena_fftconv_gate_forward(v, xs, b, h=hd)
    else:
        H = hy.hyena_filter_rfft(hd)
        y = hy.hyena_fftconv_gate_forward(v, xs, b, H=H)
    torch.cuda.synchronize()
    return host(y)


def oracle_forward(inp, h, seqs=None, route="fft"):
    """Oracle forward; seqs = list of (b, d) to compute only those rows."""
    v = inp["v"].astype(np.float64)
    x = np.stack(inp["x"]).astype(np.float64)
    b = inp["b"].astype(np.float64)
    if seqs is None:
        return oracle.hyena_forward(v, x, h, b, route=route)
    rows = []
    for (bi, di) in seqs:
        rows.append(oracle.hyena_forward(v[bi:bi + 1, di:di + 1], x[:, bi:bi + 1, di:di + 1],
                                         h[:, di:di + 1], b[:, di:di + 1], route=route)[0, 0])
    return np.stack(rows)


# ------------------------------------------------------------- filters

# covers the single-launch path (N*D <= 64), the tensor-core head (lengths
# a multiple of 4: 256-row tiles, a last tile of 192 rows, and head rows
# that are not a multiple of 16), and the SIMT head for lengths that are
# not a multiple of 4 (scalar h access)
@pytest.mark.parametrize("N,D,L", [(2, 64, 1024), (2, 768, 2048), (3, 5, 100), (1, 1, 1), (2, 3, 65536),
                                   (3, 100, 5001), (2, 256, 65536), (2, 256, 65535), (3, 27, 1024),
                                   (5, 77, 4096), (2, 40, 132)])
def test_filter_gen_matches_oracle(hy, N, D, L):
    wl, inp = random_problem(1, D, L, N, seed=11 + L)
    got = host(gpu_filters(inp, wl))
    ref = oracle_filters(inp, wl)
    assert rel_max_err(got, ref) <= 2e-5
    assert hy.LIB.hyena_device_fault_count() == 0


@pytest.mark.parametrize("N,C,H,W", [(2, 4, 16, 32), (1, 3, 7, 5), (2, 128, 256, 256), (2, 128, 255, 257)])
def test_filter_gen_2d_matches_oracle(hy, N, C, H, W):
    wl = synth.Workload("c", "2d", N=N, B=1, D=C, H=H, W=W, seed=7 + H)
    inp = synth.make_inputs(wl)
    got = host(hy.hyena_filter_gen_2d(dev(inp["W1"]), dev(inp["W2"]), dev(inp["W3"]), dev(inp["Wout"]),
                                      dev(inp["alpha"]), N, C, H, W))
    ref = oracle.filter_gen_2d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"], inp["alpha"], N, C, H, W)
    assert rel_max_err(got, ref) <= 2e-5


@pytest.mark.parametrize("L", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384,
                               32768, 65536, 262144])
def test_rfft_matches_oracle(hy, L):
    rng = np.random.default_rng(L)
    h = (rng.standard_normal((2, 3, L)) * np.exp(-np.arange(L) / (L / 4))).astype(np.float32)
    got = unpack_spectrum(hy.hyena_filter_rfft(dev(h)).cpu().numpy().astype(np.complex128))
    ref = oracle.rfft_pad2(h.astype(np.float64))
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) <= 2e-5 * np.max(np.abs(ref))


# ------------------------------------------------------------ forward

FWD_CASES = [(3, 5, L, 2, "f32") for L in (16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384)]
FWD_CASES += [(3, 5, L, 2, "bf16") for L in (16, 256, 2048, 8192)]
FWD_CASES += [(2, 7, 2048, 1, "f32"), (2, 7, 2048, 3, "f32"), (1, 3, 256, 16, "f32"),
              (1, 1, 4096, 2, "f32"), (5, 1, 1024, 2, "f32"), (4, 33, 1024, 2, "bf16")]
# four-step path (L > 16384)
FWD_CASES += [(1, 3, 32768, 2, "f32"), (2, 2, 65536, 2, "f32"), (1, 2, 131072, 3, "f32"),
              (1, 2, 65536, 2, "bf16"), (1, 1, 262144, 1, "f32")]


@pytest.mark.parametrize("B,D,L,N,io", FWD_CASES)
def test_forward_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=1000 + L + N, io=io)
    h32 = oracle_filters(inp, wl).astype(np.float32)
    got = run_forward(hy, inp, wl, h32)
    ref = oracle_forward(inp, h32.astype(np.float64))
    assert_close(got, ref, io, f"B{B} D{D} L{L} N{N} {io}")


@pytest.mark.parametrize("L", [64, 2048])
def test_forward_from_filters_equals_from_spectrum(hy, L):
    wl, inp = random_problem(2, 3, L, 2, seed=5)
    h32 = oracle_filters(inp, wl).astype(np.float32)
    a = run_forward(hy, inp, wl, h32, use_h=False)
    b = run_forward(hy, inp, wl, h32, use_h=True)
    assert np.array_equal(a, b)


def test_forward_is_deterministic(hy):
    wl, inp = random_problem(2, 9, 2048, 2, seed=6, io="bf16")
    h32 = oracle_filters(inp, wl).astype(np.float32)
    assert np.array_equal(run_forward(hy, inp, wl, h32), run_forward(hy, inp, wl, h32))


@pytest.mark.parametrize("L", [1024, 16384])
def test_delta_filters_give_the_closed_form(hy, L):
    # h_n = delta_0: y = v prod_n x_n (1 + b_n)
    wl, inp = random_problem(2, 3, L, 3, seed=8)
    h = np.zeros((3, 3, L), np.float32); h[:, :, 0] = 1.0
    got = run_forward(hy, inp, wl, h)
    ref = inp["v"].astype(np.float64)
    for n in range(3):
        ref = ref * inp["x"][n] * (1.0 + inp["b"][n].astype(np.float64))[None, :, None]
    assert_close(got, ref, "f32", "delta filters")


def test_causality(hy):
    # a change of v and x_n at t0 leaves y[:t0] unchanged up to FFT rounding
    L, t0 = 4096, 3000
    wl, inp = random_problem(1, 4, L, 2, seed=9)
    h32 = oracle_filters(inp, wl).astype(np.float32)
    y1 = run_forward(hy, inp, wl, h32)
    inp2 = dict(inp, v=inp["v"].copy(), x=[x.copy() for x in inp["x"]])
    inp2["v"][..., t0] += 100.0
    inp2["x"][0][..., t0] -= 50.0
    y2 = run_forward(hy, inp2, wl, h32)
    late = np.max(np.abs(y2[..., t0:] - y1[..., t0:]))
    early = np.max(np.abs(y2[..., :t0] - y1[..., :t0]))
    assert late > 1.0
    assert early <= 1e-5 * late


def test_linearity_in_v(hy):
    L = 2048
    wl, inp = random_problem(1, 6, L, 2, seed=10)
    h32 = oracle_filters(inp, wl).astype(np.float32)
    v2 = np.random.default_rng(3).standard_normal(inp["v"].shape).astype(np.float32)
    ya = run_forward(hy, inp, wl, h32)
    yb = run_forward(hy, dict(inp, v=v2), wl, h32)
    yc = run_forward(hy, dict(inp, v=(2 * inp["v"] - 3 * v2).astype(np.float32)), wl, h32)
    assert rel_max_err(yc, 2 * ya - 3 * yb) <= 1e-4


# ------------------------------------------- the workloads at full size

def test_c0_end_to_end(hy):
    """Order-2, B=1, D=64, L=1024, fp32: GPU filter generation, spectrum
    and forward against the oracle's filter generation and direct sums."""
    wl = synth.WORKLOADS["c0"]
    inp = synth.make_inputs(wl)
    h = gpu_filters(inp, wl)
    H = hy.hyena_filter_rfft(h)
    y = hy.hyena_fftconv_gate_forward(dev(inp["v"]), [dev(x) for x in inp["x"]], dev(inp["b"]), H=H)
    ref = oracle_forward(inp, oracle_filters(inp, wl), route="direct")
    assert_close(host(y), ref, "f32", "c0")


def _sampled_full_size(hy, name, n_samples, seed):
    """The whole workload on the GPU (filter generation, spectra, forward);
    the oracle on n_samples seeded (b, d) rows plus the first and last,
    its filters generated for just those channels."""
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl)
    h = gpu_filters(inp, wl)
    H = hy.hyena_filter_rfft(h)
    del h
    y = hy.hyena_fftconv_gate_forward(dev(inp["v"], wl.io), [dev(x, wl.io) for x in inp["x"]],
                                      dev(inp["b"]), H=H)
    torch.cuda.synchronize()
    del H
    rng = np.random.default_rng(seed)
    seqs = [(int(rng.integers(wl.B)), int(rng.integers(wl.D))) for _ in range(n_samples)]
    seqs += [(0, 0), (wl.B - 1, wl.D - 1)]
    got = np.stack([y[bi, di].float().cpu().numpy() for (bi, di) in seqs]).astype(np.float64)
    del y
    refs = []
    for (bi, di) in seqs:
        rows = [n * wl.D + di for n in range(wl.N)]
        hd = oracle.filter_gen(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["alpha"][[di]],
                               wl.N, 1, wl.L, n_bands=synth.N_BANDS, width=synth.WIDTH,
                               decay_div=synth.DECAY_DIV)
        v = inp["v"][bi:bi + 1, di:di + 1].astype(np.float64)
        x = np.stack([xx[bi:bi + 1, di:di + 1] for xx in inp["x"]]).astype(np.float64)
        refs.append(oracle.hyena_forward(v, x, hd, inp["b"][:, di:di + 1].astype(np.float64))[0, 0])
    return assert_close(got, np.stack(refs), wl.io, name)


def _full_size(hy, name):
    """The whole workload on the GPU (filter generation, spectra, forward)
    against the oracle (its own filters, FFT route) on every (b, d) row."""
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl)
    h = gpu_filters(inp, wl)
    H = hy.hyena_filter_rfft(h)
    del h
    y = hy.hyena_fftconv_gate_forward(dev(inp["v"], wl.io), [dev(x, wl.io) for x in inp["x"]],
                                      dev(inp["b"]), H=H)
    torch.cuda.synchronize()
    del H
    got = host(y)
    del y
    ref = oracle.hyena_forward(inp["v"], np.stack(inp["x"]), oracle_filters(inp, wl), inp["b"], route="fft")
    return assert_close(got, ref, wl.io, name)


def test_c1_full_size(hy):
    """Order-2, B=8, D=768, L=2048, bf16 storage: all 6144 (b, d) rows."""
    _full_size(hy, "c1")


@pytest.mark.parametrize("name", ["c2_8k", "c2_16k"])
def test_c2_full_size(hy, name):
    """Order-3, B=2, D=768, L=8192 / 16384, fp32: all 1536 (b, d) rows."""
    _full_size(hy, name)


@pytest.mark.parametrize("name", ["c3_64k", "c3_256k"])
def test_c3_full_size(hy, name):
    """Order-2, B=1, D=256, L = 64k / 256k, fp32 (the four-step path): all
    256 rows."""
    _full_size(hy, name)


def test_c3_1m_full_size_sampled(hy):
    """Order-2, B=1, D=256, L = 1M, fp32: the whole workload on the GPU, 8
    seeded channels (plus the first and last) from the oracle."""
    _sampled_full_size(hy, "c3_1m", 8, seed=3)


def test_long_forward_from_filters(hy):
    # the workspace then holds the spectra and the four-step scratch
    wl, inp = random_problem(1, 3, 65536, 2, seed=12)
    h32 = oracle_filters(inp, wl).astype(np.float32)
    a = run_forward(hy, inp, wl, h32, use_h=False)
    b = run_forward(hy, inp, wl, h32, use_h=True)
    assert np.array_equal(a, b)


def test_long_wave_boundaries(hy):
    # more sequences than one wave of the four-step scratch holds at 1M
    # (8 per 64 MB wave): 10 sequences span two waves
    wl, inp = random_problem(2, 5, 1 << 20, 1, seed=13)
    h32 = (np.random.default_rng(1).standard_normal((1, 5, 1 << 20))
           * np.exp(-np.arange(1 << 20) / 300.0)).astype(np.float32)
    got = run_forward(hy, inp, wl, h32)
    ref = oracle_forward(inp, h32.astype(np.float64), seqs=[(0, 0), (1, 4), (0, 3)])
    assert_close(got[[0, 1, 0], [0, 4, 3]], ref, "f32", "waves")
