"""GPU parity of the 1-D backward pass against the float64 oracle (-m gpu).

The oracle's backward is pinned to finite differences of its forward
(tests/test_oracle_backward_pins.py).  Tolerances: dv and dx_n as the
forward's output (1e-4 of the maximum for float32 storage, 2e-2 for bf16);
dh and dbias, accumulated in float32 from float32 intermediates, 1e-4 of
their maximum for both storage types.
"""
import numpy as np
import pytest
import torch

import oracle
from subquadratic_sequence_b200 import synth
from tests.gpu_helpers import assert_close, dev, host, random_problem, rel_max_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def filters(wl, seed):
    """Seeded decaying filters (float32), the shape the filter network gives."""
    r = np.random.default_rng(seed)
    decay = np.exp(-np.arange(wl.L) * np.linspace(0.3, 1.5, wl.D)[:, None] / 64.0)
    return (r.standard_normal((wl.N, wl.D, wl.L)) * 0.2 * decay).astype(np.float32)


def run(hy, wl, inp, h32, dy):
    io = wl.io
    H = hy.hyena_filter_rfft(dev(h32))
    dv, dxs, dh, db = hy.hyena_fftconv_gate_backward(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), H, dev(dy, io))
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
    (1, 1, 16, 1, "f32"), (2, 3, 64, 2, "f32"), (3, 5, 256, 3, "f32"), (2, 7, 1024, 2, "bf16"),
    (2, 13, 2048, 2, "f32"),        # 13 channels: a partly idle CTA at L = 2048 (6 per CTA)
    (1, 4, 4096, 4, "f32"), (2, 3, 8192, 2, "f32"), (1, 2, 16384, 2, "f32"), (3, 2, 512, 16, "f32"),
    (8, 6, 2048, 2, "bf16"),
]


@pytest.mark.parametrize("B,D,L,N,io", CASES)
def test_backward_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=300 + L + N, io=io)
    h32 = filters(wl, seed=L + N)
    dy = synth.make_output_grad(wl)
    got = run(hy, wl, inp, h32, dy)
    ref = oracle.hyena_backward(inp["v"], np.stack(inp["x"]), h32, inp["b"], dy)
    check(got, ref, io, f"B{B} D{D} L{L} N{N} {io}")


def test_backward_c1_full_size(hy):
    """Order-2, B=8, D=768, L=2048, bf16 storage: every output compared."""
    wl = synth.WORKLOADS["c1"]
    inp = synth.make_inputs(wl)
    h32 = filters(wl, seed=1)
    dy = synth.make_output_grad(wl)
    got = run(hy, wl, inp, h32, dy)
    ref = oracle.hyena_backward(inp["v"], np.stack(inp["x"]), h32, inp["b"], dy)
    check(got, ref, wl.io, "c1")


def test_backward_is_deterministic(hy):
    wl, inp = random_problem(4, 6, 1024, 2, seed=9)
    h32 = filters(wl, seed=9)
    dy = synth.make_output_grad(wl)
    a = run(hy, wl, inp, h32, dy)
    b = run(hy, wl, inp, h32, dy)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_of_delta_filters_is_the_closed_form(hy):
    # h = delta_0, N = 1: dv = dy x (1+b), dx = dy (1+b) v
    wl, inp = random_problem(2, 3, 512, 1, seed=4)
    h32 = np.zeros((1, 3, 512), np.float32)
    h32[:, :, 0] = 1.0
    dy = synth.make_output_grad(wl)
    dv, dx, _, _ = run(hy, wl, inp, h32, dy)
    gain = (1.0 + inp["b"][0].astype(np.float64))[None, :, None]
    assert rel_max_err(dv, dy * inp["x"][0] * gain) <= 1e-5
    assert rel_max_err(dx[0], dy * gain * inp["v"]) <= 1e-5


# ---------------------------------------------------- four-step (L > 16384)

LONG_CASES = [
    (1, 3, 32768, 2, "f32"), (2, 2, 65536, 2, "f32"), (1, 2, 131072, 1, "bf16"), (2, 1, 262144, 3, "f32"),
    (3, 4, 1 << 20, 1, "f32"),      # 12 sequences, 8 a wave: channel 2 spans two waves
    (1, 1, 1 << 22, 1, "f32"),      # the longest supported length
]


@pytest.mark.parametrize("B,D,L,N,io", LONG_CASES)
def test_backward_fourstep_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=700 + N, io=io)
    h32 = filters(wl, seed=L % 1000 + N)
    dy = synth.make_output_grad(wl)
    got = run(hy, wl, inp, h32, dy)
    ref = oracle.hyena_backward(inp["v"], np.stack(inp["x"]), h32, inp["b"], dy)
    check(got, ref, io, f"B{B} D{D} L{L} N{N} {io}")


def test_backward_c3_64k_full_size(hy):
    """Order-2, B=1, D=256, L=65536, fp32: every output compared."""
    wl = synth.WORKLOADS["c3_64k"]
    inp = synth.make_inputs(wl)
    h32 = filters(wl, seed=3)
    dy = synth.make_output_grad(wl)
    got = run(hy, wl, inp, h32, dy)
    ref = oracle.hyena_backward(inp["v"], np.stack(inp["x"]), h32, inp["b"], dy)
    check(got, ref, wl.io, "c3_64k")


# ------------------------------------------------- per-sample filters

PS_CASES = [(2, 3, 64, 2, "f32"), (3, 13, 2048, 2, "f32"), (2, 5, 1024, 3, "bf16"), (2, 2, 16384, 2, "f32"),
            (1, 1, 16, 1, "f32"),
            # four-step: L = 2^15 (N = 1), 2^16 in bf16, and 2^18, where a wave
            # holds 32 sequences, so channel 10's three samples straddle two waves
            (3, 2, 32768, 1, "f32"), (2, 3, 65536, 2, "bf16"), (3, 11, 262144, 1, "f32"),
            (1, 2, 32768, 2, "f32")]     # one sample: dbias still comes from the per-sample sum


@pytest.mark.parametrize("B,D,L,N,io", PS_CASES)
def test_backward_per_sample_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=700 + L + N, io=io)
    r = np.random.default_rng(L + B)
    decay = np.exp(-np.arange(L) * np.linspace(0.3, 1.5, D)[:, None] / 64.0)
    h32 = (r.standard_normal((B, N, D, L)) * 0.2 * decay).astype(np.float32)
    dy = synth.make_output_grad(wl)
    H = hy.hyena_filter_rfft(dev(h32.reshape(B * N, D, L))).reshape(B, N, D, L)
    dv, dxs, dh, db = hy.hyena_fftconv_gate_backward_per_sample(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), H, dev(dy, io))
    torch.cuda.synchronize()
    got = host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)
    ref = oracle.hyena_backward_per_sample(inp["v"], np.stack(inp["x"]), h32, inp["b"], dy)
    check(got, ref, io, f"per-sample B{B} D{D} L{L} N{N} {io}")


def test_backward_per_sample_with_equal_sets_is_the_shared_backward(hy):
    """Every sample given the same spectra: dv and dx equal the shared
    backward's bit for bit, the per-sample dh sum to its dh."""
    B, D, L, N = 4, 6, 2048, 2
    wl, inp = random_problem(B, D, L, N, seed=41, io="bf16")
    h32 = filters(wl, seed=42)
    dy = dev(synth.make_output_grad(wl), "bf16")
    H = hy.hyena_filter_rfft(dev(h32))
    v, xs, b = dev(inp["v"], "bf16"), [dev(x, "bf16") for x in inp["x"]], dev(inp["b"])
    dv, dxs, dh, db = hy.hyena_fftconv_gate_backward(v, xs, b, H, dy)
    pv, pxs, ph, pb = hy.hyena_fftconv_gate_backward_per_sample(
        v, xs, b, H.unsqueeze(0).expand(B, -1, -1, -1).contiguous(), dy)
    torch.cuda.synchronize()
    assert torch.equal(dv, pv) and all(torch.equal(a, c) for a, c in zip(dxs, pxs))
    assert rel_max_err(host(ph).sum(axis=0), host(dh)) <= 1e-5
    assert rel_max_err(host(pb), host(db)) <= 1e-5


def test_backward_per_sample_rejects_unsupported_lengths(hy):
    from subquadratic_sequence_b200.hyena import HyenaError
    for L in (8, 1 << 23, 3000):
        with pytest.raises(HyenaError):
            hy.hyena_fftconv_backward_per_sample_workspace_size(2, 4, L, 2)
