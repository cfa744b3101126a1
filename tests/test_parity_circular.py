"""GPU parity of the circular (unpadded) mode against the float64 oracle
(-m gpu): spectra at 2e-5 of their maximum, forward outputs at the storage
type's tolerance (1e-4 float32, 2e-2 bf16)."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_close, dev, host, random_problem, rel_max_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def filters(N, D, L, seed):
    r = np.random.default_rng(seed)
    return (r.standard_normal((N, D, L)) * 0.5 * np.exp(-np.arange(L) / (L / 8))).astype(np.float32)


@pytest.mark.parametrize("L", [32, 64, 256, 2048, 8192, 16384])
def test_rfft_circular_matches_oracle(hy, L):
    h = filters(2, 3, L, L)
    Hp = hy.hyena_filter_rfft_circular(dev(h)).cpu().numpy().astype(np.complex128)
    ref = oracle.rfft_circ(h)                      # bins 0..L/2
    got = np.empty_like(ref)
    got[..., 1:L // 2] = Hp[..., 1:]
    got[..., 0] = Hp[..., 0].real
    got[..., L // 2] = Hp[..., 0].imag
    assert rel_max_err(got, ref) <= 2e-5


@pytest.mark.parametrize("B,D,L,N,io", [
    (1, 1, 32, 1, "f32"), (2, 3, 64, 2, "f32"), (2, 5, 1024, 3, "bf16"), (2, 13, 4096, 2, "f32"),
    (1, 2, 16384, 2, "f32"), (3, 4, 2048, 4, "bf16"), (2, 7, 512, 2, "f32"),
])
def test_forward_circular_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=500 + L + N, io=io)
    h = filters(N, D, L, seed=L + 7)
    H = hy.hyena_filter_rfft_circular(dev(h))
    y = hy.hyena_fftconv_gate_forward_circular(dev(inp["v"], io), [dev(x, io) for x in inp["x"]],
                                               dev(inp["b"]), H)
    torch.cuda.synchronize()
    ref = oracle.hyena_forward_circular(inp["v"], np.stack(inp["x"]), h, inp["b"])
    assert_close(host(y), ref, io, f"circular B{B} D{D} L{L} N{N} {io}")


def test_circular_shift_filter_rotates(hy):
    # h = delta_k, b = 0, x = 1: y = v rotated by k per order
    B, D, L, k = 2, 3, 256, 17
    v = np.random.default_rng(1).standard_normal((B, D, L)).astype(np.float32)
    h = np.zeros((1, D, L), np.float32)
    h[:, :, k] = 1.0
    H = hy.hyena_filter_rfft_circular(dev(h))
    y = hy.hyena_fftconv_gate_forward_circular(dev(v), [dev(np.ones_like(v))], dev(np.zeros((1, D), np.float32)), H)
    torch.cuda.synchronize()
    assert rel_max_err(host(y), np.roll(v, k, axis=-1)) <= 1e-5


# ------------------------------------------------------------ backward

def check_backward(got, ref, io, name):
    dv, dx, dh, db = got
    rdv, rdx, rdh, rdb = ref
    assert_close(dv, rdv, io, f"{name} dv")
    assert_close(dx, rdx, io, f"{name} dx")
    assert rel_max_err(dh, rdh) <= 1e-4, f"{name} dh {rel_max_err(dh, rdh):.3e}"
    assert rel_max_err(db, rdb) <= 1e-4, f"{name} db {rel_max_err(db, rdb):.3e}"


@pytest.mark.parametrize("B,D,L,N,io", [
    (1, 1, 32, 1, "f32"), (2, 3, 64, 2, "f32"), (2, 5, 1024, 3, "bf16"), (2, 13, 4096, 2, "f32"),
    (1, 2, 16384, 2, "f32"), (8, 6, 2048, 2, "bf16"), (3, 2, 256, 16, "f32"),
])
def test_backward_circular_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=900 + L + N, io=io)
    h = filters(N, D, L, seed=L + 9)
    dy = np.random.default_rng(L).standard_normal((B, D, L)).astype(np.float32)
    if io == "bf16":
        from subquadratic_sequence_b200 import synth
        dy = synth.bf16_round(dy)
    H = hy.hyena_filter_rfft_circular(dev(h))
    dv, dxs, dh, db = hy.hyena_fftconv_gate_backward_circular(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), H, dev(dy, io))
    torch.cuda.synchronize()
    got = host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)
    ref = oracle.hyena_backward_circular(inp["v"], np.stack(inp["x"]), h, inp["b"], dy)
    check_backward(got, ref, io, f"circular backward B{B} D{D} L{L} N{N} {io}")


def test_backward_circular_shift_filter_closed_form(hy):
    # N = 1, h = delta_k, b = 0: y = x roll(v, k), so dv = roll(dy x, -k),
    # dx = dy roll(v, k), dh[s] = sum_b sum_t dy[t] x[t] v[(t - s) mod L]
    B, D, L, k = 2, 3, 512, 37
    r = np.random.default_rng(3)
    v, x, dy = (r.standard_normal((B, D, L)).astype(np.float32) for _ in range(3))
    h = np.zeros((1, D, L), np.float32)
    h[:, :, k] = 1.0
    H = hy.hyena_filter_rfft_circular(dev(h))
    dv, dxs, dh, db = hy.hyena_fftconv_gate_backward_circular(
        dev(v), [dev(x)], dev(np.zeros((1, D), np.float32)), H, dev(dy))
    torch.cuda.synchronize()
    e = (dy * x).astype(np.float64)
    assert rel_max_err(host(dv), np.roll(e, -k, axis=-1)) <= 1e-5
    assert rel_max_err(host(dxs[0]), dy * np.roll(v, k, axis=-1)) <= 1e-5
    ref_dh = np.stack([np.sum(e * np.roll(v, s, axis=-1), axis=(0, 2)) for s in range(L)], axis=-1)
    assert rel_max_err(host(dh)[0], ref_dh) <= 1e-4
    assert rel_max_err(host(db)[0], ref_dh[:, 0]) <= 1e-4


@pytest.mark.parametrize("B,D,L,N,io", [(2, 2, 32768, 2, "f32"), (1, 3, 65536, 1, "bf16"),
                                        (3, 11, 262144, 1, "f32")])   # channel 10 across two waves
def test_backward_circular_long_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=1200 + N, io=io)
    h = filters(N, D, L, seed=L + 19)
    dy = np.random.default_rng(L + 1).standard_normal((B, D, L)).astype(np.float32)
    if io == "bf16":
        from subquadratic_sequence_b200 import synth
        dy = synth.bf16_round(dy)
    H = hy.hyena_filter_rfft_circular(dev(h))
    dv, dxs, dh, db = hy.hyena_fftconv_gate_backward_circular(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), H, dev(dy, io))
    torch.cuda.synchronize()
    got = host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)
    ref = oracle.hyena_backward_circular(inp["v"], np.stack(inp["x"]), h, inp["b"], dy)
    check_backward(got, ref, io, f"circular backward B{B} D{D} L{L} N{N} {io}")


def test_backward_circular_rejects_unsupported_lengths(hy):
    from subquadratic_sequence_b200.hyena import HyenaError
    for L in (16, 1 << 23):
        with pytest.raises(HyenaError):
            hy.hyena_fftconv_backward_circular_workspace_size(2, 4, L, 2)


# ------------------------------------------- long sequences (four-step)

@pytest.mark.parametrize("L", [32768, 65536, 262144])
def test_rfft_circular_long_matches_oracle(hy, L):
    h = filters(2, 2, L, L)
    Hp = hy.hyena_filter_rfft_circular(dev(h)).cpu().numpy().astype(np.complex128)
    ref = oracle.rfft_circ(h)
    got = np.empty_like(ref)
    got[..., 1:L // 2] = Hp[..., 1:]
    got[..., 0] = Hp[..., 0].real
    got[..., L // 2] = Hp[..., 0].imag
    assert rel_max_err(got, ref) <= 2e-5


@pytest.mark.parametrize("B,D,L,N,io", [
    (2, 2, 32768, 2, "f32"), (1, 3, 65536, 3, "bf16"), (2, 2, 1 << 20, 1, "f32"),
    (3, 11, 262144, 2, "f32"),      # a wave holds 32 sequences: channel 10 spans two waves
])
def test_forward_circular_long_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=950 + N, io=io)
    h = filters(N, D, L, seed=L + 11)
    H = hy.hyena_filter_rfft_circular(dev(h))
    y = hy.hyena_fftconv_gate_forward_circular(dev(inp["v"], io), [dev(x, io) for x in inp["x"]],
                                               dev(inp["b"]), H)
    torch.cuda.synchronize()
    ref = oracle.hyena_forward_circular(inp["v"], np.stack(inp["x"]), h, inp["b"])
    assert_close(host(y), ref, io, f"circular B{B} D{D} L{L} N{N} {io}")


def test_circular_shift_filter_rotates_at_4m(hy):
    # L = 2^22 (the longest): h = delta_k, b = 0, x = 1 gives y = roll(v, k)
    B, D, L, k = 1, 2, 1 << 22, 123457
    v = np.random.default_rng(2).standard_normal((B, D, L)).astype(np.float32)
    h = np.zeros((1, D, L), np.float32)
    h[:, :, k] = 1.0
    H = hy.hyena_filter_rfft_circular(dev(h))
    y = hy.hyena_fftconv_gate_forward_circular(dev(v), [dev(np.ones_like(v))], dev(np.zeros((1, D), np.float32)), H)
    torch.cuda.synchronize()
    assert rel_max_err(host(y), np.roll(v, k, axis=-1)) <= 1e-5


def test_circular_long_on_zero_padded_sequences_is_the_linear_forward(hy):
    # length 2L with v, x_n and h_n zero beyond L: the circular recurrence's
    # first L outputs are the linear forward's (both through the four-step)
    B, D, L, N = 2, 3, 32768, 2
    wl, inp = random_problem(B, D, L, N, seed=77)
    h = filters(N, D, L, seed=78)
    pad = lambda a: np.concatenate([a, np.zeros_like(a)], axis=-1)
    yc = hy.hyena_fftconv_gate_forward_circular(dev(pad(inp["v"])), [dev(pad(x)) for x in inp["x"]],
                                                dev(inp["b"]), hy.hyena_filter_rfft_circular(dev(pad(h))))
    yl = hy.hyena_fftconv_gate_forward(dev(inp["v"]), [dev(x) for x in inp["x"]], dev(inp["b"]),
                                       H=hy.hyena_filter_rfft(dev(h)))
    torch.cuda.synchronize()
    assert rel_max_err(host(yc)[..., :L], host(yl).astype(np.float64)) <= 1e-5


# ------------------------------------- per-sample spectra (input-dependent)

@pytest.mark.parametrize("B,D,L,N,io", [(3, 4, 2048, 2, "f32"), (2, 3, 512, 2, "bf16"), (2, 2, 65536, 2, "f32")])
def test_forward_circular_per_sample_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=1100 + L, io=io)
    h = np.stack([filters(N, D, L, seed=L + 13 + b) for b in range(B)])          # [B][N][D][L]
    H = hy.hyena_filter_rfft_circular(dev(h.reshape(B * N, D, L))).reshape(B, N, D, L // 2)
    y = hy.hyena_fftconv_gate_forward_circular_per_sample(dev(inp["v"], io), [dev(x, io) for x in inp["x"]],
                                                          dev(inp["b"]), H)
    torch.cuda.synchronize()
    ref = oracle.hyena_forward_circular_per_sample(inp["v"], np.stack(inp["x"]), h, inp["b"])
    assert_close(host(y), ref, io, f"circular per-sample B{B} D{D} L{L} N{N} {io}")


def test_forward_circular_per_sample_with_equal_sets_is_the_shared_forward(hy):
    B, D, L, N = 3, 5, 4096, 2
    wl, inp = random_problem(B, D, L, N, seed=17)
    H = hy.hyena_filter_rfft_circular(dev(filters(N, D, L, seed=18)))
    v, xs, b = dev(inp["v"]), [dev(x) for x in inp["x"]], dev(inp["b"])
    y1 = hy.hyena_fftconv_gate_forward_circular(v, xs, b, H)
    y2 = hy.hyena_fftconv_gate_forward_circular_per_sample(v, xs, b, H.unsqueeze(0).expand(B, -1, -1, -1)
                                                           .contiguous())
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("B,D,L,N,io", [(3, 5, 2048, 2, "f32"), (2, 3, 512, 2, "bf16"), (2, 2, 65536, 2, "f32"),
                                        (1, 2, 32768, 1, "f32")])
def test_backward_circular_per_sample_matches_oracle(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=1300 + L, io=io)
    h = np.stack([filters(N, D, L, seed=L + 21 + b) for b in range(B)])
    dy = np.random.default_rng(L + 2).standard_normal((B, D, L)).astype(np.float32)
    if io == "bf16":
        from subquadratic_sequence_b200 import synth
        dy = synth.bf16_round(dy)
    H = hy.hyena_filter_rfft_circular(dev(h.reshape(B * N, D, L))).reshape(B, N, D, L // 2)
    dv, dxs, dh, db = hy.hyena_fftconv_gate_backward_circular_per_sample(
        dev(inp["v"], io), [dev(x, io) for x in inp["x"]], dev(inp["b"]), H, dev(dy, io))
    torch.cuda.synchronize()
    got = host(dv), np.stack([host(d) for d in dxs]), host(dh), host(db)
    ref = oracle.hyena_backward_circular_per_sample(inp["v"], np.stack(inp["x"]), h, inp["b"], dy)
    check_backward(got, ref, io, f"circular per-sample backward B{B} D{D} L{L} N{N} {io}")
