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
