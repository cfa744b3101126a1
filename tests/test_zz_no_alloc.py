"""GPU test of hyena_fftconv_gate_forward_noalloc, the entry point for
callers that cannot allocate device memory (its long-sequence scratch is a
16 MB array built into the library).  It runs the same kernels as
hyena_fftconv_gate_forward with a caller-provided workspace, only in
smaller waves, and every sequence's arithmetic is independent of the wave
it runs in: so its output must be bit-identical to that forward's, call
after call on the shared built-in scratch.  One case is also checked
against the float64 oracle.

Collected last (file name), so a run that stops at the first failure has
run every other test first; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import TOL, dev, host, rel_max_err

pytestmark = pytest.mark.gpu


def _inputs(B, D, L, N, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((B, D, L)).astype(np.float32)
    xs = [rng.standard_normal((B, D, L)).astype(np.float32) for _ in range(N)]
    b = rng.standard_normal((N, D)).astype(np.float32)
    h = (rng.standard_normal((N, D, L)) * np.exp(-np.arange(L) / 500.0)).astype(np.float32)
    return v, xs, b, h


def _case(B, D, L, N, io, seed):
    v, xs, b, h = _inputs(B, D, L, N, seed)
    return dev(v, io), [dev(x, io) for x in xs], dev(b), dev(h)


@pytest.mark.parametrize("B,D,L,N,io", [
    (1, 3, 1 << 16, 2, "f32"),      # four-step, one wave of the built-in scratch
    (1, 3, 1 << 20, 2, "f32"),      # 8 MB per sequence: 2 per wave, so 2 waves
    (2, 2, 1 << 17, 3, "bf16"),
    (2, 5, 2048, 2, "bf16"),        # single-CTA path (no scratch at all)
])
def test_noalloc_matches_workspace_forward_twice(B, D, L, N, io):
    from subquadratic_sequence_b200 import hyena
    v, xs, b, h = _case(B, D, L, N, io, seed=L + N)
    H = hyena.hyena_filter_rfft(h)
    ref = host(hyena.hyena_fftconv_gate_forward(v, xs, b, H=H))
    for _ in range(2):
        got = hyena.hyena_fftconv_gate_forward_noalloc(v, xs, b, H)
        torch.cuda.synchronize()
        assert np.array_equal(host(got), ref)


def test_noalloc_matches_oracle():
    from subquadratic_sequence_b200 import hyena
    B, D, L, N = 1, 2, 1 << 15, 2
    v, xs, b, h = _inputs(B, D, L, N, seed=77)
    H = hyena.hyena_filter_rfft(dev(h))
    got = host(hyena.hyena_fftconv_gate_forward_noalloc(dev(v), [dev(x) for x in xs], dev(b), H))
    ref = oracle.hyena_forward(v, np.stack(xs), h, b, route="fft")
    assert rel_max_err(got, ref) <= TOL["f32"]


def test_noalloc_rejects_sequences_longer_than_its_scratch():
    from subquadratic_sequence_b200 import hyena
    L = 1 << 22                     # 32 MB of scratch per sequence > 16 MB
    v = torch.zeros((1, 1, L), device="cuda")
    H = torch.zeros((1, 1, L), device="cuda", dtype=torch.complex64)
    b = torch.zeros((1, 1), device="cuda")
    with pytest.raises(hyena.HyenaError) as e:
        hyena.hyena_fftconv_gate_forward_noalloc(v, [v], b, H)
    assert e.value.status == hyena.HYENA_ERR_WORKSPACE
