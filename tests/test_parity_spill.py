"""GPU parity of hyena_fftconv_gate_forward_spill, the forward that writes z
to HBM between orders (one launch per order) instead of chaining the orders
on chip: against the float64 oracle, and against the fused forward, whose
arithmetic per order it repeats (both keep z in float32)."""
import numpy as np
import pytest
import torch

import oracle
from subquadratic_sequence_b200 import synth
from tests.gpu_helpers import (TOL, assert_close, dev, gpu_filters, host, oracle_filters, random_problem,
                               rel_max_err)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def _run(hy, inp, wl, h32):
    H = hy.hyena_filter_rfft(dev(h32))
    v = dev(inp["v"], wl.io)
    xs = [dev(x, wl.io) for x in inp["x"]]
    b = dev(inp["b"])
    spill = host(hy.hyena_fftconv_gate_forward_spill(v, xs, b, H))
    fused = host(hy.hyena_fftconv_gate_forward(v, xs, b, H=H))
    torch.cuda.synchronize()
    return spill, fused


@pytest.mark.parametrize("B,D,L,N,io", [
    (1, 3, 16, 2, "f32"),
    (2, 5, 64, 3, "f32"),
    (3, 7, 1024, 2, "bf16"),
    (2, 4, 2048, 3, "bf16"),
    (1, 9, 4096, 4, "f32"),
    (2, 3, 8192, 3, "f32"),
    (1, 2, 16384, 3, "f32"),
    (2, 3, 16384, 2, "bf16"),
    (3, 2, 512, 1, "f32"),       # one order: nothing to spill
])
def test_spill_matches_oracle_and_fused(hy, B, D, L, N, io):
    wl, inp = random_problem(B, D, L, N, seed=B * 1000 + L + N, io=io)
    h = oracle_filters(inp, wl)
    spill, fused = _run(hy, inp, wl, h.astype(np.float32))
    ref = oracle.hyena_forward(inp["v"], np.stack(inp["x"]), h.astype(np.float32), inp["b"], route="fft")
    assert_close(spill, ref, io, "spill vs oracle")
    # same per-order arithmetic, z float32 in both: float32 rounding at most
    assert rel_max_err(spill, fused) <= (1e-6 if io == "f32" else 1e-2)


@pytest.mark.parametrize("name", ["c2_8k", "c2_16k"])
def test_spill_c2_full_size(hy, name):
    """Order-3, B=2, D=768, L=8192 / 16384, fp32: every (b, d) row against
    the oracle, with the GPU's own filters and spectra."""
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl)
    H = hy.hyena_filter_rfft(gpu_filters(inp, wl))
    y = host(hy.hyena_fftconv_gate_forward_spill(dev(inp["v"]), [dev(x) for x in inp["x"]], dev(inp["b"]), H))
    del H
    ref = oracle.hyena_forward(inp["v"], np.stack(inp["x"]), oracle_filters(inp, wl), inp["b"], route="fft")
    assert_close(y, ref, "f32", name)


def test_spill_needs_its_workspace(hy):
    v = torch.zeros((1, 2, 256), device="cuda")
    H = torch.zeros((2, 2, 256), device="cuda", dtype=torch.complex64)
    b = torch.zeros((2, 2), device="cuda")
    small = torch.empty(16, device="cuda", dtype=torch.uint8)
    with pytest.raises(hy.HyenaError) as e:
        hy.hyena_fftconv_gate_forward_spill(v, [v.clone(), v.clone()], b, H, workspace=small)
    assert e.value.status == hy.HYENA_ERR_WORKSPACE
