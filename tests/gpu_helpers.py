"""Helpers shared by the GPU parity tests: device upload of the seeded
inputs, the packed-spectrum unpacking, and the tolerance checks.  The
expected values always come from the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from subquadratic_sequence_b200 import synth

# max |y_gpu - y_oracle| <= TOL * max |y_oracle| over the compared outputs
TOL = {"f32": 1e-4, "bf16": 2e-2}


def dev(a: np.ndarray, io: str = "f32") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if io == "bf16" else t


def host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def unpack_spectrum(Hp: np.ndarray) -> np.ndarray:
    """Packed [..., L] (slot 0 = (bin 0, bin L)) -> natural bins [..., L+1]."""
    L = Hp.shape[-1]
    out = np.empty(Hp.shape[:-1] + (L + 1,), dtype=np.complex128)
    out[..., 1:L] = Hp[..., 1:]
    out[..., 0] = Hp[..., 0].real
    out[..., L] = Hp[..., 0].imag
    return out


def rel_max_err(got, ref) -> float:
    """max |got - ref| / max |ref|, in complex128 when either side is complex."""
    cplx = np.iscomplexobj(got) or np.iscomplexobj(ref)
    dt = np.complex128 if cplx else np.float64
    got, ref = np.asarray(got, dt), np.asarray(ref, dt)
    return float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))


def assert_close(got, ref, io: str, what: str = "") -> float:
    err = rel_max_err(got, ref)
    assert err <= TOL[io], f"{what}: max|d|/max|ref| = {err:.3e} > {TOL[io]:.0e}"
    return err


def random_problem(B, D, L, N, seed, io="f32"):
    """Seeded inputs for small parity cases: the recipe of synth (normal
    activations, normal bias, FFN weights), at any shape."""
    wl = synth.Workload("case", "1d", N=N, B=B, D=D, L=L, io=io, seed=seed)
    return wl, synth.make_inputs(wl)


def gpu_filters(inp, wl, stream=None):
    from subquadratic_sequence_b200 import hyena
    return hyena.hyena_filter_gen(dev(inp["W1"]), dev(inp["W2"]), dev(inp["W3"]), dev(inp["Wout"]),
                                  dev(inp["alpha"]), wl.N, wl.D, wl.L, n_bands=synth.N_BANDS,
                                  width=synth.WIDTH, decay_div=synth.DECAY_DIV, stream=stream)


def oracle_filters(inp, wl):
    import oracle
    return oracle.filter_gen(inp["W1"], inp["W2"], inp["W3"], inp["Wout"], inp["alpha"], wl.N,
                             wl.D, wl.L, n_bands=synth.N_BANDS, width=synth.WIDTH,
                             decay_div=synth.DECAY_DIV)
