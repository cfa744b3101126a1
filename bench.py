"""Benchmark of the Hyena FFT-conv + gate path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3_1m] [--impl reference]

One step = one pass of the whole path over one batch of synthetic input:
implicit filter generation (hyena_filter_gen), the filter spectra
(hyena_filter_rfft, computed once and shared by the whole batch) and the
fused order-N forward (hyena_fftconv_gate_forward).  The metric is
channel-positions per second (B * D * L per step).  Device time comes from
CUDA events on the launching stream; L2 is flushed (a 256 MB write) before
every timed step, outside the timed events.  Under torchrun every rank runs
the same workload on its own GPU (the channel-sequences are independent, so
the ranks share no data: weak scaling) and rank 0 prints one JSON line with
the max time over ranks.

The default workload is the largest single-GPU configuration (order 2,
B=1, D=256, L=2^20, fp32).  The same run times the forward alone on every
configuration (``per_config``: c0, c1, c2 at 8k and 16k, c3 at 64k, 256k
and 1M, the 2-D c4) with its fraction of the HBM roofline.  ``e2e`` runs
the step end to end from pinned host memory (H2D of the inputs, the step,
D2H of y), pipelined over two buffer sets on three streams.

--impl reference times the float64 CPU oracle on the host cores on a
bounded sample of the same workload (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from subquadratic_sequence_b200 import synth  # noqa: E402

METRIC = "Hyena FFT-conv+gate fwd: channel-positions/s and % of B200 HBM roofline"
UNIT = "channel-positions/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def describe(wl: synth.Workload) -> dict:
    d = _describe(wl)
    if wl.circular:
        d["workload"] = re.sub(r" \(padded to [^)]*\)", "", d["workload"])
        d["workload"] += "; circular convolution on the grid itself (periodic boundaries, no padding)"
        d["circular"] = True
    return d


def _describe(wl: synth.Workload) -> dict:
    if wl.kind == "3d":
        filters = (f"implicit FFN over (z/Z, y/H, x/W) (3 sine layers of width {synth.WIDTH}, "
                   f"{synth.N_BANDS} bands per axis) x separable decay, regenerated every step")
        if wl.film:
            filters = (f"input-dependent: a filter set per sample, the {synth.WIDTH}-wide sine layers over "
                       f"(z/Z, y/H, x/W) ({synth.N_BANDS} bands per axis) FiLM-modulated per sample, first "
                       "layer at frequencies 1/2/4/8, Gaussian window; B*N*C filters and spectra "
                       "regenerated every step")
        return {"workload": f"{wl.name}: order-{wl.N} Hyena 3-D operator, B={wl.B}, C={wl.D}, "
                            f"{wl.Z}x{wl.H}x{wl.W} volumes (padded to {2 * wl.Z}x{2 * wl.H}x{2 * wl.W}), "
                            f"{wl.io} storage, fp32 compute",
                "N": wl.N, "B": wl.B, "C": wl.D, "Z": wl.Z, "H": wl.H, "W": wl.W, "io": wl.io,
                "filters": filters,
                "l2": "flushed (256 MB write) before every timed step"}
    if wl.kind == "2d":
        filters = (f"implicit FFN over (y/H, x/W) (3 sine layers of width {synth.WIDTH}, "
                   f"{synth.N_BANDS} bands per axis) x separable decay, regenerated every step")
        if wl.film:
            filters = (f"input-dependent: a filter set per sample, the {synth.WIDTH}-wide sine layers over "
                       f"(y/H, x/W) ({synth.N_BANDS} bands per axis) FiLM-modulated per sample, first layer at "
                       "frequencies 1/2/4/8, Gaussian window; B*N*C filters and spectra regenerated every step")
        return {"workload": f"{wl.name}: order-{wl.N} Hyena 2-D operator, B={wl.B}, C={wl.D}, "
                            f"{wl.H}x{wl.W} grid (padded to {2 * wl.H}x{2 * wl.W}), {wl.io} storage, fp32 compute",
                "N": wl.N, "B": wl.B, "C": wl.D, "H": wl.H, "W": wl.W, "io": wl.io,
                "filters": filters,
                "l2": "flushed (256 MB write) before every timed step"}
    filters = (f"implicit FFN (3 sine layers of width {synth.WIDTH}, {synth.N_BANDS} bands) "
               "x exponential decay, regenerated every step")
    if wl.film:
        filters = (f"input-dependent: a filter set per sample, the {synth.WIDTH}-wide sine layers "
                   "FiLM-modulated per sample, first layer at frequencies 1/2/4/8, Gaussian window; "
                   "B*N*D filters and spectra regenerated every step")
    return {"workload": f"{wl.name}: order-{wl.N} Hyena 1-D operator, B={wl.B}, D={wl.D}, "
                        f"L={wl.L}, {wl.io} storage, fp32 compute",
            "N": wl.N, "B": wl.B, "D": wl.D, "L": wl.L, "io": wl.io, "filters": filters,
            "l2": "flushed (256 MB write) before every timed step"}


def alg_bytes_forward(wl: synth.Workload) -> int:
    """Algorithmic HBM bytes of one forward call: v, x_1..x_N, y plus the
    N*D packed spectra (L complex64 slots each; 2H x W for the 2-D grid,
    2Z x 2H x W for the 3-D volume)."""
    act = (wl.N + 2) * wl.positions * wl.io_bytes
    if wl.circular:                        # spectra of the grid itself: half a slot per position
        return act + wl.N * wl.D * wl.per_channel // 2 * 8
    sets = wl.B if wl.film else 1          # filter spectra per sample, or shared by the batch
    if wl.kind == "3d":
        return act + sets * wl.N * wl.D * 4 * wl.Z * wl.H * wl.W * 8
    if wl.kind == "2d":
        return act + sets * wl.N * wl.D * 2 * wl.H * wl.W * 8
    return act + sets * wl.N * wl.D * wl.L * 8


def alg_bytes_backward(wl: synth.Workload) -> int:
    """Bytes the backward must move at least: v, x_1..x_N and dy in, dv and
    dx_1..dx_N out (storage type), the spectra H in (complex64), dh and
    dbias out (float32)."""
    io = 2 if wl.io == "bf16" else 4
    act = wl.positions * io
    if wl.kind == "3d" and wl.circular:       # Z x H x W/2 spectrum slots and Z x H x W of dh a filter
        return (2 * wl.N + 3) * act + wl.N * wl.D * wl.Z * wl.H * wl.W * (4 + 4) + wl.N * wl.D * 4
    if wl.kind == "3d":                       # 2Z x 2H x W spectrum slots and Z x H x W of dh a filter
        sets = wl.B if wl.film else 1
        return (2 * wl.N + 3) * act + sets * wl.N * wl.D * wl.Z * wl.H * wl.W * (32 + 4) + wl.N * wl.D * 4
    if wl.film and wl.kind == "2d":   # 2H x W spectrum slots and H x W of dh, per sample
        return (2 * wl.N + 3) * act + wl.B * wl.N * wl.D * wl.H * wl.W * (16 + 4) + wl.N * wl.D * 4
    if wl.film:             # spectra in and dh out per sample
        return (2 * wl.N + 3) * act + wl.B * wl.N * wl.D * wl.L * (8 + 4) + wl.N * wl.D * 4
    if wl.circular:         # half a spectrum slot and one dh value per position
        return (2 * wl.N + 3) * act + wl.N * wl.D * wl.per_channel * (4 + 4) + wl.N * wl.D * 4
    if wl.kind == "2d":     # 2H x W spectrum slots a filter, H x W of dh
        return (2 * wl.N + 3) * act + wl.N * wl.D * wl.H * wl.W * (16 + 4) + wl.N * wl.D * 4
    return (2 * wl.N + 3) * act + wl.N * wl.D * wl.L * (8 + 4) + wl.N * wl.D * 4


def long_path(wl: synth.Workload) -> bool:
    return wl.kind == "1d" and wl.L > 16384


def waves(nseq: int, L: int) -> int:
    per = max(1, (64 << 20) // (8 * L))
    return -(-nseq // min(nseq, per))


def launches_forward(wl: synth.Workload) -> int:
    """Kernel launches of one forward call."""
    if wl.circular:
        if wl.kind == "3d":
            return waves(wl.B * wl.D, wl.per_channel) * (4 * wl.N + 1)
        if wl.kind == "2d":
            return waves(wl.B * wl.D, wl.per_channel // 2) * (1 + 2 * wl.N)
        return waves(wl.B * wl.D, wl.L // 2) * (1 + 2 * wl.N) if long_path(wl) else 1
    if wl.kind == "3d":
        # per wave: rows, columns, then per order z, inverse columns, rows
        # (and forward columns before every order but the first)
        return waves(wl.B * wl.D, 2 * wl.Z * wl.H * wl.W) * (4 * wl.N + 1)
    if wl.kind == "2d":
        return waves(wl.B * wl.D, wl.H * wl.W) * (1 + 2 * wl.N)
    return waves(wl.B * wl.D, wl.L) * (1 + 2 * wl.N) if long_path(wl) else 1


def launches_rfft(wl: synth.Workload) -> int:
    if wl.circular:
        if long_path(wl):
            return waves(wl.N * wl.D, wl.L // 2) * 2
        return {"1d": 1, "2d": 2, "3d": 3}[wl.kind]
    if wl.kind == "3d":
        return 3
    if wl.kind == "2d":
        return 2
    rows = wl.N * wl.D * (wl.B if wl.film else 1)
    return waves(rows, wl.L) * 2 if long_path(wl) else 1


def launches_filter_gen(wl: synth.Workload) -> int:
    return 3 if wl.N * wl.D > 64 else 1


def forward_kernel(wl: synth.Workload) -> str:
    """The timed unit of the roofline: the forward call (one fused kernel,
    or the 2N+1 four-step kernels of each wave)."""
    if wl.circular and long_path(wl):
        return "fourstep_row_kernel+fourstep_col_kernel<PAD=false> (hyena_fftconv_gate_forward_circular, all launches)"
    if wl.circular:
        return {"1d": "fused1d_kernel<PAD=false> (hyena_fftconv_gate_forward_circular)",
                "2d": "fft2d_row_kernel+fft2d_col_kernel<PAD=false> (hyena_fftconv2d_gate_forward_circular, "
                      "all launches)",
                "3d": "fft2d_row_kernel+fft2d_col_kernel+fft3d_z_kernel<PAD=false> "
                      "(hyena_fftconv3d_gate_forward_circular, all launches)"}[wl.kind]
    if wl.kind == "3d":
        return "fft2d_row_kernel+fft2d_col_kernel+fft3d_z_kernel (hyena_fftconv3d_gate_forward, all launches)"
    if wl.kind == "2d":
        return "fft2d_row_kernel+fft2d_col_kernel (hyena_fftconv2d_gate_forward, all launches)"
    if long_path(wl):
        return "fourstep_row_kernel+fourstep_col_kernel (hyena_fftconv_gate_forward, all launches)"
    return "fused1d_kernel (hyena_fftconv_gate_forward)"


def peaks() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# source files that define each kernel measured by ncu (the traffic figure
# is dropped as soon as any of them changes)
KERNEL_SOURCES = {
    "fused1d_kernel": ["fused1d.cuh", "hyena_common.cuh"],
    "fourstep_row_kernel+fourstep_col_kernel": ["fourstep.cuh", "k_fourstep.cuh", "hyena_common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "subquadratic_sequence_b200", "csrc")
    for fn in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes (read + write) of `kernel` on `workload` from
    profiles/traffic.json, if it was captured on the current sources of that
    kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[f"{kernel}@{workload}"]
        current = kernel_source_hash(kernel)
    except Exception:
        return None
    return rec["dram_bytes_per_launch"] if rec.get("source_hash") == current else None


# ----------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ GPU arm

class Ranks:
    """One process per GPU (torchrun environment).  The ranks run the same
    workload on their own data (weak scaling) and meet only to line up the
    timed region (barriers) and to take the max time over ranks."""

    def __init__(self, backend: str):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        if backend == "nccl":
            torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": torch.device("cuda", self.local)} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        if self.world == 1:
            return x
        import torch
        import torch.distributed as dist
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


def throughput(positions_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job channel-positions per second: the units all ranks processed
    over the slowest rank's time."""
    return positions_per_rank * world * steps / (total_ms / 1e3)


class Buffers:
    """One set of device inputs and output of a step."""

    def __init__(self, wl: synth.Workload, inp: dict):
        import torch
        io = torch.bfloat16 if wl.io == "bf16" else torch.float32

        def to_dev(a, dtype=torch.float32):
            return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(dtype)

        self.v = to_dev(inp["v"], io)
        self.xs = [to_dev(x, io) for x in inp["x"]]
        self.b = to_dev(inp["b"])
        self.W = [to_dev(inp[k]) for k in WKEYS]
        self.F = [to_dev(inp[k]) for k in FILM_KEYS] if wl.film else []
        self.y = torch.empty_like(self.v)


WKEYS = ("W1", "W2", "W3", "Wout", "alpha")
FILM_KEYS = ("omega", "gamma", "beta", "sigma")


def setup_step(wl: synth.Workload, bf: Buffers, spill: bool = False):
    """The step (filter generation, spectra, forward) and the forward alone
    of one workload on one buffer set, with the filters, spectra and
    workspaces they use allocated once.  Returns (step, forward, H).
    spill: the forward that writes z to HBM between orders instead of the
    fused one (1-D workloads with a spill variant)."""
    import torch
    from subquadratic_sequence_b200 import hyena

    v, xs, b, W, F, y = bf.v, bf.xs, bf.b, bf.W, bf.F, bf.y
    if wl.circular and wl.kind == "3d":
        h = torch.empty((wl.N, wl.D, wl.Z, wl.H, wl.W), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.N, wl.D, wl.Z, wl.H, wl.W // 2), device="cuda", dtype=torch.complex64)
        ws_fwd = torch.empty(hyena.hyena_fftconv3d_circular_workspace_size(wl.B, wl.D, wl.Z, wl.H, wl.W),
                             device="cuda", dtype=torch.uint8)

        def forward():
            hyena.hyena_fftconv3d_gate_forward_circular(v, xs, b, H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen_3d(*W, wl.N, wl.D, wl.Z, wl.H, wl.W, n_bands=synth.N_BANDS,
                                      width=synth.WIDTH, decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft3d_circular(h, out=H)
            forward()
    elif wl.circular and wl.kind == "2d":
        h = torch.empty((wl.N, wl.D, wl.H, wl.W), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.N, wl.D, wl.H, wl.W // 2), device="cuda", dtype=torch.complex64)
        ws_fwd = torch.empty(hyena.hyena_fftconv2d_circular_workspace_size(wl.B, wl.D, wl.H, wl.W),
                             device="cuda", dtype=torch.uint8)

        def forward():
            hyena.hyena_fftconv2d_gate_forward_circular(v, xs, b, H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen_2d(*W, wl.N, wl.D, wl.H, wl.W, n_bands=synth.N_BANDS,
                                      width=synth.WIDTH, decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft2d_circular(h, out=H)
            forward()
    elif wl.circular:
        h = torch.empty((wl.N, wl.D, wl.L), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.N, wl.D, wl.L // 2), device="cuda", dtype=torch.complex64)
        # four-step workspaces (L > 16384), allocated once
        ws_rfft_n = hyena.LIB.hyena_filter_rfft_circular_workspace_size(wl.N, wl.D, wl.L)
        ws_fwd_n = hyena.LIB.hyena_fftconv_circular_workspace_size(wl.B, wl.D, wl.L, wl.N)
        ws_rfft = torch.empty(ws_rfft_n, device="cuda", dtype=torch.uint8) if ws_rfft_n else None
        ws_fwd = torch.empty(ws_fwd_n, device="cuda", dtype=torch.uint8) if ws_fwd_n else None

        def forward():
            hyena.hyena_fftconv_gate_forward_circular(v, xs, b, H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen(*W, wl.N, wl.D, wl.L, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                   decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft_circular(h, out=H, workspace=ws_rfft)
            forward()
    elif wl.kind == "3d" and wl.film:
        h = torch.empty((wl.B, wl.N, wl.D, wl.Z, wl.H, wl.W), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.B, wl.N, wl.D, 2 * wl.Z, 2 * wl.H, wl.W), device="cuda", dtype=torch.complex64)
        ws_n = hyena.hyena_fftconv3d_workspace_size(wl.B, wl.D, wl.Z, wl.H, wl.W, wl.N, hyena.io_dtype(v), True)
        ws_fwd = torch.empty(ws_n, device="cuda", dtype=torch.uint8)

        def forward():
            hyena.hyena_fftconv3d_gate_forward_per_sample(v, xs, b, H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen_film_3d(*W, wl.N, wl.D, wl.Z, wl.H, wl.W, B=wl.B, omega=F[0], gamma=F[1],
                                           beta=F[2], sigma=F[3], n_bands=synth.N_BANDS, width=synth.WIDTH,
                                           decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft3d(h.view(wl.B * wl.N, wl.D, wl.Z, wl.H, wl.W),
                                      out=H.view(wl.B * wl.N, wl.D, 2 * wl.Z, 2 * wl.H, wl.W))
            forward()
    elif wl.kind == "3d":
        h = torch.empty((wl.N, wl.D, wl.Z, wl.H, wl.W), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.N, wl.D, 2 * wl.Z, 2 * wl.H, wl.W), device="cuda", dtype=torch.complex64)
        ws_n = hyena.hyena_fftconv3d_workspace_size(wl.B, wl.D, wl.Z, wl.H, wl.W, wl.N, hyena.io_dtype(v), True)
        ws_fwd = torch.empty(ws_n, device="cuda", dtype=torch.uint8)

        def forward():
            hyena.hyena_fftconv3d_gate_forward(v, xs, b, Hs=H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen_3d(*W, wl.N, wl.D, wl.Z, wl.H, wl.W, n_bands=synth.N_BANDS,
                                      width=synth.WIDTH, decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft3d(h, out=H)
            forward()
    elif wl.kind == "2d" and wl.film:
        h = torch.empty((wl.B, wl.N, wl.D, wl.H, wl.W), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.B, wl.N, wl.D, 2 * wl.H, wl.W), device="cuda", dtype=torch.complex64)
        ws_n = hyena.hyena_fftconv2d_workspace_size(wl.B, wl.D, wl.H, wl.W, wl.N, hyena.io_dtype(v), True)
        ws_fwd = torch.empty(ws_n, device="cuda", dtype=torch.uint8)

        def forward():
            hyena.hyena_fftconv2d_gate_forward_per_sample(v, xs, b, H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen_film_2d(*W, wl.N, wl.D, wl.H, wl.W, B=wl.B, omega=F[0], gamma=F[1], beta=F[2],
                                           sigma=F[3], n_bands=synth.N_BANDS, width=synth.WIDTH,
                                           decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft2d(h.view(wl.B * wl.N, wl.D, wl.H, wl.W),
                                      out=H.view(wl.B * wl.N, wl.D, 2 * wl.H, wl.W))
            forward()
    elif wl.kind == "2d":
        h = torch.empty((wl.N, wl.D, wl.H, wl.W), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.N, wl.D, 2 * wl.H, wl.W), device="cuda", dtype=torch.complex64)
        ws_n = hyena.hyena_fftconv2d_workspace_size(wl.B, wl.D, wl.H, wl.W, wl.N, hyena.io_dtype(v), True)
        ws_fwd = torch.empty(ws_n, device="cuda", dtype=torch.uint8)

        def forward():
            hyena.hyena_fftconv2d_gate_forward(v, xs, b, Hs=H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen_2d(*W, wl.N, wl.D, wl.H, wl.W, n_bands=synth.N_BANDS,
                                      width=synth.WIDTH, decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft2d(h, out=H)
            forward()
    elif wl.film:
        h = torch.empty((wl.B, wl.N, wl.D, wl.L), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.B, wl.N, wl.D, wl.L), device="cuda", dtype=torch.complex64)
        ws_rfft_n = hyena.hyena_filter_rfft_workspace_size(wl.B * wl.N, wl.D, wl.L)
        ws_fwd_n = hyena.hyena_fftconv_workspace_size(wl.B, wl.D, wl.L, wl.N, hyena.io_dtype(v), True)
        ws_rfft = torch.empty(ws_rfft_n, device="cuda", dtype=torch.uint8) if ws_rfft_n else None
        ws_fwd = torch.empty(max(ws_fwd_n, 1), device="cuda", dtype=torch.uint8)

        def forward():
            hyena.hyena_fftconv_gate_forward_per_sample(v, xs, b, H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen_film(*W, wl.N, wl.D, wl.L, B=wl.B, omega=F[0], gamma=F[1], beta=F[2],
                                        sigma=F[3], n_bands=synth.N_BANDS, width=synth.WIDTH,
                                        decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft(h.view(wl.B * wl.N, wl.D, wl.L), out=H.view(wl.B * wl.N, wl.D, wl.L),
                                    workspace=ws_rfft)
            forward()
    else:
        h = torch.empty((wl.N, wl.D, wl.L), device="cuda", dtype=torch.float32)
        H = torch.empty((wl.N, wl.D, wl.L), device="cuda", dtype=torch.complex64)
        # workspaces (four-step scratch for L > 16384), allocated once
        ws_rfft_n = hyena.hyena_filter_rfft_workspace_size(wl.N, wl.D, wl.L)
        ws_fwd_n = hyena.hyena_fftconv_workspace_size(wl.B, wl.D, wl.L, wl.N, hyena.io_dtype(v), True)
        ws_rfft = torch.empty(ws_rfft_n, device="cuda", dtype=torch.uint8) if ws_rfft_n else None
        ws_fwd = torch.empty(ws_fwd_n, device="cuda", dtype=torch.uint8) if ws_fwd_n else None

        if spill:     # z spilled to HBM between orders, one launch per order
            ws_fwd = torch.empty(hyena.hyena_fftconv_spill_workspace_size(wl.B, wl.D, wl.L, wl.N),
                                 device="cuda", dtype=torch.uint8)

            def forward():
                hyena.hyena_fftconv_gate_forward_spill(v, xs, b, H, out=y, workspace=ws_fwd)
        else:
            def forward():
                hyena.hyena_fftconv_gate_forward(v, xs, b, H=H, out=y, workspace=ws_fwd)

        def step():
            hyena.hyena_filter_gen(*W, wl.N, wl.D, wl.L, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                   decay_div=synth.DECAY_DIV, out=h)
            hyena.hyena_filter_rfft(h, out=H, workspace=ws_rfft)
            forward()

    return step, forward, H


def run_e2e(args, wl: synth.Workload, inp: dict, bufs: "Buffers", step, max_over_ranks):
    """Milliseconds of args.steps end-to-end steps (pipelined over two
    buffer sets: H2D, compute and D2H on their own streams), and the H2D and
    D2H bytes of one step."""
    import torch
    io = bufs.v.dtype
    pin = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dt).pin_memory()
    hin = [pin(inp["v"], io), *[pin(x, io) for x in inp["x"]], pin(inp["b"]),
           *[pin(inp[k]) for k in WKEYS], *([pin(inp[k]) for k in FILM_KEYS] if wl.film else [])]
    hout = [torch.empty(bufs.y.shape, dtype=io).pin_memory() for _ in range(2)]
    sets = [(bufs, step)]
    bufs2 = Buffers(wl, inp)
    step2, _, _ = setup_step(wl, bufs2, spill=args.forward == "spill")
    sets.append((bufs2, step2))
    dins = [[s.v, *s.xs, s.b, *s.W, *s.F] for s, _ in sets]
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = hout[0].numel() * hout[0].element_size()
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)

    def run(nsteps: int):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        free_in = [None, None]    # compute done with the set's inputs
        free_out = [None, None]   # D2H done with the set's y
        torch.cuda.synchronize()
        start.record(s_cmp)
        s_in.wait_event(start)
        s_out.wait_event(start)
        last = None
        for i in range(nsteps):
            k = i % 2
            bf, stp = sets[k]
            with torch.cuda.stream(s_in):
                if free_in[k] is not None:
                    s_in.wait_event(free_in[k])
                for dst, src in zip(dins[k], hin):
                    dst.copy_(src, non_blocking=True)
                landed = ev()
                landed.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(landed)
                if free_out[k] is not None:
                    s_cmp.wait_event(free_out[k])
                stp()
                done = ev()
                done.record(s_cmp)
                free_in[k] = done
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                hout[k].copy_(bf.y, non_blocking=True)
                last = ev()
                last.record(s_out)
                free_out[k] = last
        s_cmp.wait_event(last)
        end.record(s_cmp)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    run(2)                                    # warm the second set and the streams
    ms = max_over_ranks(run(args.steps))
    del sets, bufs2, dins
    return ms, h2d, d2h


def has_spill(wl: synth.Workload) -> bool:
    """Workloads with a spill variant to compare against (1-D, shared
    spectra, padded, L <= 16384, more than one order)."""
    return wl.kind == "1d" and not wl.film and not wl.circular and wl.L <= 16384 and wl.N > 1


def has_noalloc_long(wl: synth.Workload) -> bool:
    """Workloads whose forward the no-workspace entry point runs on its
    built-in scratch (1-D, shared spectra, padded, 16384 < L <= 2^21)."""
    return wl.kind == "1d" and not wl.film and not wl.circular and 16384 < wl.L <= (1 << 21)


# the configurations whose forward is timed in the same run as the headline
# line (the parity configurations c0..c4 at their full sizes)
PER_CONFIG = ("c0", "c1", "c2_8k", "c2_16k", "c3_64k", "c3_256k", "c3_1m", "c4")


def per_config_forward(args, headline: synth.Workload, headline_ms: float, flush, gpu_id: str) -> dict:
    """Forward ms per call (CUDA events on the launching stream, L2 flushed
    before each call), algorithmic bytes and fraction of the HBM peak for
    every configuration, with the clocks sampled over the whole loop."""
    import torch
    peak, _ = peaks()
    stream = torch.cuda.current_stream()
    out = {}
    with ClockSampler(gpu_id) as clk:
        for name in PER_CONFIG:
            wl = synth.WORKLOADS[name]
            reps = 10 if wl.positions >= (1 << 26) else 20

            def timed(fn) -> float:
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(reps)]
                for a, b in evs:
                    flush.zero_()
                    a.record(stream)
                    fn()
                    b.record(stream)
                torch.cuda.synchronize()
                return statistics.mean(a.elapsed_time(b) for a, b in evs)

            spill_ms = noalloc_ms = None
            if wl == headline and not has_noalloc_long(wl):
                ms = headline_ms
            else:
                bufs = Buffers(wl, synth.make_inputs(wl))
                step, forward, H = setup_step(wl, bufs)
                for _ in range(3):
                    step()
                ms = headline_ms if wl == headline else timed(forward)
                if has_noalloc_long(wl):
                    # the same forward on the library's built-in 16 MB scratch
                    from subquadratic_sequence_b200 import hyena

                    def noalloc():
                        hyena.hyena_fftconv_gate_forward_noalloc(bufs.v, bufs.xs, bufs.b, H, out=bufs.y)
                    noalloc()
                    noalloc_ms = timed(noalloc)
                if has_spill(wl):
                    # the same forward with z spilled to HBM between orders
                    from subquadratic_sequence_b200 import hyena
                    ws = torch.empty(hyena.hyena_fftconv_spill_workspace_size(wl.B, wl.D, wl.L, wl.N),
                                     device="cuda", dtype=torch.uint8)

                    def spill():
                        hyena.hyena_fftconv_gate_forward_spill(bufs.v, bufs.xs, bufs.b, H, out=bufs.y,
                                                               workspace=ws)
                    spill()
                    spill_ms = timed(spill)
                    del ws
                del bufs, step, forward, H
                torch.cuda.empty_cache()
            nbytes = alg_bytes_forward(wl)
            out[name] = {"kernel": forward_kernel(wl), "ms_per_launch": ms, "alg_bytes_per_launch": nbytes,
                         "achieved_gbs": nbytes / (ms / 1e3) / 1e9, "frac": nbytes / (ms / 1e3) / 1e9 / peak,
                         "value": wl.positions / (ms / 1e3), "unit": UNIT}
            if noalloc_ms is not None:
                out[name]["noalloc"] = {
                    "kernel": "fourstep_col_kernel+fourstep_row_kernel (hyena_fftconv_gate_forward_noalloc, "
                              "16 MB built-in scratch)",
                    "ms_per_call": noalloc_ms, "frac": nbytes / (noalloc_ms / 1e3) / 1e9 / peak,
                    "slowdown": noalloc_ms / ms}
            if spill_ms is not None:
                moved = nbytes + 2 * (wl.N - 1) * wl.positions * 4
                out[name]["spill"] = {
                    "kernel": "fused1d_order_kernel x N (hyena_fftconv_gate_forward_spill)",
                    "ms_per_call": spill_ms, "frac": nbytes / (spill_ms / 1e3) / 1e9 / peak,
                    "bytes_moved_per_call": moved, "fused_speedup": spill_ms / ms}
    out["clocks"] = clk.summary()
    return out


def run_gpu(args, wl: synth.Workload) -> dict | None:
    import torch

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the path has no CPU fallback)")
    from subquadratic_sequence_b200 import hyena

    ranks = Ranks("nccl")
    world, rank, local = ranks.world, ranks.rank, ranks.local
    barrier, max_over_ranks = ranks.barrier, ranks.max

    inp = synth.make_inputs(wl)
    io = torch.bfloat16 if wl.io == "bf16" else torch.float32

    def to_dev(a, dtype=torch.float32):
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(dtype)

    bufs = Buffers(wl, inp)
    v, xs, b, y = bufs.v, bufs.xs, bufs.b, bufs.y
    flush = torch.empty(L2_FLUSH_BYTES, device="cuda", dtype=torch.uint8)
    stream = torch.cuda.current_stream()
    step, forward, H = setup_step(wl, bufs, spill=args.forward == "spill")
    launches_per_step = (launches_filter_gen(wl) + launches_rfft(wl)
                         + (wl.N if args.forward == "spill" else launches_forward(wl)))
    fwd_name = ("fused1d_order_kernel x N (hyena_fftconv_gate_forward_spill)" if args.forward == "spill"
                else forward_kernel(wl))

    # ---- warm-up
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed steps (device time; L2 flushed before each, outside the events)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    gpu_uuid = str(torch.cuda.get_device_properties(local).uuid)
    gpu_id = gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}"
    with ClockSampler(gpu_id) as clk:
        barrier()
        torch.cuda.synchronize()
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        wall = time.perf_counter() - t_wall
        # keep sampling clocks over the same work when the timed region was
        # shorter than a few samples
        t_end = time.perf_counter() + max(0.0, 1.5 - wall)
        while time.perf_counter() < t_end:
            for _ in range(20):
                flush.zero_()
                step()
            torch.cuda.synchronize()
    step_ms = [a.elapsed_time(bb) for a, bb in ev]
    total_ms = max_over_ranks(sum(step_ms))

    # ---- the dominant kernel alone: the fused forward, per launch
    fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(max(args.steps, 10))]
    step()
    for i in range(len(fev)):
        flush.zero_()
        fev[i][0].record(stream)
        forward()
        fev[i][1].record(stream)
    torch.cuda.synchronize()
    fwd_ms = max_over_ranks(statistics.mean(a.elapsed_time(bb) for a, bb in fev))

    # ---- end to end through the C ABI with host buffers: every step copies
    # its inputs from pinned host memory (H2D), runs the whole path and reads
    # its result back (D2H).  Steps run as a pipeline over two buffer sets on
    # three streams, as a stream of batches would be served: the H2D of step
    # i+1 and the D2H of step i-1 overlap the compute of step i.  Every copy
    # and launch lies inside the timed region.
    e2e_ms, h2d, d2h = run_e2e(args, wl, inp, bufs, step, max_over_ranks)

    # ---- the backward pass: one call per timed repetition
    bwd = None
    if wl.kind in ("1d", "2d", "3d"):
        dy = to_dev(synth.make_output_grad(wl), io)
        if wl.kind == "3d":
            size_fn = (hyena.hyena_fftconv3d_backward_circular_workspace_size if wl.circular
                       else hyena.hyena_fftconv3d_backward_per_sample_workspace_size if wl.film
                       else hyena.hyena_fftconv3d_backward_workspace_size)
            ws_b = torch.empty(size_fn(wl.B, wl.D, wl.Z, wl.H, wl.W, wl.N), device="cuda", dtype=torch.uint8)
            bwd_fn = (hyena.hyena_fftconv3d_gate_backward_circular if wl.circular
                      else hyena.hyena_fftconv3d_gate_backward_per_sample if wl.film
                      else hyena.hyena_fftconv3d_gate_backward)
            bwd_kernel = ("fft2d_bwd_row_kernel+fft2d_col_kernel+fft3d_bwd_z_kernel (" + bwd_fn.__name__ +
                          ", all launches)")

            def backward():
                bwd_fn(v, xs, b, H, dy, workspace=ws_b)
        elif wl.film and wl.kind == "2d":
            ws_b = torch.empty(hyena.hyena_fftconv2d_backward_per_sample_workspace_size(wl.B, wl.D, wl.H, wl.W,
                                                                                        wl.N),
                               device="cuda", dtype=torch.uint8)
            bwd_kernel = ("fft2d_bwd_row_kernel+fft2d_bwd_col_kernel (hyena_fftconv2d_gate_backward_per_sample, "
                          "all launches)")

            def backward():
                hyena.hyena_fftconv2d_gate_backward_per_sample(v, xs, b, H, dy, workspace=ws_b)
        elif wl.circular and wl.kind == "2d":
            ws_b = torch.empty(hyena.hyena_fftconv2d_backward_circular_workspace_size(wl.B, wl.D, wl.H, wl.W,
                                                                                      wl.N),
                               device="cuda", dtype=torch.uint8)
            bwd_kernel = ("fft2d_bwd_row_kernel+fft2d_bwd_col_kernel<PAD=false> "
                          "(hyena_fftconv2d_gate_backward_circular, all launches)")

            def backward():
                hyena.hyena_fftconv2d_gate_backward_circular(v, xs, b, H, dy, workspace=ws_b)
        elif wl.circular:
            ws_b = torch.empty(hyena.hyena_fftconv_backward_circular_workspace_size(wl.B, wl.D, wl.L, wl.N),
                               device="cuda", dtype=torch.uint8)
            bwd_kernel = ("fourstep_bwd_row_kernel+fourstep_bwd_col_kernel<PAD=false> "
                          "(hyena_fftconv_gate_backward_circular, all launches)" if long_path(wl) else
                          "backward1d_kernel<PAD=false> (hyena_fftconv_gate_backward_circular)")

            def backward():
                hyena.hyena_fftconv_gate_backward_circular(v, xs, b, H, dy, workspace=ws_b)
        elif wl.film:
            ws_b = torch.empty(hyena.hyena_fftconv_backward_per_sample_workspace_size(wl.B, wl.D, wl.L, wl.N),
                               device="cuda", dtype=torch.uint8)
            bwd_kernel = "backward1d_kernel<PS> (hyena_fftconv_gate_backward_per_sample)"

            def backward():
                hyena.hyena_fftconv_gate_backward_per_sample(v, xs, b, H, dy, workspace=ws_b)
        elif wl.kind == "2d":
            ws_b = torch.empty(hyena.hyena_fftconv2d_backward_workspace_size(wl.B, wl.D, wl.H, wl.W, wl.N),
                               device="cuda", dtype=torch.uint8)
            bwd_kernel = "fft2d_bwd_row_kernel+fft2d_bwd_col_kernel (hyena_fftconv2d_gate_backward, all launches)"

            def backward():
                hyena.hyena_fftconv2d_gate_backward(v, xs, b, H, dy, workspace=ws_b)
        else:
            ws_b = torch.empty(hyena.hyena_fftconv_backward_workspace_size(wl.B, wl.D, wl.L, wl.N),
                               device="cuda", dtype=torch.uint8)
            bwd_kernel = ("fourstep_bwd_row_kernel+fourstep_bwd_col_kernel (hyena_fftconv_gate_backward, "
                          "all launches)" if long_path(wl) else "backward1d_kernel (hyena_fftconv_gate_backward)")

            def backward():
                hyena.hyena_fftconv_gate_backward(v, xs, b, H, dy, workspace=ws_b)

        for _ in range(3):
            backward()
        bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(max(args.steps // 5, 5))]
        for i in range(len(bev)):
            flush.zero_()
            bev[i][0].record(stream)
            backward()
            bev[i][1].record(stream)
        torch.cuda.synchronize()
        bwd_ms = max_over_ranks(statistics.mean(a.elapsed_time(bb) for a, bb in bev))
        bwd = {"kernel": bwd_kernel, "ms_per_call": bwd_ms,
               "value": wl.positions * world / (bwd_ms / 1e3), "unit": UNIT,
               "alg_bytes_per_call": alg_bytes_backward(wl),
               "achieved_gbs": alg_bytes_backward(wl) / (bwd_ms / 1e3) / 1e9}

    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = per_config_forward(args, wl, fwd_ms, flush, gpu_id)

    ranks.close()
    if rank != 0:
        return None

    positions = wl.positions * world
    value = throughput(wl.positions, world, args.steps, total_ms)
    peak, peak_kind = peaks()
    achieved = alg_bytes_forward(wl) / (fwd_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": {**describe(wl), **({"forward": "spill: z in HBM between orders"}
                                                            if args.forward == "spill" else {})},
        "roofline": {"bound": "hbm", "kernel": fwd_name,
                     "achieved": achieved, "peak": peak, "peak_source": peak_kind,
                     "unit": "GB/s", "frac": achieved / peak,
                     "traffic": ncu_traffic(fwd_name.split()[0], wl.name),
                     "alg_bytes_per_launch": alg_bytes_forward(wl), "ms_per_launch": fwd_ms},
        "forward_only": {"value": wl.positions * world / (fwd_ms / 1e3), "unit": UNIT},
        "e2e": {"value": positions * args.steps / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if bwd is not None:
        bwd["frac"] = bwd["achieved_gbs"] / peak
        line["backward"] = bwd
    if per_config is not None:
        line["per_config"] = per_config
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_seconds)
    return line


# ------------------------------------------------------- oracle (CPU)

def oracle_sample(wl: synth.Workload, inp: dict, channels: np.ndarray, threads: int) -> float:
    """Seconds the oracle takes for the whole path (filter generation for the
    sampled channels, then the order-N forward by its FFT route) on all B
    batch elements of the sampled channels."""
    import oracle
    rows = np.concatenate([n * wl.D + channels for n in range(wl.N)])
    t0 = time.perf_counter()
    v = inp["v"][:, channels].astype(np.float64)
    x = np.stack([xx[:, channels] for xx in inp["x"]]).astype(np.float64)
    bias = inp["b"][:, channels].astype(np.float64)
    if wl.kind == "3d" and wl.film:
        h = oracle.filter_gen_film_3d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["omega"],
                                      inp["gamma"], inp["beta"], inp["sigma"][channels], True, wl.N,
                                      len(channels), wl.Z, wl.H, wl.W, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                      decay_div=synth.DECAY_DIV, threads=threads)
        oracle.hyena_forward_3d_per_sample(v, x, h, bias, route="fft")
        return time.perf_counter() - t0
    if wl.kind == "3d":
        h = oracle.filter_gen_3d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["alpha"][channels],
                                 wl.N, len(channels), wl.Z, wl.H, wl.W, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                 decay_div=synth.DECAY_DIV, threads=threads)
        if wl.circular:
            oracle.hyena_forward_circular_nd(v, x, h, bias, route="fft")
        else:
            oracle.hyena_forward_3d(v, x, h, bias, route="fft")
        return time.perf_counter() - t0
    if wl.circular and wl.kind == "2d":
        h = oracle.filter_gen_2d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["alpha"][channels],
                                 wl.N, len(channels), wl.H, wl.W, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                 decay_div=synth.DECAY_DIV, threads=threads)
        oracle.hyena_forward_circular_nd(v, x, h, bias, route="fft")
        return time.perf_counter() - t0
    if wl.circular:
        h = oracle.filter_gen(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["alpha"][channels],
                              wl.N, len(channels), wl.L, n_bands=synth.N_BANDS, width=synth.WIDTH,
                              decay_div=synth.DECAY_DIV, threads=threads)
        oracle.hyena_forward_circular(v, x, h, bias, route="fft", threads=threads)
        return time.perf_counter() - t0
    if wl.kind == "2d" and wl.film:
        h = oracle.filter_gen_film_2d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["omega"],
                                      inp["gamma"], inp["beta"], inp["sigma"][channels], True, wl.N,
                                      len(channels), wl.H, wl.W, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                      decay_div=synth.DECAY_DIV, threads=threads)
        oracle.hyena_forward_2d_per_sample(v, x, h, bias, route="fft", threads=threads)
        return time.perf_counter() - t0
    if wl.kind == "2d":
        h = oracle.filter_gen_2d(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["alpha"][channels],
                                 wl.N, len(channels), wl.H, wl.W, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                 decay_div=synth.DECAY_DIV, threads=threads)
        oracle.hyena_forward_2d(v, x, h, bias, route="fft", threads=threads)
        return time.perf_counter() - t0
    if wl.film:
        h = oracle.filter_gen_film(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["omega"],
                                   inp["gamma"], inp["beta"], inp["sigma"][channels], True, wl.N,
                                   len(channels), wl.L, n_bands=synth.N_BANDS, width=synth.WIDTH,
                                   decay_div=synth.DECAY_DIV, threads=threads)
        oracle.hyena_forward_per_sample(v, x, h, inp["b"][:, channels].astype(np.float64), route="fft",
                                        threads=threads)
        return time.perf_counter() - t0
    h = oracle.filter_gen(inp["W1"], inp["W2"], inp["W3"], inp["Wout"][rows], inp["alpha"][channels],
                          wl.N, len(channels), wl.L, n_bands=synth.N_BANDS, width=synth.WIDTH,
                          decay_div=synth.DECAY_DIV, threads=threads)
    oracle.hyena_forward(v, x, h, inp["b"][:, channels].astype(np.float64), route="fft",
                         threads=threads)
    return time.perf_counter() - t0


def extent(wl: synth.Workload) -> str:
    if wl.kind == "3d":
        return f"{wl.Z}x{wl.H}x{wl.W}"
    if wl.kind == "2d":
        return f"{wl.H}x{wl.W}"
    return f"L={wl.L}"


def one_thread(wl: synth.Workload) -> bool:
    """The 3-D oracle and the circular 2-D/3-D oracle are single-threaded."""
    return wl.kind == "3d" or (wl.circular and wl.kind == "2d")


def stages(wl: synth.Workload) -> str:
    circ = "circular " if wl.circular else ""
    if wl.kind == "3d":
        return f"3-D filter generation (all cores) + order-{wl.N} {circ}forward (one thread)"
    if one_thread(wl):
        return f"filter generation (all cores) + order-{wl.N} {circ}forward (one thread)"
    if wl.circular:
        return f"filter generation + order-{wl.N} circular forward"
    return f"filter generation + order-{wl.N} forward"


def cpu_baseline(wl: synth.Workload, budget_s: float = 15.0, inp: dict | None = None) -> dict:
    import oracle
    inp = inp or synth.make_inputs(wl)
    threads = oracle.default_threads()
    rng = np.random.default_rng(0)
    n = 1 if one_thread(wl) else max(1, min(wl.D, threads))   # the N-D oracles below run on one thread
    t = oracle_sample(wl, inp, np.sort(rng.choice(wl.D, n, replace=False)), threads)
    # grow the sample to about budget_s of CPU work
    n2 = int(min(wl.D, max(n, n * budget_s / max(t, 1e-3))))
    if n2 > n:
        n = n2
        t = oracle_sample(wl, inp, np.sort(rng.choice(wl.D, n, replace=False)), threads)
    positions = wl.B * n * wl.per_channel
    cores = threads
    return {"value": positions / t, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} of {wl.D} channels x all {wl.B} batch elements x {extent(wl)} "
                      f"({stages(wl)}, float64 FFT route), {t:.1f} s"}


def run_reference(args, wl: synth.Workload) -> dict | None:
    """The reference arm: the float64 CPU oracle, each step a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import oracle
    inp = synth.make_inputs(wl)
    threads = oracle.default_threads()
    rng = np.random.default_rng(0)
    n = 1 if one_thread(wl) else max(1, min(wl.D, threads))   # the N-D oracles below run on one thread
    probe = oracle_sample(wl, inp, np.sort(rng.choice(wl.D, n, replace=False)), threads)
    # size each step so that warm-up + timed steps end within ~2 minutes
    per_step_budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(wl.D, max(1, n * per_step_budget / max(probe, 1e-3))))
    chans = [np.sort(rng.choice(wl.D, n, replace=False)) for _ in range(args.steps + args.warmup)]
    for i in range(args.warmup):
        oracle_sample(wl, inp, chans[i], threads)
    total = sum(oracle_sample(wl, inp, chans[args.warmup + i], threads) for i in range(args.steps))
    positions = wl.B * n * wl.per_channel
    value = positions * args.steps / total
    sample = (f"{n} of {wl.D} channels x all {wl.B} batch elements x {extent(wl)} per step "
              f"({stages(wl)}, float64 FFT route)")

    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {**describe(wl), **({"forward": "spill: z in HBM between orders"}
                                                            if args.forward == "spill" else {})},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_dft32(args) -> dict:
    """One radix-32 FFT level on the FP32 pipes and on the tensor cores
    (hyena_dft32_stage): device time per level per point, L2-resident input
    (each vector is read once and transformed `reps` times)."""
    import torch
    from subquadratic_sequence_b200 import hyena
    count, reps = 148 * 2 * 128 * 4, 64
    rng = np.random.default_rng(5)
    x = torch.from_numpy((rng.standard_normal((count, 32)) + 1j * rng.standard_normal((count, 32)))
                         .astype(np.complex64)).cuda()
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    out = {"experiment": "one radix-32 FFT level: FP32 pipes vs tcgen05 tensor cores (3xTF32)",
           "vectors": count, "reps": reps, "points_per_level": count * 32}
    for method, name in ((0, "simt"), (1, "tcgen05_3xtf32")):
        for _ in range(3):
            hyena.hyena_dft32_stage(x, reps, method, out=y)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
        for a, b in evs:
            a.record(stream)
            hyena.hyena_dft32_stage(x, reps, method, out=y)
            b.record(stream)
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        out[name] = {"ms_per_call": ms, "ps_per_point_per_level": ms * 1e9 / (count * 32 * reps)}
    out["simt_speedup"] = out["tcgen05_3xtf32"]["ms_per_call"] / out["simt"]["ms_per_call"]
    out["device_faults"] = hyena.LIB.hyena_device_fault_count()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c3_1m", choices=list(synth.WORKLOADS))
    ap.add_argument("--channels", type=int, default=0,
                    help="run the workload with this many channels instead (small profiling cases)")
    ap.add_argument("--forward", default="fused", choices=["fused", "spill"],
                    help="spill: the forward that writes z to HBM between orders (L <= 16384)")
    ap.add_argument("--experiment", choices=["dft32"], default=None,
                    help="dft32: time one radix-32 FFT level on the FP32 pipes and on the tensor cores")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the forward timing of every configuration")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("bench.py: at least 3 warm-up steps are required")
    if args.experiment == "dft32":
        print(json.dumps(run_dft32(args)), flush=True)
        return
    wl = synth.WORKLOADS[args.workload]
    if args.forward == "spill" and not has_spill(wl):
        raise SystemExit(f"bench.py: {wl.name} has no spill variant (1-D, shared spectra, L <= 16384, N > 1)")
    if args.channels:
        wl = wl.with_(D=args.channels, name=f"{wl.name}_D{args.channels}")
        args.no_per_config = True
    line = run_reference(args, wl) if args.impl == "reference" else run_gpu(args, wl)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
