#!/usr/bin/env python3
"""Benchmark of the selective-scan hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-extra] [--no-cpu-baseline]

One step = the Mamba-1 selective scan forward + backward over one batch of the
Mamba-2.8B-layer-shaped workload (bf16 storage, f32 accumulation; batch 4,
d_inner 5120, d_state 16, L 4096, final state returned), inputs resident in
HBM.  Metric:
tokens*channels per second (B*L*D per step / step time), whole job over all
ranks.  Under torchrun each rank runs its own batch (independent problems, no
data-path collective: weak scaling); timing is taken with CUDA events on the
launching stream, bracketed by a barrier and a synchronize, max over ranks.

The JSON line also carries: the roofline of the dominant launch (algorithmic
bytes / measured duration vs the measured HBM copy bandwidth), the e2e figure
(the same step through the C ABI starting from pinned host buffers, copies
inside the timed region), the compute ceiling of the Mamba-1 kernels (their
2^x count over the SFU rate measured by the library's probe in the same run),
the CPU oracle timed on a bounded sample, SM clocks sampled during the timed
region, and per-workload figures for the other workloads (130M-layer-shaped
Mamba-1, Mamba-3 SISO, decode steps, conv, discretisation).

--impl reference runs the f64 CPU oracle (the reference arm of this build) on a
bounded sample of the same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_14_b200 import workloads as W  # noqa: E402

METRIC = "selective-scan tokens·channels/s (fwd+bwd) and achieved HBM GB/s vs ~8 TB/s peak"
UNIT = "tokens*channels/s"
HEADLINE = "m1_bf16_b4_d5120_n16_l4096"
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


# ---------------------------------------------------------------------------
# algorithmic bytes (inputs read once + outputs written once)
# ---------------------------------------------------------------------------
def m1_bytes(Bsz, D, N, L, io_bytes, G=1):
    tc = Bsz * D * L
    bt = Bsz * G * L
    params = D * N * 4 + 2 * D * 4
    fwd = 4 * io_bytes * tc + 2 * N * io_bytes * bt + params + Bsz * D * N * 4  # x,dt,z,out; B,C; final
    bwd = 7 * io_bytes * tc + 2 * N * io_bytes * bt + 2 * N * 4 * bt + params + D * N * 4 + 2 * D * 4
    return fwd, bwd


def m1_sfu_ops(Bsz, D, N, L):
    """SFU operations of the Mamba-1 kernels: one 2^x per state element and
    step (its decay; the backward recomputes it once), plus per token the
    forward's softplus (2^x and a reciprocal or logarithm) and silu gate
    (2^x and a reciprocal), and the backward's softplus, sigmoid of the gate
    and sigmoid of the delta pre-activation (two each)."""
    tc = Bsz * D * L
    return tc * (N + 4), tc * (N + 6)


def m3_bytes(Bsz, L, H, P, N, G, K, io_bytes):
    tc = Bsz * L * H * P
    th = Bsz * L * H
    bt = Bsz * L * G
    fwd = 3 * io_bytes * tc + (3 + K) * io_bytes * th + 2 * N * io_bytes * bt + Bsz * H * P * N * 4
    bwd = (5 * io_bytes * tc + (3 + K) * io_bytes * th + 2 * N * io_bytes * bt
           + (3 + K) * 4 * th + 2 * N * 4 * bt + H * 4)
    return fwd, bwd


def su_bytes(Bsz, D, N, io_bytes, G=1):
    return Bsz * D * (2 * N * 4 + 4 * io_bytes) + 2 * Bsz * G * N * io_bytes


def m3su_bytes(Bsz, H, P, N, G, K, io_bytes):
    """One Mamba-3 decode step: the carried state, last input, last rotated key
    and angles read and written (f32); x, z, out, alpha, beta, gamma, theta per
    (b, h) and B, C per (b, g) in io."""
    per_head = 2 * 4 * (P * N + P + N + K) + io_bytes * (3 * P + 3 + K)
    return Bsz * H * per_head + 2 * Bsz * G * N * io_bytes


def m3su_raw_bytes(Bsz, H, P, N, G, K, io_bytes):
    """The Mamba-3 decode step from raw values: the plain step's bytes with
    alpha, beta, gamma, theta per (b, h) and the normalised B, C replaced by
    dd_dt, dd_a, trap per (b, h), the angles per b and the raw B, C (same
    size); dt_bias is small."""
    return (m3su_bytes(Bsz, H, P, N, G, K, io_bytes) - Bsz * H * (3 + K) * io_bytes
            + Bsz * H * 3 * io_bytes + Bsz * K * io_bytes)


# ---------------------------------------------------------------------------
# DRAM traffic of the dominant kernel from an ncu capture (dram__bytes_read.sum
# + dram__bytes_write.sum, one launch of the named workload), valid only for
# the kernel source it was taken on: reported when the source file's hash
# still matches, else null.
# ---------------------------------------------------------------------------
NCU_TRAFFIC = {
    # kernel source file: (sha256 prefix of the file, workload, bytes per launch)
    "m1_bwd.cu": ("aa9e576ab0269254", "m1_bf16_b4_d5120_n16_l4096", 1350000000 + 592440000),
    "m1_fwd.cu": ("cb6f1bfb350b55cd", "m1_bf16_b4_d5120_n16_l4096", 505620000 + 792910000),
}


def ncu_traffic(src_name, workload):
    import hashlib
    ent = NCU_TRAFFIC.get(src_name)
    if ent is None or ent[1] != workload:
        return None
    path = os.path.join(ROOT, "selective_state_space_14_b200", "csrc", src_name)
    try:
        with open(path, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return ent[2] if digest.startswith(ent[0]) else None


# ---------------------------------------------------------------------------
# clocks sampling
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and throttle reasons of one GPU, polled through NVML every
    ``period_s`` from a thread while the timed region runs (read-only)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index, period_s=0.002):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self.err = None
        self._stop = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 -- no NVML: report it, keep the run
            self.nvml = None
            self.err = f"nvml unavailable: {e}"[:120]

    def _poll(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, rs))
            except Exception as e:  # noqa: BLE001
                self.err = str(e)[:120]
                return
            time.sleep(self.period)

    def start(self):
        if self.nvml is None:
            return
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def stop(self):
        if self.nvml is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=[self.err])
        self._stop.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return dict(sm_mhz=None, sm_max_mhz=self.max_mhz, reasons=["no samples"])
        reasons = sorted({name for _, rs in self.samples for name, bit in self.REASONS.items()
                          if rs & bit})
        return dict(sm_mhz=statistics.median(s for s, _ in self.samples), sm_max_mhz=self.max_mhz,
                    reasons=reasons, samples=len(self.samples))


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; no data-path collective)
# ---------------------------------------------------------------------------
def dist_init(n_gpus, backend="nccl"):
    """Rank, world size and local rank from the launcher's environment; one
    process group (short timeout) when there is more than one rank."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch one process per GPU")
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value, device="cuda"):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def to_dev(t):
    import torch
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return torch.from_numpy(np.ascontiguousarray(t, dtype=np.float32)).cuda()
    if t.dtype == "bf16":
        return torch.from_numpy(t.data.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(t.data).cuda()


def to_pinned(t):
    import torch
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return torch.from_numpy(np.ascontiguousarray(t, dtype=np.float32)).pin_memory()
    if t.dtype == "bf16":
        return torch.from_numpy(t.data.view(np.int16)).view(torch.bfloat16).pin_memory()
    return torch.from_numpy(t.data).pin_memory()


class M1Step:
    """Device-resident Mamba-1 fwd+bwd step with all buffers preallocated."""

    def __init__(self, p, msc):
        import torch
        self.msc = msc
        self.p = p
        self.a = dict(u=to_dev(p.u), delta=to_dev(p.delta), A=to_dev(p.A), B=to_dev(p.B),
                      C=to_dev(p.C), D=to_dev(p.D), delta_bias=to_dev(p.delta_bias),
                      z=to_dev(p.z), h0=None, delta_softplus=p.delta_softplus)
        self.dout = to_dev(p.dout)
        u = self.a["u"]
        Bsz, D, L, N, G = p.batch, p.dim, p.seqlen, p.dstate, p.ngroups
        f32 = dict(device="cuda", dtype=torch.float32)
        self.out = torch.empty_like(u)
        self.fs = torch.empty((Bsz, D, N), **f32)
        self.saved = torch.empty((Bsz, D, (L + msc.MSC_M1_SAVE_INTERVAL - 1) // msc.MSC_M1_SAVE_INTERVAL, N), **f32)
        self.grads = dict(du=torch.empty_like(u), ddelta=torch.empty_like(u), dz=torch.empty_like(u),
                          dA=torch.empty((D, N), **f32), dB=torch.empty((Bsz, G, N, L), **f32),
                          dC=torch.empty((Bsz, G, N, L), **f32), dD=torch.empty((D,), **f32),
                          ddelta_bias=torch.empty((D,), **f32), dh0=None)
        self.ws = torch.empty(max(msc.msc_selective_scan_bwd_workspace_bytes(Bsz, D, N, L, G), 16),
                              device="cuda", dtype=torch.uint8)

    def fwd(self):
        self.msc.msc_selective_scan_fwd(**self.a, out=self.out, final_state=self.fs,
                                        saved_states=self.saved)

    def bwd(self):
        self.msc.msc_selective_scan_bwd(**self.a, saved_states=self.saved, dout=self.dout,
                                        workspace=self.ws, grads=self.grads, want_dh0=False)


class M1ConvStep:
    """Device-resident causal conv1d + Mamba-1 scan: the fused forward, the
    unfused forward (conv, then scan), and the two backward calls."""

    def __init__(self, q, msc):
        import torch
        self.msc = msc
        self.q = q
        self.st = M1Step(q.scan, msc)  # its u is the conv's input x
        self.x = self.st.a["u"]
        self.w, self.bias = to_dev(q.w), to_dev(q.bias)
        self.u = torch.empty_like(self.x)
        Bsz, D = q.scan.batch, q.scan.dim
        self.xs = torch.empty((Bsz, D, q.width - 1), device="cuda", dtype=torch.float32)
        self.scan_a = {k: v for k, v in self.st.a.items() if k != "u"}
        self.cws = torch.empty(max(msc.msc_causal_conv1d_bwd_workspace_bytes(
            Bsz, D, q.scan.seqlen, q.width), 16), device="cuda", dtype=torch.uint8)
        self.cgrads = None

    def fused_fwd(self):
        """One launch: u = silu(conv(x)) feeds the scan in shared memory (u is
        also written out for the backward pass)."""
        self.msc.msc_selective_scan_conv_fwd(
            self.x, self.w, conv_bias=self.bias, **self.scan_a, u_out=self.u,
            conv_state_out=self.xs, out=self.st.out, final_state=self.st.fs,
            saved_states=self.st.saved)

    def conv_fwd(self):
        self.msc.msc_causal_conv1d_fwd(self.x, self.w, bias=self.bias, u=self.u,
                                       conv_state_out=self.xs)

    def scan_fwd(self):
        self.msc.msc_selective_scan_fwd(u=self.u, **self.scan_a, out=self.st.out,
                                        final_state=self.st.fs, saved_states=self.st.saved)

    def scan_bwd(self):
        self.msc.msc_selective_scan_bwd(u=self.u, **self.scan_a, saved_states=self.st.saved,
                                        dout=self.st.dout, workspace=self.st.ws,
                                        grads=self.st.grads, want_dh0=False)

    def conv_bwd(self):
        self.cgrads = self.msc.msc_causal_conv1d_bwd(
            self.x, self.w, self.st.grads["du"], bias=self.bias, workspace=self.cws,
            grads=self.cgrads)


class M3DiscStep:
    """Device-resident Mamba-3 step from the raw projections: discretisation
    and BCNorm, the scan forward and backward, the discretisation backward."""

    def __init__(self, q, msc):
        import torch
        self.msc, self.q = msc, q
        s = q.scan
        self.raw = dict(dd_dt=to_dev(q.dd_dt), dd_a=to_dev(q.dd_a), trap=to_dev(q.trap),
                        angles=to_dev(q.angles), B_raw=to_dev(q.B_raw), C_raw=to_dev(q.C_raw))
        self.kw = dict(dt_bias=to_dev(q.dt_bias), A_floor=q.A_floor, eps=q.eps)
        self.o = msc.msc_mamba3_siso_discretize(**self.raw, **self.kw)
        self.a = dict(x=to_dev(s.x), B=self.o["B"], C=self.o["C"], alpha=self.o["alpha"],
                      beta=self.o["beta"], gamma=self.o["gamma"], theta=self.o["theta"],
                      D=to_dev(s.D), z=to_dev(s.z), h0=None)
        self.dout = to_dev(s.dout)
        self.out, _, self.saved = msc.msc_mamba3_siso_scan_fwd(**self.a)
        self.ws = torch.empty(max(msc.msc_mamba3_siso_scan_bwd_workspace_bytes(
            s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.nangles), 16),
            device="cuda", dtype=torch.uint8)
        self.gs = msc.msc_mamba3_siso_scan_bwd(**self.a, saved_states=self.saved, dout=self.dout,
                                               workspace=self.ws)
        self.gd = None
        self.disc_bwd()
        # the same step through the fused entry points (the derived inputs are
        # made inside the scan's kernels and never stored)
        self.c = dict(x=self.a["x"], D=self.a["D"], z=self.a["z"], h0=None)
        self.ws_f = torch.empty(max(msc.msc_mamba3_siso_scan_fwd_raw_workspace_bytes(
            s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.nangles), 16),
            device="cuda", dtype=torch.uint8)
        self.out_r, _, self.saved_r = msc.msc_mamba3_siso_scan_fwd_raw(
            **self.c, **self.raw, **self.kw, workspace=self.ws_f)
        self.ws_r = torch.empty(max(msc.msc_mamba3_siso_scan_bwd_raw_workspace_bytes(
            s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.nangles), 16),
            device="cuda", dtype=torch.uint8)
        self.gr = None
        self.fused_bwd()

    def fused_fwd(self):
        self.msc.msc_mamba3_siso_scan_fwd_raw(**self.c, **self.raw, **self.kw, out=self.out_r,
                                              saved_states=self.saved_r, workspace=self.ws_f)

    def fused_bwd(self):
        self.gr = self.msc.msc_mamba3_siso_scan_bwd_raw(
            **self.c, **self.raw, **self.kw, saved_states=self.saved_r, dout=self.dout,
            workspace=self.ws_r, grads=self.gr)

    def disc_fwd(self):
        self.msc.msc_mamba3_siso_discretize(**self.raw, **self.kw, outs=self.o)

    def scan_fwd(self):
        self.msc.msc_mamba3_siso_scan_fwd(**self.a, out=self.out, saved_states=self.saved)

    def scan_bwd(self):
        self.msc.msc_mamba3_siso_scan_bwd(**self.a, saved_states=self.saved, dout=self.dout,
                                          workspace=self.ws, grads=self.gs)

    def disc_bwd(self):
        g = self.gs
        self.gd = self.msc.msc_mamba3_siso_discretize_bwd(
            **self.raw, dalpha=g["dalpha"], dbeta=g["dbeta"], dgamma=g["dgamma"],
            dtheta=g["dtheta"], dB=g["dB"], dC=g["dC"], **self.kw, grads=self.gd)


def m3disc_bytes(Bsz, L, H, N, G, K, io_bytes):
    """Algorithmic HBM bytes of the discretisation: forward reads dd_dt, dd_a,
    trap, angles, B_raw, C_raw and writes alpha, beta, gamma, theta, B, C (io);
    backward reads the raw inputs (io) and the f32 upstream gradients, writes
    f32 gradients of the raw inputs."""
    tok = Bsz * L
    raw = tok * (3 * H + K + 2 * G * N) * io_bytes
    fwd = raw + tok * (3 * H + H * K + 2 * G * N) * io_bytes
    bwd = raw + tok * (3 * H + H * K + 2 * G * N) * 4 + tok * (3 * H + K + 2 * G * N) * 4
    return fwd, bwd


def conv_bytes(Bsz, D, L, W, io_bytes):
    """Algorithmic HBM bytes of the standalone conv: forward reads x, writes u;
    backward reads x and du, writes dx (weights, states and the per-run dw
    partials are small and left out)."""
    n = Bsz * D * L * io_bytes
    return 2 * n, 3 * n


def graphed(fn):
    """fn captured once in a CUDA graph; returns its replay.  For launches
    shorter than the Python binding's host time, so that CUDA events measure
    the device, not the gaps between launches.  fn must allocate nothing."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g.replay


def time_steps(step_fns, steps, warmup, world, sampler=None):
    """Run warmup, then time `steps` iterations; per-phase CUDA-event times.
    A clock sampler, if given, runs during the timed region only."""
    import torch
    for _ in range(warmup):
        for f in step_fns:
            f()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(step_fns) + 1)]
          for _ in range(steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if sampler is not None:
        sampler.start()
    start.record(stream)
    for k in range(steps):
        ev[k][0].record(stream)
        for i, f in enumerate(step_fns):
            f()
            ev[k][i + 1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.clocks = sampler.stop()
    barrier(world)
    total_ms = start.elapsed_time(end)
    phase_ms = [sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps)) / steps
                for i in range(len(step_fns))]
    return total_ms, phase_ms


def measure_rates(msc, reps=3):
    """The SFU's 2^x rate and the FMA pipe's (scalar and packed) on this GPU,
    from the library's probes: 8 CTAs of 256 threads per SM, best of ``reps``
    CUDA-event timed launches after one warm-up (a burst rate, like the
    measured copy bandwidth the HBM fraction divides by)."""
    import torch
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    blocks = props.multi_processor_count * 8
    out = torch.empty(blocks * int(msc.lib().msc_probe_threads_per_block()), device="cuda",
                      dtype=torch.float32)
    stream = torch.cuda.current_stream()
    rates = {}
    for kind, iters in (("ex2", 2048), ("ffma", 16384), ("ffma2", 8192)):
        msc.msc_probe(kind, out, blocks, iters)
        best = None
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ops = msc.msc_probe(kind, out, blocks, iters)
            b.record(stream)
            b.synchronize()
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
        rates[kind] = ops / (best / 1e3)
    return dict(sfu_ex2_per_s=round(rates["ex2"], 1), ffma_per_s=round(rates["ffma"], 1),
                ffma2_elem_per_s=round(rates["ffma2"], 1), sms=props.multi_processor_count,
                how="libmsc probes: 8 CTAs x 256 threads per SM, 8 independent chains per "
                    "thread, best of 3 CUDA-event timed launches")


def cpu_baseline(budget_s=12.0):
    """The f64 oracle (as it stands) on a bounded sample of the headline workload:
    batch row 0 (all its channels, all steps), forward + backward, repeated for
    about ``budget_s`` seconds."""
    import oracle
    p = W.make(HEADLINE)
    nch = p.dim
    sub = W.M1Problem(1, nch, p.dstate, p.seqlen, 1, p.io, p.delta_softplus,
                      W.Tensor(p.io, p.u.data[:1, :nch]), W.Tensor(p.io, p.delta.data[:1, :nch]),
                      p.A[:nch], W.Tensor(p.io, p.B.data[:1]), W.Tensor(p.io, p.C.data[:1]),
                      p.D[:nch], p.delta_bias[:nch], W.Tensor(p.io, p.z.data[:1, :nch]), None,
                      W.Tensor(p.io, p.dout.data[:1, :nch]))
    args = oracle.m1_problem_args(sub)
    dout = sub.dout.as_f64()
    threads = oracle.default_threads()
    reps, t_total = 0, 0.0
    while t_total < budget_s and reps < 1000:
        t0 = time.perf_counter()
        oracle.m1_fwd(**args, nthreads=threads)
        oracle.m1_bwd(dout=dout, **args, nthreads=threads)
        t_total += time.perf_counter() - t0
        reps += 1
    units = nch * p.seqlen * reps
    # one host thread, forward only, on the first 128 channels of the same row
    few = {k: (v[:, :128] if k in ("u", "delta", "z") else
               v[:128] if k in ("A", "D", "delta_bias") else v) for k, v in args.items()}
    t0 = time.perf_counter()
    oracle.m1_fwd(**few, nthreads=1)
    t1 = time.perf_counter() - t0
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            model = next((ln.split(":", 1)[1].strip() for ln in f if ln.startswith("model name")),
                         "")
    except OSError:
        pass
    return dict(value=units / t_total, unit=UNIT, cores=threads, kind="oracle",
                sample=f"batch row 0, channels 0..{nch - 1}, L={p.seqlen}, fwd+bwd, {reps} reps, "
                       f"{t_total:.1f} s",
                fwd_1thread=dict(value=round(128 * p.seqlen / t1, 1), unit=UNIT,
                                 sample=f"batch row 0, channels 0..127, L={p.seqlen}, fwd only"),
                cpu_model=model)


def _rate(fn, budget_s):
    """Calls of fn per second over about budget_s seconds (at least one call)."""
    reps, t = 0, 0.0
    while reps == 0 or (t < budget_s and reps < 1000):
        t0 = time.perf_counter()
        fn()
        t += time.perf_counter() - t0
        reps += 1
    return reps / t, reps, t


def oracle_beside(res, budget_s=1.5):
    """The f64 oracle, as it stands, timed on the host beside each extra
    workload, on a bounded sample (stated): one row or sequence of the
    workload's shape drawn with its generator and distributions, in the
    workload's unit."""
    import oracle
    f64 = lambda a: None if a is None else np.asarray(a, np.float64)
    thr = oracle.default_threads()
    BF = "bf16"

    def put(name, units_per_call, fn, sample):
        if name not in res or "error" in res[name]:
            return
        r, reps, t = _rate(fn, budget_s)
        res[name]["oracle"] = dict(value=round(units_per_call * r, 1), unit=res[name]["unit"],
                                   cores=thr, kind="oracle",
                                   sample=f"{sample}; {reps} reps, {t:.1f} s")

    # Mamba-1, 130M-layer rows: one batch row of 256 channels, L 2048, fwd+bwd
    p = W.m1_problem(1, 256, 16, 2048, io=BF, bias=True)
    a = oracle.m1_problem_args(p)
    dout = p.dout.as_f64()
    put("m1_bf16_b8_d1536_n16_l2048", 256 * 2048,
        lambda: (oracle.m1_fwd(**a), oracle.m1_bwd(dout=dout, **a)),
        "one batch row of 256 channels, L 2048, fwd+bwd")
    # Mamba-1 decode: 64 channels of one sequence, 10 steps
    q = W.su_problem(1, 64, 16, n_pool=10)
    steps = [{k: v.as_f64() for k, v in s_.items()} for s_ in q.steps]

    def su():
        st = q.state0.astype(np.float64)
        for s_ in steps:
            st, _ = oracle.ssm_state_update(st, s_["x"], s_["delta"], f64(q.A), s_["B"], s_["C"],
                                            D=f64(q.D), delta_bias=f64(q.delta_bias), z=s_["z"])
    put("su_bf16_b256_d5120_n16_x1000", 64 * 10, su, "64 channels of one sequence, 10 steps")
    # Mamba-3 SISO: one sequence, one head (P64 N64 K32), L 2048, fwd+bwd
    m3 = W.m3_problem(1, 2048, 1, 64, 64, nangles=32, io=BF)
    ms = oracle.m3_problem_args(m3)
    mdout = m3.dout.as_f64()
    put("m3_bf16_b8_h24_p64_n64_k32_l2048", 2048 * 64,
        lambda: (oracle.m3_fwd(**ms), oracle.m3_bwd(dout=mdout, **ms)),
        "one sequence, one head, L 2048, fwd+bwd")
    # Mamba-3 decode: one sequence (24 heads), 10 steps
    q3 = W.m3su_problem(1, 24, 64, 64, nangles=32, n_pool=10)
    st3 = [{k: v.as_f64() for k, v in s_.items()} for s_ in q3.steps]

    def su3():
        c = [v.astype(np.float64) for v in (q3.state0, q3.x_prev0, q3.bt_prev0, q3.phi0)]
        for s_ in st3:
            *c, _ = oracle.m3_state_update(*c, *[s_[k] for k in ("x", "B", "C", "alpha", "beta",
                                                                "gamma", "theta")],
                                           D=f64(q3.D), z=s_["z"])
    put("m3su_bf16_b256_h24_p64_n64_k32_x1000", 24 * 64 * 10, su3,
        "one sequence (24 heads), 10 steps")
    # the same decode from raw values: the oracle's discretisation of the token
    # (values rounded to bf16 as stored) ahead of its step
    raw_steps, rdtb = W.m3su_raw_steps(1, 24, 64, nangles=32, n_pool=10)
    rsteps = [{k: v.as_f64()[:, None] for k, v in s_.items()} for s_ in raw_steps]

    def su3_raw():
        c = [v.astype(np.float64) for v in (q3.state0, q3.x_prev0, q3.bt_prev0, q3.phi0)]
        for s_, r_ in zip(st3, rsteps):
            d_ = oracle.m3_discretize(**r_, dt_bias=f64(rdtb), A_floor=1e-4, eps=1e-5)
            d_ = {k: W.store(v[:, 0].astype(np.float32), BF).as_f64() for k, v in d_.items()}
            *c, _ = oracle.m3_state_update(*c, s_["x"], d_["B"], d_["C"], d_["alpha"], d_["beta"],
                                           d_["gamma"], d_["theta"], D=f64(q3.D), z=s_["z"])
    put("m3su_raw_bf16_b256_h24_p64_n64_k32_x1000", 24 * 64 * 10, su3_raw,
        "one sequence (24 heads), 10 steps from raw values")
    # Mamba-3 from raw projections: one sequence; the discretisation fwd+bwd of
    # all 24 heads and the scan fwd+bwd of one head, per token-channel of one head
    d = W.m3disc_problem(1, 2048, 24, 64, 64, nangles=32, io=BF)
    raw = {k: getattr(d, k).as_f64() for k in ("dd_dt", "dd_a", "trap", "angles", "B_raw",
                                                "C_raw")}
    kw = dict(dt_bias=f64(d.dt_bias), A_floor=d.A_floor, eps=d.eps)
    rng = np.random.default_rng(0)
    up = dict(dalpha=rng.standard_normal((1, 2048, 24)), dbeta=rng.standard_normal((1, 2048, 24)),
              dgamma=rng.standard_normal((1, 2048, 24)),
              dtheta=rng.standard_normal((1, 2048, 24, 32)),
              dB=rng.standard_normal((1, 2048, 1, 64)), dC=rng.standard_normal((1, 2048, 1, 64)))
    name = "m3disc_bf16_b8_h24_p64_n64_k32_l2048"
    if name in res and "error" not in res[name]:
        # seconds per token-channel: the discretisation's share (all 24 heads)
        # plus one head's scan
        rd, nd, td = _rate(lambda: (oracle.m3_discretize(**raw, **kw),
                                    oracle.m3_discretize_bwd(**raw, **up, **kw)), budget_s)
        rs, ns, ts = _rate(lambda: (oracle.m3_fwd(**ms), oracle.m3_bwd(dout=mdout, **ms)),
                           budget_s)
        per = 1.0 / (rd * 24 * 2048 * 64) + 1.0 / (rs * 2048 * 64)
        res[name]["oracle"] = dict(
            value=round(1.0 / per, 1), unit=res[name]["unit"], cores=thr, kind="oracle",
            sample=f"one sequence: discretisation fwd+bwd of its 24 heads ({nd} reps, {td:.1f} s) "
                   f"and scan fwd+bwd of one head ({ns} reps, {ts:.1f} s), combined per "
                   f"token-channel")
    # conv + Mamba-1 scan: one batch row of 128 channels, conv and scan fwd+bwd
    c = W.m1conv_problem(1, 128, 16, 2048)
    cs = oracle.m1_problem_args(c.scan)
    cx, cw, cb = cs["u"], f64(c.w), f64(c.bias)
    cdout = c.scan.dout.as_f64()

    def conv_step():
        u, _ = oracle.conv1d_fwd(cx, cw, bias=cb)
        sa = dict(cs, u=u)
        oracle.m1_fwd(**sa)
        g = oracle.m1_bwd(dout=cdout, **sa)
        oracle.conv1d_bwd(cx, cw, g["du"], bias=cb)
    put("m1conv_bf16_b8_d1536_n16_l2048_w4", 128 * 2048, conv_step,
        "one batch row of 128 channels, conv fwd+bwd and scan fwd+bwd")


def run_e2e(p, msc, steps, warmup, world):
    """The step through the C ABI from pinned host buffers, pipelined the way a
    training input pipeline runs: every step copies its inputs host to device
    and every gradient and the output back, inside the timed region, with the
    uploads of step k+1 and the downloads of step k-1 overlapping the compute
    of step k (three streams, two device buffer sets)."""
    import torch
    sets = [M1Step(p, msc), M1Step(p, msc)]
    host_in = dict(u=to_pinned(p.u), delta=to_pinned(p.delta), z=to_pinned(p.z), B=to_pinned(p.B),
                   C=to_pinned(p.C), dout=to_pinned(p.dout))
    dev_in = [dict(u=st.a["u"], delta=st.a["delta"], z=st.a["z"], B=st.a["B"], C=st.a["C"],
                   dout=st.dout) for st in sets]
    outs = [[st.out] + [v for v in st.grads.values() if v is not None] for st in sets]
    host_out = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in os_] for os_ in outs]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(o.numel() * o.element_size() for o in host_out[0])
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_comp + ev_out:
        e.record(comp)

    def run(n):
        for k in range(n):
            i = k % 2
            s_in.wait_event(ev_comp[i])  # set i's last compute no longer reads its inputs
            with torch.cuda.stream(s_in):
                for name, v in host_in.items():
                    dev_in[i][name].copy_(v, non_blocking=True)
                ev_in[i].record(s_in)
            comp.wait_event(ev_in[i])
            comp.wait_event(ev_out[i])  # set i's last results have left the device
            sets[i].fwd()
            sets[i].bwd()
            ev_comp[i].record(comp)
            s_out.wait_event(ev_comp[i])
            with torch.cuda.stream(s_out):
                for d, hbuf in zip(outs[i], host_out[i]):
                    hbuf.copy_(d, non_blocking=True)
                ev_out[i].record(s_out)

    run(warmup)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    run(steps)
    for e in ev_out:
        comp.wait_event(e)  # the timed region ends when the last results are on the host
    end.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(world, start.elapsed_time(end))
    return total_ms / steps, h2d, d2h


def run_ours(args):
    import torch
    world, rank, local = dist_init(args.gpus)
    torch.cuda.set_device(local)
    from selective_state_space_14_b200 import msc
    msc.lib()
    peaks = load_peaks()
    p = W.make(HEADLINE, shard=rank)  # each rank its own batch of the same shape
    st = M1Step(p, msc)
    sampler = ClockSampler(local)
    total_ms, (fwd_ms, bwd_ms) = time_steps([st.fwd, st.bwd], args.steps, args.warmup, world,
                                            sampler=sampler)
    clocks = sampler.clocks
    total_ms = max_over_ranks(world, total_ms)
    ms_per_step = total_ms / args.steps
    units = p.token_channels
    value = units * world / (ms_per_step / 1e3)
    fwd_b, bwd_b = m1_bytes(p.batch, p.dim, p.dstate, p.seqlen, 2)
    dom = "bwd" if bwd_ms >= fwd_ms else "fwd"
    dom_ms, dom_b = (bwd_ms, bwd_b) if dom == "bwd" else (fwd_ms, fwd_b)
    achieved = dom_b / (dom_ms / 1e3) / 1e9
    # the compute side: the kernels' 2^x count over the measured SFU rate
    rates = measure_rates(msc)
    fwd_ops, bwd_ops = m1_sfu_ops(p.batch, p.dim, p.dstate, p.seqlen)
    sfu = rates["sfu_ex2_per_s"]

    def compute(ops, ms):
        floor_ms = ops / sfu * 1e3
        return dict(bound="sfu", sfu_ops=ops, floor_ms=round(floor_ms, 4),
                    achieved_ops_per_s=round(ops / (ms / 1e3), 1), peak_ops_per_s=sfu,
                    frac=round(floor_ms / ms, 4))
    compute_fwd, compute_bwd = compute(fwd_ops, fwd_ms), compute(bwd_ops, bwd_ms)
    roofline = dict(bound="hbm", achieved=round(achieved, 1), peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=round(achieved / peaks["hbm_gbs"], 4),
                    traffic=ncu_traffic("m1_bwd.cu" if dom == "bwd" else "m1_fwd.cu", HEADLINE),
                    kernel=("msc_selective_scan_bwd (m1_bwd_kernel + m1_bwd_reduce_kernel)"
                            if dom == "bwd" else "msc_selective_scan_fwd (m1_fwd_kernel)"),
                    algorithmic_bytes=dom_b, launch_ms=round(dom_ms, 4),
                    peak_source=peaks["source"],
                    compute=compute_bwd if dom == "bwd" else compute_fwd)
    e2e_ms, h2d, d2h = run_e2e(p, msc, max(2, args.steps // 2), 3, world)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": HEADLINE, "batch": p.batch, "d_inner": p.dim, "d_state": p.dstate,
                   "seq_len": p.seqlen, "io": "bf16 storage, f32 accumulation",
                   "parallelism": f"independent batch per rank x{world}",
                   "l2": "per-step working set > 126 MB L2 (inputs larger than L2)"},
        "phases_ms": {"fwd": round(fwd_ms, 4), "bwd": round(bwd_ms, 4)},
        "achieved_gbs": {"fwd": round(fwd_b / fwd_ms / 1e6, 1), "bwd": round(bwd_b / bwd_ms / 1e6, 1)},
        "hbm_frac": {"fwd": round(fwd_b / fwd_ms / 1e6 / peaks["hbm_gbs"], 4),
                     "bwd": round(bwd_b / bwd_ms / 1e6 / peaks["hbm_gbs"], 4)},
        "compute_frac": {"fwd": compute_fwd["frac"], "bwd": compute_bwd["frac"]},
        "compute": {"fwd": compute_fwd, "bwd": compute_bwd},
        "rates": rates,
        "roofline": roofline,
        "e2e": {"value": round(units * world / (e2e_ms / 1e3), 1), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "pipeline": "uploads of step k+1 and downloads of step k-1 overlap step k"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if not args.no_extra:
        args.sfu_rate = rates["sfu_ex2_per_s"]
        line["workloads"] = extra_workloads(msc, args, world, peaks)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            oracle_beside(line["workloads"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def extra_workloads(msc, args, world, peaks):
    """Per-workload figures beside the headline (each timed like the headline)."""
    import torch
    res = {}
    # Mamba-130M-layer-shaped Mamba-1 scan (bf16, B8 D1536 N16 L2048)
    name = "m1_bf16_b8_d1536_n16_l2048"
    p = W.make(name)
    st = M1Step(p, msc)
    total_ms, (fwd_ms, bwd_ms) = time_steps([st.fwd, st.bwd], max(3, args.steps), 3, world)
    fb, bb = m1_bytes(p.batch, p.dim, p.dstate, p.seqlen, 2)
    fo, bo = m1_sfu_ops(p.batch, p.dim, p.dstate, p.seqlen)
    sfu = getattr(args, "sfu_rate", None)
    res[name] = dict(
        fwd_ms=round(fwd_ms, 4), bwd_ms=round(bwd_ms, 4),
        value=round(p.token_channels / ((fwd_ms + bwd_ms) / 1e3), 1), unit=UNIT,
        fwd_hbm_frac=round(fb / fwd_ms / 1e6 / peaks["hbm_gbs"], 4),
        bwd_hbm_frac=round(bb / bwd_ms / 1e6 / peaks["hbm_gbs"], 4),
        bwd_traffic=ncu_traffic("m1_bwd.cu", name))
    if sfu:
        res[name]["fwd_compute_frac"] = round(fo / sfu / (fwd_ms / 1e3), 4)
        res[name]["bwd_compute_frac"] = round(bo / sfu / (bwd_ms / 1e3), 4)
    del st
    torch.cuda.empty_cache()
    # decode step (B256 D5120 N16, 1000 consecutive steps cycling 8 input sets)
    q = W.make("su_bf16_b256_d5120_n16_x1000")
    state = torch.from_numpy(q.state0).cuda()
    A, Dp, bias = to_dev(q.A), to_dev(q.D), to_dev(q.delta_bias)
    pool = [{k: to_dev(v) for k, v in s.items()} for s in q.steps]
    outs = [torch.empty_like(pool[0]["x"]) for _ in range(8)]

    def decode_1000():
        for t in range(1000):
            s = pool[t % 8]
            msc.msc_ssm_state_update(state, s["x"], s["delta"], A, s["B"], s["C"], D=Dp,
                                     delta_bias=bias, z=s["z"], out=outs[t % 8])

    total_ms, (ms,) = time_steps([decode_1000], 2, 1, world)
    sb = su_bytes(q.batch, q.dim, q.dstate, 2)
    res["su_bf16_b256_d5120_n16_x1000"] = dict(
        ms_per_1000_steps=round(ms, 3), us_per_step=round(ms, 3),
        value=round(q.batch * q.dim * 1000 / (ms / 1e3), 1), unit="channel-steps/s",
        hbm_frac=round(sb * 1000 / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        note="84 MB state can stay L2-resident between steps")
    # Mamba-3 SISO decode step (B256 H24 P64 N64 K32, 1000 steps cycling 8 input sets)
    q3 = W.make("m3su_bf16_b256_h24_p64_n64_k32_x1000")
    carried = [torch.from_numpy(v).cuda() for v in (q3.state0, q3.x_prev0, q3.bt_prev0, q3.phi0)]
    D3 = to_dev(q3.D)
    pool3 = [{k: to_dev(v) for k, v in s.items()} for s in q3.steps]
    outs3 = [torch.empty_like(pool3[0]["x"]) for _ in range(8)]

    def m3_decode_1000():
        for t in range(1000):
            s = pool3[t % 8]
            msc.msc_mamba3_siso_state_update(*carried, s["x"], s["B"], s["C"], s["alpha"],
                                             s["beta"], s["gamma"], s["theta"], D=D3, z=s["z"],
                                             out=outs3[t % 8])

    total_ms, (ms,) = time_steps([m3_decode_1000], 2, 1, world)
    sb3 = m3su_bytes(q3.batch, q3.nheads, q3.headdim, q3.dstate, q3.ngroups, q3.nangles, 2)
    res["m3su_bf16_b256_h24_p64_n64_k32_x1000"] = dict(
        ms_per_1000_steps=round(ms, 3), us_per_step=round(ms, 3),
        value=round(q3.batch * q3.nheads * q3.headdim * 1000 / (ms / 1e3), 1),
        unit="token-channel steps/s",
        hbm_frac=round(sb3 * 1000 / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        note="101 MB state: most of it can stay in the 126 MB L2 between steps")
    # the same decode from raw values: the discretisation fused into the step,
    # against the discretisation kernel (one token) followed by the plain step
    raw_steps, dtb = W.m3su_raw_steps(q3.batch, q3.nheads, q3.dstate, nangles=q3.nangles)
    rawd = [{k: to_dev(v) for k, v in s_.items()} for s_ in raw_steps]
    dtb_d = to_dev(dtb)
    one = lambda t: t.view(t.shape[0], 1, *t.shape[1:])
    disc_out = msc.msc_mamba3_siso_discretize(one(rawd[0]["dd_dt"]), one(rawd[0]["dd_a"]),
                                              one(rawd[0]["trap"]), one(rawd[0]["angles"]),
                                              one(rawd[0]["B_raw"]), one(rawd[0]["C_raw"]),
                                              dt_bias=dtb_d)
    sq = {k: v[:, 0] for k, v in disc_out.items()}

    def m3_decode_raw_1000():
        for t in range(1000):
            r = rawd[t % 8]
            msc.msc_mamba3_siso_disc_state_update(
                *carried, pool3[t % 8]["x"], r["dd_dt"], r["dd_a"], r["trap"], r["angles"],
                r["B_raw"], r["C_raw"], dt_bias=dtb_d, D=D3, z=pool3[t % 8]["z"],
                out=outs3[t % 8])

    def m3_decode_raw_unfused_1000():
        for t in range(1000):
            r = rawd[t % 8]
            msc.msc_mamba3_siso_discretize(one(r["dd_dt"]), one(r["dd_a"]), one(r["trap"]),
                                           one(r["angles"]), one(r["B_raw"]), one(r["C_raw"]),
                                           dt_bias=dtb_d, outs=disc_out)
            msc.msc_mamba3_siso_state_update(*carried, pool3[t % 8]["x"], sq["B"], sq["C"],
                                             sq["alpha"], sq["beta"], sq["gamma"], sq["theta"],
                                             D=D3, z=pool3[t % 8]["z"], out=outs3[t % 8])

    _, (ms_f,) = time_steps([m3_decode_raw_1000], 2, 1, world)
    _, (ms_u,) = time_steps([m3_decode_raw_unfused_1000], 2, 1, world)
    rb3 = m3su_raw_bytes(q3.batch, q3.nheads, q3.headdim, q3.dstate, q3.ngroups, q3.nangles, 2)
    res["m3su_raw_bf16_b256_h24_p64_n64_k32_x1000"] = dict(
        us_per_step=round(ms_f, 3), unfused_us_per_step=round(ms_u, 3),
        value=round(q3.batch * q3.nheads * q3.headdim * 1000 / (ms_f / 1e3), 1),
        unit="token-channel steps/s",
        hbm_frac=round(rb3 * 1000 / (ms_f / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        note="decode from raw dd_dt, dd_a, trap, angles, B_raw, C_raw: the discretisation "
             "fused into the step vs its own kernel ahead of the plain step")
    del carried, pool3, outs3
    torch.cuda.empty_cache()
    # Mamba-3 SISO
    try:
        m3 = W.make("m3_bf16_b8_h24_p64_n64_k32_l2048")
        a = dict(x=to_dev(m3.x), B=to_dev(m3.B), C=to_dev(m3.C), alpha=to_dev(m3.alpha),
                 beta=to_dev(m3.beta), gamma=to_dev(m3.gamma), theta=to_dev(m3.theta),
                 D=to_dev(m3.D), z=to_dev(m3.z), h0=None)
        dout = to_dev(m3.dout)
        holder = {}

        def f3():
            holder["o"] = msc.msc_mamba3_siso_scan_fwd(**a, out=holder.get("out"),
                                                       saved_states=holder.get("saved"))
            holder["out"], holder["saved"] = holder["o"][0], holder["o"][2]

        f3()
        ws = torch.empty(max(msc.msc_mamba3_siso_scan_bwd_workspace_bytes(
            m3.batch, m3.seqlen, m3.nheads, m3.headdim, m3.dstate, m3.ngroups, m3.nangles), 16),
            device="cuda", dtype=torch.uint8)
        grads = msc.msc_mamba3_siso_scan_bwd(**a, saved_states=holder["saved"], dout=dout,
                                             workspace=ws)

        def b3():
            msc.msc_mamba3_siso_scan_bwd(**a, saved_states=holder["saved"], dout=dout,
                                         workspace=ws, grads=grads)

        total_ms, (f_ms, b_ms) = time_steps([f3, b3], max(3, args.steps // 2), 3, world)
        fb, bb = m3_bytes(m3.batch, m3.seqlen, m3.nheads, m3.headdim, m3.dstate, m3.ngroups,
                          m3.nangles, 2)
        res["m3_bf16_b8_h24_p64_n64_k32_l2048"] = dict(
            fwd_ms=round(f_ms, 4), bwd_ms=round(b_ms, 4),
            value=round(m3.token_channels / ((f_ms + b_ms) / 1e3), 1), unit=UNIT,
            fwd_hbm_frac=round(fb / f_ms / 1e6 / peaks["hbm_gbs"], 4),
            bwd_hbm_frac=round(bb / b_ms / 1e6 / peaks["hbm_gbs"], 4))
    except Exception as e:  # noqa: BLE001 -- report, keep the headline line
        res["m3_bf16_b8_h24_p64_n64_k32_l2048"] = dict(error=str(e)[:200])
    torch.cuda.empty_cache()
    # Mamba-3 from the raw projections: discretisation + BCNorm around the scan
    name = "m3disc_bf16_b8_h24_p64_n64_k32_l2048"
    try:
        ds = M3DiscStep(W.make(name), msc)
        n = max(3, args.steps // 2)
        _, (dfw, sfw, sbw, dbw) = time_steps([graphed(ds.disc_fwd), ds.scan_fwd, ds.scan_bwd,
                                              graphed(ds.disc_bwd)], n, 3, world)
        _, (ffw, fbw) = time_steps([ds.fused_fwd, ds.fused_bwd], n, 3, world)
        s = ds.q.scan
        fb, bb = m3disc_bytes(s.batch, s.seqlen, s.nheads, s.dstate, s.ngroups, s.nangles, 2)
        res[name] = dict(
            fused_fwd_ms=round(ffw, 4), fused_bwd_ms=round(fbw, 4),
            disc_fwd_ms=round(dfw, 4), scan_fwd_ms=round(sfw, 4), scan_bwd_ms=round(sbw, 4),
            disc_bwd_ms=round(dbw, 4),
            value=round(s.token_channels / ((ffw + fbw) / 1e3), 1), unit=UNIT,
            unfused_value=round(s.token_channels / ((dfw + sfw + sbw + dbw) / 1e3), 1),
            disc_fwd_hbm_frac=round(fb / dfw / 1e6 / peaks["hbm_gbs"], 4),
            disc_bwd_hbm_frac=round(bb / dbw / 1e6 / peaks["hbm_gbs"], 4),
            note="value: scan forward + backward from raw projections (fused entry points); "
                 "unfused_value: discretisation + scan forward + scan backward + "
                 "discretisation backward as four calls")
        del ds
    except Exception as e:  # noqa: BLE001 -- report, keep the headline line
        res[name] = dict(error=str(e)[:200])
    torch.cuda.empty_cache()
    # causal conv1d (width 4) + SiLU ahead of the Mamba-1 scan, the headline's sizes
    name = "m1conv_bf16_b8_d1536_n16_l2048_w4"
    try:
        q = W.make(name)
        cs = M1ConvStep(q, msc)
        cs.fused_fwd()
        cs.scan_bwd()
        cs.conv_bwd()
        n = max(3, args.steps // 2)
        _, (fused_ms, sbwd_ms, cbwd_ms) = time_steps([cs.fused_fwd, cs.scan_bwd,
                                                      graphed(cs.conv_bwd)], n, 3, world)
        _, (conv_ms, sfwd_ms) = time_steps([graphed(cs.conv_fwd), cs.scan_fwd], n, 3, world)
        sp = q.scan
        fb, _ = m1_bytes(sp.batch, sp.dim, sp.dstate, sp.seqlen, 2)
        cfb, cbb = conv_bytes(sp.batch, sp.dim, sp.seqlen, q.width, 2)
        res[name] = dict(
            fused_fwd_ms=round(fused_ms, 4), unfused_fwd_ms=round(conv_ms + sfwd_ms, 4),
            conv_fwd_ms=round(conv_ms, 4), scan_fwd_ms=round(sfwd_ms, 4),
            scan_bwd_ms=round(sbwd_ms, 4), conv_bwd_ms=round(cbwd_ms, 4),
            value=round(sp.token_channels / ((fused_ms + sbwd_ms + cbwd_ms) / 1e3), 1),
            unit=UNIT,
            fused_fwd_hbm_frac=round((fb + sp.batch * sp.dim * sp.seqlen * 2) / fused_ms / 1e6
                                     / peaks["hbm_gbs"], 4),
            conv_fwd_hbm_frac=round(cfb / conv_ms / 1e6 / peaks["hbm_gbs"], 4),
            conv_bwd_hbm_frac=round(cbb / cbwd_ms / 1e6 / peaks["hbm_gbs"], 4),
            note="value: fused forward + scan backward + conv backward")
        del cs
    except Exception as e:  # noqa: BLE001 -- report, keep the headline line
        res[name] = dict(error=str(e)[:200])
    return res


# ---------------------------------------------------------------------------
# one phase alone (for profilers): launches only that phase's kernels
# ---------------------------------------------------------------------------
def run_only(args):
    """``--only PHASE``: the named phase of ``--workload`` (default: the headline
    Mamba-1 workload, or the Mamba-3 one for m3 phases), ``warmup`` untimed and
    ``steps`` timed launches; prints one JSON line with the per-launch time.  Not
    a bench line: the setup launches (e.g. the forward whose saved states a
    backward needs) run before the warm-up."""
    import torch
    from selective_state_space_14_b200 import msc
    msc.lib()
    phase = args.only
    if phase in ("m1_fwd", "m1_bwd"):
        p = W.make(args.workload or HEADLINE)
        st = M1Step(p, msc)
        st.fwd()
        fn = st.fwd if phase == "m1_fwd" else st.bwd
        units = p.token_channels
    elif phase in ("m3_fwd", "m3_bwd"):
        m3 = W.make(args.workload or "m3_bf16_b8_h24_p64_n64_k32_l2048")
        a = dict(x=to_dev(m3.x), B=to_dev(m3.B), C=to_dev(m3.C), alpha=to_dev(m3.alpha),
                 beta=to_dev(m3.beta), gamma=to_dev(m3.gamma), theta=to_dev(m3.theta),
                 D=to_dev(m3.D), z=to_dev(m3.z), h0=None)
        dout = to_dev(m3.dout)
        out, _, saved = msc.msc_mamba3_siso_scan_fwd(**a)
        ws = torch.empty(max(msc.msc_mamba3_siso_scan_bwd_workspace_bytes(
            m3.batch, m3.seqlen, m3.nheads, m3.headdim, m3.dstate, m3.ngroups, m3.nangles), 16),
            device="cuda", dtype=torch.uint8)
        grads = msc.msc_mamba3_siso_scan_bwd(**a, saved_states=saved, dout=dout, workspace=ws)
        if phase == "m3_fwd":
            def fn():
                msc.msc_mamba3_siso_scan_fwd(**a, out=out, saved_states=saved)
        else:
            def fn():
                msc.msc_mamba3_siso_scan_bwd(**a, saved_states=saved, dout=dout, workspace=ws,
                                             grads=grads)
        units = m3.token_channels
    elif phase in ("m3_disc_fwd", "m3_disc_bwd", "m3_raw_fwd", "m3_raw_bwd"):
        ds = M3DiscStep(W.make(args.workload or "m3disc_bf16_b8_h24_p64_n64_k32_l2048"), msc)
        fn = {"m3_disc_fwd": ds.disc_fwd, "m3_disc_bwd": ds.disc_bwd, "m3_raw_fwd": ds.fused_fwd,
              "m3_raw_bwd": ds.fused_bwd}[phase]
        units = ds.q.scan.token_channels
    elif phase in ("m1_conv_fwd", "conv_fwd", "conv_bwd"):
        q = W.make(args.workload or "m1conv_bf16_b8_d1536_n16_l2048_w4")
        cs = M1ConvStep(q, msc)
        cs.fused_fwd()
        cs.scan_bwd()
        cs.conv_bwd()
        fn = {"m1_conv_fwd": cs.fused_fwd, "conv_fwd": cs.conv_fwd, "conv_bwd": cs.conv_bwd}[phase]
        units = q.scan.token_channels
    elif phase == "m3_decode_raw":
        q = W.make(args.workload or "m3su_bf16_b256_h24_p64_n64_k32_x1000")
        carried = [torch.from_numpy(v).cuda() for v in (q.state0, q.x_prev0, q.bt_prev0, q.phi0)]
        D3 = to_dev(q.D)
        s = {k: to_dev(v) for k, v in q.steps[0].items()}
        raw_steps, dtb = W.m3su_raw_steps(q.batch, q.nheads, q.dstate, nangles=q.nangles)
        r = {k: to_dev(v) for k, v in raw_steps[0].items()}
        dtb_d = to_dev(dtb)
        out = torch.empty_like(s["x"])

        def fn():
            msc.msc_mamba3_siso_disc_state_update(*carried, s["x"], r["dd_dt"], r["dd_a"],
                                                  r["trap"], r["angles"], r["B_raw"], r["C_raw"],
                                                  dt_bias=dtb_d, D=D3, z=s["z"], out=out)
        units = q.batch * q.nheads * q.headdim
    elif phase == "m3_decode":
        q = W.make(args.workload or "m3su_bf16_b256_h24_p64_n64_k32_x1000")
        carried = [torch.from_numpy(v).cuda() for v in (q.state0, q.x_prev0, q.bt_prev0, q.phi0)]
        D3 = to_dev(q.D)
        s = {k: to_dev(v) for k, v in q.steps[0].items()}
        out = torch.empty_like(s["x"])

        def fn():
            msc.msc_mamba3_siso_state_update(*carried, s["x"], s["B"], s["C"], s["alpha"],
                                             s["beta"], s["gamma"], s["theta"], D=D3, z=s["z"],
                                             out=out)
        units = q.batch * q.nheads * q.headdim
    else:  # decode
        q = W.make(args.workload or "su_bf16_b256_d5120_n16_x1000")
        state = torch.from_numpy(q.state0).cuda()
        A, Dp, bias = to_dev(q.A), to_dev(q.D), to_dev(q.delta_bias)
        s = {k: to_dev(v) for k, v in q.steps[0].items()}
        out = torch.empty_like(s["x"])

        def fn():
            msc.msc_ssm_state_update(state, s["x"], s["delta"], A, s["B"], s["C"], D=Dp,
                                     delta_bias=bias, z=s["z"], out=out)
        units = q.batch * q.dim
    torch.cuda.synchronize()
    if args.graph:
        fn = graphed(fn)
    total_ms, (ms,) = time_steps([fn], args.steps, args.warmup, 1)
    print(json.dumps({"only": phase, "workload": args.workload, "ms_per_launch": round(ms, 5),
                      "units_per_s": round(units / (ms / 1e3), 1)}), flush=True)


# ---------------------------------------------------------------------------
# reference arm: the f64 CPU oracle
# ---------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    p = W.make(HEADLINE)
    nch = 256  # channels of batch row 0 per step: a step is ~50 ms of oracle work
    sub = W.M1Problem(1, nch, p.dstate, p.seqlen, 1, p.io, p.delta_softplus,
                      W.Tensor(p.io, p.u.data[:1, :nch]), W.Tensor(p.io, p.delta.data[:1, :nch]),
                      p.A[:nch], W.Tensor(p.io, p.B.data[:1]), W.Tensor(p.io, p.C.data[:1]),
                      p.D[:nch], p.delta_bias[:nch], W.Tensor(p.io, p.z.data[:1, :nch]), None,
                      W.Tensor(p.io, p.dout.data[:1, :nch]))
    a = oracle.m1_problem_args(sub)
    dout = sub.dout.as_f64()
    threads = oracle.default_threads()
    for _ in range(args.warmup):
        oracle.m1_fwd(**a, nthreads=threads)
        oracle.m1_bwd(dout=dout, **a, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.m1_fwd(**a, nthreads=threads)
        oracle.m1_bwd(dout=dout, **a, nthreads=threads)
    dt = time.perf_counter() - t0
    units = nch * p.seqlen * args.steps
    value = units / dt
    sample = f"batch row 0, channels 0..{nch - 1} of {HEADLINE}, fwd+bwd per step"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE, "sample": sample},
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["m1_fwd", "m1_bwd", "m3_fwd", "m3_bwd", "decode",
                                       "m3_decode", "m1_conv_fwd", "conv_fwd", "conv_bwd",
                                       "m3_disc_fwd", "m3_disc_bwd", "m3_raw_fwd", "m3_raw_bwd",
                                       "m3_decode_raw"],
                    help="time one phase alone (for profiling); prints no bench line")
    ap.add_argument("--workload", default=None, help="workload name for --only")
    ap.add_argument("--graph", action="store_true",
                    help="with --only: replay the launch from a CUDA graph (device time alone)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.only:
        run_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
