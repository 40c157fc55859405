"""Seeded synthetic inputs for the selective-scan library and for its oracle.

This module is the one piece shared by the CUDA path's tests/benchmark and the
f64 oracle.  It draws random tensors and rounds them to the storage dtype; it
holds none of the scan's arithmetic.  The only transforms applied here are the
input *distributions* the workloads are defined with:

* Mamba-1: x, z, B, C, D, dout ~ N(0,1); delta_raw = 0.5*N(0,1) - 2 (softplus is
  applied by the scan, not here); A[c, n] = -exp(log(n + 1)); the delta bias of
  the model-shaped workloads ~ U(ln 1e-3, ln 1e-1), the "targeted range" the
  state-spaces/mamba README ("Troubleshooting / Initialization") describes.
* Mamba-3 SISO: x, z, dout ~ N(0,1); B, C ~ N(0,1) then RMS-normalised over
  d_state (the BCNorm stage that precedes the scan in the mamba-rs 0.4.2
  ``Mamba3Scratch`` stage list, B5); alpha = exp(-softplus(N(0,1))); beta,
  gamma ~ U(0, 0.5); theta (per-step rotation angle increments) ~ U(0, 0.1);
  D ~ N(0,1) per head.

Values are drawn in float32 from numpy's PCG64 with a fixed seed and rounded
to the io dtype with round-to-nearest-even.  ``as_f64`` widens the rounded
values, so the GPU path and the oracle see bit-identical inputs.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np

SEED_BASE = 20261202

F32 = "f32"
BF16 = "bf16"
F16 = "f16"


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round-to-nearest-even.

    The sum below fits in 32 bits for every finite value and every infinity
    (the largest pattern, 0xFF800000, plus 0x8000 stays below 2^32); only NaN
    payloads near 0xFFFFFFFF would wrap, and the generators draw none."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    bits = f.view(np.uint32)
    r = (bits >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += bits
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Tensor:
    """A stored tensor: its io dtype and its payload.

    ``data`` is float32 for f32 tensors, uint16 bit patterns for bf16 and
    float16 for f16 (IEEE binary16, numpy's round-to-nearest-even cast).
    """

    dtype: str
    data: np.ndarray

    @property
    def shape(self):
        return self.data.shape

    def as_f32(self) -> np.ndarray:
        if self.dtype == BF16:
            return bf16_bits_to_f32(self.data)
        if self.dtype == F16:
            return self.data.astype(np.float32)
        return self.data

    def as_f64(self) -> np.ndarray:
        return self.as_f32().astype(np.float64)

    @property
    def nbytes(self) -> int:
        return self.data.nbytes


def store(x: np.ndarray, dtype: str) -> Tensor:
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == BF16:
        return Tensor(BF16, round_to_bf16_bits(x))
    if dtype == F32:
        return Tensor(F32, x)
    if dtype == F16:
        return Tensor(F16, x.astype(np.float16))
    raise ValueError(dtype)


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _uniform(rng, lo, hi, shape):
    return (lo + (hi - lo) * rng.random(size=shape, dtype=np.float32)).astype(np.float32)


# --------------------------------------------------------------------------
# Mamba-1 selective scan
# --------------------------------------------------------------------------
@dataclass
class M1Problem:
    batch: int
    dim: int
    dstate: int
    seqlen: int
    ngroups: int
    io: str
    delta_softplus: bool
    u: Tensor
    delta: Tensor
    A: np.ndarray            # float32 [D, N]
    B: Tensor                # [B, G, N, L]
    C: Tensor                # [B, G, N, L]
    D: Optional[np.ndarray]  # float32 [D]
    delta_bias: Optional[np.ndarray]  # float32 [D]
    z: Optional[Tensor]
    h0: Optional[np.ndarray]  # float32 [B, D, N]
    dout: Tensor
    meta: Dict[str, object] = field(default_factory=dict)

    @property
    def token_channels(self) -> int:
        return self.batch * self.dim * self.seqlen


def m1_problem(batch, dim, dstate, seqlen, io=F32, seed=SEED_BASE, ngroups=1,
               bias=False, with_z=True, with_D=True, with_h0=False,
               delta_softplus=True) -> M1Problem:
    """Mamba-1 scan inputs.

    bias=False follows the small parity workload (no delta bias);
    bias=True follows the model-shaped workloads (bias ~ U(ln 1e-3, ln 1e-1)).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    Bsz, D, N, L, G = batch, dim, dstate, seqlen, ngroups
    u = store(_normal(rng, (Bsz, D, L)), io)
    delta = store(0.5 * _normal(rng, (Bsz, D, L)) - 2.0, io)
    z = store(_normal(rng, (Bsz, D, L)), io) if with_z else None
    Bm = store(_normal(rng, (Bsz, G, N, L)), io)
    Cm = store(_normal(rng, (Bsz, G, N, L)), io)
    A = np.ascontiguousarray(
        np.broadcast_to(-np.exp(np.log(np.arange(1, N + 1, dtype=np.float64))), (D, N))
    ).astype(np.float32)
    Dp = _normal(rng, (D,)) if with_D else None
    db = _uniform(rng, np.log(1e-3), np.log(1e-1), (D,)) if bias else None
    h0 = _normal(rng, (Bsz, D, N)) if with_h0 else None
    dout = store(_normal(rng, (Bsz, D, L)), io)
    return M1Problem(Bsz, D, N, L, G, io, delta_softplus, u, delta, A, Bm, Cm, Dp, db, z,
                     h0, dout)


# --------------------------------------------------------------------------
# Mamba-3 SISO scan
# --------------------------------------------------------------------------
@dataclass
class M3Problem:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    nangles: int
    io: str
    x: Tensor          # [B, L, H, P]
    z: Optional[Tensor]
    B: Tensor          # [B, L, G, N]
    C: Tensor          # [B, L, G, N]
    alpha: Tensor      # [B, L, H]
    beta: Tensor       # [B, L, H]
    gamma: Tensor      # [B, L, H]
    theta: Tensor      # [B, L, H, K]
    D: Optional[np.ndarray]  # float32 [H]
    h0: Optional[np.ndarray]  # float32 [B, H, P, N]
    dout: Tensor

    @property
    def token_channels(self) -> int:
        return self.batch * self.seqlen * self.nheads * self.headdim


def _rms_normalise(v: np.ndarray, eps=1e-5) -> np.ndarray:
    v64 = v.astype(np.float64)
    return (v64 / np.sqrt(np.mean(v64 * v64, axis=-1, keepdims=True) + eps)).astype(np.float32)


def m3_problem(batch, seqlen, nheads, headdim, dstate, ngroups=1, nangles=None, io=F32,
               seed=SEED_BASE + 3, with_z=True, with_D=True, with_h0=False) -> M3Problem:
    rng = np.random.Generator(np.random.PCG64(seed))
    Bsz, L, H, P, N, G = batch, seqlen, nheads, headdim, dstate, ngroups
    K = N // 2 if nangles is None else nangles
    x = store(_normal(rng, (Bsz, L, H, P)), io)
    z = store(_normal(rng, (Bsz, L, H, P)), io) if with_z else None
    Bm = store(_rms_normalise(_normal(rng, (Bsz, L, G, N))), io)
    Cm = store(_rms_normalise(_normal(rng, (Bsz, L, G, N))), io)
    r = _normal(rng, (Bsz, L, H)).astype(np.float64)
    alpha = store(np.exp(-np.logaddexp(0.0, r)), io)
    beta = store(_uniform(rng, 0.0, 0.5, (Bsz, L, H)), io)
    gamma = store(_uniform(rng, 0.0, 0.5, (Bsz, L, H)), io)
    theta = store(_uniform(rng, 0.0, 0.1, (Bsz, L, H, K)), io)
    Dp = _normal(rng, (H,)) if with_D else None
    h0 = _normal(rng, (Bsz, H, P, N)) if with_h0 else None
    dout = store(_normal(rng, (Bsz, L, H, P)), io)
    return M3Problem(Bsz, L, H, P, N, G, K, io, x, z, Bm, Cm, alpha, beta, gamma, theta, Dp,
                     h0, dout)


@dataclass
class M3DiscProblem:
    """Mamba-3 inputs before the discretisation and BCNorm stages: the scan
    problem ``scan`` (its x, z, D, h0, dout are used; its alpha .. theta, B, C
    are not) and the raw per-token values those stages take."""
    scan: M3Problem
    dd_dt: Tensor      # [B, L, H]
    dd_a: Tensor       # [B, L, H]
    trap: Tensor       # [B, L, H]
    angles: Tensor     # [B, L, K]
    B_raw: Tensor      # [B, L, G, N]
    C_raw: Tensor      # [B, L, G, N]
    dt_bias: np.ndarray  # float32 [H]
    A_floor: float
    eps: float


def m3disc_problem(batch, seqlen, nheads, headdim, dstate, ngroups=1, nangles=None, io=F32,
                   seed=SEED_BASE + 7, with_h0=False, A_floor=1e-4, eps=1e-5) -> M3DiscProblem:
    """Raw projections ~ N(0, 1) (dd_dt scaled by 1/2, as Mamba-1's delta);
    dt_bias = softplus^-1(dt0) with dt0 log-uniform on [1e-3, 1e-1], the Mamba
    dt initialisation, so that dt starts in that range."""
    scan = m3_problem(batch, seqlen, nheads, headdim, dstate, ngroups, nangles, io=io, seed=seed,
                      with_h0=with_h0)
    rng = np.random.Generator(np.random.PCG64(seed + 500))
    Bsz, L, H, N, G, K = batch, seqlen, nheads, dstate, ngroups, scan.nangles
    dt0 = np.exp(_uniform(rng, np.log(1e-3), np.log(1e-1), (H,)).astype(np.float64))
    dt_bias = np.log(np.expm1(dt0)).astype(np.float32)
    return M3DiscProblem(
        scan, store(0.5 * _normal(rng, (Bsz, L, H)), io), store(_normal(rng, (Bsz, L, H)), io),
        store(_normal(rng, (Bsz, L, H)), io), store(_normal(rng, (Bsz, L, K)), io),
        store(_normal(rng, (Bsz, L, G, N)), io), store(_normal(rng, (Bsz, L, G, N)), io),
        dt_bias, A_floor, eps)


# --------------------------------------------------------------------------
# Single-token state update (decode)
# --------------------------------------------------------------------------
@dataclass
class SUProblem:
    batch: int
    dim: int
    dstate: int
    ngroups: int
    io: str
    delta_softplus: bool
    A: np.ndarray
    D: Optional[np.ndarray]
    delta_bias: Optional[np.ndarray]
    state0: np.ndarray           # float32 [B, D, N]
    steps: list                  # list of dicts: x, delta, z, B, C (Tensors)


def su_problem(batch, dim, dstate, io=BF16, seed=SEED_BASE + 4, n_pool=8, ngroups=1,
               random_state=False) -> SUProblem:
    """Decode-step inputs: a pool of ``n_pool`` step input sets, cycled by the caller."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Bsz, D, N, G = batch, dim, dstate, ngroups
    A = np.ascontiguousarray(
        np.broadcast_to(-np.exp(np.log(np.arange(1, N + 1, dtype=np.float64))), (D, N))
    ).astype(np.float32)
    Dp = _normal(rng, (D,))
    db = _uniform(rng, np.log(1e-3), np.log(1e-1), (D,))
    state0 = _normal(rng, (Bsz, D, N)) if random_state else np.zeros((Bsz, D, N), np.float32)
    steps = []
    for _ in range(n_pool):
        steps.append(dict(
            x=store(_normal(rng, (Bsz, D)), io),
            delta=store(0.5 * _normal(rng, (Bsz, D)) - 2.0, io),
            z=store(_normal(rng, (Bsz, D)), io),
            B=store(_normal(rng, (Bsz, G, N)), io),
            C=store(_normal(rng, (Bsz, G, N)), io),
        ))
    return SUProblem(Bsz, D, N, G, io, True, A, Dp, db, state0, steps)


@dataclass
class M3SUProblem:
    """Mamba-3 SISO decode: the carried state and a pool of step inputs."""
    batch: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    nangles: int
    io: str
    D: Optional[np.ndarray]      # float32 [H]
    state0: np.ndarray           # float32 [B, H, P, N]
    x_prev0: np.ndarray          # float32 [B, H, P]
    bt_prev0: np.ndarray         # float32 [B, H, N]
    phi0: np.ndarray             # float32 [B, H, K]
    steps: list                  # dicts: x, z [B,H,P]; B, C [B,G,N]; alpha, beta, gamma [B,H]; theta [B,H,K]


def m3su_problem(batch, nheads, headdim, dstate, ngroups=1, nangles=None, io=BF16,
                 seed=SEED_BASE + 5, n_pool=8, random_state=False, with_z=True,
                 with_D=True) -> M3SUProblem:
    """Mamba-3 decode-step inputs with the distributions of the Mamba-3 scan
    workload, a pool of ``n_pool`` step input sets cycled by the caller.  The
    carried state starts at zero (a fresh sequence) or, with ``random_state``,
    at random values (the middle of a sequence: N(0,1) state and last input,
    a unit-RMS last rotated key, angles in [0, 10))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Bsz, H, P, N, G = batch, nheads, headdim, dstate, ngroups
    K = N // 2 if nangles is None else nangles
    Dp = _normal(rng, (H,)) if with_D else None
    if random_state:
        state0 = _normal(rng, (Bsz, H, P, N))
        x_prev0 = _normal(rng, (Bsz, H, P))
        bt_prev0 = _rms_normalise(_normal(rng, (Bsz, H, N)))
        phi0 = _uniform(rng, 0.0, 10.0, (Bsz, H, K))
    else:
        state0 = np.zeros((Bsz, H, P, N), np.float32)
        x_prev0 = np.zeros((Bsz, H, P), np.float32)
        bt_prev0 = np.zeros((Bsz, H, N), np.float32)
        phi0 = np.zeros((Bsz, H, K), np.float32)
    steps = []
    for _ in range(n_pool):
        r = _normal(rng, (Bsz, H)).astype(np.float64)
        steps.append(dict(
            x=store(_normal(rng, (Bsz, H, P)), io),
            z=store(_normal(rng, (Bsz, H, P)), io) if with_z else None,
            B=store(_rms_normalise(_normal(rng, (Bsz, G, N))), io),
            C=store(_rms_normalise(_normal(rng, (Bsz, G, N))), io),
            alpha=store(np.exp(-np.logaddexp(0.0, r)), io),
            beta=store(_uniform(rng, 0.0, 0.5, (Bsz, H)), io),
            gamma=store(_uniform(rng, 0.0, 0.5, (Bsz, H)), io),
            theta=store(_uniform(rng, 0.0, 0.1, (Bsz, H, K)), io),
        ))
    return M3SUProblem(Bsz, H, P, N, G, K, io, Dp, state0, x_prev0, bt_prev0, phi0, steps)


def m3su_raw_steps(batch, nheads, dstate, ngroups=1, nangles=None, io=BF16, seed=SEED_BASE + 8,
                   n_pool=8):
    """Raw per-token values for the Mamba-3 decode step with the discretisation
    fused ahead, drawn like the raw-input scan workload: a pool of ``n_pool``
    step sets (dd_dt, dd_a, trap [B, H], angles [B, K], B_raw, C_raw [B, G, N])
    and dt_bias [H]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Bsz, H, N, G = batch, nheads, dstate, ngroups
    K = N // 2 if nangles is None else nangles
    dt0 = np.exp(_uniform(rng, np.log(1e-3), np.log(1e-1), (H,)).astype(np.float64))
    dt_bias = np.log(np.expm1(dt0)).astype(np.float32)
    steps = [dict(dd_dt=store(0.5 * _normal(rng, (Bsz, H)), io),
                  dd_a=store(_normal(rng, (Bsz, H)), io), trap=store(_normal(rng, (Bsz, H)), io),
                  angles=store(_normal(rng, (Bsz, K)), io),
                  B_raw=store(_normal(rng, (Bsz, G, N)), io),
                  C_raw=store(_normal(rng, (Bsz, G, N)), io)) for _ in range(n_pool)]
    return steps, dt_bias


# --------------------------------------------------------------------------
# The causal conv1d ahead of the Mamba-1 scan
# --------------------------------------------------------------------------
@dataclass
class M1ConvProblem:
    """Conv + scan inputs: ``scan`` is a Mamba-1 problem whose ``u`` is the
    conv's input x; w f32 [D, W] and bias f32 [D] are the conv's parameters."""
    scan: M1Problem
    width: int
    w: np.ndarray
    bias: np.ndarray


def m1conv_problem(batch, dim, dstate, seqlen, width=4, io=BF16, seed=SEED_BASE + 6,
                   ngroups=1) -> M1ConvProblem:
    """The scan inputs of a model-shaped Mamba-1 workload, and conv weights and
    bias drawn like a fresh depthwise Conv1d layer's: U(-1/sqrt(W), 1/sqrt(W))
    (one input channel per group, so the fan-in is the width)."""
    scan = m1_problem(batch, dim, dstate, seqlen, io=io, seed=seed, ngroups=ngroups, bias=True)
    rng = np.random.Generator(np.random.PCG64(seed + 500))
    k = 1.0 / np.sqrt(width)
    w = _uniform(rng, -k, k, (dim, width))
    bias = _uniform(rng, -k, k, (dim,))
    return M1ConvProblem(scan, width, w, bias)


# --------------------------------------------------------------------------
# The named workloads
# --------------------------------------------------------------------------
WORKLOADS = {
    "m1_f32_b1_d64_n16_l256": dict(kind="m1", batch=1, dim=64, dstate=16, seqlen=256, io=F32,
                                   bias=False, seed=SEED_BASE + 0),
    "m1_bf16_b8_d1536_n16_l2048": dict(kind="m1", batch=8, dim=1536, dstate=16, seqlen=2048,
                                       io=BF16, bias=True, seed=SEED_BASE + 1),
    "m1_bf16_b4_d5120_n16_l4096": dict(kind="m1", batch=4, dim=5120, dstate=16, seqlen=4096,
                                       io=BF16, bias=True, seed=SEED_BASE + 2),
    # one sequence of few channels: the scans split time into segments
    "m1_bf16_b1_d256_n16_l4096": dict(kind="m1", batch=1, dim=256, dstate=16, seqlen=4096,
                                      io=BF16, bias=True, seed=SEED_BASE + 9),
    "m3_bf16_b8_h24_p64_n64_k32_l2048": dict(kind="m3", batch=8, seqlen=2048, nheads=24,
                                             headdim=64, dstate=64, nangles=32, io=BF16,
                                             seed=SEED_BASE + 3),
    "su_bf16_b256_d5120_n16_x1000": dict(kind="su", batch=256, dim=5120, dstate=16, io=BF16,
                                         steps=1000, seed=SEED_BASE + 4),
    "m3su_bf16_b256_h24_p64_n64_k32_x1000": dict(kind="m3su", batch=256, nheads=24, headdim=64,
                                                 dstate=64, nangles=32, io=BF16, steps=1000,
                                                 seed=SEED_BASE + 5),
    "m3disc_bf16_b8_h24_p64_n64_k32_l2048": dict(kind="m3disc", batch=8, seqlen=2048,
                                                 nheads=24, headdim=64, dstate=64, nangles=32,
                                                 io=BF16, seed=SEED_BASE + 7),
    "m1conv_bf16_b8_d1536_n16_l2048_w4": dict(kind="m1conv", batch=8, dim=1536, dstate=16,
                                              seqlen=2048, width=4, io=BF16,
                                              seed=SEED_BASE + 6),
}


def make(name: str, shard: int = 0):
    """The named workload.  ``shard`` > 0 draws another batch of the same shape
    and distributions (seed + 1000 * shard): one per rank when ranks process
    independent batches."""
    w = dict(WORKLOADS[name])
    kind = w.pop("kind")
    w["seed"] += 1000 * shard
    if kind == "m1":
        return m1_problem(w["batch"], w["dim"], w["dstate"], w["seqlen"], io=w["io"],
                          seed=w["seed"], bias=w["bias"])
    if kind == "m3":
        return m3_problem(w["batch"], w["seqlen"], w["nheads"], w["headdim"], w["dstate"],
                          nangles=w["nangles"], io=w["io"], seed=w["seed"])
    if kind == "su":
        return su_problem(w["batch"], w["dim"], w["dstate"], io=w["io"], seed=w["seed"])
    if kind == "m3disc":
        return m3disc_problem(w["batch"], w["seqlen"], w["nheads"], w["headdim"], w["dstate"],
                              nangles=w["nangles"], io=w["io"], seed=w["seed"])
    if kind == "m1conv":
        return m1conv_problem(w["batch"], w["dim"], w["dstate"], w["seqlen"], width=w["width"],
                              io=w["io"], seed=w["seed"])
    if kind == "m3su":
        return m3su_problem(w["batch"], w["nheads"], w["headdim"], w["dstate"],
                            nangles=w["nangles"], io=w["io"], seed=w["seed"])
    raise ValueError(kind)
