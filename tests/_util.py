"""Helpers shared by the GPU parity tests: moving generated inputs to the
device, and the parity metric.

Parity metric, per tensor, with g the GPU result (widened to f64) and o the
f64 oracle:
  * primary: the max relative error  max_i |g_i - o_i| / max_i |o_i|
    (infinity-norm relative error), limit 1e-5 for f32 storage and 2e-2 for
    bf16 storage with f32 accumulation; 5e-3 for f16 storage, ten times the
    2^-11 relative rounding of an f16 output;
  * secondary, element by element: max_i |g_i - o_i| / max(|o_i|, 1e-3 max_j |o_j|),
    limit 1e-2 for f32 and f16 storage and 2e-2 for bf16.
Elementwise relative error of a sum that cancels is not bounded by the
arithmetic's rounding (a plain sequential f32 evaluation of the Mamba-1 scan
already scores ~1e-4 on it while its normwise error is ~6e-7; the chunked
Mamba-3 form, with 64-term f32 sums, reaches ~2e-3 on entries near the floor),
so the 1e-5 bar is applied normwise and the elementwise check only guards
small entries against gross errors (a dropped term, a wrong sign or index).
"""
import numpy as np

TOL = {"f32": 1e-5, "f16": 5e-3, "bf16": 2e-2}
TOL_ELEM = {"f32": 1e-2, "f16": 1e-2, "bf16": 2e-2}


def norm_rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    m = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (m if m > 0 else 1.0)


def max_rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    floor = 1e-3 * float(np.max(np.abs(ref)))
    den = np.maximum(np.abs(ref), floor if floor > 0 else 1e-30)
    return float(np.max(np.abs(got - ref) / den))


def assert_close(name, got, ref, tol):
    """tol is TOL[io]; the elementwise guard uses the matching TOL_ELEM."""
    e = norm_rel_err(got, ref)
    assert e <= tol, f"{name}: max relative error {e:.3e} > {tol:.1e}"
    io = "f32" if tol <= TOL["f32"] else ("f16" if tol <= TOL["f16"] else "bf16")
    elem_tol = TOL_ELEM[io]
    ee = max_rel_err(got, ref)
    assert ee <= elem_tol, f"{name}: elementwise relative error {ee:.3e} > {elem_tol:.1e}"
    return e


def dev(t, device="cuda"):
    """workloads.Tensor / float32 ndarray / None -> contiguous torch tensor on the GPU."""
    import torch
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return torch.from_numpy(np.ascontiguousarray(t, dtype=np.float32)).to(device)
    if t.dtype == "bf16":
        return torch.from_numpy(t.data.view(np.int16)).to(device).view(torch.bfloat16)
    if t.dtype == "f16":
        return torch.from_numpy(np.ascontiguousarray(t.data)).to(device)
    return torch.from_numpy(t.data).to(device)


def host(x):
    """torch tensor (any dtype) -> float64 numpy array."""
    return x.detach().float().cpu().numpy().astype(np.float64)


def m1_device_args(p):
    return dict(u=dev(p.u), delta=dev(p.delta), A=dev(p.A), B=dev(p.B), C=dev(p.C), D=dev(p.D),
                delta_bias=dev(p.delta_bias), z=dev(p.z), h0=dev(p.h0),
                delta_softplus=p.delta_softplus)


def m3_device_args(p):
    return dict(x=dev(p.x), B=dev(p.B), C=dev(p.C), alpha=dev(p.alpha), beta=dev(p.beta),
                gamma=dev(p.gamma), theta=dev(p.theta), D=dev(p.D), z=dev(p.z), h0=dev(p.h0))
