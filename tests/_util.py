"""Helpers shared by the GPU parity tests: moving generated inputs to the
device, and the parity metric.

Parity metric, per tensor, with g the GPU result (widened to f64) and o the
f64 oracle:
  * primary: the max relative error  max_i |g_i - o_i| / max_i |o_i|
    (infinity-norm relative error), limit 1e-5 for f32 storage and 2e-2 for
    bf16 storage with f32 accumulation; 5e-3 for f16 storage, ten times the
    2^-11 relative rounding of an f16 output;
  * secondary, element by element: max_i |g_i - o_i| / max(|o_i|, 1e-3 max_j |o_j|),
    limit 2e-2 for bf16 storage and 1e-2 for f16; for f32 storage the limit is
    derived per tensor from a committed measurement (below).
Elementwise relative error of a sum that cancels is not bounded by the
arithmetic's rounding, so the 1e-5 bar is applied normwise.  The f32
elementwise guard comes from ``tests/golden/f32_error_floor.json``, written
by ``tests/golden/f32_error_floor.py`` from the oracle and an independent
plain f32 evaluation of each recurrence (sequential in time, numpy float32
arithmetic, correctly rounded exp) on the seeded inputs of the f32 parity
cases: for a Mamba-1 or Mamba-3 output tensor the limit is F32_ELEM_FACTOR
times the largest error that evaluation makes on that tensor over the cases,
and for the tensors it does not cover (the conv's, the discretisation's, the
decode steps') F32_ELEM_FACTOR times the largest over the family.  The factor
16 covers what the kernels may do differently and still be honest f32
arithmetic: the hardware 2^x has a relative error up to 2^-22 (four times an
f32 rounding), and sums are taken in chunked or tree order rather than step
by step.
"""
import json
import os

import numpy as np

TOL = {"f32": 1e-5, "f16": 5e-3, "bf16": 2e-2}
TOL_ELEM = {"f16": 1e-2, "bf16": 2e-2}
F32_ELEM_FACTOR = 16.0

_FLOOR_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                           "f32_error_floor.json")


def _load_floor():
    """(family, tensor) -> the largest elementwise error of the plain f32
    evaluation over the recorded cases; (family, None) -> over all tensors."""
    with open(_FLOOR_PATH) as f:
        rec = json.load(f)
    floor = {}
    for fam in ("m1", "m3"):
        for case in rec[fam].values():
            for tensor, e in case.items():
                floor[(fam, tensor)] = max(floor.get((fam, tensor), 0.0), e["elem"])
                floor[(fam, None)] = max(floor.get((fam, None), 0.0), e["elem"])
    return floor


F32_FLOOR = _load_floor()


def f32_elem_tol(family, name):
    """The f32 elementwise limit for tensor `name` (a prefix before a space,
    '@' or '[' is ignored) of the family's recurrence."""
    if family not in ("m1", "m3"):
        raise ValueError(f"f32 comparisons name their recurrence family, got {family!r}")
    base = name.split(" ")[0].split("@")[0].split("[")[0]
    return F32_ELEM_FACTOR * F32_FLOOR.get((family, base), F32_FLOOR[(family, None)])


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


def _log(name, io, e, ee):
    """With MSC_PARITY_LOG set, every comparison appends one JSON line (the
    test, the tensor, both errors) to that file: the record the parity
    figures of the documentation are read from."""
    path = os.environ.get("MSC_PARITY_LOG")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
                            "tensor": name, "io": io, "norm": e, "elem": ee}) + "\n")


def assert_close(name, got, ref, tol, family=None):
    """tol is TOL[io]; the elementwise guard uses the matching TOL_ELEM, or
    for f32 the derived limit of tensor `name` of `family` ("m1" or "m3")."""
    e = norm_rel_err(got, ref)
    io = "f32" if tol <= TOL["f32"] else ("f16" if tol <= TOL["f16"] else "bf16")
    ee = max_rel_err(got, ref)
    _log(name, io, e, ee)
    assert e <= tol, f"{name}: max relative error {e:.3e} > {tol:.1e}"
    elem_tol = f32_elem_tol(family, name) if io == "f32" else TOL_ELEM[io]
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
