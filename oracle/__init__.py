"""Python front end of the f64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the package's ``smoke()`` check and the
benchmark's CPU-baseline leg call this; the library itself never does.  It
shares no code with the CUDA path.  Every function takes float64 numpy arrays
(the io-rounded inputs, widened) and returns float64 numpy arrays.

The recurrences are documented in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, IEEE semantics, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", _SRC, "-o", _LIB,
               "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        i64, ci, dp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        _lib.oracle_m1_fwd.argtypes = [i64] * 5 + [ci] + [dp] * 12 + [ci]
        _lib.oracle_m1_fwd_tree.argtypes = [i64] * 5 + [ci] + [dp] * 11 + [ci]
        _lib.oracle_m1_bwd.argtypes = [i64] * 5 + [ci] + [dp] * 19 + [ci]
        _lib.oracle_ssm_state_update.argtypes = [i64] * 4 + [ci] + [dp] * 10
        _lib.oracle_m3_fwd.argtypes = [i64] * 7 + [dp] * 12 + [ci]
        _lib.oracle_m3_bwd.argtypes = [i64] * 7 + [dp] * 21 + [ci]
        _lib.oracle_m3_state_update.argtypes = [i64] * 6 + [dp] * 14
        _lib.oracle_conv1d_fwd.argtypes = [i64] * 4 + [dp] * 6
        _lib.oracle_conv1d_bwd.argtypes = [i64] * 4 + [dp] * 9
        for f in (_lib.oracle_m1_fwd, _lib.oracle_m1_fwd_tree, _lib.oracle_m1_bwd,
                  _lib.oracle_ssm_state_update, _lib.oracle_m3_fwd, _lib.oracle_m3_bwd,
                  _lib.oracle_m3_state_update, _lib.oracle_conv1d_fwd, _lib.oracle_conv1d_bwd):
            f.restype = ctypes.c_int
        _lib.oracle_default_threads.restype = ctypes.c_int
    return _lib


def default_threads() -> int:
    return int(_load().oracle_default_threads())


def _in(a: Optional[np.ndarray]):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data


def _out(shape):
    a = np.zeros(shape, dtype=np.float64)
    return a, a.ctypes.data


def _check(rc):
    if rc != 0:
        raise ValueError("oracle rejected the problem dimensions")


# ---------------------------------------------------------------------------
# Mamba-1
# ---------------------------------------------------------------------------
def m1_fwd(u, delta, A, B, C, D=None, delta_bias=None, z=None, h0=None, delta_softplus=True,
           nthreads=0, tree=False, want_y=False):
    """Mamba-1 forward.  u, delta, z: [B, D, L]; A: [D, N]; B, C: [B, G, N, L].

    Returns dict(out [B,D,L], final_state [B,D,N][, y pre-gate [B,D,L]]).
    tree=True evaluates the time recurrence as a Hillis-Steele scan instead.
    """
    lib = _load()
    Bsz, Dm, L = u.shape
    G, N = B.shape[1], B.shape[2]
    keep = [_in(x) for x in (u, delta, A, B, C, D, delta_bias, z, h0)]
    out, po = _out((Bsz, Dm, L))
    fs, pf = _out((Bsz, Dm, N))
    res = dict(out=out, final_state=fs)
    if tree:
        _check(lib.oracle_m1_fwd_tree(Bsz, Dm, N, L, G, int(delta_softplus),
                                      *[k[1] for k in keep], po, pf, nthreads))
    else:
        y, py = _out((Bsz, Dm, L)) if want_y else (None, None)
        _check(lib.oracle_m1_fwd(Bsz, Dm, N, L, G, int(delta_softplus), *[k[1] for k in keep],
                                 po, pf, py, nthreads))
        if want_y:
            res["y"] = y
    return res


def m1_bwd(u, delta, A, B, C, dout, D=None, delta_bias=None, z=None, h0=None,
           delta_softplus=True, nthreads=0):
    """Mamba-1 backward.  Returns du, ddelta, dA, dB, dC, dD, ddelta_bias, dz, dh0."""
    lib = _load()
    Bsz, Dm, L = u.shape
    G, N = B.shape[1], B.shape[2]
    keep = [_in(x) for x in (u, delta, A, B, C, D, delta_bias, z, h0, dout)]
    du, p1 = _out((Bsz, Dm, L))
    dd, p2 = _out((Bsz, Dm, L))
    dA, p3 = _out((Dm, N))
    dB, p4 = _out((Bsz, G, N, L))
    dC, p5 = _out((Bsz, G, N, L))
    dD, p6 = _out((Dm,))
    dbias, p7 = _out((Dm,))
    dz, p8 = _out((Bsz, Dm, L))
    dh0, p9 = _out((Bsz, Dm, N))
    _check(lib.oracle_m1_bwd(Bsz, Dm, N, L, G, int(delta_softplus), *[k[1] for k in keep],
                             p1, p2, p3, p4, p5, p6, p7, p8, p9, nthreads))
    return dict(du=du, ddelta=dd, dA=dA, dB=dB, dC=dC, dD=dD, ddelta_bias=dbias, dz=dz, dh0=dh0)


def ssm_state_update(state, x, delta, A, B, C, D=None, delta_bias=None, z=None,
                     delta_softplus=True):
    """One decode step.  state [B, D, N] (returned updated copy); x, delta, z [B, D];
    B, C [B, G, N].  Returns (new_state, out [B, D])."""
    lib = _load()
    st = np.array(state, dtype=np.float64, copy=True)
    Bsz, Dm, N = st.shape
    G = B.shape[1]
    keep = [_in(v) for v in (x, delta, A, B, C, D, delta_bias, z)]
    out, po = _out((Bsz, Dm))
    _check(lib.oracle_ssm_state_update(Bsz, Dm, N, G, int(delta_softplus), st.ctypes.data,
                                       *[k[1] for k in keep], po))
    return st, out


# ---------------------------------------------------------------------------
# Mamba-3 SISO
# ---------------------------------------------------------------------------
def m3_fwd(x, B, C, alpha, beta, gamma, theta, D=None, z=None, h0=None, nthreads=0):
    """Mamba-3 SISO forward.  x, z: [B, L, H, P]; B, C: [B, L, G, N];
    alpha/beta/gamma: [B, L, H]; theta: [B, L, H, K].  Returns out, final_state."""
    lib = _load()
    Bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    K = theta.shape[3]
    keep = [_in(v) for v in (x, z, B, C, alpha, beta, gamma, theta, D, h0)]
    out, po = _out((Bsz, L, H, P))
    fs, pf = _out((Bsz, H, P, N))
    _check(lib.oracle_m3_fwd(Bsz, L, H, P, N, G, K, *[k[1] for k in keep], po, pf, nthreads))
    return dict(out=out, final_state=fs)


def m3_bwd(x, B, C, alpha, beta, gamma, theta, dout, D=None, z=None, h0=None, nthreads=0):
    """Mamba-3 SISO backward.  Returns dx, dz, dB, dC, dalpha, dbeta, dgamma, dtheta, dD, dh0."""
    lib = _load()
    Bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    K = theta.shape[3]
    keep = [_in(v) for v in (x, z, B, C, alpha, beta, gamma, theta, D, h0, dout)]
    dx, p1 = _out((Bsz, L, H, P))
    dz, p2 = _out((Bsz, L, H, P))
    dB, p3 = _out((Bsz, L, G, N))
    dC, p4 = _out((Bsz, L, G, N))
    da, p5 = _out((Bsz, L, H))
    db, p6 = _out((Bsz, L, H))
    dg, p7 = _out((Bsz, L, H))
    dth, p8 = _out((Bsz, L, H, K))
    dD, p9 = _out((H,))
    dh0, p10 = _out((Bsz, H, P, N))
    _check(lib.oracle_m3_bwd(Bsz, L, H, P, N, G, K, *[k[1] for k in keep],
                             p1, p2, p3, p4, p5, p6, p7, p8, p9, p10, nthreads))
    return dict(dx=dx, dz=dz, dB=dB, dC=dC, dalpha=da, dbeta=db, dgamma=dg, dtheta=dth, dD=dD,
                dh0=dh0)


def m3_state_update(state, x_prev, bt_prev, phi, x, B, C, alpha, beta, gamma, theta, D=None,
                    z=None):
    """One Mamba-3 SISO decode step.  state [B, H, P, N], x_prev [B, H, P],
    bt_prev [B, H, N], phi [B, H, K] (updated copies are returned); x, z [B, H, P];
    B, C [B, G, N]; alpha/beta/gamma [B, H]; theta [B, H, K].
    Returns (state, x_prev, bt_prev, phi, out [B, H, P])."""
    lib = _load()
    carried = [np.array(a, dtype=np.float64, copy=True) for a in (state, x_prev, bt_prev, phi)]
    Bsz, H, P, N = carried[0].shape
    G = B.shape[1]
    K = carried[3].shape[2]
    keep = [_in(v) for v in (x, z, B, C, alpha, beta, gamma, theta, D)]
    out, po = _out((Bsz, H, P))
    _check(lib.oracle_m3_state_update(Bsz, H, P, N, G, K, *[a.ctypes.data for a in carried],
                                      *[k[1] for k in keep], po))
    return (*carried, out)


# ---------------------------------------------------------------------------
# causal conv1d (+ SiLU) ahead of the Mamba-1 scan
# ---------------------------------------------------------------------------
def conv1d_fwd(x, w, bias=None, xs0=None):
    """x [B, D, L]; w [D, W]; bias [D]; xs0 [B, D, W-1].  Returns (u, xs_final)."""
    lib = _load()
    Bsz, Dm, L = x.shape
    W = w.shape[1]
    keep = [_in(v) for v in (x, w, bias, xs0)]
    u, pu = _out((Bsz, Dm, L))
    xs, px = _out((Bsz, Dm, max(W - 1, 0)))
    _check(lib.oracle_conv1d_fwd(Bsz, Dm, L, W, *[k[1] for k in keep], pu, px))
    return u, xs


def conv1d_bwd(x, w, du, bias=None, xs0=None):
    """Gradients of u = silu(conv(x)) for an upstream du [B, D, L].
    Returns dx, dw, dbias, dxs0."""
    lib = _load()
    Bsz, Dm, L = x.shape
    W = w.shape[1]
    keep = [_in(v) for v in (x, w, bias, xs0, du)]
    dx, p1 = _out((Bsz, Dm, L))
    dw, p2 = _out((Dm, W))
    db, p3 = _out((Dm,))
    dxs, p4 = _out((Bsz, Dm, max(W - 1, 0)))
    _check(lib.oracle_conv1d_bwd(Bsz, Dm, L, W, *[k[1] for k in keep], p1, p2, p3, p4))
    return dict(dx=dx, dw=dw, dbias=db, dxs0=dxs)


# ---------------------------------------------------------------------------
# Mamba-3 SISO discretisation and BCNorm (the stages ahead of the scan)
# ---------------------------------------------------------------------------
# Mamba3Scratch (mamba-rs 0.4.2 src/mamba3_siso/cpu/scratch.rs) names the
# stages: B6 "discretization" turns per-token, per-head dd_dt, dd_a, trap
# [T * nheads] and per-token raw angles [T * n_angles] into the scan's
# coefficients, B5 "BCNorm" normalises the raw B and C [T * ngroups *
# d_state].  The pages print no formulas; these are the exponential-trapezoid
# discretisation of the cited Mamba-3 paper (Lahoti et al., 2026), read in its
# plainest form:
#   dt    = softplus(dd_dt + dt_bias[h])
#   A     = min(-softplus(dd_a), -A_floor)
#   alpha = exp(dt * A)
#   lam   = sigmoid(trap)
#   beta  = (1 - lam) * dt * alpha      (the x_{t-1} end of the trapezoid,
#                                        carried through one step of decay)
#   gamma = lam * dt                    (the x_t end)
#   theta[k] = dt * angles[k]           (per head: dt is per head)
#   B = B_raw / sqrt(mean_n B_raw^2 + eps),  C likewise (RMS norm over
#   d_state per (token, group), no weight)
def _softplus(v):
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def _sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def m3_discretize(dd_dt, dd_a, trap, angles, B_raw, C_raw, dt_bias=None, A_floor=0.0,
                  eps=1e-5):
    """dd_dt, dd_a, trap [B, L, H]; angles [B, L, K]; B_raw, C_raw [B, L, G, N];
    dt_bias [H].  Returns alpha, beta, gamma [B, L, H], theta [B, L, H, K], B, C
    (all float64)."""
    u = dd_dt + (0.0 if dt_bias is None else dt_bias[None, None, :])
    dt = _softplus(u)
    A = np.minimum(-_softplus(dd_a), -A_floor)
    alpha = np.exp(dt * A)
    lam = _sigmoid(trap)
    beta = (1.0 - lam) * dt * alpha
    gamma = lam * dt
    theta = dt[..., None] * angles[:, :, None, :]
    B = B_raw / np.sqrt(np.mean(B_raw * B_raw, axis=-1, keepdims=True) + eps)
    C = C_raw / np.sqrt(np.mean(C_raw * C_raw, axis=-1, keepdims=True) + eps)
    return dict(alpha=alpha, beta=beta, gamma=gamma, theta=theta, B=B, C=C)


def _rms_norm_bwd(v, g, eps):
    """Gradient of v / sqrt(mean(v^2) + eps) (last axis) for an upstream g."""
    r = 1.0 / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    vh = v * r
    return r * (g - vh * np.mean(g * vh, axis=-1, keepdims=True))


def m3_discretize_bwd(dd_dt, dd_a, trap, angles, B_raw, C_raw, dalpha, dbeta, dgamma, dtheta,
                      dB, dC, dt_bias=None, A_floor=0.0, eps=1e-5):
    """Chain rule through m3_discretize for upstream gradients of its outputs.
    Returns ddd_dt, ddd_a, dtrap [B, L, H], dangles [B, L, K], ddt_bias [H],
    dB_raw, dC_raw [B, L, G, N]."""
    u = dd_dt + (0.0 if dt_bias is None else dt_bias[None, None, :])
    dt = _softplus(u)
    sa = _softplus(dd_a)
    clamped = -sa > -A_floor          # A = -A_floor there: no gradient to dd_a
    A = np.where(clamped, -A_floor, -sa)
    alpha = np.exp(dt * A)
    lam = _sigmoid(trap)
    # alpha reaches the loss directly and through beta
    g_alpha = dalpha + dbeta * (1.0 - lam) * dt
    d_dt = (g_alpha * alpha * A + dbeta * (1.0 - lam) * alpha + dgamma * lam
            + np.sum(dtheta * angles[:, :, None, :], axis=-1))
    d_A = g_alpha * alpha * dt
    d_lam = dgamma * dt - dbeta * dt * alpha
    ddd_dt = d_dt * _sigmoid(u)
    ddd_a = np.where(clamped, 0.0, -d_A * _sigmoid(dd_a))
    dtrap = d_lam * lam * (1.0 - lam)
    dangles = np.sum(dtheta * dt[..., None], axis=2)
    ddt_bias = ddd_dt.sum(axis=(0, 1))
    return dict(ddd_dt=ddd_dt, ddd_a=ddd_a, dtrap=dtrap, dangles=dangles, ddt_bias=ddt_bias,
                dB_raw=_rms_norm_bwd(B_raw, dB, eps), dC_raw=_rms_norm_bwd(C_raw, dC, eps))


# ---------------------------------------------------------------------------
# convenience: run on a generated problem (workloads.M1Problem / M3Problem)
# ---------------------------------------------------------------------------
def m1_problem_args(p):
    f = lambda t: None if t is None else t.as_f64()
    w = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    return dict(u=f(p.u), delta=f(p.delta), A=w(p.A), B=f(p.B), C=f(p.C), D=w(p.D),
                delta_bias=w(p.delta_bias), z=f(p.z), h0=w(p.h0),
                delta_softplus=p.delta_softplus)


def m3_problem_args(p):
    f = lambda t: None if t is None else t.as_f64()
    w = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    return dict(x=f(p.x), B=f(p.B), C=f(p.C), alpha=f(p.alpha), beta=f(p.beta),
                gamma=f(p.gamma), theta=f(p.theta), D=w(p.D), z=f(p.z), h0=w(p.h0))
