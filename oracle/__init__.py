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
