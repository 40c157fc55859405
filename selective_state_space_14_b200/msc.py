"""Thin Python binding of libmsc.so (the C ABI declared in include/msc.h).

Argument marshalling only: every step of the scans runs in the library's CUDA
kernels.  torch supplies device memory and the current stream.  There is no
CPU fallback: if libmsc.so is missing or cannot be loaded, every call raises.

The functions carry the C entry points' names and take torch tensors laid out
as msc.h states (contiguous, on the current CUDA device).  Outputs not passed
in are allocated with torch and returned.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsc.so")

MSC_F32, MSC_BF16, MSC_F16 = 0, 1, 2
MSC_M1_SAVE_INTERVAL = 8

STATUS = {0: "MSC_OK", 1: "MSC_ERR_INVALID_ARG", 2: "MSC_ERR_UNSUPPORTED", 3: "MSC_ERR_ALIGNMENT",
          4: "MSC_ERR_CUDA", 5: "MSC_ERR_WORKSPACE"}


class MscError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_u32 = ctypes.c_uint32


class SsFwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("dim", _i64),
                ("dstate", _i64), ("seqlen", _i64), ("ngroups", _i64), ("delta_softplus", _i32),
                ("u", _vp), ("delta", _vp), ("A", _vp), ("Bm", _vp), ("Cm", _vp), ("D", _vp),
                ("delta_bias", _vp), ("z", _vp), ("h0", _vp), ("out", _vp), ("final_state", _vp),
                ("saved_states", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class SsConvArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("width", _i64), ("w", _vp), ("bias", _vp),
                ("conv_state_in", _vp), ("conv_state_out", _vp), ("u_out", _vp)]


class SsBwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("dim", _i64),
                ("dstate", _i64), ("seqlen", _i64), ("ngroups", _i64), ("delta_softplus", _i32),
                ("u", _vp), ("delta", _vp), ("A", _vp), ("Bm", _vp), ("Cm", _vp), ("D", _vp),
                ("delta_bias", _vp), ("z", _vp), ("h0", _vp), ("saved_states", _vp),
                ("dout", _vp), ("du", _vp), ("ddelta", _vp), ("dz", _vp), ("dA", _vp),
                ("dB", _vp), ("dC", _vp), ("dD", _vp), ("ddelta_bias", _vp), ("dh0", _vp)]


class SuArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("dim", _i64),
                ("dstate", _i64), ("ngroups", _i64), ("delta_softplus", _i32), ("state", _vp),
                ("x", _vp), ("delta", _vp), ("A", _vp), ("Bm", _vp), ("Cm", _vp), ("D", _vp),
                ("delta_bias", _vp), ("z", _vp), ("out", _vp)]


class M3FwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("seqlen", _i64),
                ("nheads", _i64), ("headdim", _i64), ("dstate", _i64), ("ngroups", _i64),
                ("nangles", _i64), ("x", _vp), ("z", _vp), ("Bm", _vp), ("Cm", _vp),
                ("alpha", _vp), ("beta", _vp), ("gamma", _vp), ("theta", _vp), ("D", _vp),
                ("h0", _vp), ("out", _vp), ("final_state", _vp), ("saved_states", _vp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class M3BwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("seqlen", _i64),
                ("nheads", _i64), ("headdim", _i64), ("dstate", _i64), ("ngroups", _i64),
                ("nangles", _i64), ("x", _vp), ("z", _vp), ("Bm", _vp), ("Cm", _vp),
                ("alpha", _vp), ("beta", _vp), ("gamma", _vp), ("theta", _vp), ("D", _vp),
                ("h0", _vp), ("saved_states", _vp), ("dout", _vp), ("dx", _vp), ("dz", _vp),
                ("dB", _vp), ("dC", _vp), ("dalpha", _vp), ("dbeta", _vp), ("dgamma", _vp),
                ("dtheta", _vp), ("dD", _vp), ("dh0", _vp)]


class M3SuArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("nheads", _i64),
                ("headdim", _i64), ("dstate", _i64), ("ngroups", _i64), ("nangles", _i64),
                ("state", _vp), ("x_prev", _vp), ("bt_prev", _vp), ("phi", _vp), ("x", _vp),
                ("z", _vp), ("Bm", _vp), ("Cm", _vp), ("alpha", _vp), ("beta", _vp),
                ("gamma", _vp), ("theta", _vp), ("D", _vp), ("out", _vp)]


class M3DiscStepArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("A_floor", ctypes.c_float), ("eps", ctypes.c_float),
                ("dd_dt", _vp), ("dd_a", _vp), ("trap", _vp), ("angles", _vp), ("dt_bias", _vp),
                ("B_raw", _vp), ("C_raw", _vp)]


class M3DiscArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("seqlen", _i64),
                ("nheads", _i64), ("dstate", _i64), ("ngroups", _i64), ("nangles", _i64),
                ("A_floor", ctypes.c_float), ("eps", ctypes.c_float), ("dd_dt", _vp),
                ("dd_a", _vp), ("trap", _vp), ("angles", _vp), ("dt_bias", _vp),
                ("B_raw", _vp), ("C_raw", _vp), ("alpha", _vp), ("beta", _vp), ("gamma", _vp),
                ("theta", _vp), ("Bm", _vp), ("Cm", _vp)]


class M3DiscBwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("seqlen", _i64),
                ("nheads", _i64), ("dstate", _i64), ("ngroups", _i64), ("nangles", _i64),
                ("A_floor", ctypes.c_float), ("eps", ctypes.c_float), ("dd_dt", _vp),
                ("dd_a", _vp), ("trap", _vp), ("angles", _vp), ("dt_bias", _vp),
                ("B_raw", _vp), ("C_raw", _vp), ("dalpha", _vp), ("dbeta", _vp),
                ("dgamma", _vp), ("dtheta", _vp), ("dB", _vp), ("dC", _vp), ("ddd_dt", _vp),
                ("ddd_a", _vp), ("dtrap", _vp), ("dangles", _vp), ("ddt_bias", _vp),
                ("dB_raw", _vp), ("dC_raw", _vp)]


class M3RawArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("A_floor", ctypes.c_float), ("eps", ctypes.c_float),
                ("dd_dt", _vp), ("dd_a", _vp), ("trap", _vp), ("angles", _vp), ("dt_bias", _vp),
                ("B_raw", _vp), ("C_raw", _vp)]


class M3RawGrads(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("ddd_dt", _vp), ("ddd_a", _vp), ("dtrap", _vp),
                ("dangles", _vp), ("ddt_bias", _vp), ("dB_raw", _vp), ("dC_raw", _vp)]


class ConvFwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("dim", _i64),
                ("seqlen", _i64), ("width", _i64), ("x", _vp), ("w", _vp), ("bias", _vp),
                ("conv_state_in", _vp), ("u", _vp), ("conv_state_out", _vp)]


class ConvBwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", _u32), ("io_dtype", _i32), ("batch", _i64), ("dim", _i64),
                ("seqlen", _i64), ("width", _i64), ("x", _vp), ("w", _vp), ("bias", _vp),
                ("conv_state_in", _vp), ("du", _vp), ("dx", _vp), ("dw", _vp), ("dbias", _vp),
                ("dconv_state_in", _vp)]


EXPORTS = ["msc_last_error", "msc_version", "msc_selective_scan_saved_states_bytes",
           "msc_selective_scan_fwd_workspace_bytes", "msc_selective_scan_fwd", "msc_selective_scan_bwd_workspace_bytes",
           "msc_selective_scan_bwd", "msc_selective_scan_bwd_static", "msc_ssm_state_update",
           "msc_mamba3_siso_saved_states_bytes", "msc_mamba3_siso_scan_fwd_workspace_bytes",
           "msc_mamba3_siso_scan_fwd", "msc_mamba3_siso_scan_bwd_workspace_bytes",
           "msc_mamba3_siso_scan_bwd", "msc_mamba3_siso_state_update", "msc_causal_conv1d_fwd",
           "msc_causal_conv1d_bwd_workspace_bytes", "msc_causal_conv1d_bwd",
           "msc_selective_scan_conv_fwd", "msc_mamba3_siso_discretize",
           "msc_mamba3_siso_discretize_bwd", "msc_mamba3_siso_disc_state_update",
           "msc_probe_threads_per_block", "msc_probe_sfu_ex2", "msc_probe_ffma",
           "msc_mamba3_siso_scan_fwd_raw", "msc_mamba3_siso_scan_fwd_raw_workspace_bytes",
           "msc_mamba3_siso_scan_bwd_raw_workspace_bytes",
           "msc_mamba3_siso_scan_bwd_raw"]

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmsc.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m selective_state_space_14_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.msc_last_error.restype = ctypes.c_char_p
        L.msc_version.restype = ctypes.c_char_p
        for name, argt in (("msc_selective_scan_fwd", [ctypes.POINTER(SsFwdArgs), _vp]),
                           ("msc_selective_scan_conv_fwd",
                            [ctypes.POINTER(SsFwdArgs), ctypes.POINTER(SsConvArgs), _vp]),
                           ("msc_selective_scan_bwd",
                            [ctypes.POINTER(SsBwdArgs), _vp, ctypes.c_size_t, _vp]),
                           ("msc_selective_scan_bwd_static", [ctypes.POINTER(SsBwdArgs), _vp]),
                           ("msc_ssm_state_update", [ctypes.POINTER(SuArgs), _vp]),
                           ("msc_mamba3_siso_scan_fwd", [ctypes.POINTER(M3FwdArgs), _vp]),
                           ("msc_mamba3_siso_scan_bwd",
                            [ctypes.POINTER(M3BwdArgs), _vp, ctypes.c_size_t, _vp]),
                           ("msc_mamba3_siso_state_update", [ctypes.POINTER(M3SuArgs), _vp]),
                           ("msc_mamba3_siso_discretize", [ctypes.POINTER(M3DiscArgs), _vp]),
                           ("msc_mamba3_siso_disc_state_update",
                            [ctypes.POINTER(M3SuArgs), ctypes.POINTER(M3DiscStepArgs), _vp]),
                           ("msc_mamba3_siso_discretize_bwd",
                            [ctypes.POINTER(M3DiscBwdArgs), _vp]),
                           ("msc_mamba3_siso_scan_fwd_raw",
                            [ctypes.POINTER(M3FwdArgs), ctypes.POINTER(M3RawArgs), _vp]),
                           ("msc_mamba3_siso_scan_bwd_raw",
                            [ctypes.POINTER(M3BwdArgs), ctypes.POINTER(M3RawArgs),
                             ctypes.POINTER(M3RawGrads), _vp, ctypes.c_size_t, _vp]),
                           ("msc_causal_conv1d_fwd", [ctypes.POINTER(ConvFwdArgs), _vp]),
                           ("msc_causal_conv1d_bwd",
                            [ctypes.POINTER(ConvBwdArgs), _vp, ctypes.c_size_t, _vp])):
            f = getattr(L, name)
            f.argtypes = argt
            f.restype = ctypes.c_int
        L.msc_selective_scan_saved_states_bytes.argtypes = [_i64] * 4
        L.msc_selective_scan_saved_states_bytes.restype = ctypes.c_size_t
        L.msc_selective_scan_fwd_workspace_bytes.argtypes = [_i64] * 4
        L.msc_selective_scan_fwd_workspace_bytes.restype = ctypes.c_size_t
        L.msc_selective_scan_bwd_workspace_bytes.argtypes = [_i64] * 5
        L.msc_selective_scan_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.msc_mamba3_siso_saved_states_bytes.argtypes = [_i64] * 5
        L.msc_mamba3_siso_saved_states_bytes.restype = ctypes.c_size_t
        L.msc_mamba3_siso_scan_fwd_workspace_bytes.argtypes = [_i64] * 5
        L.msc_mamba3_siso_scan_fwd_workspace_bytes.restype = ctypes.c_size_t
        L.msc_causal_conv1d_bwd_workspace_bytes.argtypes = [_i64] * 4
        L.msc_causal_conv1d_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.msc_mamba3_siso_scan_bwd_workspace_bytes.argtypes = [_i64] * 7
        L.msc_mamba3_siso_scan_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.msc_mamba3_siso_scan_fwd_raw_workspace_bytes.argtypes = [_i64] * 7
        L.msc_mamba3_siso_scan_fwd_raw_workspace_bytes.restype = ctypes.c_size_t
        L.msc_mamba3_siso_scan_bwd_raw_workspace_bytes.argtypes = [_i64] * 7
        L.msc_mamba3_siso_scan_bwd_raw_workspace_bytes.restype = ctypes.c_size_t
        L.msc_probe_threads_per_block.argtypes = []
        L.msc_probe_threads_per_block.restype = _i64
        L.msc_probe_sfu_ex2.argtypes = [_vp, _i64, _i64, ctypes.POINTER(_i64), _vp]
        L.msc_probe_sfu_ex2.restype = ctypes.c_int
        L.msc_probe_ffma.argtypes = [_vp, _i64, _i64, ctypes.c_int32, ctypes.POINTER(_i64), _vp]
        L.msc_probe_ffma.restype = ctypes.c_int
        _lib = L
    return _lib


def version() -> str:
    return lib().msc_version().decode()


def _check(status: int):
    if status != 0:
        raise MscError(status, lib().msc_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmsc must be contiguous")
    return t.data_ptr()


def _io(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MSC_BF16
    if t.dtype == torch.float32:
        return MSC_F32
    if t.dtype == torch.float16:
        return MSC_F16
    raise TypeError(f"unsupported io dtype {t.dtype}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# Mamba-1 selective scan
# ---------------------------------------------------------------------------
def msc_selective_scan_saved_states_bytes(batch, dim, dstate, seqlen) -> int:
    return int(lib().msc_selective_scan_saved_states_bytes(batch, dim, dstate, seqlen))


def msc_selective_scan_bwd_workspace_bytes(batch, dim, dstate, seqlen, ngroups=1) -> int:
    return int(lib().msc_selective_scan_bwd_workspace_bytes(batch, dim, dstate, seqlen, ngroups))


def msc_probe(kind, out, blocks, iters, stream=None) -> int:
    """Launch one rate probe ("ex2", "ffma" or "ffma2") into the float32 device
    tensor ``out`` (blocks * msc_probe_threads_per_block() elements); returns
    the number of operations the launch performs."""
    ops = _i64(0)
    n = int(lib().msc_probe_threads_per_block()) * blocks
    if out.numel() < n:
        raise ValueError(f"out holds {out.numel()} floats, the probe writes {n}")
    if kind == "ex2":
        st = lib().msc_probe_sfu_ex2(out.data_ptr(), blocks, iters, ctypes.byref(ops), _stream(stream))
    else:
        st = lib().msc_probe_ffma(out.data_ptr(), blocks, iters, 1 if kind == "ffma2" else 0,
                                  ctypes.byref(ops), _stream(stream))
    _check(st)
    return int(ops.value)


def msc_selective_scan_fwd_workspace_bytes(batch, dim, dstate, seqlen) -> int:
    return int(lib().msc_selective_scan_fwd_workspace_bytes(batch, dim, dstate, seqlen))


def msc_selective_scan_fwd(u, delta, A, B, C, D=None, delta_bias=None, z=None, h0=None,
                           delta_softplus=True, out=None, final_state=None, saved_states=None,
                           want_final_state=True, want_saved_states=True, workspace=None,
                           stream=None):
    """Mamba-1 forward.  u, delta, z: [B, D, L]; A: f32 [D, N]; B, C: [B, G, N, L].
    Above 64 states a workspace is needed (allocated here if not given).

    Returns (out, final_state, saved_states)."""
    a, out, final_state, saved_states, ws = _ss_fwd_args(
        u, delta, A, B, C, D, delta_bias, z, h0, delta_softplus, out, final_state, saved_states,
        want_final_state, want_saved_states, workspace)
    _check(lib().msc_selective_scan_fwd(ctypes.byref(a), _stream(stream)))
    return out, final_state, saved_states


def msc_selective_scan_conv_fwd(x, conv_w, delta, A, B, C, conv_bias=None, conv_state=None,
                                D=None, delta_bias=None, z=None, h0=None, delta_softplus=True,
                                want_u=True, want_conv_state=True, want_final_state=True,
                                want_saved_states=True, u_out=None, conv_state_out=None,
                                out=None, final_state=None, saved_states=None, workspace=None,
                                stream=None):
    """The causal conv1d + SiLU fused ahead of the Mamba-1 forward: x [B, D, L]
    is the conv's input, conv_w f32 [D, W], conv_bias f32 [D], conv_state
    f32 [B, D, W-1] (the inputs before x).

    Returns (out, final_state, saved_states, u, conv_state_out); u is the
    scan's input silu(conv(x)) (what the backward pass takes as u).  Output
    tensors may be given (u_out, conv_state_out, out, final_state,
    saved_states); the missing ones are allocated when wanted."""
    a, out, final_state, saved_states, ws = _ss_fwd_args(
        x, delta, A, B, C, D, delta_bias, z, h0, delta_softplus, out, final_state, saved_states,
        want_final_state, want_saved_states, workspace)
    Bsz, Dm, _L = x.shape
    W = conv_w.shape[1]
    u = u_out if u_out is not None else (torch.empty_like(x) if want_u else None)
    xs_out = conv_state_out
    if xs_out is None and want_conv_state:
        xs_out = torch.empty((Bsz, Dm, max(W - 1, 0)), device=x.device, dtype=torch.float32)
    c = SsConvArgs(ctypes.sizeof(SsConvArgs), W, _ptr(conv_w), _ptr(conv_bias),
                   _ptr(conv_state), _ptr(xs_out), _ptr(u))
    _check(lib().msc_selective_scan_conv_fwd(ctypes.byref(a), ctypes.byref(c), _stream(stream)))
    return out, final_state, saved_states, u, xs_out


def _ss_fwd_args(u, delta, A, B, C, D, delta_bias, z, h0, delta_softplus, out, final_state,
                 saved_states, want_final_state, want_saved_states, workspace):
    Bsz, Dm, L = u.shape
    G, N = B.shape[1], B.shape[2]
    dev = u.device
    if out is None:
        out = torch.empty_like(u)
    if final_state is None and want_final_state:
        final_state = torch.empty((Bsz, Dm, N), device=dev, dtype=torch.float32)
    if saved_states is None and want_saved_states:
        n_save = (L + MSC_M1_SAVE_INTERVAL - 1) // MSC_M1_SAVE_INTERVAL
        saved_states = torch.empty((Bsz, Dm, max(n_save, 1), N), device=dev, dtype=torch.float32)
    need = msc_selective_scan_fwd_workspace_bytes(Bsz, Dm, N, L)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    a = SsFwdArgs(ctypes.sizeof(SsFwdArgs), _io(u), Bsz, Dm, N, L, G, int(delta_softplus),
                  _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(delta_bias),
                  _ptr(z), _ptr(h0), _ptr(out), _ptr(final_state), _ptr(saved_states),
                  _ptr(workspace), workspace.numel() * workspace.element_size()
                  if workspace is not None else 0)
    return a, out, final_state, saved_states, workspace


def msc_selective_scan_bwd(u, delta, A, B, C, saved_states, dout, D=None, delta_bias=None, z=None,
                           h0=None, delta_softplus=True, workspace=None, want_dh0=True,
                           grads=None, stream=None):
    """Mamba-1 backward.  Returns dict du, ddelta, dA, dB, dC, dD, ddelta_bias, dz, dh0."""
    Bsz, Dm, L = u.shape
    G, N = B.shape[1], B.shape[2]
    dev = u.device
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(grads or {})
    if "du" not in g:
        g["du"] = torch.empty_like(u)
    if "ddelta" not in g:
        g["ddelta"] = torch.empty_like(u)
    if "dA" not in g:
        g["dA"] = torch.empty((Dm, N), **f32)
    if "dB" not in g:
        g["dB"] = torch.empty((Bsz, G, N, L), **f32)
    if "dC" not in g:
        g["dC"] = torch.empty((Bsz, G, N, L), **f32)
    if "dD" not in g:
        g["dD"] = torch.empty((Dm,), **f32)
    if "ddelta_bias" not in g:
        g["ddelta_bias"] = torch.empty((Dm,), **f32)
    if "dz" not in g:
        g["dz"] = torch.empty_like(u) if z is not None else None
    if "dh0" not in g:
        g["dh0"] = torch.empty((Bsz, Dm, N), **f32) if want_dh0 else None
    need = msc_selective_scan_bwd_workspace_bytes(Bsz, Dm, N, L, G)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    a = SsBwdArgs(ctypes.sizeof(SsBwdArgs), _io(u), Bsz, Dm, N, L, G, int(delta_softplus),
                  _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(delta_bias),
                  _ptr(z), _ptr(h0), _ptr(saved_states), _ptr(dout), _ptr(g["du"]),
                  _ptr(g["ddelta"]), _ptr(g["dz"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
                  _ptr(g["dD"]), _ptr(g["ddelta_bias"]), _ptr(g["dh0"]))
    _check(lib().msc_selective_scan_bwd(ctypes.byref(a), _ptr(workspace), workspace.numel(),
                                        _stream(stream)))
    return g


MSC_STATIC_SCRATCH_BYTES = 64 << 20


def msc_selective_scan_bwd_static(u, delta, A, B, C, saved_states, dout, D=None,
                                  delta_bias=None, z=None, h0=None, delta_softplus=True,
                                  want_dh0=True, grads=None, stream=None):
    """Mamba-1 backward with the library's static scratch instead of a workspace
    (for callers that may not allocate device memory; see msc.h)."""
    Bsz, Dm, L = u.shape
    G, N = B.shape[1], B.shape[2]
    dev = u.device
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(grads or {})
    for k, shape in (("dA", (Dm, N)), ("dB", (Bsz, G, N, L)), ("dC", (Bsz, G, N, L)),
                     ("dD", (Dm,)), ("ddelta_bias", (Dm,))):
        if k not in g:
            g[k] = torch.empty(shape, **f32)
    if "du" not in g:
        g["du"] = torch.empty_like(u)
    if "ddelta" not in g:
        g["ddelta"] = torch.empty_like(u)
    if "dz" not in g:
        g["dz"] = torch.empty_like(u) if z is not None else None
    if "dh0" not in g:
        g["dh0"] = torch.empty((Bsz, Dm, N), **f32) if want_dh0 else None
    a = SsBwdArgs(ctypes.sizeof(SsBwdArgs), _io(u), Bsz, Dm, N, L, G, int(delta_softplus),
                  _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(delta_bias),
                  _ptr(z), _ptr(h0), _ptr(saved_states), _ptr(dout), _ptr(g["du"]),
                  _ptr(g["ddelta"]), _ptr(g["dz"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
                  _ptr(g["dD"]), _ptr(g["ddelta_bias"]), _ptr(g["dh0"]))
    _check(lib().msc_selective_scan_bwd_static(ctypes.byref(a), _stream(stream)))
    return g


# ---------------------------------------------------------------------------
# single-token state update
# ---------------------------------------------------------------------------
def msc_ssm_state_update(state, x, delta, A, B, C, D=None, delta_bias=None, z=None,
                         delta_softplus=True, out=None, stream=None):
    """In-place decode step.  state f32 [B, D, N]; x, delta, z [B, D]; B, C [B, G, N]."""
    Bsz, Dm, N = state.shape
    G = B.shape[1]
    if out is None:
        out = torch.empty_like(x)
    a = SuArgs(ctypes.sizeof(SuArgs), _io(x), Bsz, Dm, N, G, int(delta_softplus), _ptr(state),
               _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(delta_bias),
               _ptr(z), _ptr(out))
    _check(lib().msc_ssm_state_update(ctypes.byref(a), _stream(stream)))
    return out


# ---------------------------------------------------------------------------
# Mamba-3 SISO
# ---------------------------------------------------------------------------
def msc_mamba3_siso_saved_states_bytes(batch, seqlen, nheads, headdim, dstate) -> int:
    return int(lib().msc_mamba3_siso_saved_states_bytes(batch, seqlen, nheads, headdim, dstate))


def msc_mamba3_siso_scan_bwd_workspace_bytes(batch, seqlen, nheads, headdim, dstate, ngroups,
                                             nangles) -> int:
    return int(lib().msc_mamba3_siso_scan_bwd_workspace_bytes(batch, seqlen, nheads, headdim,
                                                                 dstate, ngroups, nangles))


def msc_mamba3_siso_scan_fwd_workspace_bytes(batch, seqlen, nheads, headdim, dstate) -> int:
    return int(lib().msc_mamba3_siso_scan_fwd_workspace_bytes(batch, seqlen, nheads, headdim,
                                                                 dstate))


def msc_mamba3_siso_scan_fwd(x, B, C, alpha, beta, gamma, theta, D=None, z=None, h0=None,
                             out=None, final_state=None, saved_states=None,
                             want_final_state=True, want_saved_states=True, workspace=None,
                             stream=None):
    """Mamba-3 SISO forward.  x, z [B, L, H, P]; B, C [B, L, G, N]; alpha, beta, gamma
    [B, L, H]; theta [B, L, H, K].  Returns (out, final_state, saved_states)."""
    Bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    K = theta.shape[3]
    dev = x.device
    if out is None:
        out = torch.empty_like(x)
    if final_state is None and want_final_state:
        final_state = torch.empty((Bsz, H, P, N), device=dev, dtype=torch.float32)
    if saved_states is None and want_saved_states:
        nb = msc_mamba3_siso_saved_states_bytes(Bsz, L, H, P, N)
        saved_states = torch.empty(max(nb // 4, 4), device=dev, dtype=torch.float32)
    need = msc_mamba3_siso_scan_fwd_workspace_bytes(Bsz, L, H, P, N)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    a = M3FwdArgs(ctypes.sizeof(M3FwdArgs), _io(x), Bsz, L, H, P, N, G, K, _ptr(x), _ptr(z),
                  _ptr(B), _ptr(C), _ptr(alpha), _ptr(beta), _ptr(gamma), _ptr(theta), _ptr(D),
                  _ptr(h0), _ptr(out), _ptr(final_state), _ptr(saved_states), _ptr(workspace),
                  workspace.numel() * workspace.element_size() if workspace is not None else 0)
    _check(lib().msc_mamba3_siso_scan_fwd(ctypes.byref(a), _stream(stream)))
    return out, final_state, saved_states


def msc_mamba3_siso_scan_bwd(x, B, C, alpha, beta, gamma, theta, saved_states, dout, D=None,
                             z=None, h0=None, workspace=None, want_dh0=True, grads=None,
                             stream=None):
    """Mamba-3 SISO backward.  Returns dict dx, dz, dB, dC, dalpha, dbeta, dgamma, dtheta, dD, dh0."""
    Bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    K = theta.shape[3]
    dev = x.device
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(grads or {})
    if "dx" not in g:
        g["dx"] = torch.empty_like(x)
    if "dz" not in g:
        g["dz"] = torch.empty_like(x) if z is not None else None
    if "dB" not in g:
        g["dB"] = torch.empty((Bsz, L, G, N), **f32)
    if "dC" not in g:
        g["dC"] = torch.empty((Bsz, L, G, N), **f32)
    if "dalpha" not in g:
        g["dalpha"] = torch.empty((Bsz, L, H), **f32)
    if "dbeta" not in g:
        g["dbeta"] = torch.empty((Bsz, L, H), **f32)
    if "dgamma" not in g:
        g["dgamma"] = torch.empty((Bsz, L, H), **f32)
    if "dtheta" not in g:
        g["dtheta"] = torch.empty((Bsz, L, H, K), **f32)
    if "dD" not in g:
        g["dD"] = torch.empty((H,), **f32)
    if "dh0" not in g:
        g["dh0"] = torch.empty((Bsz, H, P, N), **f32) if want_dh0 else None
    need = msc_mamba3_siso_scan_bwd_workspace_bytes(Bsz, L, H, P, N, G, K)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    a = M3BwdArgs(ctypes.sizeof(M3BwdArgs), _io(x), Bsz, L, H, P, N, G, K, _ptr(x), _ptr(z),
                  _ptr(B), _ptr(C), _ptr(alpha), _ptr(beta), _ptr(gamma), _ptr(theta), _ptr(D),
                  _ptr(h0), _ptr(saved_states), _ptr(dout), _ptr(g["dx"]), _ptr(g["dz"]),
                  _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dalpha"]), _ptr(g["dbeta"]),
                  _ptr(g["dgamma"]), _ptr(g["dtheta"]), _ptr(g["dD"]), _ptr(g["dh0"]))
    _check(lib().msc_mamba3_siso_scan_bwd(ctypes.byref(a), _ptr(workspace), workspace.numel(),
                                          _stream(stream)))
    return g


def _m3_raw(dd_dt, dd_a, trap, angles, B_raw, C_raw, dt_bias, A_floor, eps):
    return M3RawArgs(ctypes.sizeof(M3RawArgs), A_floor, eps, _ptr(dd_dt), _ptr(dd_a), _ptr(trap),
                     _ptr(angles), _ptr(dt_bias), _ptr(B_raw), _ptr(C_raw))


def msc_mamba3_siso_scan_fwd_raw_workspace_bytes(batch, seqlen, nheads, headdim, dstate,
                                                 ngroups, nangles) -> int:
    return int(lib().msc_mamba3_siso_scan_fwd_raw_workspace_bytes(
        batch, seqlen, nheads, headdim, dstate, ngroups, nangles))


def msc_mamba3_siso_scan_fwd_raw(x, dd_dt, dd_a, trap, angles, B_raw, C_raw, dt_bias=None,
                                 A_floor=1e-4, eps=1e-5, D=None, z=None, h0=None, out=None,
                                 final_state=None, saved_states=None, want_final_state=True,
                                 want_saved_states=True, workspace=None, stream=None):
    """Mamba-3 SISO forward from raw projections (bf16, d_state 16, 32 or 64):
    dd_dt, dd_a, trap [B, L, H]; angles [B, L, K]; B_raw, C_raw [B, L, G, N].
    Returns (out, final_state, saved_states); equals msc_mamba3_siso_discretize
    followed by msc_mamba3_siso_scan_fwd bit for bit."""
    Bsz, L, H, P = x.shape
    G, N = B_raw.shape[2], B_raw.shape[3]
    K = angles.shape[2] if angles is not None else 0
    dev = x.device
    if out is None:
        out = torch.empty_like(x)
    if final_state is None and want_final_state:
        final_state = torch.empty((Bsz, H, P, N), device=dev, dtype=torch.float32)
    if saved_states is None and want_saved_states:
        nb = msc_mamba3_siso_saved_states_bytes(Bsz, L, H, P, N)
        saved_states = torch.empty(max(nb // 4, 4), device=dev, dtype=torch.float32)
    if workspace is None:
        need = msc_mamba3_siso_scan_fwd_raw_workspace_bytes(Bsz, L, H, P, N, G, K)
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    a = M3FwdArgs(ctypes.sizeof(M3FwdArgs), _io(x), Bsz, L, H, P, N, G, K, _ptr(x), _ptr(z),
                  None, None, None, None, None, None, _ptr(D), _ptr(h0), _ptr(out),
                  _ptr(final_state), _ptr(saved_states), _ptr(workspace), workspace.numel())
    r = _m3_raw(dd_dt, dd_a, trap, angles, B_raw, C_raw, dt_bias, A_floor, eps)
    _check(lib().msc_mamba3_siso_scan_fwd_raw(ctypes.byref(a), ctypes.byref(r), _stream(stream)))
    return out, final_state, saved_states


def msc_mamba3_siso_scan_bwd_raw_workspace_bytes(batch, seqlen, nheads, headdim, dstate,
                                                 ngroups, nangles) -> int:
    return int(lib().msc_mamba3_siso_scan_bwd_raw_workspace_bytes(
        batch, seqlen, nheads, headdim, dstate, ngroups, nangles))


def msc_mamba3_siso_scan_bwd_raw(x, dd_dt, dd_a, trap, angles, B_raw, C_raw, saved_states, dout,
                                 dt_bias=None, A_floor=1e-4, eps=1e-5, D=None, z=None, h0=None,
                                 workspace=None, want_dh0=True, grads=None, stream=None):
    """Mamba-3 SISO backward from raw projections (bf16, d_state 16, 32 or 64).
    Returns dict dx, dz, dD, dh0 and ddd_dt, ddd_a, dtrap, dangles, ddt_bias,
    dB_raw, dC_raw; equals the scan's backward followed by
    msc_mamba3_siso_discretize_bwd bit for bit."""
    Bsz, L, H, P = x.shape
    G, N = B_raw.shape[2], B_raw.shape[3]
    K = angles.shape[2] if angles is not None else 0
    dev = x.device
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(grads or {})
    defaults = dict(dx=lambda: torch.empty_like(x),
                    dz=lambda: torch.empty_like(x) if z is not None else None,
                    dD=lambda: torch.empty((H,), **f32),
                    dh0=lambda: torch.empty((Bsz, H, P, N), **f32) if want_dh0 else None,
                    ddd_dt=lambda: torch.empty((Bsz, L, H), **f32),
                    ddd_a=lambda: torch.empty((Bsz, L, H), **f32),
                    dtrap=lambda: torch.empty((Bsz, L, H), **f32),
                    dangles=lambda: torch.empty((Bsz, L, K), **f32) if K > 0 else None,
                    ddt_bias=lambda: torch.empty((H,), **f32),
                    dB_raw=lambda: torch.empty((Bsz, L, G, N), **f32),
                    dC_raw=lambda: torch.empty((Bsz, L, G, N), **f32))
    for k, mk in defaults.items():
        if k not in g:
            g[k] = mk()
    need = msc_mamba3_siso_scan_bwd_raw_workspace_bytes(Bsz, L, H, P, N, G, K)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    a = M3BwdArgs(ctypes.sizeof(M3BwdArgs), _io(x), Bsz, L, H, P, N, G, K, _ptr(x), _ptr(z),
                  None, None, None, None, None, None, _ptr(D), _ptr(h0), _ptr(saved_states),
                  _ptr(dout), _ptr(g["dx"]), _ptr(g["dz"]), None, None, None, None, None, None,
                  _ptr(g["dD"]), _ptr(g["dh0"]))
    r = _m3_raw(dd_dt, dd_a, trap, angles, B_raw, C_raw, dt_bias, A_floor, eps)
    gr = M3RawGrads(ctypes.sizeof(M3RawGrads), _ptr(g["ddd_dt"]), _ptr(g["ddd_a"]),
                    _ptr(g["dtrap"]), _ptr(g["dangles"]), _ptr(g["ddt_bias"]), _ptr(g["dB_raw"]),
                    _ptr(g["dC_raw"]))
    _check(lib().msc_mamba3_siso_scan_bwd_raw(ctypes.byref(a), ctypes.byref(r), ctypes.byref(gr),
                                              _ptr(workspace), workspace.numel(),
                                              _stream(stream)))
    return g


def msc_mamba3_siso_state_update(state, x_prev, bt_prev, phi, x, B, C, alpha, beta, gamma,
                                 theta, D=None, z=None, out=None, stream=None):
    """In-place Mamba-3 SISO decode step.  Carried: state f32 [B, H, P, N], x_prev f32
    [B, H, P], bt_prev f32 [B, H, N], phi f32 [B, H, K].  Step inputs: x, z [B, H, P];
    B, C [B, G, N]; alpha, beta, gamma [B, H]; theta [B, H, K].  Returns out [B, H, P]."""
    Bsz, H, P, N = state.shape
    G = B.shape[1]
    K = phi.shape[2]
    if out is None:
        out = torch.empty_like(x)
    a = M3SuArgs(ctypes.sizeof(M3SuArgs), _io(x), Bsz, H, P, N, G, K, _ptr(state), _ptr(x_prev),
                 _ptr(bt_prev), _ptr(phi) if K > 0 else None, _ptr(x), _ptr(z), _ptr(B), _ptr(C),
                 _ptr(alpha), _ptr(beta), _ptr(gamma), _ptr(theta) if K > 0 else None, _ptr(D),
                 _ptr(out))
    _check(lib().msc_mamba3_siso_state_update(ctypes.byref(a), _stream(stream)))
    return out


def msc_mamba3_siso_disc_state_update(state, x_prev, bt_prev, phi, x, dd_dt, dd_a, trap, angles,
                                      B_raw, C_raw, dt_bias=None, A_floor=1e-4, eps=1e-5, D=None,
                                      z=None, out=None, stream=None):
    """The Mamba-3 decode step from this token's raw values (the discretisation
    and BCNorm fused ahead).  Carried state as msc_mamba3_siso_state_update;
    dd_dt, dd_a, trap [B, H]; angles [B, K]; B_raw, C_raw [B, G, N] (io);
    dt_bias f32 [H].  Returns out [B, H, P]."""
    Bsz, H, P, N = state.shape
    G = B_raw.shape[1]
    K = phi.shape[2]
    if out is None:
        out = torch.empty_like(x)
    a = M3SuArgs(ctypes.sizeof(M3SuArgs), _io(x), Bsz, H, P, N, G, K, _ptr(state), _ptr(x_prev),
                 _ptr(bt_prev), _ptr(phi) if K > 0 else None, _ptr(x), _ptr(z), None, None,
                 None, None, None, None, _ptr(D), _ptr(out))
    r = M3DiscStepArgs(ctypes.sizeof(M3DiscStepArgs), A_floor, eps, _ptr(dd_dt), _ptr(dd_a),
                       _ptr(trap), _ptr(angles) if K > 0 else None, _ptr(dt_bias), _ptr(B_raw),
                       _ptr(C_raw))
    _check(lib().msc_mamba3_siso_disc_state_update(ctypes.byref(a), ctypes.byref(r),
                                                   _stream(stream)))
    return out


def msc_mamba3_siso_discretize(dd_dt, dd_a, trap, angles, B_raw, C_raw, dt_bias=None,
                               A_floor=1e-4, eps=1e-5, outs=None, stream=None):
    """Discretisation and BCNorm ahead of the Mamba-3 scan.  dd_dt, dd_a, trap
    [B, L, H]; angles [B, L, K]; B_raw, C_raw [B, L, G, N] (io); dt_bias f32 [H].
    Returns dict alpha, beta, gamma, theta, B, C (io, the scan's inputs)."""
    Bsz, L, H = dd_dt.shape
    G, N = B_raw.shape[2], B_raw.shape[3]
    K = angles.shape[2] if angles is not None else 0
    o = dict(outs or {})
    for k in ("alpha", "beta", "gamma"):
        if k not in o:
            o[k] = torch.empty_like(dd_dt)
    if "theta" not in o:
        o["theta"] = torch.empty((Bsz, L, H, K), device=dd_dt.device, dtype=dd_dt.dtype)
    if "B" not in o:
        o["B"] = torch.empty_like(B_raw)
    if "C" not in o:
        o["C"] = torch.empty_like(C_raw)
    a = M3DiscArgs(ctypes.sizeof(M3DiscArgs), _io(dd_dt), Bsz, L, H, N, G, K, A_floor, eps,
                   _ptr(dd_dt), _ptr(dd_a), _ptr(trap), _ptr(angles) if K > 0 else None,
                   _ptr(dt_bias), _ptr(B_raw), _ptr(C_raw), _ptr(o["alpha"]), _ptr(o["beta"]),
                   _ptr(o["gamma"]), _ptr(o["theta"]) if K > 0 else None, _ptr(o["B"]),
                   _ptr(o["C"]))
    _check(lib().msc_mamba3_siso_discretize(ctypes.byref(a), _stream(stream)))
    return o


def msc_mamba3_siso_discretize_bwd(dd_dt, dd_a, trap, angles, B_raw, C_raw, dalpha, dbeta,
                                   dgamma, dtheta, dB, dC, dt_bias=None, A_floor=1e-4,
                                   eps=1e-5, want_ddt_bias=True, grads=None, stream=None):
    """Backward of msc_mamba3_siso_discretize for f32 upstream gradients (as the
    scan backward returns them).  Returns dict ddd_dt, ddd_a, dtrap, dangles,
    ddt_bias, dB_raw, dC_raw (f32)."""
    Bsz, L, H = dd_dt.shape
    G, N = B_raw.shape[2], B_raw.shape[3]
    K = angles.shape[2] if angles is not None else 0
    f32 = dict(device=dd_dt.device, dtype=torch.float32)
    g = dict(grads or {})
    for k in ("ddd_dt", "ddd_a", "dtrap"):
        if k not in g:
            g[k] = torch.empty((Bsz, L, H), **f32)
    if "dangles" not in g:
        g["dangles"] = torch.empty((Bsz, L, K), **f32)
    if "ddt_bias" not in g:
        g["ddt_bias"] = torch.empty((H,), **f32) if want_ddt_bias else None
    if "dB_raw" not in g:
        g["dB_raw"] = torch.empty((Bsz, L, G, N), **f32)
    if "dC_raw" not in g:
        g["dC_raw"] = torch.empty((Bsz, L, G, N), **f32)
    a = M3DiscBwdArgs(ctypes.sizeof(M3DiscBwdArgs), _io(dd_dt), Bsz, L, H, N, G, K, A_floor,
                      eps, _ptr(dd_dt), _ptr(dd_a), _ptr(trap), _ptr(angles) if K > 0 else None,
                      _ptr(dt_bias), _ptr(B_raw), _ptr(C_raw), _ptr(dalpha), _ptr(dbeta),
                      _ptr(dgamma), _ptr(dtheta) if K > 0 else None, _ptr(dB), _ptr(dC),
                      _ptr(g["ddd_dt"]), _ptr(g["ddd_a"]), _ptr(g["dtrap"]),
                      _ptr(g["dangles"]) if K > 0 else None, _ptr(g["ddt_bias"]),
                      _ptr(g["dB_raw"]), _ptr(g["dC_raw"]))
    _check(lib().msc_mamba3_siso_discretize_bwd(ctypes.byref(a), _stream(stream)))
    return g


# ---------------------------------------------------------------------------
# causal conv1d + SiLU ahead of the Mamba-1 scan
# ---------------------------------------------------------------------------
def msc_causal_conv1d_fwd(x, w, bias=None, conv_state_in=None, u=None, conv_state_out=None,
                          want_state=True, stream=None):
    """u = silu(causal depthwise conv of x).  x [B, D, L] (io); w f32 [D, W];
    bias f32 [D]; conv states f32 [B, D, W-1].  Returns (u, conv_state_out)."""
    Bsz, Dm, L = x.shape
    W = w.shape[1]
    if u is None:
        u = torch.empty_like(x)
    if conv_state_out is None and want_state and W > 1:
        conv_state_out = torch.empty((Bsz, Dm, W - 1), device=x.device, dtype=torch.float32)
    a = ConvFwdArgs(ctypes.sizeof(ConvFwdArgs), _io(x), Bsz, Dm, L, W, _ptr(x), _ptr(w),
                    _ptr(bias), _ptr(conv_state_in), _ptr(u), _ptr(conv_state_out))
    _check(lib().msc_causal_conv1d_fwd(ctypes.byref(a), _stream(stream)))
    return u, conv_state_out


def msc_causal_conv1d_bwd_workspace_bytes(batch, dim, seqlen, width) -> int:
    return int(lib().msc_causal_conv1d_bwd_workspace_bytes(batch, dim, seqlen, width))


def msc_causal_conv1d_bwd(x, w, du, bias=None, conv_state_in=None, workspace=None,
                          want_dstate=True, grads=None, stream=None):
    """Backward of msc_causal_conv1d_fwd for the upstream du.  Returns dict dx, dw,
    dbias, dconv_state_in."""
    Bsz, Dm, L = x.shape
    W = w.shape[1]
    f32 = dict(device=x.device, dtype=torch.float32)
    g = dict(grads or {})
    if "dx" not in g:
        g["dx"] = torch.empty_like(x)
    if "dw" not in g:
        g["dw"] = torch.empty((Dm, W), **f32)
    if "dbias" not in g:
        g["dbias"] = torch.empty((Dm,), **f32) if bias is not None else None
    if "dconv_state_in" not in g:
        g["dconv_state_in"] = (torch.empty((Bsz, Dm, W - 1), **f32)
                               if want_dstate and W > 1 else None)
    if workspace is None:
        need = msc_causal_conv1d_bwd_workspace_bytes(Bsz, Dm, L, W)
        workspace = torch.empty(max(need, 16), device=x.device, dtype=torch.uint8)
    a = ConvBwdArgs(ctypes.sizeof(ConvBwdArgs), _io(x), Bsz, Dm, L, W, _ptr(x), _ptr(w),
                    _ptr(bias), _ptr(conv_state_in), _ptr(du), _ptr(g["dx"]), _ptr(g["dw"]),
                    _ptr(g["dbias"]), _ptr(g["dconv_state_in"]))
    _check(lib().msc_causal_conv1d_bwd(ctypes.byref(a), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)))
    return g
