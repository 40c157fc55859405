"""The C ABI on the host: the library loads without a GPU, exports every
function include/msc.h declares, and refuses bad arguments with the documented
status and a message naming the argument, before touching the device."""
import ctypes
import os
import re

import pytest

from selective_state_space_14_b200 import msc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, ALIGNMENT, CUDA, WORKSPACE = 0, 1, 2, 3, 4, 5


def _header_functions():
    text = open(os.path.join(ROOT, "include", "msc.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(msc_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert _header_functions() == sorted(msc.EXPORTS)


def test_library_exports_every_declared_function():
    lib = ctypes.CDLL(msc.LIB_PATH)
    for name in _header_functions():
        assert hasattr(lib, name), name


def test_version_string():
    assert msc.lib().msc_version().decode().startswith("msc ")


def _err():
    return msc.lib().msc_last_error().decode()


def _fwd_args(**kw):
    a = msc.SsFwdArgs()
    a.struct_size = ctypes.sizeof(msc.SsFwdArgs)
    # 2 x 4096 channels fill the GPU with channel blocks: a single pass over
    # time, which needs no workspace
    a.io_dtype, a.batch, a.dim, a.dstate, a.seqlen, a.ngroups, a.delta_softplus = (
        msc.MSC_BF16, 2, 4096, 16, 128, 1, 1)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    for f in ("u", "delta", "A", "Bm", "Cm", "out"):
        setattr(a, f, fake)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _call_fwd(a):
    return msc.lib().msc_selective_scan_fwd(ctypes.byref(a) if a is not None else None, None)


def test_fwd_rejects_null_args():
    assert _call_fwd(None) == INVALID and "args is NULL" in _err()


def test_fwd_rejects_short_struct():
    assert _call_fwd(_fwd_args(struct_size=8)) == INVALID and "struct_size" in _err()


def test_fwd_rejects_bad_dtype():
    assert _call_fwd(_fwd_args(io_dtype=7)) == INVALID and "io_dtype" in _err()
    assert _call_fwd(_fwd_args(io_dtype=3)) == INVALID and "MSC_F16" in _err()


def test_f16_is_an_io_dtype():
    """MSC_F16 passes the dtype check: the call goes on to the pointer checks
    (a NULL u stops it there, before any launch)."""
    assert _call_fwd(_fwd_args(io_dtype=msc.MSC_F16, u=None)) == INVALID
    assert "io_dtype" not in _err() and "u is NULL" in _err()


@pytest.mark.parametrize("field,value,status,word", [
    ("batch", -1, INVALID, "batch"),
    ("seqlen", -5, INVALID, "seqlen"),
    ("dstate", 0, UNSUPPORTED, "dstate"),
    ("dstate", 257, UNSUPPORTED, "dstate"),
    ("ngroups", 3, INVALID, "ngroups"),
    ("delta_softplus", 2, INVALID, "delta_softplus"),
])
def test_fwd_rejects_bad_sizes(field, value, status, word):
    assert _call_fwd(_fwd_args(**{field: value})) == status
    assert word in _err()


def test_fwd_wide_state_needs_a_workspace():
    """Above 64 states the forward runs in slabs and needs its workspace; the
    call stops at that check (no launch)."""
    assert msc.msc_selective_scan_fwd_workspace_bytes(8, 1536, 64, 128) == 0
    assert msc.msc_selective_scan_fwd_workspace_bytes(2, 64, 65, 128) == 4 * 2 * 64 * 128
    assert _call_fwd(_fwd_args(dstate=128)) == WORKSPACE and "workspace" in _err()


def test_fwd_accepts_the_struct_without_workspace_fields():
    """A struct that ends before the workspace fields is still read (a NULL u
    stops the call at the pointer checks, before any launch)."""
    short = msc.SsFwdArgs.workspace.offset
    assert _call_fwd(_fwd_args(struct_size=short, u=None)) == INVALID and "u is NULL" in _err()
    assert _call_fwd(_fwd_args(struct_size=short - 8)) == INVALID and "struct_size" in _err()


def test_fwd_rejects_missing_input():
    assert _call_fwd(_fwd_args(u=None)) == INVALID and "u" in _err()


def test_fwd_rejects_misaligned_pointer():
    assert _call_fwd(_fwd_args(A=ctypes.c_void_p((1 << 20) + 2))) == ALIGNMENT
    assert "A" in _err()


def test_bwd_rejects_small_workspace():
    a = msc.SsBwdArgs()
    a.struct_size = ctypes.sizeof(msc.SsBwdArgs)
    a.io_dtype, a.batch, a.dim, a.dstate, a.seqlen, a.ngroups, a.delta_softplus = (
        msc.MSC_F32, 1, 64, 16, 64, 1, 1)
    fake = ctypes.c_void_p(1 << 20)
    for f in ("u", "delta", "A", "Bm", "Cm", "saved_states", "dout", "du", "ddelta", "dA",
              "dB", "dC"):
        setattr(a, f, fake)
    need = msc.msc_selective_scan_bwd_workspace_bytes(1, 64, 16, 64, 1)
    st = msc.lib().msc_selective_scan_bwd(ctypes.byref(a), fake, need - 256, None)
    assert st == WORKSPACE and "workspace" in _err()


def test_m3_rejects_unsupported_headdim():
    a = msc.M3FwdArgs()
    a.struct_size = ctypes.sizeof(msc.M3FwdArgs)
    a.io_dtype, a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, 1, 64, 2, 24, 64, 1, 8)
    st = msc.lib().msc_mamba3_siso_scan_fwd(ctypes.byref(a), None)
    assert st == UNSUPPORTED and "headdim" in _err()


def test_m3_wide_state_needs_a_workspace():
    """d_state 128 runs as slabs; the forward then needs its workspace (the call
    stops at that check, before any launch)."""
    assert msc.msc_mamba3_siso_scan_fwd_workspace_bytes(2, 100, 3, 64, 64) == 0
    assert msc.msc_mamba3_siso_scan_fwd_workspace_bytes(2, 100, 3, 64, 128) == 4 * 2 * 100 * 3 * 64
    a = msc.M3FwdArgs()
    a.struct_size = ctypes.sizeof(msc.M3FwdArgs)
    a.io_dtype, a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, 1, 64, 2, 64, 128, 1, 8)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the workspace check fails first
    for f in ("x", "Bm", "Cm", "alpha", "beta", "gamma", "theta", "out"):
        setattr(a, f, fake)
    assert msc.lib().msc_mamba3_siso_scan_fwd(ctypes.byref(a), None) == WORKSPACE
    assert "workspace" in _err()


def test_m3_rejects_too_many_angles():
    a = msc.M3FwdArgs()
    a.struct_size = ctypes.sizeof(msc.M3FwdArgs)
    a.io_dtype, a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, 1, 64, 2, 64, 16, 1, 9)
    st = msc.lib().msc_mamba3_siso_scan_fwd(ctypes.byref(a), None)
    assert st == INVALID and "nangles" in _err()


def test_state_update_rejects_null():
    assert msc.lib().msc_ssm_state_update(None, None) == INVALID


def _m3su_args(**kw):
    a = msc.M3SuArgs()
    a.struct_size = ctypes.sizeof(msc.M3SuArgs)
    a.io_dtype, a.batch, a.nheads, a.headdim, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, 2, 4, 64, 64, 1, 32)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,status,word", [
    ("headdim", 48, UNSUPPORTED, "headdim"),
    ("dstate", 96, UNSUPPORTED, "dstate"),
    ("dstate", 320, UNSUPPORTED, "dstate"),
    ("nangles", 33, INVALID, "nangles"),
    ("ngroups", 3, INVALID, "ngroups"),
    ("nheads", 0, INVALID, "nheads"),
    ("io_dtype", 7, INVALID, "io_dtype"),
    ("struct_size", 8, INVALID, "struct_size"),
])
def test_m3_state_update_rejects_bad_sizes(field, value, status, word):
    st = msc.lib().msc_mamba3_siso_state_update(ctypes.byref(_m3su_args(**{field: value})), None)
    assert st == status and word in _err()


def test_m3_state_update_rejects_missing_and_misaligned():
    assert msc.lib().msc_mamba3_siso_state_update(None, None) == INVALID
    st = msc.lib().msc_mamba3_siso_state_update(ctypes.byref(_m3su_args()), None)
    assert st == INVALID and "state" in _err()
    a = _m3su_args(state=0x1000, x_prev=0x2000, bt_prev=0x3008)
    st = msc.lib().msc_mamba3_siso_state_update(ctypes.byref(a), None)
    assert st == ALIGNMENT and "bt_prev" in _err()


def test_m3_state_update_empty_batch_is_a_no_op():
    assert msc.lib().msc_mamba3_siso_state_update(ctypes.byref(_m3su_args(batch=0)), None) == 0


def test_size_functions():
    # saved states: f32 [B, D, ceil(L / 8), N]
    assert msc.msc_selective_scan_saved_states_bytes(2, 3, 16, 17) == 4 * 2 * 3 * 3 * 16
    # M3 saved states: f32 [B, H, ceil(L / 64), P, N] + angles f32 [B, H, ceil(L / 64), N / 2]
    assert int(msc.lib().msc_mamba3_siso_saved_states_bytes(2, 65, 3, 16, 32)) == \
        4 * 2 * 3 * 2 * (16 * 32 + 16)
    assert msc.msc_selective_scan_bwd_workspace_bytes(8, 1536, 16, 2048, 1) <= \
        msc.MSC_STATIC_SCRATCH_BYTES


def test_fwd_time_segments_workspace():
    """The forward runs in time segments when its (batch, channel) grid has
    fewer CTAs than SMs: two floats per segment and state element.  B1 D64
    N16 L256 gives 4 channel blocks, so 4 segments of 64 steps; grids of 148
    or more blocks, and d_state above 64 (slabs), take none."""
    assert msc.msc_selective_scan_fwd_workspace_bytes(1, 64, 16, 256) == 4 * 2 * 4 * 64 * 16
    assert msc.msc_selective_scan_fwd_workspace_bytes(8, 1536, 16, 2048) == 0
    assert msc.msc_selective_scan_fwd_workspace_bytes(1, 64, 16, 63) == 0  # too short to split
    assert msc.msc_selective_scan_fwd_workspace_bytes(1, 8, 128, 4096) == 4 * 1 * 8 * 4096


def test_bwd_workspace_holds_the_time_segments():
    """A grid of few (batch, channel) blocks splits the backward into time
    segments: the workspace then holds per-segment partials and summaries; a
    model-shaped grid does not split."""
    def base(B, D, N, L, n_part, n_seg=1):
        up = lambda v: (v + 255) // 256 * 256
        return up(4 * n_part * B * 2 * N * L) + up(4 * n_seg * B * D * (N + 2))
    # 8 CTAs of 12 channels (one cluster): 4 segments of 64 steps
    got = msc.msc_selective_scan_bwd_workspace_bytes(1, 64, 16, 256, 1)
    assert got == base(1, 64, 16, 256, 1, 4) + 4 * 2 * 4 * 1 * 64 * 16
    # the 130M-layer shape fills the GPU: no segments (ceil(1536 / 12) = 128
    # CTAs per batch row, one partial per cluster of 8)
    assert msc.msc_selective_scan_bwd_workspace_bytes(8, 1536, 16, 2048, 1) == \
        base(8, 1536, 16, 2048, 128 // 8)


def test_bwd_workspace_query_refuses_bad_groups():
    """ngroups < 1 or not a divisor of dim needs no workspace (the backward
    refuses it); the query must not divide by it."""
    assert msc.msc_selective_scan_bwd_workspace_bytes(2, 64, 16, 128, 0) == 0
    assert msc.msc_selective_scan_bwd_workspace_bytes(2, 64, 16, 128, -2) == 0
    assert msc.msc_selective_scan_bwd_workspace_bytes(2, 64, 16, 128, 3) == 0
    assert msc.msc_selective_scan_bwd_workspace_bytes(2, 64, 300, 128, 1) == 0


@pytest.mark.parametrize("field,value,status,word", [
    ("ngroups", 0, INVALID, "ngroups"),
    ("ngroups", -1, INVALID, "ngroups"),
    ("ngroups", 3, INVALID, "ngroups"),
    ("dstate", 0, UNSUPPORTED, "dstate"),
    ("io_dtype", 9, INVALID, "io_dtype"),
    ("delta_softplus", 2, INVALID, "delta_softplus"),
])
def test_static_backward_checks_arguments_before_sizing(field, value, status, word):
    """The allocation-free backward validates its arguments the way the
    workspace backward does, before the scratch size is computed (no host
    division by ngroups = 0); nothing is launched, so no GPU is needed."""
    a = msc.SsBwdArgs()
    a.struct_size = ctypes.sizeof(msc.SsBwdArgs)
    a.io_dtype, a.batch, a.dim, a.dstate, a.seqlen, a.ngroups = msc.MSC_BF16, 2, 64, 16, 128, 1
    a.delta_softplus = 1
    setattr(a, field, value)
    st = msc.lib().msc_selective_scan_bwd_static(ctypes.byref(a), None)
    assert st == status and word in _err()


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    """No silent fallback: without libmsc.so the binding raises."""
    monkeypatch.setattr(msc, "LIB_PATH", str(tmp_path / "missing" / "libmsc.so"))
    monkeypatch.setattr(msc, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        msc.lib()


def _conv_args(cls, **kw):
    a = cls()
    a.struct_size = ctypes.sizeof(cls)
    a.io_dtype, a.batch, a.dim, a.seqlen, a.width = msc.MSC_BF16, 2, 8, 64, 4
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,status,word", [
    ("width", 0, UNSUPPORTED, "width"),
    ("width", 5, UNSUPPORTED, "width"),
    ("seqlen", -1, INVALID, "seqlen"),
    ("io_dtype", 9, INVALID, "io_dtype"),
    ("struct_size", 4, INVALID, "struct_size"),
])
def test_conv_rejects_bad_sizes(field, value, status, word):
    st = msc.lib().msc_causal_conv1d_fwd(ctypes.byref(_conv_args(msc.ConvFwdArgs, **{field: value})),
                                         None)
    assert st == status and word in _err()


def test_conv_rejects_missing_weights_and_workspace():
    """No weights: rejected; backward without a workspace: rejected (the calls
    stop at the checks, before any launch)."""
    assert msc.lib().msc_causal_conv1d_fwd(ctypes.byref(_conv_args(msc.ConvFwdArgs)), None) == INVALID
    assert "w is NULL" in _err()
    fake = ctypes.c_void_p(1 << 20)
    a = _conv_args(msc.ConvBwdArgs, w=fake, x=fake, du=fake, dx=fake, dw=fake)
    assert msc.lib().msc_causal_conv1d_bwd(ctypes.byref(a), None, 0, None) == WORKSPACE
    # one f32 partial of (dw, dbias) per row and segment slot: one slot while a
    # row fits 256 runs of 16 steps, at most 64 slots
    assert msc.msc_causal_conv1d_bwd_workspace_bytes(2, 8, 64, 4) == 4 * 2 * 8 * 5
    assert msc.msc_causal_conv1d_bwd_workspace_bytes(2, 8, 8192, 4) == 4 * 2 * 2 * 8 * 5
    assert msc.msc_causal_conv1d_bwd_workspace_bytes(2, 8, 1 << 20, 3) == 4 * 64 * 2 * 8 * 4


def _ss_conv_args(**kw):
    c = msc.SsConvArgs()
    c.struct_size = ctypes.sizeof(msc.SsConvArgs)
    c.width = 4
    c.w = ctypes.c_void_p(1 << 20)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,status,word", [
    ("width", 0, UNSUPPORTED, "width"),
    ("width", 5, UNSUPPORTED, "width"),
    ("struct_size", 8, INVALID, "struct_size"),
    ("w", None, INVALID, "w is NULL"),
])
def test_fused_conv_fwd_rejects_bad_conv_args(field, value, status, word):
    c = _ss_conv_args(**{field: value})
    st = msc.lib().msc_selective_scan_conv_fwd(ctypes.byref(_fwd_args()), ctypes.byref(c), None)
    assert st == status and word in _err() and "msc_selective_scan_conv_fwd" in _err()


def test_fused_conv_fwd_checks_scan_args_and_null_conv():
    """A missing conv is rejected; so is a scan argument the plain forward
    rejects (the call stops at the checks, before any launch)."""
    st = msc.lib().msc_selective_scan_conv_fwd(ctypes.byref(_fwd_args()), None, None)
    assert st == INVALID and "conv is NULL" in _err()
    st = msc.lib().msc_selective_scan_conv_fwd(ctypes.byref(_fwd_args(A=None)),
                                               ctypes.byref(_ss_conv_args()), None)
    assert st == INVALID and "A is NULL" in _err()
    st = msc.lib().msc_selective_scan_conv_fwd(ctypes.byref(_fwd_args(dstate=300)),
                                               ctypes.byref(_ss_conv_args()), None)
    assert st == UNSUPPORTED


def _disc_args(cls=None, **kw):
    cls = cls or msc.M3DiscArgs
    a = cls()
    a.struct_size = ctypes.sizeof(cls)
    a.io_dtype, a.batch, a.seqlen, a.nheads, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, 2, 64, 4, 64, 1, 32)
    a.A_floor, a.eps = 1e-4, 1e-5
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,status,word", [
    ("struct_size", 8, INVALID, "struct_size"),
    ("io_dtype", 7, INVALID, "io_dtype"),
    ("nheads", 0, INVALID, "nheads"),
    ("nangles", 33, INVALID, "nangles"),
    ("eps", -1.0, INVALID, "eps"),
    ("nheads", 200, UNSUPPORTED, "6144"),
])
def test_disc_rejects_bad_sizes(field, value, status, word):
    for fn, cls in (("msc_mamba3_siso_discretize", msc.M3DiscArgs),
                    ("msc_mamba3_siso_discretize_bwd", msc.M3DiscBwdArgs)):
        st = getattr(msc.lib(), fn)(ctypes.byref(_disc_args(cls, **{field: value})), None)
        assert st == status and word in _err() and fn in _err()


def test_disc_rejects_missing_pointers():
    """Inputs, outputs and upstream gradients are required (the calls stop at
    the checks, before any launch); no tokens is a no-op."""
    fake = ctypes.c_void_p(1 << 20)
    st = msc.lib().msc_mamba3_siso_discretize(ctypes.byref(_disc_args()), None)
    assert st == INVALID and "dd_dt is NULL" in _err()
    a = _disc_args(dd_dt=fake, dd_a=fake, trap=fake, angles=fake, B_raw=fake, C_raw=fake)
    assert msc.lib().msc_mamba3_siso_discretize(ctypes.byref(a), None) == INVALID
    assert "alpha is NULL" in _err()
    a.angles = ctypes.c_void_p((1 << 20) + 4)
    assert msc.lib().msc_mamba3_siso_discretize(ctypes.byref(a), None) == ALIGNMENT
    b = _disc_args(msc.M3DiscBwdArgs, dd_dt=fake, dd_a=fake, trap=fake, angles=fake, B_raw=fake,
                   C_raw=fake, dalpha=fake, dbeta=fake, dgamma=fake, dB=fake, dC=fake)
    assert msc.lib().msc_mamba3_siso_discretize_bwd(ctypes.byref(b), None) == INVALID
    assert "ddd_dt is NULL" in _err()
    assert msc.lib().msc_mamba3_siso_discretize(ctypes.byref(_disc_args(batch=0)), None) == OK


def test_fused_decode_checks_raw_args():
    """The fused decode step rejects a missing raw struct or raw input before
    any launch; the plain step's alpha .. Cm are not required."""
    fake = ctypes.c_void_p(1 << 20)
    a = msc.M3SuArgs()
    a.struct_size = ctypes.sizeof(msc.M3SuArgs)
    a.io_dtype, a.batch, a.nheads, a.headdim, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, 2, 4, 64, 64, 1, 32)
    for f in ("state", "x_prev", "bt_prev", "phi", "x", "out"):
        setattr(a, f, fake)
    fn = msc.lib().msc_mamba3_siso_disc_state_update
    assert fn(ctypes.byref(a), None, None) == INVALID and "raw is NULL" in _err()
    r = msc.M3DiscStepArgs()
    r.struct_size = ctypes.sizeof(msc.M3DiscStepArgs)
    r.A_floor, r.eps = 1e-4, 1e-5
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "dd_dt is NULL" in _err()
    r.dd_dt = r.dd_a = r.trap = r.angles = r.B_raw = fake
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "C_raw is NULL" in _err()
    r.eps = -1.0
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "eps" in _err()
    r.eps, r.struct_size = 1e-5, 4
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "struct_size" in _err()


def _m3_raw_scan_args(**kw):
    a = msc.M3FwdArgs()
    a.struct_size = ctypes.sizeof(msc.M3FwdArgs)
    a.io_dtype, a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, 2, 128, 4, 64, 64, 1, 32)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    a.x = a.out = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _m3_raw(**kw):
    r = msc.M3RawArgs()
    r.struct_size = ctypes.sizeof(msc.M3RawArgs)
    r.A_floor, r.eps = 1e-4, 1e-5
    fake = ctypes.c_void_p(1 << 20)
    r.dd_dt = r.dd_a = r.trap = r.angles = r.B_raw = r.C_raw = fake
    for k, v in kw.items():
        setattr(r, k, v)
    return r


@pytest.mark.parametrize("field,value,word", [
    ("io_dtype", msc.MSC_F32, "bf16"),
    ("io_dtype", msc.MSC_F16, "bf16"),
    ("dstate", 128, "dstate"),   # a shape the plain scan takes as slabs
    ("dstate", 48, "dstate"),
])
def test_fused_raw_scan_rejects_what_it_does_not_fuse(field, value, word):
    """The scan from raw projections takes bf16 io and d_state 16, 32 or 64; other
    shapes are MSC_ERR_UNSUPPORTED (the two-call chain serves them)."""
    a = _m3_raw_scan_args(**{field: value})
    st = msc.lib().msc_mamba3_siso_scan_fwd_raw(ctypes.byref(a), ctypes.byref(_m3_raw()), None)
    assert st == UNSUPPORTED and word in _err()


def test_fused_raw_scan_checks_raw_args():
    fn = msc.lib().msc_mamba3_siso_scan_fwd_raw
    a = _m3_raw_scan_args()
    assert fn(ctypes.byref(a), None, None) == INVALID and "raw is NULL" in _err()
    r = _m3_raw(trap=None)
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "trap is NULL" in _err()
    r = _m3_raw(C_raw=None)
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "C_raw is NULL" in _err()
    r = _m3_raw(angles=ctypes.c_void_p((1 << 20) + 2))
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == ALIGNMENT and "angles" in _err()
    r = _m3_raw(eps=-1.0)
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "eps" in _err()
    r = _m3_raw(struct_size=4)
    assert fn(ctypes.byref(a), ctypes.byref(r), None) == INVALID and "struct_size" in _err()
    # the scan struct is checked first
    a.struct_size = 4
    assert fn(ctypes.byref(a), ctypes.byref(_m3_raw()), None) == INVALID
    assert "struct_size" in _err()


def test_fused_raw_fwd_needs_the_bcnorm_workspace():
    """BCNorm's rows (bf16 B and C, once per row) live in the forward's
    workspace; without it the call is refused before any launch."""
    B, L, H, P, N, G, K = 2, 128, 4, 64, 64, 1, 32
    need = msc.msc_mamba3_siso_scan_fwd_raw_workspace_bytes(B, L, H, P, N, G, K)
    assert need >= 2 * 2 * B * L * G * N
    assert msc.msc_mamba3_siso_scan_fwd_raw_workspace_bytes(B, L, H, P, N, 0, K) == 0
    fn = msc.lib().msc_mamba3_siso_scan_fwd_raw
    a = _m3_raw_scan_args()
    assert fn(ctypes.byref(a), ctypes.byref(_m3_raw()), None) == WORKSPACE
    assert "workspace" in _err()
    a.workspace, a.workspace_bytes = ctypes.c_void_p(1 << 20), need - 16
    assert fn(ctypes.byref(a), ctypes.byref(_m3_raw()), None) == WORKSPACE
    a.workspace, a.workspace_bytes = ctypes.c_void_p((1 << 20) + 8), need
    assert fn(ctypes.byref(a), ctypes.byref(_m3_raw()), None) == ALIGNMENT
    # the scan's pointers are checked before BCNorm launches
    a.workspace, a.x = ctypes.c_void_p(1 << 20), None
    assert fn(ctypes.byref(a), ctypes.byref(_m3_raw()), None) == INVALID and "x is NULL" in _err()


def test_fused_raw_bwd_workspace_and_grads():
    """The backward from raw projections needs the scan's workspace plus room for
    the scan's gradients of the derived inputs, and its raw-gradient struct."""
    B, L, H, P, N, G, K = 2, 128, 4, 64, 64, 1, 32
    scan = msc.msc_mamba3_siso_scan_bwd_workspace_bytes(B, L, H, P, N, G, K)
    need = msc.msc_mamba3_siso_scan_bwd_raw_workspace_bytes(B, L, H, P, N, G, K)
    derived = 4 * B * L * (3 * H + H * K + 2 * G * N) + 2 * 2 * B * L * G * N  # + BCNorm's rows
    assert need >= scan + derived
    assert msc.msc_mamba3_siso_scan_bwd_raw_workspace_bytes(B, L, H, P, N, 0, K) == 0
    fake = ctypes.c_void_p(1 << 20)
    a = msc.M3BwdArgs()
    a.struct_size = ctypes.sizeof(msc.M3BwdArgs)
    a.io_dtype, a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.nangles = (
        msc.MSC_BF16, B, L, H, P, N, G, K)
    a.x = a.saved_states = a.dout = a.dx = fake
    fn = msc.lib().msc_mamba3_siso_scan_bwd_raw
    r = _m3_raw()
    assert fn(ctypes.byref(a), ctypes.byref(r), None, fake, need, None) == INVALID
    assert "grads is NULL" in _err()
    g = msc.M3RawGrads()
    g.struct_size = ctypes.sizeof(msc.M3RawGrads)
    g.ddd_dt = g.ddd_a = g.dtrap = g.dangles = g.dB_raw = g.dC_raw = fake
    assert fn(ctypes.byref(a), ctypes.byref(r), ctypes.byref(g), fake, need - 16, None) == WORKSPACE
    g.dangles = None
    assert fn(ctypes.byref(a), ctypes.byref(r), ctypes.byref(g), fake, need, None) == INVALID
    assert "dangles is NULL" in _err()
