"""GPU parity of the causal conv1d (+ SiLU) ahead of the Mamba-1 scan against
the f64 oracle, through the C ABI: forward, backward, the conv feeding the
scan (forward and backward chained), continuation and determinism."""
import numpy as np
import pytest

import oracle
from selective_state_space_14_b200 import workloads as W
from tests._util import TOL, assert_close, dev, host, m1_device_args

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# f32 elementwise guards of the Mamba-1 recurrences (tests/_util.py)
FAMILY = "m1"


@pytest.fixture(scope="module")
def msc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_14_b200 import msc as m
    m.lib()
    return m


def _problem(Bsz, Dm, L, Wd, io, seed, bias=True, state=False):
    rng = np.random.default_rng(seed)
    x = W.store(rng.standard_normal((Bsz, Dm, L)).astype(np.float32), io)
    w = (rng.standard_normal((Dm, Wd)) / np.sqrt(Wd)).astype(np.float32)
    b = rng.standard_normal(Dm).astype(np.float32) if bias else None
    xs0 = rng.standard_normal((Bsz, Dm, Wd - 1)).astype(np.float32) if state and Wd > 1 else None
    du = W.store(rng.standard_normal((Bsz, Dm, L)).astype(np.float32), io)
    return x, w, b, xs0, du


CASES = [
    # (B, D, L, W, io, bias, state)
    (1, 3, 1, 4, "f32", True, False),
    (2, 5, 17, 4, "f32", True, True),
    (1, 8, 64, 3, "f32", False, True),
    (2, 16, 130, 2, "f32", True, False),
    (1, 4, 33, 1, "f32", True, False),
    (2, 96, 1000, 4, "bf16", True, True),
    (1, 40, 257, 4, "bf16", True, False),
    (3, 24, 64, 3, "f16", True, True),
    (2, 3, 8195, 4, "f32", True, True),      # two segments per row
    (1, 2, 270007, 4, "bf16", True, True),   # 64 segment slots, CTAs loop
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}D{c[1]}L{c[2]}W{c[3]}{c[4]}" for c in CASES])
def test_conv_fwd_bwd_parity(msc, case):
    Bsz, Dm, L, Wd, io, bias, state = case
    x, w, b, xs0, du = _problem(Bsz, Dm, L, Wd, io, 3 + L + Dm, bias, state)
    u, xs = msc.msc_causal_conv1d_fwd(dev(x), dev(w), bias=dev(b), conv_state_in=dev(xs0))
    g = msc.msc_causal_conv1d_bwd(dev(x), dev(w), dev(du), bias=dev(b), conv_state_in=dev(xs0))
    torch.cuda.synchronize()
    f64 = lambda a: None if a is None else np.asarray(a, np.float64)
    u_ref, xs_ref = oracle.conv1d_fwd(x.as_f64(), f64(w), bias=f64(b), xs0=f64(xs0))
    r = oracle.conv1d_bwd(x.as_f64(), f64(w), du.as_f64(), bias=f64(b), xs0=f64(xs0))
    assert_close("u", host(u), u_ref, TOL[io], FAMILY)
    if Wd > 1:
        assert_close("conv_state_out", host(xs), xs_ref, TOL["f32"], FAMILY)
    assert_close("dx", host(g["dx"]), r["dx"], TOL[io], FAMILY)
    assert_close("dw", host(g["dw"]), r["dw"], TOL[io], FAMILY)
    if bias:
        assert_close("dbias", host(g["dbias"]), r["dbias"], TOL[io], FAMILY)
    if Wd > 1:
        assert_close("dconv_state_in", host(g["dconv_state_in"]), r["dxs0"], TOL[io], FAMILY)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_feeding_the_scan(msc, io):
    """x -> conv + SiLU -> Mamba-1 scan, forward and backward chained on the GPU,
    against the same chain in the oracle."""
    p = W.m1_problem(2, 48, 16, 300, io=io, seed=12, bias=True, with_h0=True)
    x, w, b, xs0, _ = _problem(2, 48, 300, 4, io, 5, True, True)
    a = m1_device_args(p)
    u, _ = msc.msc_causal_conv1d_fwd(dev(x), dev(w), bias=dev(b), conv_state_in=dev(xs0))
    a["u"] = u
    out, fs, saved = msc.msc_selective_scan_fwd(**a)
    gs = msc.msc_selective_scan_bwd(saved_states=saved, dout=dev(p.dout), **a)
    gc = msc.msc_causal_conv1d_bwd(dev(x), dev(w), gs["du"], bias=dev(b),
                                   conv_state_in=dev(xs0))
    torch.cuda.synchronize()
    f64 = lambda a_: np.asarray(a_, np.float64)
    u_ref, _ = oracle.conv1d_fwd(x.as_f64(), f64(w), bias=f64(b), xs0=f64(xs0))
    ra = oracle.m1_problem_args(p)
    # the scan consumes u as the io dtype stores it
    ra["u"] = W.store(u_ref.astype(np.float32), io).as_f64()
    ref = oracle.m1_fwd(**ra)
    refg = oracle.m1_bwd(dout=p.dout.as_f64(), **ra)
    du_stored = W.store(refg["du"].astype(np.float32), io).as_f64()
    rc = oracle.conv1d_bwd(x.as_f64(), f64(w), du_stored, bias=f64(b), xs0=f64(xs0))
    assert_close("out", host(out), ref["out"], TOL[io], FAMILY)
    assert_close("dx", host(gc["dx"]), rc["dx"], TOL[io], FAMILY)
    assert_close("dw", host(gc["dw"]), rc["dw"], TOL[io], FAMILY)
    assert_close("dbias", host(gc["dbias"]), rc["dbias"], TOL[io], FAMILY)


def test_conv_continuation(msc):
    """Two calls chained through the conv state equal one call over both halves."""
    x, w, b, _, _ = _problem(2, 32, 200, 4, "f32", 9)
    xd = dev(x)
    u, xs = msc.msc_causal_conv1d_fwd(xd, dev(w), bias=dev(b))
    u1, xs1 = msc.msc_causal_conv1d_fwd(xd[:, :, :120].contiguous(), dev(w), bias=dev(b))
    u2, xs2 = msc.msc_causal_conv1d_fwd(xd[:, :, 120:].contiguous(), dev(w), bias=dev(b),
                                        conv_state_in=xs1)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([u1, u2], dim=2), u)
    assert torch.equal(xs2, xs)


def test_conv_deterministic(msc):
    x, w, b, xs0, du = _problem(4, 64, 2048, 4, "bf16", 2, True, True)
    runs = []
    for _ in range(3):
        g = msc.msc_causal_conv1d_bwd(dev(x), dev(w), dev(du), bias=dev(b),
                                      conv_state_in=dev(xs0))
        torch.cuda.synchronize()
        runs.append(g)
    for r in runs[1:]:
        for k in ("dx", "dw", "dbias", "dconv_state_in"):
            assert torch.equal(r[k], runs[0][k]), k


# ---------------------------------------------------------------------------
# the conv fused ahead of the scan forward (one launch)
FUSED_CASES = [
    # (B, D, N, L, G, W, io, state)
    (1, 8, 16, 1, 1, 4, "f32", False),
    (2, 40, 16, 300, 1, 4, "f32", True),
    (2, 72, 32, 129, 2, 3, "f32", True),
    (1, 48, 64, 200, 1, 2, "f32", False),
    (2, 24, 16, 70, 1, 1, "f32", False),
    (2, 96, 16, 513, 1, 4, "bf16", True),
    (1, 64, 128, 130, 1, 4, "bf16", True),
    (2, 48, 16, 257, 3, 4, "f16", True),
]


def _fused_inputs(case, seed):
    Bsz, Dm, N, L, G, Wd, io, state = case
    p = W.m1_problem(Bsz, Dm, N, L, io=io, seed=seed, ngroups=G, bias=True, with_h0=state)
    x, w, b, xs0, _ = _problem(Bsz, Dm, L, Wd, io, seed + 1, True, state)
    return p, x, w, b, xs0


@pytest.mark.parametrize("case", FUSED_CASES,
                         ids=[f"B{c[0]}D{c[1]}N{c[2]}L{c[3]}G{c[4]}W{c[5]}{c[6]}"
                              for c in FUSED_CASES])
def test_fused_conv_scan_fwd_parity(msc, case):
    """One launch of conv + SiLU + scan against the oracle's conv followed by
    its scan (u rounded to the io type between them, as it is stored)."""
    Bsz, Dm, N, L, G, Wd, io, state = case
    p, x, w, b, xs0 = _fused_inputs(case, 40 + L)
    a = m1_device_args(p)
    a.pop("u")
    out, fs, saved, u, xs = msc.msc_selective_scan_conv_fwd(
        dev(x), dev(w), conv_bias=dev(b), conv_state=dev(xs0), **a)
    torch.cuda.synchronize()
    f64 = lambda a_: None if a_ is None else np.asarray(a_, np.float64)
    u_ref, xs_ref = oracle.conv1d_fwd(x.as_f64(), f64(w), bias=f64(b), xs0=f64(xs0))
    ra = oracle.m1_problem_args(p)
    ra["u"] = W.store(u_ref.astype(np.float32), io).as_f64()
    ref = oracle.m1_fwd(**ra)
    assert_close("u", host(u), u_ref, TOL[io], FAMILY)
    assert_close("out", host(out), ref["out"], TOL[io], FAMILY)
    assert_close("final_state", host(fs), ref["final_state"], TOL[io], FAMILY)
    if Wd > 1:
        assert_close("conv_state_out", host(xs), xs_ref, TOL["f32"], FAMILY)


@pytest.mark.parametrize("case", [FUSED_CASES[1], FUSED_CASES[5], FUSED_CASES[6], FUSED_CASES[7]],
                         ids=["f32", "bf16", "bf16_n128", "f16_g3"])
def test_fused_equals_unfused(msc, case):
    """The fused forward gives, bit for bit, what the standalone conv followed
    by the scan forward gives."""
    Bsz, Dm, N, L, G, Wd, io, state = case
    p, x, w, b, xs0 = _fused_inputs(case, 7)
    a = m1_device_args(p)
    a.pop("u")
    out, fs, saved, u, xs = msc.msc_selective_scan_conv_fwd(
        dev(x), dev(w), conv_bias=dev(b), conv_state=dev(xs0), **a)
    u2, xs2 = msc.msc_causal_conv1d_fwd(dev(x), dev(w), bias=dev(b), conv_state_in=dev(xs0))
    out2, fs2, saved2 = msc.msc_selective_scan_fwd(u=u2, **a)
    torch.cuda.synchronize()
    assert torch.equal(u, u2)
    assert torch.equal(xs, xs2)
    assert torch.equal(out, out2)
    assert torch.equal(fs, fs2)
    assert torch.equal(saved, saved2)


def test_fused_conv_scan_train_step(msc):
    """Fused forward, then the scan backward on its u and the conv backward on
    the scan's du, against the oracle's chain."""
    case = (2, 48, 16, 300, 1, 4, "bf16", True)
    p, x, w, b, xs0 = _fused_inputs(case, 21)
    a = m1_device_args(p)
    a.pop("u")
    out, fs, saved, u, _ = msc.msc_selective_scan_conv_fwd(
        dev(x), dev(w), conv_bias=dev(b), conv_state=dev(xs0), **a)
    gs = msc.msc_selective_scan_bwd(u=u, saved_states=saved, dout=dev(p.dout), **a)
    gc = msc.msc_causal_conv1d_bwd(dev(x), dev(w), gs["du"], bias=dev(b), conv_state_in=dev(xs0))
    torch.cuda.synchronize()
    f64 = lambda a_: np.asarray(a_, np.float64)
    u_ref, _ = oracle.conv1d_fwd(x.as_f64(), f64(w), bias=f64(b), xs0=f64(xs0))
    ra = oracle.m1_problem_args(p)
    ra["u"] = W.store(u_ref.astype(np.float32), "bf16").as_f64()
    refg = oracle.m1_bwd(dout=p.dout.as_f64(), **ra)
    du_stored = W.store(refg["du"].astype(np.float32), "bf16").as_f64()
    rc = oracle.conv1d_bwd(x.as_f64(), f64(w), du_stored, bias=f64(b), xs0=f64(xs0))
    assert_close("dA", host(gs["dA"]), refg["dA"], TOL["bf16"], FAMILY)
    assert_close("dx", host(gc["dx"]), rc["dx"], TOL["bf16"], FAMILY)
    assert_close("dw", host(gc["dw"]), rc["dw"], TOL["bf16"], FAMILY)
    assert_close("dconv_state_in", host(gc["dconv_state_in"]), rc["dxs0"], TOL["bf16"], FAMILY)


def test_fused_continuation(msc):
    """Two fused calls chained through the conv state and the scan state equal
    one call over both halves."""
    case = (2, 40, 16, 256, 1, 4, "f32", False)
    p, x, w, b, _ = _fused_inputs(case, 33)
    a = m1_device_args(p)
    for k in ("u", "h0"):
        a.pop(k)
    xd, dd, zd = dev(x), a.pop("delta"), a.pop("z")
    Bd, Cd = a.pop("B"), a.pop("C")
    cut = 96
    half = lambda t, lo, hi: t[..., lo:hi].contiguous()
    out, fs, _, _, xs = msc.msc_selective_scan_conv_fwd(xd, dev(w), dd, B=Bd, C=Cd, z=zd,
                                                        conv_bias=dev(b), **a)
    o1, fs1, _, _, xs1 = msc.msc_selective_scan_conv_fwd(
        half(xd, 0, cut), dev(w), half(dd, 0, cut), B=half(Bd, 0, cut), C=half(Cd, 0, cut),
        z=half(zd, 0, cut), conv_bias=dev(b), **a)
    o2, fs2, _, _, xs2 = msc.msc_selective_scan_conv_fwd(
        half(xd, cut, 256), dev(w), half(dd, cut, 256), B=half(Bd, cut, 256),
        C=half(Cd, cut, 256), z=half(zd, cut, 256), conv_bias=dev(b), conv_state=xs1, h0=fs1,
        **a)
    torch.cuda.synchronize()
    assert torch.equal(xs2, xs)
    assert torch.allclose(torch.cat([o1, o2], dim=2), out, rtol=1e-5, atol=1e-5)
    assert torch.allclose(fs2, fs, rtol=1e-5, atol=1e-5)


def test_conv_workload_full_size(msc):
    """The conv + scan workload (bf16, B8 D1536 N16 L2048, width 4) at full size
    in the launches the bench times: the fused forward against the oracle's
    conv followed by its scan over the whole problem, and the standalone conv
    backward against the oracle's."""
    q = W.make("m1conv_bf16_b8_d1536_n16_l2048_w4")
    a = m1_device_args(q.scan)
    x = a.pop("u")
    out, fs, _, u, xs = msc.msc_selective_scan_conv_fwd(x, dev(q.w), conv_bias=dev(q.bias), **a)
    g = msc.msc_causal_conv1d_bwd(x, dev(q.w), dev(q.scan.dout), bias=dev(q.bias))
    torch.cuda.synchronize()
    f64 = lambda a_: np.asarray(a_, np.float64)
    u_ref, xs_ref = oracle.conv1d_fwd(q.scan.u.as_f64(), f64(q.w), bias=f64(q.bias))
    ra = oracle.m1_problem_args(q.scan)
    ra["u"] = W.store(u_ref.astype(np.float32), "bf16").as_f64()
    ref = oracle.m1_fwd(**ra)
    assert_close("u", host(u), u_ref, TOL["bf16"], FAMILY)
    assert_close("out", host(out), ref["out"], TOL["bf16"], FAMILY)
    assert_close("final_state", host(fs), ref["final_state"], TOL["bf16"], FAMILY)
    assert_close("conv_state_out", host(xs), xs_ref, TOL["f32"], FAMILY)
    rc = oracle.conv1d_bwd(q.scan.u.as_f64(), f64(q.w), q.scan.dout.as_f64(), bias=f64(q.bias))
    for k, rk in (("dx", "dx"), ("dw", "dw"), ("dbias", "dbias")):
        assert_close(k, host(g[k]), rc[rk], TOL["bf16"], FAMILY)


def test_conv_empty_sequences(msc):
    """L = 0: the conv state passes through (or becomes zeros), the gradients of
    the weights are zero; the fused forward also passes the scan state."""
    x = torch.empty(2, 3, 0, device="cuda")
    w = torch.randn(3, 4, device="cuda")
    xs0 = torch.randn(2, 3, 3, device="cuda")
    _, xs = msc.msc_causal_conv1d_fwd(x, w, conv_state_in=xs0)
    _, xz = msc.msc_causal_conv1d_fwd(x, w)
    g = msc.msc_causal_conv1d_bwd(x, w, x, bias=torch.randn(3, device="cuda"), conv_state_in=xs0)
    A = -torch.ones(3, 16, device="cuda")
    Be = torch.empty(2, 1, 16, 0, device="cuda")
    h0 = torch.randn(2, 3, 16, device="cuda")
    out, fs, _, u, xs2 = msc.msc_selective_scan_conv_fwd(x, w, x, A, Be, Be, conv_state=xs0, h0=h0)
    torch.cuda.synchronize()
    assert torch.equal(xs, xs0) and float(xz.abs().sum()) == 0.0
    assert float(g["dw"].abs().sum()) == 0.0 and float(g["dbias"].abs().sum()) == 0.0
    assert float(g["dconv_state_in"].abs().sum()) == 0.0
    assert torch.equal(fs, h0) and torch.equal(xs2, xs0)
