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
    assert_close("u", host(u), u_ref, TOL[io])
    if Wd > 1:
        assert_close("conv_state_out", host(xs), xs_ref, TOL["f32"])
    assert_close("dx", host(g["dx"]), r["dx"], TOL[io])
    assert_close("dw", host(g["dw"]), r["dw"], TOL[io])
    if bias:
        assert_close("dbias", host(g["dbias"]), r["dbias"], TOL[io])
    if Wd > 1:
        assert_close("dconv_state_in", host(g["dconv_state_in"]), r["dxs0"], TOL[io])


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
    assert_close("out", host(out), ref["out"], TOL[io])
    assert_close("dx", host(gc["dx"]), rc["dx"], TOL[io])
    assert_close("dw", host(gc["dw"]), rc["dw"], TOL[io])
    assert_close("dbias", host(gc["dbias"]), rc["dbias"], TOL[io])


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
