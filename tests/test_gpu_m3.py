"""GPU parity of the Mamba-3 SISO scan (forward, backward) against the f64
oracle, through the C ABI (libmsc.so via its binding)."""
import numpy as np
import pytest

import oracle
from selective_state_space_14_b200 import workloads as W
from tests._util import TOL, assert_close, dev, host, m3_device_args

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

M3_GRADS = ("dx", "dz", "dB", "dC", "dalpha", "dbeta", "dgamma", "dtheta", "dD", "dh0")


@pytest.fixture(scope="module")
def msc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_14_b200 import msc as m
    m.lib()
    return m


def _gpu_fwd(msc, p):
    a = m3_device_args(p)
    out, fs, saved = msc.msc_mamba3_siso_scan_fwd(**a)
    torch.cuda.synchronize()
    return dict(out=host(out), final_state=host(fs)), a, saved


def _oracle_fwd(p):
    return oracle.m3_fwd(**oracle.m3_problem_args(p))


FWD_CASES = [
    # (B, L, H, P, N, G, K, io, z, D, h0)
    (1, 1, 1, 16, 16, 1, 8, "f32", True, True, False),
    (2, 7, 2, 16, 16, 1, 4, "f32", True, True, True),
    (1, 64, 2, 32, 16, 1, 8, "f32", False, False, False),
    (1, 65, 3, 16, 32, 3, 16, "f32", True, True, True),
    (2, 200, 4, 64, 64, 2, 32, "f32", True, True, True),
    (1, 130, 2, 32, 64, 1, 0, "f32", True, False, True),
    (2, 300, 4, 64, 64, 1, 32, "bf16", True, True, False),
    (1, 129, 2, 64, 32, 1, 10, "bf16", True, True, True),
    (1, 1, 1, 16, 16, 1, 8, "bf16", True, True, True),
    (2, 7, 2, 16, 32, 1, 4, "bf16", True, True, True),
    (1, 65, 3, 32, 64, 3, 16, "bf16", False, False, True),
    (2, 200, 4, 64, 64, 2, 32, "bf16", True, True, True),
    (1, 130, 2, 32, 16, 1, 0, "bf16", True, False, True),
    (1, 640, 2, 64, 64, 1, 32, "bf16", True, True, True),
]


@pytest.mark.parametrize("case", FWD_CASES,
                         ids=[f"B{c[0]}L{c[1]}H{c[2]}P{c[3]}N{c[4]}G{c[5]}K{c[6]}{c[7]}" for c in FWD_CASES])
def test_fwd_parity_shapes(msc, case):
    Bsz, L, H, P, N, G, K, io, z, Dp, h0 = case
    p = W.m3_problem(Bsz, L, H, P, N, ngroups=G, nangles=K, io=io, seed=77 + L + H, with_z=z,
                     with_D=Dp, with_h0=h0)
    g, _, _ = _gpu_fwd(msc, p)
    r = _oracle_fwd(p)
    assert_close("out", g["out"], r["out"], TOL[io])
    assert_close("final_state", g["final_state"], r["final_state"], TOL[io])


@pytest.mark.parametrize("case", [c for c in FWD_CASES if c[7] == "bf16"],
                         ids=[f"B{c[0]}L{c[1]}H{c[2]}P{c[3]}N{c[4]}G{c[5]}K{c[6]}" for c in FWD_CASES
                              if c[7] == "bf16"])
def test_fwd_without_saved_states(msc, case):
    """bf16 forward without saved states against the oracle, and against the
    same forward with saved states."""
    Bsz, L, H, P, N, G, K, io, z, Dp, h0 = case
    p = W.m3_problem(Bsz, L, H, P, N, ngroups=G, nangles=K, io=io, seed=77 + L + H, with_z=z,
                     with_D=Dp, with_h0=h0)
    a = m3_device_args(p)
    out1, fs1, sv = msc.msc_mamba3_siso_scan_fwd(**a, want_saved_states=False)
    out2, fs2, _ = msc.msc_mamba3_siso_scan_fwd(**a)
    torch.cuda.synchronize()
    assert sv is None
    r = _oracle_fwd(p)
    assert_close("out", host(out1), r["out"], TOL[io])
    assert_close("final_state", host(fs1), r["final_state"], TOL[io])
    assert torch.equal(out1, out2) and torch.equal(fs1, fs2)


def test_fwd_determinism(msc):
    p = W.m3_problem(2, 150, 3, 64, 64, nangles=32, io="bf16", seed=3)
    a = m3_device_args(p)
    outs = []
    for _ in range(3):
        o, fs, sv = msc.msc_mamba3_siso_scan_fwd(**a)
        torch.cuda.synchronize()
        outs.append((o.clone(), fs.clone(), sv.clone()))
    for o in outs[1:]:
        for x, y in zip(o, outs[0]):
            assert torch.equal(x, y)


def test_fwd_empty(msc):
    h0 = torch.randn(2, 3, 16, 16, device="cuda")
    e = torch.empty(2, 0, 3, 16, device="cuda")
    Be = torch.empty(2, 0, 1, 16, device="cuda")
    s3 = torch.empty(2, 0, 3, device="cuda")
    th = torch.empty(2, 0, 3, 4, device="cuda")
    out, fs, _ = msc.msc_mamba3_siso_scan_fwd(e, Be, Be, s3, s3, s3, th, h0=h0)
    torch.cuda.synchronize()
    assert torch.equal(fs, h0)


def test_fwd_model_shaped_full_size(msc):
    """The Mamba-3 SISO workload (bf16, B8 H24 P64 N64 K32 L2048) at full size,
    compared with the f64 oracle on every output."""
    p = W.make("m3_bf16_b8_h24_p64_n64_k32_l2048")
    g, _, _ = _gpu_fwd(msc, p)
    r = _oracle_fwd(p)
    assert_close("out", g["out"], r["out"], TOL["bf16"])
    assert_close("final_state", g["final_state"], r["final_state"], TOL["bf16"])


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
def _gpu_bwd(msc, p):
    a = m3_device_args(p)
    out, fs, saved = msc.msc_mamba3_siso_scan_fwd(**a)
    g = msc.msc_mamba3_siso_scan_bwd(saved_states=saved, dout=dev(p.dout), **a)
    torch.cuda.synchronize()
    return {k: host(v) for k, v in g.items() if v is not None}


def _oracle_bwd(p):
    return oracle.m3_bwd(dout=p.dout.as_f64(), **oracle.m3_problem_args(p))


BWD_CASES = [
    # (B, L, H, P, N, G, K, io, z, D, h0)
    (1, 1, 1, 16, 16, 1, 8, "f32", True, True, True),
    (2, 7, 2, 16, 16, 1, 4, "f32", True, True, True),
    (1, 64, 2, 32, 16, 1, 8, "f32", False, False, False),
    (1, 65, 3, 16, 32, 3, 16, "f32", True, True, True),
    (2, 200, 4, 64, 64, 2, 32, "f32", True, True, True),
    (1, 130, 2, 32, 64, 1, 0, "f32", True, False, True),
    (2, 300, 4, 64, 64, 1, 32, "bf16", True, True, False),
]


@pytest.mark.parametrize("case", BWD_CASES,
                         ids=[f"B{c[0]}L{c[1]}H{c[2]}P{c[3]}N{c[4]}G{c[5]}K{c[6]}{c[7]}" for c in BWD_CASES])
def test_bwd_parity_shapes(msc, case):
    Bsz, L, H, P, N, G, K, io, z, Dp, h0 = case
    p = W.m3_problem(Bsz, L, H, P, N, ngroups=G, nangles=K, io=io, seed=91 + L + H, with_z=z,
                     with_D=Dp, with_h0=h0)
    g = _gpu_bwd(msc, p)
    r = _oracle_bwd(p)
    for k in M3_GRADS:
        if k not in g:
            continue
        if k == "dtheta" and K == 0:
            continue
        if k == "dz" and not z:
            continue
        if k == "dD" and not Dp:
            continue
        assert_close(k, g[k], r[k], TOL[io])


def test_bwd_determinism(msc):
    p = W.m3_problem(2, 150, 3, 64, 64, nangles=32, io="bf16", seed=4, with_h0=True)
    runs = [_gpu_bwd(msc, p) for _ in range(3)]
    for r in runs[1:]:
        for k in runs[0]:
            np.testing.assert_array_equal(r[k], runs[0][k], err_msg=k)


def test_bwd_model_shaped_full_size(msc):
    """The Mamba-3 SISO workload at full size (bf16, B8 H24 P64 N64 K32 L2048):
    the GPU runs all of it; the oracle recomputes batch row 0 (all 24 heads, so
    the group sums of dB and dC are complete) and that row is compared."""
    p = W.make("m3_bf16_b8_h24_p64_n64_k32_l2048")
    g = _gpu_bwd(msc, p)
    T = lambda t: W.Tensor(t.dtype, t.data[:1])
    p0 = W.M3Problem(1, p.seqlen, p.nheads, p.headdim, p.dstate, p.ngroups, p.nangles, p.io,
                     T(p.x), T(p.z), T(p.B), T(p.C), T(p.alpha), T(p.beta), T(p.gamma),
                     T(p.theta), p.D, None, T(p.dout))
    r = _oracle_bwd(p0)
    for k in ("dx", "dz", "dB", "dC", "dalpha", "dbeta", "dgamma", "dtheta", "dh0"):
        assert_close(k, g[k][:1], r[k], TOL["bf16"])
