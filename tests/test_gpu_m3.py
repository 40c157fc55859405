"""GPU parity of the Mamba-3 SISO scan (forward, backward) against the f64
oracle, through the C ABI (libmsc.so via its binding)."""
import numpy as np
import pytest

import oracle
from selective_state_space_14_b200 import workloads as W
from tests._util import TOL, assert_close, dev, host, m3_device_args

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# f32 elementwise guards of the Mamba-3 recurrences (tests/_util.py)
FAMILY = "m3"

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
    (2, 200, 4, 64, 64, 2, 32, "f16", True, True, True),
    (1, 65, 3, 16, 32, 3, 16, "f16", False, True, True),
    # d_state above 64: slabs of 64 states (angle pairs split across the slabs,
    # a slab without angles, a slab with a few)
    (1, 130, 2, 64, 128, 1, 64, "bf16", True, True, True),
    (1, 129, 2, 64, 128, 1, 10, "bf16", True, True, False),
    (2, 70, 2, 32, 256, 2, 100, "f32", True, True, True),
    (1, 65, 2, 16, 192, 1, 96, "bf16", False, False, True),
    (1, 64, 2, 64, 128, 1, 10, "f16", True, True, True),
]


@pytest.mark.parametrize("case", FWD_CASES,
                         ids=[f"B{c[0]}L{c[1]}H{c[2]}P{c[3]}N{c[4]}G{c[5]}K{c[6]}{c[7]}" for c in FWD_CASES])
def test_fwd_parity_shapes(msc, case):
    Bsz, L, H, P, N, G, K, io, z, Dp, h0 = case
    p = W.m3_problem(Bsz, L, H, P, N, ngroups=G, nangles=K, io=io, seed=77 + L + H, with_z=z,
                     with_D=Dp, with_h0=h0)
    g, _, _ = _gpu_fwd(msc, p)
    r = _oracle_fwd(p)
    assert_close("out", g["out"], r["out"], TOL[io], FAMILY)
    assert_close("final_state", g["final_state"], r["final_state"], TOL[io], FAMILY)


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
    assert_close("out", host(out1), r["out"], TOL[io], FAMILY)
    assert_close("final_state", host(fs1), r["final_state"], TOL[io], FAMILY)
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
    assert_close("out", g["out"], r["out"], TOL["bf16"], FAMILY)
    assert_close("final_state", g["final_state"], r["final_state"], TOL["bf16"], FAMILY)


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
    (1, 130, 2, 32, 64, 1, 10, "f16", True, True, True),
    (2, 70, 2, 64, 64, 1, 32, "f16", True, False, True),
    (1, 130, 2, 64, 128, 1, 64, "bf16", True, True, True),
    (1, 70, 2, 32, 256, 1, 100, "f32", True, True, True),
    (2, 65, 2, 16, 128, 2, 20, "f16", True, True, True),
    (1, 100, 2, 64, 192, 1, 40, "bf16", False, True, False),
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
        assert_close(k, g[k], r[k], TOL[io], FAMILY)


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
        assert_close(k, g[k][:1], r[k], TOL["bf16"], FAMILY)


# ---------------------------------------------------------------------------
# single-token state update (decode)
# ---------------------------------------------------------------------------
def _su_device_state(q):
    return [torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
            for a in (q.state0, q.x_prev0, q.bt_prev0, q.phi0)]


SU_CASES = [
    # (B, H, P, N, G, K, io, random_state, z, D, steps)
    (3, 4, 64, 64, 1, 32, "f32", True, True, True, 12),
    (2, 6, 16, 16, 2, 8, "f32", True, True, False, 12),
    (5, 3, 32, 64, 3, 5, "f32", False, False, True, 12),
    (4, 8, 64, 64, 2, 32, "bf16", True, True, True, 40),
    (7, 3, 16, 32, 1, 16, "bf16", True, True, True, 20),
    (3, 5, 64, 16, 1, 0, "bf16", False, True, False, 20),
    (9, 2, 16, 16, 1, 8, "bf16", True, False, True, 20),
    (2, 4, 32, 32, 4, 16, "bf16", True, True, True, 20),
    (3, 4, 64, 64, 1, 32, "f16", True, True, True, 12),
    (2, 6, 16, 32, 2, 8, "f16", False, True, True, 12),
    (2, 3, 64, 128, 1, 64, "bf16", True, True, True, 10),
    (2, 4, 16, 256, 2, 100, "f32", True, True, True, 8),
    (3, 2, 32, 192, 1, 20, "bf16", False, True, True, 8),
]


@pytest.mark.parametrize("case", SU_CASES,
                         ids=[f"B{c[0]}H{c[1]}P{c[2]}N{c[3]}G{c[4]}K{c[5]}{c[6]}" for c in SU_CASES])
def test_m3_state_update_chain(msc, case):
    """Chained decode steps against the oracle's chained steps: every output
    and, at the end, the four carried tensors."""
    Bsz, H, P, N, G, K, io, rs, z, Dp, n = case
    q = W.m3su_problem(Bsz, H, P, N, ngroups=G, nangles=K, io=io, seed=11 + Bsz + N, n_pool=n,
                       random_state=rs, with_z=z, with_D=Dp)
    S, xp, bp, ph = _su_device_state(q)
    ref = [a.astype(np.float64) for a in (q.state0, q.x_prev0, q.bt_prev0, q.phi0)]
    D = dev(q.D)
    for s in q.steps:
        o = msc.msc_mamba3_siso_state_update(S, xp, bp, ph, dev(s["x"]), dev(s["B"]), dev(s["C"]),
                                             dev(s["alpha"]), dev(s["beta"]), dev(s["gamma"]),
                                             dev(s["theta"]), D=D, z=dev(s["z"]))
        f = lambda t: None if t is None else t.as_f64()
        *ref, o_ref = oracle.m3_state_update(*ref, f(s["x"]), f(s["B"]), f(s["C"]),
                                             f(s["alpha"]), f(s["beta"]), f(s["gamma"]),
                                             f(s["theta"]),
                                             D=None if q.D is None else q.D.astype(np.float64),
                                             z=f(s["z"]))
        assert_close("out", host(o), o_ref, TOL[io], FAMILY)
    for name, g, r in zip(("state", "x_prev", "bt_prev", "phi"), (S, xp, bp, ph), ref):
        assert_close(name, host(g), r, TOL[io], FAMILY)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_m3_state_update_chain_equals_scan(msc, io):
    """Decoding a sequence token by token from a fresh carried state (the state
    set to h0) gives the outputs and final state of the scan of the same
    tokens, within the storage tolerance (the scan's chunked tile products and
    the step's per-row sums round differently)."""
    p = W.m3_problem(2, 150, 4, 64, 64, ngroups=2, nangles=32, io=io, seed=5, with_h0=True)
    a = m3_device_args(p)
    out, fs, _ = msc.msc_mamba3_siso_scan_fwd(**a, want_saved_states=False)
    S = a["h0"].clone()
    xp = torch.zeros((2, 4, 64), device="cuda")
    bp = torch.zeros((2, 4, 64), device="cuda")
    ph = torch.zeros((2, 4, 32), device="cuda")
    outs = []
    for t in range(p.seqlen):
        c = lambda k: a[k][:, t].contiguous()
        outs.append(msc.msc_mamba3_siso_state_update(
            S, xp, bp, ph, c("x"), c("B"), c("C"), c("alpha"), c("beta"), c("gamma"), c("theta"),
            D=a["D"], z=c("z")))
    torch.cuda.synchronize()
    assert_close("out", host(torch.stack(outs, dim=1)), host(out), TOL[io], FAMILY)
    assert_close("final_state", host(S), host(fs), TOL[io], FAMILY)


def test_m3_state_update_deterministic(msc):
    q = W.m3su_problem(4, 8, 64, 64, nangles=32, io="bf16", seed=2, n_pool=3, random_state=True)
    runs = []
    for _ in range(2):
        S, xp, bp, ph = _su_device_state(q)
        for s in q.steps:
            o = msc.msc_mamba3_siso_state_update(S, xp, bp, ph, dev(s["x"]), dev(s["B"]),
                                                 dev(s["C"]), dev(s["alpha"]), dev(s["beta"]),
                                                 dev(s["gamma"]), dev(s["theta"]), D=dev(q.D),
                                                 z=dev(s["z"]))
        torch.cuda.synchronize()
        runs.append((o.clone(), S.clone(), bp.clone(), ph.clone()))
    for x, y in zip(*runs):
        assert torch.equal(x, y)


def test_m3_state_update_workload_sampled(msc):
    """The Mamba-3 decode workload (B256 H24 P64 N64 K32, bf16 inputs, f32
    state, 1000 steps cycling a pool of 8 input sets) on the GPU; the oracle
    follows 6 fixed (b, h) rows through all 1000 steps (rows are independent)."""
    q = W.make("m3su_bf16_b256_h24_p64_n64_k32_x1000")
    S, xp, bp, ph = _su_device_state(q)
    D = dev(q.D)
    steps = [{k: dev(v) for k, v in s.items()} for s in q.steps]
    rows = [(0, 0), (17, 5), (100, 23), (128, 12), (201, 7), (255, 23)]
    bi = np.array([r[0] for r in rows])
    hi = np.array([r[1] for r in rows])
    outs = []
    for t in range(1000):
        s = steps[t % 8]
        o = msc.msc_mamba3_siso_state_update(S, xp, bp, ph, s["x"], s["B"], s["C"], s["alpha"],
                                             s["beta"], s["gamma"], s["theta"], D=D, z=s["z"])
        if t % 250 == 249:
            outs.append((t, host(o)[bi, hi]))
    torch.cuda.synchronize()
    # oracle: the sampled rows as one problem of 6 batch rows with one head each
    f = lambda t: t.as_f64()
    pool = [dict(x=f(s["x"])[bi, hi][:, None], z=f(s["z"])[bi, hi][:, None],
                 B=f(s["B"])[bi], C=f(s["C"])[bi], alpha=f(s["alpha"])[bi, hi][:, None],
                 beta=f(s["beta"])[bi, hi][:, None], gamma=f(s["gamma"])[bi, hi][:, None],
                 theta=f(s["theta"])[bi, hi][:, None]) for s in q.steps]
    Dh = q.D.astype(np.float64)[hi]
    ref = [np.zeros((6, 1, 64, 64)), np.zeros((6, 1, 64)), np.zeros((6, 1, 64)),
           np.zeros((6, 1, 32))]
    k = 0
    for t in range(1000):
        s = pool[t % 8]
        # per-row D: run each row as its own head-0 problem with its own D
        new = [np.empty_like(r) for r in ref]
        o_ref = np.empty((6, 1, 64))
        for r in range(6):
            res = oracle.m3_state_update(*[a[r:r + 1] for a in ref], s["x"][r:r + 1],
                                         s["B"][r:r + 1], s["C"][r:r + 1], s["alpha"][r:r + 1],
                                         s["beta"][r:r + 1], s["gamma"][r:r + 1],
                                         s["theta"][r:r + 1], D=Dh[r:r + 1], z=s["z"][r:r + 1])
            for a, b_ in zip(new, res[:4]):
                a[r:r + 1] = b_
            o_ref[r:r + 1] = res[4]
        ref = new
        if k < len(outs) and outs[k][0] == t:
            assert_close(f"out@{t}", outs[k][1], o_ref[:, 0], TOL["bf16"], FAMILY)
            k += 1
    assert_close("state", host(S)[bi, hi], ref[0][:, 0], TOL["bf16"], FAMILY)
    assert_close("phi", host(ph)[bi, hi], ref[3][:, 0], TOL["bf16"], FAMILY)
