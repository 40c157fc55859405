"""GPU parity of the Mamba-3 discretisation and BCNorm stages (forward and
backward) against the f64 oracle, through the C ABI, and chained with the
scan: raw projections -> discretisation -> scan -> scan backward ->
discretisation backward."""
import numpy as np
import pytest

import oracle
from selective_state_space_14_b200 import workloads as W
from tests._util import TOL, assert_close, dev, host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# f32 elementwise guards of the Mamba-3 recurrences (tests/_util.py)
FAMILY = "m3"

DISC_OUT = ("alpha", "beta", "gamma", "theta", "B", "C")
DISC_GRADS = ("ddd_dt", "ddd_a", "dtrap", "dangles", "ddt_bias", "dB_raw", "dC_raw")


@pytest.fixture(scope="module")
def msc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_14_b200 import msc as m
    m.lib()
    return m


def _raw(q):
    return dict(dd_dt=q.dd_dt, dd_a=q.dd_a, trap=q.trap, angles=q.angles, B_raw=q.B_raw,
                C_raw=q.C_raw)


def _oracle_raw(q, bias=True):
    a = {k: v.as_f64() for k, v in _raw(q).items()}
    a["dt_bias"] = q.dt_bias.astype(np.float64) if bias else None
    return a


CASES = [
    # (B, L, H, N, G, K, io, bias, A_floor)
    (1, 1, 1, 16, 1, 8, "f32", True, 1e-4),
    (2, 37, 3, 16, 1, 8, "f32", True, 0.3),      # the floor holds for part of the entries
    (1, 70, 40, 64, 2, 32, "f32", False, 1e-4),  # more heads than lanes
    (2, 33, 4, 17, 1, 3, "f32", True, 1e-4),     # odd d_state
    (1, 20, 2, 32, 2, 0, "f32", True, 1e-4),     # no angles
    (2, 130, 24, 64, 1, 32, "bf16", True, 1e-4),
    (1, 65, 6, 128, 3, 64, "bf16", True, 1e-4),
    (2, 48, 8, 64, 2, 16, "f16", True, 1e-4),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}L{c[1]}H{c[2]}N{c[3]}G{c[4]}K{c[5]}{c[6]}"
                                             for c in CASES])
def test_disc_fwd_bwd_parity(msc, case):
    Bsz, L, H, N, G, K, io, bias, A_floor = case
    q = W.m3disc_problem(Bsz, L, H, 16, N, ngroups=G, nangles=K, io=io, seed=L + H,
                         A_floor=A_floor)
    d = {k: dev(v) for k, v in _raw(q).items()}
    if K == 0:
        d["angles"] = None
    dtb = dev(q.dt_bias) if bias else None
    o = msc.msc_mamba3_siso_discretize(**d, dt_bias=dtb, A_floor=A_floor, eps=q.eps)
    rng = np.random.default_rng(L)
    up = dict(dalpha=rng.standard_normal((Bsz, L, H)), dbeta=rng.standard_normal((Bsz, L, H)),
              dgamma=rng.standard_normal((Bsz, L, H)),
              dtheta=rng.standard_normal((Bsz, L, H, K)),
              dB=rng.standard_normal((Bsz, L, G, N)), dC=rng.standard_normal((Bsz, L, G, N)))
    up = {k: v.astype(np.float32) for k, v in up.items()}
    g = msc.msc_mamba3_siso_discretize_bwd(**d, **{k: dev(v) for k, v in up.items()},
                                           dt_bias=dtb, A_floor=A_floor, eps=q.eps)
    torch.cuda.synchronize()
    ra = _oracle_raw(q, bias)
    ref = oracle.m3_discretize(**ra, A_floor=A_floor, eps=q.eps)
    refg = oracle.m3_discretize_bwd(**ra, **{k: v.astype(np.float64) for k, v in up.items()},
                                    A_floor=A_floor, eps=q.eps)
    for k in DISC_OUT:
        assert_close(k, host(o[k]), ref[k], TOL[io], FAMILY)
    # the gradients are f32 from io-rounded inputs: f32 arithmetic throughout
    for k in DISC_GRADS:
        assert_close(k, host(g[k]), refg[k], TOL["f32"], FAMILY)


def test_disc_chained_with_the_scan(msc):
    """Raw projections through the discretisation, the scan forward and
    backward, and the discretisation backward, against the oracle's chain (the
    scan consuming the discretised values as the io dtype stores them)."""
    q = W.m3disc_problem(2, 130, 4, 32, 64, nangles=32, io="bf16", seed=5, with_h0=True)
    s = q.scan
    d = {k: dev(v) for k, v in _raw(q).items()}
    o = msc.msc_mamba3_siso_discretize(**d, dt_bias=dev(q.dt_bias), A_floor=q.A_floor, eps=q.eps)
    a = dict(x=dev(s.x), B=o["B"], C=o["C"], alpha=o["alpha"], beta=o["beta"], gamma=o["gamma"],
             theta=o["theta"], D=dev(s.D), z=dev(s.z), h0=dev(s.h0))
    out, fs, saved = msc.msc_mamba3_siso_scan_fwd(**a)
    gs = msc.msc_mamba3_siso_scan_bwd(**a, saved_states=saved, dout=dev(s.dout))
    g = msc.msc_mamba3_siso_discretize_bwd(**d, dalpha=gs["dalpha"], dbeta=gs["dbeta"],
                                           dgamma=gs["dgamma"], dtheta=gs["dtheta"], dB=gs["dB"],
                                           dC=gs["dC"], dt_bias=dev(q.dt_bias), A_floor=q.A_floor,
                                           eps=q.eps)
    torch.cuda.synchronize()
    ra = _oracle_raw(q)
    disc = oracle.m3_discretize(**ra, A_floor=q.A_floor, eps=q.eps)
    stored = {k: W.store(v.astype(np.float32), "bf16").as_f64() for k, v in disc.items()}
    f64 = lambda a_: None if a_ is None else np.asarray(a_, np.float64)
    sa = dict(x=s.x.as_f64(), B=stored["B"], C=stored["C"], alpha=stored["alpha"],
              beta=stored["beta"], gamma=stored["gamma"], theta=stored["theta"], D=f64(s.D),
              z=s.z.as_f64(), h0=f64(s.h0))
    ref = oracle.m3_fwd(**sa)
    refs = oracle.m3_bwd(**sa, dout=s.dout.as_f64())
    refg = oracle.m3_discretize_bwd(**ra, dalpha=refs["dalpha"], dbeta=refs["dbeta"],
                                    dgamma=refs["dgamma"], dtheta=refs["dtheta"], dB=refs["dB"],
                                    dC=refs["dC"], A_floor=q.A_floor, eps=q.eps)
    assert_close("out", host(out), ref["out"], TOL["bf16"], FAMILY)
    for k in DISC_GRADS:
        assert_close(k, host(g[k]), refg[k], TOL["bf16"], FAMILY)


def test_disc_full_size_sampled(msc):
    """The full-size workload (B8 L2048 H24 N64 K32, bf16) through the launch
    the bench times; a sample of tokens against the oracle (tokens are
    independent in the forward, so the sample is exact)."""
    q = W.make("m3disc_bf16_b8_h24_p64_n64_k32_l2048")
    d = {k: dev(v) for k, v in _raw(q).items()}
    o = msc.msc_mamba3_siso_discretize(**d, dt_bias=dev(q.dt_bias), A_floor=q.A_floor, eps=q.eps)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    bs, ts = rng.integers(0, 8, 64), rng.integers(0, 2048, 64)
    ra = {k: v[bs, ts][:, None] for k, v in _oracle_raw(q).items() if k != "dt_bias"}
    ref = oracle.m3_discretize(**ra, dt_bias=q.dt_bias.astype(np.float64), A_floor=q.A_floor,
                               eps=q.eps)
    for k in DISC_OUT:
        got = host(o[k])[bs, ts][:, None]
        assert_close(k, got, ref[k], TOL["bf16"], FAMILY)


def test_disc_bwd_deterministic(msc):
    q = W.m3disc_problem(4, 512, 24, 16, 64, nangles=32, io="bf16", seed=3)
    d = {k: dev(v) for k, v in _raw(q).items()}
    gen = torch.Generator(device="cuda").manual_seed(0)
    sh = dict(dalpha=(4, 512, 24), dbeta=(4, 512, 24), dgamma=(4, 512, 24),
              dtheta=(4, 512, 24, 32), dB=(4, 512, 1, 64), dC=(4, 512, 1, 64))
    up = {k: torch.randn(v, device="cuda", generator=gen) for k, v in sh.items()}
    runs = [msc.msc_mamba3_siso_discretize_bwd(**d, **up, dt_bias=dev(q.dt_bias)) for _ in range(3)]
    torch.cuda.synchronize()
    for r in runs[1:]:
        for k in DISC_GRADS:
            assert torch.equal(r[k], runs[0][k]), k


def test_disc_bwd_full_size(msc):
    """The full-size workload's discretisation backward (B8 L2048 H24 N64 K32,
    bf16 inputs, f32 upstream gradients) against the oracle on the whole
    problem (ddt_bias sums all 16384 tokens)."""
    q = W.make("m3disc_bf16_b8_h24_p64_n64_k32_l2048")
    d = {k: dev(v) for k, v in _raw(q).items()}
    rng = np.random.default_rng(2)
    Bsz, L, H, K, G, N = 8, 2048, 24, 32, 1, 64
    up = dict(dalpha=rng.standard_normal((Bsz, L, H)), dbeta=rng.standard_normal((Bsz, L, H)),
              dgamma=rng.standard_normal((Bsz, L, H)),
              dtheta=rng.standard_normal((Bsz, L, H, K)),
              dB=rng.standard_normal((Bsz, L, G, N)), dC=rng.standard_normal((Bsz, L, G, N)))
    up = {k: v.astype(np.float32) for k, v in up.items()}
    g = msc.msc_mamba3_siso_discretize_bwd(**d, **{k: dev(v) for k, v in up.items()},
                                           dt_bias=dev(q.dt_bias), A_floor=q.A_floor, eps=q.eps)
    torch.cuda.synchronize()
    refg = oracle.m3_discretize_bwd(**_oracle_raw(q),
                                    **{k: v.astype(np.float64) for k, v in up.items()},
                                    A_floor=q.A_floor, eps=q.eps)
    for k in DISC_GRADS:
        assert_close(k, host(g[k]), refg[k], TOL["f32"], FAMILY)


def test_disc_empty_sequence(msc):
    """L = 0: nothing to discretise; the bias gradient is zero."""
    e3 = torch.empty(2, 0, 4, device="cuda")
    ang = torch.empty(2, 0, 8, device="cuda")
    raw = torch.empty(2, 0, 1, 16, device="cuda")
    dtb = torch.randn(4, device="cuda")
    msc.msc_mamba3_siso_discretize(e3, e3, e3, ang, raw, raw, dt_bias=dtb)
    g = msc.msc_mamba3_siso_discretize_bwd(e3, e3, e3, ang, raw, raw, e3, e3, e3,
                                           torch.empty(2, 0, 4, 8, device="cuda"), raw, raw,
                                           dt_bias=dtb)
    torch.cuda.synchronize()
    assert float(g["ddt_bias"].abs().sum()) == 0.0


# ---------------------------------------------------------------------------
# the decode step with the discretisation fused ahead
# ---------------------------------------------------------------------------
def _raw_steps(Bsz, H, N, G, K, io, n, seed):
    rng = np.random.default_rng(seed)
    st = lambda *sh, s=1.0: W.store((s * rng.standard_normal(sh)).astype(np.float32), io)
    return [dict(x=None, dd_dt=st(Bsz, H, s=0.5), dd_a=st(Bsz, H), trap=st(Bsz, H),
                 angles=st(Bsz, K), B_raw=st(Bsz, G, N), C_raw=st(Bsz, G, N), z=None)
            for _ in range(n)]


def _carried(Bsz, H, P, N, K, seed):
    rng = np.random.default_rng(seed)
    f = lambda *sh: (0.5 * rng.standard_normal(sh)).astype(np.float32)
    return [f(Bsz, H, P, N), f(Bsz, H, P), f(Bsz, H, N), f(Bsz, H, K)]


DEC_CASES = [
    # (B, H, P, N, G, K, io)
    (2, 4, 16, 16, 1, 8, "f32"),
    (3, 6, 64, 64, 2, 32, "bf16"),
    (2, 4, 32, 128, 1, 48, "bf16"),
    (2, 3, 64, 192, 3, 96, "f16"),
    (1, 2, 16, 32, 1, 0, "f32"),
]


@pytest.mark.parametrize("case", DEC_CASES, ids=[f"B{c[0]}H{c[1]}P{c[2]}N{c[3]}G{c[4]}K{c[5]}{c[6]}"
                                                 for c in DEC_CASES])
def test_fused_decode_equals_unfused(msc, case):
    """Ten chained decode steps from raw values: the fused step gives the bits
    of the discretisation kernel (one token) followed by the plain step."""
    Bsz, H, P, N, G, K, io = case
    rng = np.random.default_rng(N + H)
    steps = _raw_steps(Bsz, H, N, G, K, io, 10, N)
    xs = [W.store(rng.standard_normal((Bsz, H, P)).astype(np.float32), io) for _ in steps]
    zs = [W.store(rng.standard_normal((Bsz, H, P)).astype(np.float32), io) for _ in steps]
    dtb = dev(rng.standard_normal(H).astype(np.float32))
    Dp = dev(rng.standard_normal(H).astype(np.float32))
    c0 = _carried(Bsz, H, P, N, K, 3)
    ca = [dev(v) for v in c0]
    cb = [dev(v) for v in c0]
    for s, x, z in zip(steps, xs, zs):
        r = {k: dev(v) for k, v in s.items() if v is not None}
        if K == 0:
            r["angles"] = None
        oa = msc.msc_mamba3_siso_disc_state_update(*ca, dev(x), r["dd_dt"], r["dd_a"], r["trap"],
                                                   r["angles"], r["B_raw"], r["C_raw"],
                                                   dt_bias=dtb, A_floor=0.05, eps=1e-5, D=Dp,
                                                   z=dev(z))
        one = lambda t: None if t is None else t.unsqueeze(1).contiguous()
        d = msc.msc_mamba3_siso_discretize(one(r["dd_dt"]), one(r["dd_a"]), one(r["trap"]),
                                           one(r["angles"]) if K else None, one(r["B_raw"]),
                                           one(r["C_raw"]), dt_bias=dtb, A_floor=0.05, eps=1e-5)
        ob = msc.msc_mamba3_siso_state_update(*cb, dev(x), d["B"][:, 0].contiguous(),
                                              d["C"][:, 0].contiguous(), d["alpha"][:, 0].contiguous(),
                                              d["beta"][:, 0].contiguous(), d["gamma"][:, 0].contiguous(),
                                              d["theta"][:, 0].contiguous(), D=Dp, z=dev(z))
        torch.cuda.synchronize()
        assert torch.equal(oa, ob)
    for u, v in zip(ca, cb):
        assert torch.equal(u, v)


def test_fused_decode_vs_oracle(msc):
    """Chained fused decode steps against the oracle's discretisation (each
    value rounded to the io type, as stored) followed by its decode step."""
    Bsz, H, P, N, G, K, io = 2, 4, 64, 64, 1, 32, "bf16"
    rng = np.random.default_rng(9)
    steps = _raw_steps(Bsz, H, N, G, K, io, 8, 1)
    dtb = rng.standard_normal(H).astype(np.float32)
    Dp = rng.standard_normal(H).astype(np.float32)
    c0 = _carried(Bsz, H, P, N, K, 5)
    cg = [dev(v) for v in c0]
    cr = [v.astype(np.float64) for v in c0]
    for s in steps:
        x = W.store(rng.standard_normal((Bsz, H, P)).astype(np.float32), io)
        z = W.store(rng.standard_normal((Bsz, H, P)).astype(np.float32), io)
        o = msc.msc_mamba3_siso_disc_state_update(
            *cg, dev(x), dev(s["dd_dt"]), dev(s["dd_a"]), dev(s["trap"]), dev(s["angles"]),
            dev(s["B_raw"]), dev(s["C_raw"]), dt_bias=dev(dtb), A_floor=1e-4, eps=1e-5,
            D=dev(Dp), z=dev(z))
        one = lambda t: t.as_f64()[:, None]
        d = oracle.m3_discretize(one(s["dd_dt"]), one(s["dd_a"]), one(s["trap"]),
                                 one(s["angles"]), one(s["B_raw"]), one(s["C_raw"]),
                                 dt_bias=dtb.astype(np.float64), A_floor=1e-4, eps=1e-5)
        d = {k: W.store(v[:, 0].astype(np.float32), io).as_f64() for k, v in d.items()}
        *cr, o_ref = oracle.m3_state_update(*cr, x.as_f64(), d["B"], d["C"], d["alpha"],
                                            d["beta"], d["gamma"], d["theta"],
                                            D=Dp.astype(np.float64), z=z.as_f64())
        torch.cuda.synchronize()
        assert_close("out", host(o), o_ref, TOL["bf16"], FAMILY)
    assert_close("state", host(cg[0]), cr[0], TOL["bf16"], FAMILY)


# --------------------------------------------------------------------------
# The scan from raw projections (the per-head discretisation fused into the
# forward kernel, BCNorm once per row ahead of it; the backward re-deriving
# both): bit for bit the two-call chain, and so the oracle's chain
# --------------------------------------------------------------------------
SCAN_OUT = ("dx", "dz", "dD", "dh0")


def _chain_and_fused(msc, q, bias=True, h0=True, z=True, D=True):
    """Run discretise -> scan forward -> scan backward -> discretise backward and
    the two fused entry points on the same inputs."""
    s = q.scan
    d = {k: dev(v) for k, v in _raw(q).items()}
    if s.nangles == 0:
        d["angles"] = None
    dtb = dev(q.dt_bias) if bias else None
    kw = dict(dt_bias=dtb, A_floor=q.A_floor, eps=q.eps)
    com = dict(x=dev(s.x), D=dev(s.D) if D else None, z=dev(s.z) if z else None,
               h0=dev(s.h0) if h0 else None)
    dout = dev(s.dout)
    o = msc.msc_mamba3_siso_discretize(**d, **kw)
    der = dict(B=o["B"], C=o["C"], alpha=o["alpha"], beta=o["beta"], gamma=o["gamma"],
               theta=o["theta"])
    out, fs, saved = msc.msc_mamba3_siso_scan_fwd(**com, **der)
    gs = msc.msc_mamba3_siso_scan_bwd(**com, **der, saved_states=saved, dout=dout)
    g = msc.msc_mamba3_siso_discretize_bwd(**d, dalpha=gs["dalpha"], dbeta=gs["dbeta"],
                                           dgamma=gs["dgamma"], dtheta=gs["dtheta"],
                                           dB=gs["dB"], dC=gs["dC"], **kw)
    chain = dict(out=out, final_state=fs, saved=saved, **{k: gs[k] for k in SCAN_OUT}, **g)
    out_r, fs_r, saved_r = msc.msc_mamba3_siso_scan_fwd_raw(**com, **d, **kw)
    gr = msc.msc_mamba3_siso_scan_bwd_raw(**com, **d, **kw, saved_states=saved_r, dout=dout)
    fused = dict(out=out_r, final_state=fs_r, saved=saved_r, **gr)
    torch.cuda.synchronize()
    return chain, fused


def _assert_bit_equal(chain, fused, keys):
    for k in keys:
        a, b = chain[k], fused[k]
        if a is None or b is None:  # absent (no angles, no h0): absent or empty on both sides
            assert all(v is None or v.numel() == 0 for v in (a, b)), k
            continue
        assert torch.equal(a, b), (k, (a.float() - b.float()).abs().max().item())


FUSED_CASES = [
    # (B, L, H, P, N, G, K, bias, h0, z, D)
    (2, 130, 4, 64, 64, 1, 32, True, True, True, True),   # ragged last chunk
    (1, 200, 6, 32, 32, 2, 16, False, False, True, False),
    (2, 64, 4, 16, 16, 1, 0, True, True, False, True),    # no angles, one chunk
    (1, 1, 2, 64, 64, 1, 8, True, False, True, True),     # one step
    (1, 257, 8, 64, 16, 4, 8, True, True, True, True),    # four groups
]


@pytest.mark.parametrize("case", FUSED_CASES,
                         ids=[f"B{c[0]}L{c[1]}H{c[2]}P{c[3]}N{c[4]}G{c[5]}K{c[6]}"
                              for c in FUSED_CASES])
def test_fused_raw_equals_the_chain(msc, case):
    Bsz, L, H, P, N, G, K, bias, h0, z, D = case
    q = W.m3disc_problem(Bsz, L, H, P, N, ngroups=G, nangles=K, io="bf16", seed=L + 3 * H,
                         with_h0=h0)
    chain, fused = _chain_and_fused(msc, q, bias=bias, h0=h0, z=z, D=D)
    _assert_bit_equal(chain, fused, ("out", "final_state", "saved") + SCAN_OUT + DISC_GRADS)


def test_fused_raw_against_the_oracle(msc):
    """The fused entry points against the oracle's chain directly (the scan taking
    the discretised values as bf16 stores them)."""
    q = W.m3disc_problem(2, 130, 4, 64, 64, nangles=32, io="bf16", seed=11, with_h0=True)
    _, fused = _chain_and_fused(msc, q)
    s = q.scan
    ra = _oracle_raw(q)
    disc = oracle.m3_discretize(**ra, A_floor=q.A_floor, eps=q.eps)
    stored = {k: W.store(v.astype(np.float32), "bf16").as_f64() for k, v in disc.items()}
    sa = dict(x=s.x.as_f64(), B=stored["B"], C=stored["C"], alpha=stored["alpha"],
              beta=stored["beta"], gamma=stored["gamma"], theta=stored["theta"],
              D=np.asarray(s.D, np.float64), z=s.z.as_f64(), h0=np.asarray(s.h0, np.float64))
    ref = oracle.m3_fwd(**sa)
    refs = oracle.m3_bwd(**sa, dout=s.dout.as_f64())
    refg = oracle.m3_discretize_bwd(**ra, dalpha=refs["dalpha"], dbeta=refs["dbeta"],
                                    dgamma=refs["dgamma"], dtheta=refs["dtheta"], dB=refs["dB"],
                                    dC=refs["dC"], A_floor=q.A_floor, eps=q.eps)
    assert_close("out", host(fused["out"]), ref["out"], TOL["bf16"], FAMILY)
    assert_close("final_state", host(fused["final_state"]), ref["final_state"], TOL["bf16"],
                 FAMILY)
    for k in ("dx", "dz"):
        assert_close(k, host(fused[k]), refs[k], TOL["bf16"], FAMILY)
    for k in ("dD", "dh0"):
        assert_close(k, host(fused[k]), refs[k], TOL["bf16"], FAMILY)
    for k in DISC_GRADS:
        assert_close(k, host(fused[k]), refg[k], TOL["bf16"], FAMILY)


def test_fused_raw_full_size_equals_the_chain(msc):
    """At the full training shape (B8 L2048 H24 P64 N64 K32, bf16), the launch the
    bench times: every output bit for bit the two-call chain's, whose own parity
    the scan's full-size tests establish."""
    q = W.make("m3disc_bf16_b8_h24_p64_n64_k32_l2048")
    chain, fused = _chain_and_fused(msc, q, h0=False)
    _assert_bit_equal(chain, fused, ("out", "final_state", "saved") + SCAN_OUT + DISC_GRADS)


def test_fused_raw_empty_sequence(msc):
    """L = 0 from raw projections: the final state is h0; dD, dh0 and the dt
    bias gradient are zero; nothing else is touched."""
    Bsz, H, P, N, K = 2, 3, 64, 64, 16
    bf = dict(device="cuda", dtype=torch.bfloat16)
    x = torch.empty(Bsz, 0, H, P, **bf)
    raw = dict(dd_dt=torch.empty(Bsz, 0, H, **bf), dd_a=torch.empty(Bsz, 0, H, **bf),
               trap=torch.empty(Bsz, 0, H, **bf), angles=torch.empty(Bsz, 0, K, **bf),
               B_raw=torch.empty(Bsz, 0, 1, N, **bf), C_raw=torch.empty(Bsz, 0, 1, N, **bf))
    h0 = torch.randn(Bsz, H, P, N, device="cuda")
    dtb = torch.randn(H, device="cuda")
    out, fs, saved = msc.msc_mamba3_siso_scan_fwd_raw(x, **raw, dt_bias=dtb, h0=h0)
    g = msc.msc_mamba3_siso_scan_bwd_raw(x, **raw, dt_bias=dtb, h0=h0, saved_states=saved,
                                         dout=torch.empty_like(x),
                                         D=torch.randn(H, device="cuda"))
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(fs, h0)
    assert torch.count_nonzero(g["dD"]) == 0 and torch.count_nonzero(g["dh0"]) == 0
    assert torch.count_nonzero(g["ddt_bias"]) == 0
