"""GPU parity of the Mamba-1 selective scan (forward, backward) and the decode
step against the f64 oracle, through the C ABI (libmsc.so via its binding)."""
import numpy as np
import pytest

import oracle
from selective_state_space_14_b200 import workloads as W
from tests._util import TOL, assert_close, dev, host, m1_device_args

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# f32 elementwise guards of the Mamba-1 recurrences (tests/_util.py)
FAMILY = "m1"

M1_GRADS = ("du", "ddelta", "dA", "dB", "dC", "dD", "ddelta_bias", "dz", "dh0")


@pytest.fixture(scope="module")
def msc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_14_b200 import msc as m
    m.lib()
    return m


def _run_gpu(msc, p, backward=True):
    a = m1_device_args(p)
    out, fs, saved = msc.msc_selective_scan_fwd(**a)
    res = dict(out=host(out), final_state=host(fs))
    if backward:
        g = msc.msc_selective_scan_bwd(saved_states=saved, dout=dev(p.dout), **a)
        for k in M1_GRADS:
            if g.get(k) is not None:
                res[k] = host(g[k])
    torch.cuda.synchronize()
    return res


def _run_oracle(p, backward=True):
    args = oracle.m1_problem_args(p)
    r = oracle.m1_fwd(**args)
    res = dict(out=r["out"], final_state=r["final_state"])
    if backward:
        res.update(oracle.m1_bwd(dout=p.dout.as_f64(), **args))
    return res


def _compare(gpu, ref, tol, skip=()):
    errs = {}
    for k, v in gpu.items():
        if k in skip or k not in ref:
            continue
        errs[k] = assert_close(k, v, ref[k], tol, FAMILY)
    return errs


def test_small_f32_workload(msc):
    """The small Mamba-1 workload: f32, batch 1, d_inner 64, d_state 16, L 256."""
    p = W.make("m1_f32_b1_d64_n16_l256")
    _compare(_run_gpu(msc, p), _run_oracle(p), TOL["f32"])


CASES = [
    # (B, D, N, L, G, io, bias, z, D, h0, softplus)
    (1, 3, 1, 1, 1, "f32", False, True, True, False, True),
    (2, 5, 3, 7, 1, "f32", True, True, True, True, True),
    (1, 4, 16, 255, 1, "f32", True, False, False, True, True),
    (1, 4, 16, 257, 1, "f32", True, True, True, True, False),
    (2, 65, 16, 600, 1, "f32", True, True, True, True, True),
    (1, 8, 64, 300, 1, "f32", True, True, True, True, True),
    (1, 7, 5, 513, 1, "f32", False, True, True, False, True),
    (2, 256, 8, 130, 2, "f32", True, True, True, True, True),
    (2, 96, 16, 700, 1, "bf16", True, True, True, True, True),
    (1, 40, 16, 9, 1, "bf16", True, True, True, False, True),
    # 16-byte-aligned rows (cp.async staging) with a ragged last block, groups
    # that do not fill whole CTAs or clusters, d_state 32 and 64
    (2, 100, 32, 1000, 2, "bf16", True, True, True, True, True),
    (1, 24, 64, 96, 1, "bf16", True, True, True, True, True),
    (3, 36, 16, 1024, 3, "bf16", True, False, True, True, True),
    (1, 20, 16, 40, 1, "f32", True, True, True, True, True),
    # f16 storage: aligned rows with a ragged block, d_state 64, unaligned rows
    (2, 96, 16, 700, 1, "f16", True, True, True, True, True),
    (1, 24, 64, 96, 1, "f16", True, True, True, True, True),
    (1, 7, 5, 513, 1, "f16", False, True, True, False, True),
    (2, 100, 32, 1000, 2, "f16", True, True, True, True, True),
    # d_state above 64: slabs of 64 states (first + last, first + middles + last,
    # a narrow last slab)
    (1, 8, 128, 300, 1, "f32", True, True, True, True, True),
    (2, 12, 100, 257, 1, "f32", False, True, True, True, True),
    (1, 16, 256, 130, 2, "bf16", True, True, True, True, True),
    (2, 40, 96, 1000, 1, "bf16", True, False, True, True, True),
    (1, 8, 200, 64, 1, "f16", True, True, True, True, True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}D{c[1]}N{c[2]}L{c[3]}G{c[4]}{c[5]}" for c in CASES])
def test_parity_shapes(msc, case):
    Bsz, D, N, L, G, io, bias, z, Dp, h0, sp = case
    p = W.m1_problem(Bsz, D, N, L, io=io, seed=1000 + L + D, ngroups=G, bias=bias, with_z=z,
                     with_D=Dp, with_h0=h0, delta_softplus=sp)
    if not sp:  # softplus off: keep delta positive (no bias) so the state stays bounded
        p.delta = W.store(np.abs(p.delta.as_f32()) * 0.2, io)
        p.delta_bias = None
    _compare(_run_gpu(msc, p), _run_oracle(p), TOL[io])


SEG_CASES = [
    # (B, D, N, L, io): grids of few (batch, channel) blocks, so the forward
    # runs in time segments combined by the warp-shuffle scan
    (1, 64, 16, 256, "f32"),
    (1, 16, 16, 1024, "f32"),
    # 4096 steps in bf16: over that many steps a step-by-step f32 evaluation
    # with correctly rounded exp already leaves the final state 1.75e-5 from
    # the oracle (normwise), above the f32 bound
    (1, 16, 16, 4096, "bf16"),
    (2, 40, 32, 2000, "bf16"),
    (1, 8, 64, 777, "f32"),
    (1, 512, 16, 2048, "bf16"),
]


SEG_VARIANT_CASES = [
    # (B, D, N, L, io, G, z, bias, softplus, h0): the branches of the segment
    # summaries -- groups of B/C, no gate, no bias, raw delta, f16 storage
    (1, 96, 16, 1024, "bf16", 2, True, True, True, False),
    (1, 48, 16, 700, "f32", 1, False, False, True, True),
    (1, 32, 32, 900, "f32", 1, True, False, False, True),
    (2, 24, 16, 1500, "f16", 3, True, True, True, True),
]


@pytest.mark.parametrize("case", SEG_VARIANT_CASES,
                         ids=[f"B{c[0]}D{c[1]}N{c[2]}L{c[3]}{c[4]}G{c[5]}z{int(c[6])}b{int(c[7])}"
                              f"sp{int(c[8])}" for c in SEG_VARIANT_CASES])
def test_time_segments_variants(msc, case):
    """Both scans in time segments with groups, without the gate or the bias,
    with softplus off, and in f16, against the oracle."""
    Bsz, D, N, L, io, G, z, bias, sp, h0 = case
    assert msc.msc_selective_scan_fwd_workspace_bytes(Bsz, D, N, L) > 0
    p = W.m1_problem(Bsz, D, N, L, io=io, seed=3100 + L, ngroups=G, bias=bias, with_z=z,
                     with_h0=h0, delta_softplus=sp)
    if not sp:  # softplus off: keep delta positive (no bias) so the state stays bounded
        p.delta = W.store(np.abs(p.delta.as_f32()) * 0.2, io)
        p.delta_bias = None
    _compare(_run_gpu(msc, p), _run_oracle(p), TOL[io])


@pytest.mark.parametrize("case", SEG_CASES, ids=[f"B{c[0]}D{c[1]}N{c[2]}L{c[3]}{c[4]}" for c in SEG_CASES])
def test_time_segments_parity(msc, case):
    """Forward and backward in time segments against the oracle: the grids of
    (batch, channel) blocks are small enough that both split time (the
    forward's workspace query is > 0; the backward's includes the segments'
    summaries), the summaries composed by the warp-shuffle scan."""
    Bsz, D, N, L, io = case
    assert msc.msc_selective_scan_fwd_workspace_bytes(Bsz, D, N, L) > 0
    p = W.m1_problem(Bsz, D, N, L, io=io, seed=3000 + L, bias=True, with_h0=True)
    _compare(_run_gpu(msc, p), _run_oracle(p), TOL[io])


def test_determinism(msc):
    """Same inputs, same bits: five runs of forward and backward."""
    p = W.m1_problem(2, 130, 16, 700, io="bf16", seed=5, bias=True, with_h0=True)
    runs = [_run_gpu(msc, p) for _ in range(5)]
    for r in runs[1:]:
        for k in runs[0]:
            np.testing.assert_array_equal(r[k], runs[0][k], err_msg=k)


def test_resume_is_bit_continuous(msc):
    """A scan over L equals a scan over L1 followed by one over L - L1 started
    from the first one's final state; bit-equal when L1 is a multiple of the
    forward's 32-step chunk (and so of the 8-step saved-state interval).  The
    sizes fill the GPU with (batch, channel) blocks, so the forward walks time
    in one pass (no time segments, whose composition rounds differently)."""
    assert msc.msc_selective_scan_fwd_workspace_bytes(2, 1184, 16, 1536) == 0
    p = W.m1_problem(2, 1184, 16, 1536, io="f32", seed=9, bias=True)
    a = m1_device_args(p)
    full, fs_full, _ = msc.msc_selective_scan_fwd(**a)
    L1 = 1024  # a multiple of the 32-step chunk
    part = {k: (v[..., :L1].contiguous() if k in ("u", "delta", "z") else v) for k, v in a.items()}
    part["B"], part["C"] = a["B"][..., :L1].contiguous(), a["C"][..., :L1].contiguous()
    o1, fs1, _ = msc.msc_selective_scan_fwd(**part)
    rest = {k: (v[..., L1:].contiguous() if k in ("u", "delta", "z") else v) for k, v in a.items()}
    rest["B"], rest["C"] = a["B"][..., L1:].contiguous(), a["C"][..., L1:].contiguous()
    rest["h0"] = fs1
    o2, fs2, _ = msc.msc_selective_scan_fwd(**rest)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([o1, o2], -1), full)
    assert torch.equal(fs2, fs_full)


def test_empty_inputs(msc):
    """L = 0: no steps, the final state is h0; the backward gives zero gradients."""
    h0 = torch.randn(2, 3, 4, device="cuda")
    A = -torch.rand(3, 4, device="cuda")
    e = torch.empty(2, 3, 0, device="cuda")
    Be = torch.empty(2, 1, 4, 0, device="cuda")
    out, fs, saved = msc.msc_selective_scan_fwd(e, e, A, Be, Be, h0=h0)
    torch.cuda.synchronize()
    assert torch.equal(fs, h0)
    g = msc.msc_selective_scan_bwd(e, e, A, Be, Be, saved, e, h0=h0)
    torch.cuda.synchronize()
    assert float(g["dA"].abs().sum()) == 0.0 and float(g["dh0"].abs().sum()) == 0.0


def test_model_shaped_full_size(msc):
    """The Mamba-130M-layer-shaped workload (bf16, B8 D1536 N16 L2048) at full
    size, in the launch configuration the benchmark times; every output
    compared with the f64 oracle on the whole problem."""
    p = W.make("m1_bf16_b8_d1536_n16_l2048")
    _compare(_run_gpu(msc, p), _run_oracle(p), TOL["bf16"])


def test_2p8b_shaped_full_size_sampled(msc):
    """The Mamba-2.8B-layer-shaped workload (bf16, B4 D5120 N16 L4096) at full
    size on the GPU; the oracle recomputes batch row 0 (all 5120 channels, so
    dB/dC are exact sums) and the outputs of that row are compared."""
    p = W.make("m1_bf16_b4_d5120_n16_l4096")
    g = _run_gpu(msc, p)
    p0 = W.M1Problem(1, p.dim, p.dstate, p.seqlen, p.ngroups, p.io, p.delta_softplus,
                     W.Tensor(p.io, p.u.data[:1]), W.Tensor(p.io, p.delta.data[:1]), p.A,
                     W.Tensor(p.io, p.B.data[:1]), W.Tensor(p.io, p.C.data[:1]), p.D,
                     p.delta_bias, W.Tensor(p.io, p.z.data[:1]), None,
                     W.Tensor(p.io, p.dout.data[:1]))
    ref = _run_oracle(p0)
    for k in ("out", "final_state", "du", "ddelta", "dz", "dh0", "dB", "dC"):
        assert_close(k, g[k][:1], ref[k], TOL["bf16"], FAMILY)


# ---------------------------------------------------------------------------
# decode step
# ---------------------------------------------------------------------------
def test_state_update_equals_scan_step_bitwise(msc):
    """The decode step and a forward scan of length 1 give identical bits."""
    p = W.m1_problem(4, 96, 16, 1, io="bf16", seed=77, bias=True, with_h0=True)
    a = m1_device_args(p)
    out, fs, _ = msc.msc_selective_scan_fwd(**a)
    st = a["h0"].clone()
    o = msc.msc_ssm_state_update(st, a["u"][..., 0].contiguous(), a["delta"][..., 0].contiguous(),
                                 a["A"], a["B"][..., 0].contiguous(), a["C"][..., 0].contiguous(),
                                 D=a["D"], delta_bias=a["delta_bias"],
                                 z=a["z"][..., 0].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(o, out[..., 0])
    assert torch.equal(st, fs)


@pytest.mark.parametrize("io", ["f32", "bf16", "f16"])
def test_state_update_chain(msc, io):
    """60 chained decode steps against the oracle's chained steps."""
    q = W.su_problem(3, 70, 16, io=io, seed=3, random_state=True, n_pool=60)
    st = torch.from_numpy(q.state0).cuda()
    st_ref = q.state0.astype(np.float64)
    A, Dp, bias = dev(q.A), dev(q.D), dev(q.delta_bias)
    for s in q.steps:
        o = msc.msc_ssm_state_update(st, dev(s["x"]), dev(s["delta"]), A, dev(s["B"]),
                                     dev(s["C"]), D=Dp, delta_bias=bias, z=dev(s["z"]))
        st_ref, o_ref = oracle.ssm_state_update(st_ref, s["x"].as_f64(), s["delta"].as_f64(),
                                                q.A.astype(np.float64), s["B"].as_f64(),
                                                s["C"].as_f64(), D=q.D.astype(np.float64),
                                                delta_bias=q.delta_bias.astype(np.float64),
                                                z=s["z"].as_f64())
        assert_close("out", host(o), o_ref, TOL[io], FAMILY)
    assert_close("state", host(st), st_ref, TOL[io], FAMILY)


def test_state_update_wide_state(msc):
    """The decode step with 200 states (the step has no d_state limit below 256)."""
    q = W.su_problem(2, 24, 200, io="bf16", seed=8, random_state=True, n_pool=6)
    st = torch.from_numpy(q.state0).cuda()
    st_ref = q.state0.astype(np.float64)
    A, Dp, bias = dev(q.A), dev(q.D), dev(q.delta_bias)
    for s in q.steps:
        o = msc.msc_ssm_state_update(st, dev(s["x"]), dev(s["delta"]), A, dev(s["B"]),
                                     dev(s["C"]), D=Dp, delta_bias=bias, z=dev(s["z"]))
        st_ref, o_ref = oracle.ssm_state_update(st_ref, s["x"].as_f64(), s["delta"].as_f64(),
                                                q.A.astype(np.float64), s["B"].as_f64(),
                                                s["C"].as_f64(), D=q.D.astype(np.float64),
                                                delta_bias=q.delta_bias.astype(np.float64),
                                                z=s["z"].as_f64())
        assert_close("out", host(o), o_ref, TOL["bf16"], FAMILY)
    assert_close("state", host(st), st_ref, TOL["bf16"], FAMILY)


def test_state_update_decode_workload_sampled(msc):
    """The decode workload (B256 D5120 N16, f32 state, bf16 inputs, 1000 steps
    cycling a pool of 8 input sets) on the GPU; the oracle follows 64 fixed
    (b, c) rows through all 1000 steps (rows are independent, so this is exact
    for them)."""
    q = W.make("su_bf16_b256_d5120_n16_x1000")
    st = torch.from_numpy(q.state0).cuda()
    A, Dp, bias = dev(q.A), dev(q.D), dev(q.delta_bias)
    steps = [{k: dev(v) for k, v in s.items()} for s in q.steps]
    rng = np.random.default_rng(0)
    rows_b = rng.integers(0, q.batch, 64)
    rows_c = rng.integers(0, q.dim, 64)
    st_ref = np.zeros((64, 1, q.dstate))
    A64 = q.A[rows_c].astype(np.float64)
    outs = []
    for t in range(1000):
        s = steps[t % 8]
        o = msc.msc_ssm_state_update(st, s["x"], s["delta"], A, s["B"], s["C"], D=Dp,
                                     delta_bias=bias, z=s["z"])
        if t % 100 == 99 or t == 999:
            outs.append((t, host(o)[rows_b, rows_c]))
    final = host(st)[rows_b, rows_c]
    # oracle: each sampled row as its own (batch=1, dim=1) problem; the pool's
    # sampled rows are widened to f64 once
    pool = [dict(x=s["x"].as_f64()[rows_b, rows_c], delta=s["delta"].as_f64()[rows_b, rows_c],
                 z=s["z"].as_f64()[rows_b, rows_c], B=s["B"].as_f64()[rows_b],
                 C=s["C"].as_f64()[rows_b]) for s in q.steps]
    D64 = q.D.astype(np.float64)[rows_c]
    bias64 = q.delta_bias.astype(np.float64)[rows_c]
    for t in range(1000):
        s = pool[t % 8]
        ref_out = np.zeros(64)
        for r in range(64):
            ns, o = oracle.ssm_state_update(
                st_ref[r:r + 1], s["x"][r:r + 1, None], s["delta"][r:r + 1, None], A64[r:r + 1],
                s["B"][r:r + 1], s["C"][r:r + 1], D=D64[r:r + 1], delta_bias=bias64[r:r + 1],
                z=s["z"][r:r + 1, None])
            st_ref[r:r + 1] = ns
            ref_out[r] = o[0, 0]
        for (tt, got) in outs:
            if tt == t:
                assert_close(f"out@{t}", got, ref_out, TOL["bf16"], FAMILY)
    assert_close("state", final, st_ref[:, 0, :], TOL["bf16"], FAMILY)
