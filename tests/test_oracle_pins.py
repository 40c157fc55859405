"""Pins of the f64 oracle against facts that do not come from the oracle itself.

Each test fixes part of the oracle with a closed form, a brute-force evaluation
written independently here with numpy, an invariant of the recurrence, or
central finite differences.  A plausible slip in the oracle (a dropped term, a
sign, an off-by-one in the time index, a transposed operand) fails at least
one of them.  CPU only.
"""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(7)


def _rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def _silu(v):
    return v / (1.0 + np.exp(-v))


# ---------------------------------------------------------------------------
# Mamba-1 forward
# ---------------------------------------------------------------------------
def test_m1_geometric_series():
    """N=1, constant delta, A, B, x; C=1, D=0, no gate, h0=0:
    h_t = delta B x (1 - a^{t+1}) / (1 - a),  a = exp(delta A)."""
    L, dt, A, Bv, x = 50, 0.3, -0.7, 1.3, -0.8
    u = np.full((1, 1, L), x)
    delta = np.full((1, 1, L), dt)
    r = oracle.m1_fwd(u, delta, np.array([[A]]), np.full((1, 1, 1, L), Bv),
                      np.ones((1, 1, 1, L)), delta_softplus=False)
    a = np.exp(dt * A)
    t = np.arange(L)
    expect = dt * Bv * x * (1 - a ** (t + 1)) / (1 - a)
    np.testing.assert_allclose(r["out"][0, 0], expect, rtol=1e-13, atol=0)
    np.testing.assert_allclose(r["final_state"][0, 0, 0], expect[-1], rtol=1e-13)


def test_m1_softplus_values():
    """softplus(v) = log(1 + e^v); with N=1, A=0 (a=1), B=C=x=1, L=1: y = softplus(v)."""
    v = np.array([-30.0, -5.0, -1e-3, 0.0, 0.7, 5.0, 30.0])
    L = 1
    for vv in v:
        r = oracle.m1_fwd(np.ones((1, 1, L)), np.full((1, 1, L), vv), np.zeros((1, 1)),
                          np.ones((1, 1, 1, L)), np.ones((1, 1, 1, L)), delta_softplus=True)
        assert r["out"][0, 0, 0] == pytest.approx(np.log1p(np.exp(vv)) if vv < 30 else vv + np.log1p(np.exp(-vv)), rel=1e-14)


def test_m1_delta_zero_keeps_state():
    """delta = 0 (softplus off, no bias): h stays h0, so out = (C.h0 + D x) silu(z)."""
    Bsz, D, N, L = 2, 3, 4, 9
    h0 = _rand(Bsz, D, N)
    u, z = _rand(Bsz, D, L), _rand(Bsz, D, L)
    Bm, Cm = _rand(Bsz, 1, N, L), _rand(Bsz, 1, N, L)
    Dp, A = _rand(D), -np.abs(_rand(D, N))
    r = oracle.m1_fwd(u, np.zeros((Bsz, D, L)), A, Bm, Cm, D=Dp, z=z, h0=h0,
                      delta_softplus=False)
    y = np.einsum("bnl,bdn->bdl", Cm[:, 0], h0) + Dp[None, :, None] * u
    np.testing.assert_allclose(r["out"], y * _silu(z), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(r["final_state"], h0, rtol=0, atol=0)
    # and with h0 = 0 it is D x silu(z)
    r0 = oracle.m1_fwd(u, np.zeros((Bsz, D, L)), A, Bm, Cm, D=Dp, z=z, delta_softplus=False)
    np.testing.assert_allclose(r0["out"], Dp[None, :, None] * u * _silu(z), rtol=1e-14)


def test_m1_tree_order_equals_sequential():
    """The Hillis-Steele evaluation with (a,b)o(a',b') = (aa', a'b + b') equals the loop."""
    Bsz, D, N, L, G = 2, 5, 6, 77, 1
    args = dict(u=_rand(Bsz, D, L), delta=0.5 * _rand(Bsz, D, L) - 2, A=-np.abs(_rand(D, N)),
                B=_rand(Bsz, G, N, L), C=_rand(Bsz, G, N, L), D=_rand(D),
                delta_bias=_rand(D, scale=0.1), z=_rand(Bsz, D, L), h0=_rand(Bsz, D, N))
    s = oracle.m1_fwd(**args)
    t = oracle.m1_fwd(**args, tree=True)
    np.testing.assert_allclose(t["out"], s["out"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(t["final_state"], s["final_state"], rtol=1e-12, atol=1e-12)


def _m1_bruteforce(u, delta_raw, A, Bm, Cm, Dp, bias, z, h0, G):
    """y_t = sum_n C_t (prod_{r=0..t} a_r) h0 + sum_{s<=t} sum_n C_t (prod_{r=s+1..t} a_r)
    delta_s B_s x_s + D x_t, evaluated from materialised decay products (O(L^2))."""
    Bsz, D, L = u.shape
    N = A.shape[1]
    out = np.zeros_like(u)
    for b in range(Bsz):
        for c in range(D):
            g = c // (D // G)
            dt = np.log1p(np.exp(delta_raw[b, c] + bias[c]))
            a = np.exp(dt[:, None] * A[c][None, :])  # [L, N]
            for t in range(L):
                y = 0.0
                for n in range(N):
                    y += Cm[b, g, n, t] * np.prod(a[: t + 1, n]) * h0[b, c, n]
                    for s in range(t + 1):
                        y += Cm[b, g, n, t] * np.prod(a[s + 1: t + 1, n]) * dt[s] * Bm[b, g, n, s] * u[b, c, s]
                y += Dp[c] * u[b, c, t]
                out[b, c, t] = y * _silu(z[b, c, t])
    return out


def test_m1_bruteforce_convolution_form():
    Bsz, D, N, L, G = 2, 4, 3, 11, 2
    u, d = _rand(Bsz, D, L), 0.5 * _rand(Bsz, D, L) - 1
    A, Bm, Cm = -np.abs(_rand(D, N)), _rand(Bsz, G, N, L), _rand(Bsz, G, N, L)
    Dp, bias, z, h0 = _rand(D), _rand(D, scale=0.3), _rand(Bsz, D, L), _rand(Bsz, D, N)
    r = oracle.m1_fwd(u, d, A, Bm, Cm, D=Dp, delta_bias=bias, z=z, h0=h0)
    np.testing.assert_allclose(r["out"], _m1_bruteforce(u, d, A, Bm, Cm, Dp, bias, z, h0, G),
                               rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# State update
# ---------------------------------------------------------------------------
def test_state_update_equals_one_scan_step():
    Bsz, D, N, G = 3, 6, 5, 1
    st = _rand(Bsz, D, N)
    x, d, z = _rand(Bsz, D), _rand(Bsz, D) * 0.5 - 2, _rand(Bsz, D)
    Bm, Cm, A, Dp, bias = _rand(Bsz, G, N), _rand(Bsz, G, N), -np.abs(_rand(D, N)), _rand(D), _rand(D)
    new, out = oracle.ssm_state_update(st, x, d, A, Bm, Cm, D=Dp, delta_bias=bias, z=z)
    r = oracle.m1_fwd(x[..., None], d[..., None], A, Bm[..., None], Cm[..., None], D=Dp,
                      delta_bias=bias, z=z[..., None], h0=st)
    np.testing.assert_array_equal(out, r["out"][..., 0])
    np.testing.assert_array_equal(new, r["final_state"])


def test_state_update_chain_equals_scan():
    """T chained single-token updates equal one scan over T steps."""
    Bsz, D, N, T = 2, 3, 4, 1000
    u, d, z = _rand(Bsz, D, T), 0.5 * _rand(Bsz, D, T) - 2, _rand(Bsz, D, T)
    Bm, Cm, A, Dp = _rand(Bsz, 1, N, T), _rand(Bsz, 1, N, T), -np.abs(_rand(D, N)), _rand(D)
    r = oracle.m1_fwd(u, d, A, Bm, Cm, D=Dp, z=z)
    st = np.zeros((Bsz, D, N))
    outs = []
    for t in range(T):
        st, o = oracle.ssm_state_update(st, u[..., t], d[..., t], A, Bm[..., t], Cm[..., t],
                                        D=Dp, z=z[..., t])
        outs.append(o)
    np.testing.assert_allclose(np.stack(outs, -1), r["out"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st, r["final_state"], rtol=1e-12, atol=1e-12)


def test_state_update_geometric():
    """Chained updates with constant inputs and N=1 follow the geometric series."""
    dt, A, Bv, x = 0.2, -1.5, 0.9, 1.7
    st = np.zeros((1, 1, 1))
    a = np.exp(dt * A)
    for t in range(30):
        st, o = oracle.ssm_state_update(st, np.array([[x]]), np.array([[dt]]), np.array([[A]]),
                                        np.array([[[Bv]]]), np.array([[[1.0]]]),
                                        delta_softplus=False)
        assert o[0, 0] == pytest.approx(dt * Bv * x * (1 - a ** (t + 1)) / (1 - a), rel=1e-13)


# ---------------------------------------------------------------------------
# Mamba-1 backward: finite differences, adjoint identity, closed forms
# ---------------------------------------------------------------------------
def _m1_tiny(G=1):
    Bsz, D, N, L = 1, 2, 3, 7
    return dict(u=_rand(Bsz, D, L), delta=0.5 * _rand(Bsz, D, L) - 1, A=-np.abs(_rand(D, N)),
                B=_rand(Bsz, G, N, L), C=_rand(Bsz, G, N, L), D=_rand(D),
                delta_bias=_rand(D, scale=0.3), z=_rand(Bsz, D, L), h0=_rand(Bsz, D, N))


def _close(got, fd, key):
    """Central differences carry roundoff of order eps_machine * |loss| / step, so the
    absolute floor scales with the largest gradient entry."""
    np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-6 * max(1.0, np.abs(fd).max()),
                               err_msg=key)


def _fd(loss, args, key, eps=1e-6):
    base = args[key]
    g = np.zeros_like(base)
    it = np.nditer(base, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        p = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in args.items()}
        p[key][i] = base[i] + eps
        lp = loss(p)
        p[key][i] = base[i] - eps
        lm = loss(p)
        g[i] = (lp - lm) / (2 * eps)
    return g


M1_GRAD_OF = dict(u="du", delta="ddelta", A="dA", B="dB", C="dC", D="dD",
                  delta_bias="ddelta_bias", z="dz", h0="dh0")


@pytest.mark.parametrize("softplus", [True, False])
def test_m1_backward_finite_differences(softplus):
    args = _m1_tiny()
    dout = _rand(*args["u"].shape)
    loss = lambda p: float(np.sum(dout * oracle.m1_fwd(**p, delta_softplus=softplus)["out"]))
    g = oracle.m1_bwd(dout=dout, delta_softplus=softplus, **args)
    for key, gname in M1_GRAD_OF.items():
        _close(g[gname], _fd(loss, args, key), key)


def test_m1_backward_groups_finite_differences():
    args = _m1_tiny(G=2)
    dout = _rand(*args["u"].shape)
    loss = lambda p: float(np.sum(dout * oracle.m1_fwd(**p)["out"]))
    g = oracle.m1_bwd(dout=dout, **args)
    for key in ("B", "C", "u"):
        _close(g[M1_GRAD_OF[key]], _fd(loss, args, key), key)


def test_m1_adjoint_identity():
    """<dout, J v> = <J^T dout, v> for a random direction v over every input."""
    Bsz, D, N, L = 2, 3, 4, 20
    args = dict(u=_rand(Bsz, D, L), delta=0.5 * _rand(Bsz, D, L) - 1, A=-np.abs(_rand(D, N)),
                B=_rand(Bsz, 1, N, L), C=_rand(Bsz, 1, N, L), D=_rand(D),
                delta_bias=_rand(D, scale=0.3), z=_rand(Bsz, D, L), h0=_rand(Bsz, D, N))
    dout = _rand(Bsz, D, L)
    v = {k: _rand(*a.shape) for k, a in args.items()}
    eps = 1e-6
    plus = {k: args[k] + eps * v[k] for k in args}
    minus = {k: args[k] - eps * v[k] for k in args}
    jv = (oracle.m1_fwd(**plus)["out"] - oracle.m1_fwd(**minus)["out"]) / (2 * eps)
    g = oracle.m1_bwd(dout=dout, **args)
    lhs = float(np.sum(dout * jv))
    rhs = sum(float(np.sum(g[M1_GRAD_OF[k]] * v[k])) for k in args)
    assert lhs == pytest.approx(rhs, rel=1e-7)


def test_m1_dD_closed_form():
    args = _m1_tiny()
    dout = _rand(*args["u"].shape)
    g = oracle.m1_bwd(dout=dout, **args)
    expect = np.sum(dout * _silu(args["z"]) * args["u"], axis=(0, 2))
    np.testing.assert_allclose(g["dD"], expect, rtol=1e-13)


# ---------------------------------------------------------------------------
# Mamba-3 SISO
# ---------------------------------------------------------------------------
def _rot(v, phi, K):
    out = v.copy()
    for k in range(K):
        c, s = np.cos(phi[k]), np.sin(phi[k])
        out[2 * k] = c * v[2 * k] - s * v[2 * k + 1]
        out[2 * k + 1] = s * v[2 * k] + c * v[2 * k + 1]
    return out


def _m3_masked_quadratic(x, Bm, Cm, al, be, ga, th, Dp, z, G):
    """y = (W o (Ct Bt^T)) X + D x with w_tt = gamma_t and, for s < t,
    w_ts = prod_{r=s+2..t} alpha_r (alpha_{s+1} gamma_s + beta_{s+1})  (h0 = 0)."""
    Bsz, L, H, P = x.shape
    N, K = Bm.shape[3], th.shape[3]
    out = np.zeros_like(x)
    for b in range(Bsz):
        for h in range(H):
            g = h // (H // G)
            phi = np.cumsum(th[b, :, h, :], axis=0)
            Bt = np.stack([_rot(Bm[b, t, g], phi[t], K) for t in range(L)])
            Ct = np.stack([_rot(Cm[b, t, g], phi[t], K) for t in range(L)])
            W = np.zeros((L, L))
            for t in range(L):
                W[t, t] = ga[b, t, h]
                for s in range(t):
                    W[t, s] = np.prod(al[b, s + 2: t + 1, h]) * (al[b, s + 1, h] * ga[b, s, h] + be[b, s + 1, h])
            Y = (W * (Ct @ Bt.T)) @ x[b, :, h, :] + Dp[h] * x[b, :, h, :]
            out[b, :, h, :] = Y * _silu(z[b, :, h, :])
    return out


def _m3_tiny(Bsz=1, L=7, H=2, P=3, N=4, K=2, G=1, h0=True):
    return dict(x=_rand(Bsz, L, H, P), B=_rand(Bsz, L, G, N), C=_rand(Bsz, L, G, N),
                alpha=np.exp(-np.logaddexp(0, _rand(Bsz, L, H))),
                beta=RNG.uniform(0, 0.5, (Bsz, L, H)), gamma=RNG.uniform(0, 0.5, (Bsz, L, H)),
                theta=RNG.uniform(0, 0.5, (Bsz, L, H, K)), D=_rand(H), z=_rand(Bsz, L, H, P),
                h0=_rand(Bsz, H, P, N) if h0 else None)


def test_m3_masked_quadratic_form():
    a = _m3_tiny(Bsz=2, L=13, H=4, P=3, N=6, K=2, G=2, h0=False)
    r = oracle.m3_fwd(**a)
    q = _m3_masked_quadratic(a["x"], a["B"], a["C"], a["alpha"], a["beta"], a["gamma"],
                             a["theta"], a["D"], a["z"], 2)
    np.testing.assert_allclose(r["out"], q, rtol=1e-11, atol=1e-12)


def test_m3_scalar_decay_special_case():
    """theta = 0, beta = 0: h_t = alpha_t h_{t-1} + gamma_t x_t B_t^T, y_t = h_t C_t + D x_t
    (the scalar-decay SSD form), checked by a direct loop written here."""
    a = _m3_tiny(Bsz=1, L=9, H=2, P=3, N=4, K=2, h0=True)
    a["theta"] = np.zeros_like(a["theta"])
    a["beta"] = np.zeros_like(a["beta"])
    r = oracle.m3_fwd(**a)
    for h in range(2):
        S = a["h0"][0, h].copy()
        for t in range(9):
            S = a["alpha"][0, t, h] * S + a["gamma"][0, t, h] * np.outer(a["x"][0, t, h], a["B"][0, t, 0])
            y = S @ a["C"][0, t, 0] + a["D"][h] * a["x"][0, t, h]
            np.testing.assert_allclose(r["out"][0, t, h], y * _silu(a["z"][0, t, h]), rtol=1e-12)


def test_m3_trapezoid_sum():
    """alpha = 1, beta = gamma = 1/2, constant k = x B^T: S_t = (t + 1/2) k."""
    L, P, N = 12, 2, 4
    x = np.tile(np.array([0.7, -1.2]), (1, L, 1, 1))
    Bv = np.array([0.3, -0.5, 1.1, 0.2])
    r = oracle.m3_fwd(x, np.tile(Bv, (1, L, 1, 1)), np.tile(np.eye(N)[0], (1, L, 1, 1)),
                      np.ones((1, L, 1)), np.full((1, L, 1), 0.5), np.full((1, L, 1), 0.5),
                      np.zeros((1, L, 1, 2)))
    k = np.outer(x[0, 0, 0], Bv)
    np.testing.assert_allclose(r["final_state"][0, 0], (L - 1 + 0.5) * k, rtol=1e-14)
    t = np.arange(L)
    np.testing.assert_allclose(r["out"][0, :, 0, :], (t[:, None] + 0.5) * k[None, :, 0],
                               rtol=1e-14)


def test_m3_relative_angle_invariance():
    """Adding one constant to every head's first angle increment leaves y unchanged
    (h0 = 0): Ct_t . Bt_s depends only on phi_t - phi_s."""
    a = _m3_tiny(Bsz=1, L=10, H=3, P=2, N=6, K=3, h0=False)
    r1 = oracle.m3_fwd(**a)
    b = dict(a)
    b["theta"] = a["theta"].copy()
    b["theta"][:, 0] += 1.234
    r2 = oracle.m3_fwd(**b)
    np.testing.assert_allclose(r2["out"], r1["out"], rtol=1e-11, atol=1e-12)


def test_m3_rotation_preserves_norm():
    """With C = B and one step, y = gamma x |Bt|^2 = gamma x |B|^2 for any angle."""
    N, K = 6, 3
    Bv = _rand(N)
    for ang in (0.0, 0.3, 2.0):
        th = np.full((1, 1, 1, K), ang)
        r = oracle.m3_fwd(np.ones((1, 1, 1, 1)), Bv.reshape(1, 1, 1, N), Bv.reshape(1, 1, 1, N),
                          np.ones((1, 1, 1)), np.zeros((1, 1, 1)), np.ones((1, 1, 1)), th)
        assert r["out"][0, 0, 0, 0] == pytest.approx(float(Bv @ Bv), rel=1e-14)


M3_GRAD_OF = dict(x="dx", z="dz", B="dB", C="dC", alpha="dalpha", beta="dbeta",
                  gamma="dgamma", theta="dtheta", D="dD", h0="dh0")


@pytest.mark.parametrize("G,H", [(1, 2), (2, 2)])
def test_m3_backward_finite_differences(G, H):
    a = _m3_tiny(G=G, H=H)
    dout = _rand(*a["x"].shape)
    loss = lambda p: float(np.sum(dout * oracle.m3_fwd(**p)["out"]))
    g = oracle.m3_bwd(dout=dout, **a)
    for key, gname in M3_GRAD_OF.items():
        _close(g[gname], _fd(loss, a, key), key)


def test_m3_adjoint_identity():
    a = _m3_tiny(Bsz=2, L=16, H=2, P=3, N=6, K=2)
    dout = _rand(*a["x"].shape)
    v = {k: _rand(*x.shape) for k, x in a.items()}
    eps = 1e-6
    jv = (oracle.m3_fwd(**{k: a[k] + eps * v[k] for k in a})["out"]
          - oracle.m3_fwd(**{k: a[k] - eps * v[k] for k in a})["out"]) / (2 * eps)
    g = oracle.m3_bwd(dout=dout, **a)
    lhs = float(np.sum(dout * jv))
    rhs = sum(float(np.sum(g[M3_GRAD_OF[k]] * v[k])) for k in a)
    assert lhs == pytest.approx(rhs, rel=1e-7)


def test_m3_dD_closed_form():
    a = _m3_tiny()
    dout = _rand(*a["x"].shape)
    g = oracle.m3_bwd(dout=dout, **a)
    np.testing.assert_allclose(g["dD"], np.sum(dout * _silu(a["z"]) * a["x"], axis=(0, 1, 3)),
                               rtol=1e-13)


# ---------------------------------------------------------------------------
# Mamba-3 single-token state update
# ---------------------------------------------------------------------------
def _m3_decode_chain(a, G, state0=None):
    """Run the oracle's decode step over every token of the scan inputs `a`
    (x [B,L,H,P], ...) from a fresh carried state; returns outs [B,L,H,P] and
    the final carried state."""
    Bsz, L, H, P = a["x"].shape
    N, K = a["B"].shape[3], a["theta"].shape[3]
    S = np.zeros((Bsz, H, P, N)) if state0 is None else state0.copy()
    xp, bp, ph = np.zeros((Bsz, H, P)), np.zeros((Bsz, H, N)), np.zeros((Bsz, H, K))
    outs = np.zeros_like(a["x"])
    for t in range(L):
        S, xp, bp, ph, o = oracle.m3_state_update(
            S, xp, bp, ph, a["x"][:, t], a["B"][:, t], a["C"][:, t], a["alpha"][:, t],
            a["beta"][:, t], a["gamma"][:, t], a["theta"][:, t], D=a["D"], z=a["z"][:, t])
        outs[:, t] = o
    return outs, S, xp, bp, ph


@pytest.mark.parametrize("G,H", [(1, 2), (2, 4)])
def test_m3_state_update_chain_equals_scan(G, H):
    """L decode steps from a fresh carried state (S = h0, no last key, zero
    angles) reproduce the scan's outputs and final state: the step carries
    exactly K_{t-1} and the cumulative angles."""
    a = _m3_tiny(Bsz=2, L=9, H=H, P=3, N=6, K=2, G=G, h0=True)
    r = oracle.m3_fwd(**a)
    outs, S, xp, bp, ph = _m3_decode_chain(a, G, state0=a["h0"])
    np.testing.assert_allclose(outs, r["out"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, r["final_state"], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(xp, a["x"][:, -1])
    np.testing.assert_allclose(ph, np.cumsum(a["theta"], axis=1)[:, -1], rtol=1e-14)
    for b in range(2):
        for h in range(H):
            g = h // (H // G)
            np.testing.assert_allclose(bp[b, h], _rot(a["B"][b, -1, g], ph[b, h], 2), rtol=1e-13)


def test_m3_state_update_identity_step():
    """alpha = 1, beta = gamma = 0 leaves S as it was; y = S R(phi+theta) C + D x,
    and the carried x and rotated B become this step's."""
    Bsz, H, P, N, K = 1, 2, 3, 4, 2
    S0, xp0, bp0 = _rand(Bsz, H, P, N), _rand(Bsz, H, P), _rand(Bsz, H, N)
    ph0, th = _rand(Bsz, H, K), _rand(Bsz, H, K)
    x, Bm, Cm, D = _rand(Bsz, H, P), _rand(Bsz, 1, N), _rand(Bsz, 1, N), _rand(H)
    S, xp, bp, ph, out = oracle.m3_state_update(
        S0, xp0, bp0, ph0, x, Bm, Cm, np.ones((Bsz, H)), np.zeros((Bsz, H)), np.zeros((Bsz, H)),
        th, D=D)
    np.testing.assert_array_equal(S, S0)
    for h in range(H):
        Ct = _rot(Cm[0, 0], ph0[0, h] + th[0, h], K)
        np.testing.assert_allclose(out[0, h], S0[0, h] @ Ct + D[h] * x[0, h], rtol=1e-13)
        np.testing.assert_allclose(bp[0, h], _rot(Bm[0, 0], ph0[0, h] + th[0, h], K), rtol=1e-14)
    np.testing.assert_array_equal(xp, x)


def test_m3_state_update_angle_offset_invariance():
    """From a fresh state, adding one constant to the carried angles changes no
    output: only differences of cumulative angles reach y."""
    a = _m3_tiny(Bsz=1, L=6, H=2, P=2, N=4, K=2, h0=False)
    o1 = _m3_decode_chain(a, 1)[0]
    Bsz, L, H, P = a["x"].shape
    S, xp, bp = np.zeros((1, H, P, 4)), np.zeros((1, H, P)), np.zeros((1, H, 4))
    ph = np.full((1, H, 2), 2.5)
    for t in range(L):
        S, xp, bp, ph, o = oracle.m3_state_update(
            S, xp, bp, ph, a["x"][:, t], a["B"][:, t], a["C"][:, t], a["alpha"][:, t],
            a["beta"][:, t], a["gamma"][:, t], a["theta"][:, t], D=a["D"], z=a["z"][:, t])
        np.testing.assert_allclose(o, o1[:, t], rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# causal conv1d (+ SiLU) ahead of the Mamba-1 scan
# ---------------------------------------------------------------------------
def test_conv1d_identity_kernel():
    """w = (0, ..., 0, 1), no bias: u = silu(x)."""
    x = _rand(2, 3, 11)
    w = np.zeros((3, 4))
    w[:, -1] = 1.0
    u, xs = oracle.conv1d_fwd(x, w)
    np.testing.assert_allclose(u, _silu(x), rtol=1e-15)
    np.testing.assert_array_equal(xs, x[:, :, -3:])


def test_conv1d_equals_numpy_convolve():
    """The pre-activation is the causal (zero-padded) convolution of each row
    with its kernel: numpy.convolve of the row with the kernel taps reversed
    (tap W-1 multiplies the current step), first L outputs, plus the bias."""
    Bsz, Dm, L, W = 2, 3, 13, 4
    x, w, bias = _rand(Bsz, Dm, L), _rand(Dm, W), _rand(Dm)
    u, _ = oracle.conv1d_fwd(x, w, bias=bias)
    for b in range(Bsz):
        for c in range(Dm):
            v = np.convolve(x[b, c], w[c, ::-1])[:L] + bias[c]
            np.testing.assert_allclose(u[b, c], _silu(v), rtol=1e-13, atol=1e-15)


def test_conv1d_continuation():
    """Convolving [x1, x2] equals convolving x1, then x2 from x1's final conv state."""
    Bsz, Dm, W = 1, 4, 4
    x1, x2, w, bias = _rand(Bsz, Dm, 9), _rand(Bsz, Dm, 7), _rand(Dm, W), _rand(Dm)
    u, xs = oracle.conv1d_fwd(np.concatenate([x1, x2], axis=2), w, bias=bias)
    u1, xs1 = oracle.conv1d_fwd(x1, w, bias=bias)
    u2, xs2 = oracle.conv1d_fwd(x2, w, bias=bias, xs0=xs1)
    np.testing.assert_allclose(np.concatenate([u1, u2], axis=2), u, rtol=1e-14)
    np.testing.assert_allclose(xs2, xs, rtol=1e-15)


def test_conv1d_backward_finite_differences():
    Bsz, Dm, L, W = 2, 2, 6, 3
    x, w, bias, xs0 = _rand(Bsz, Dm, L), _rand(Dm, W), _rand(Dm), _rand(Bsz, Dm, W - 1)
    du = _rand(Bsz, Dm, L)
    g = oracle.conv1d_bwd(x, w, du, bias=bias, xs0=xs0)
    args = dict(x=x, w=w, bias=bias, xs0=xs0)
    loss = lambda a: float(np.sum(oracle.conv1d_fwd(a["x"], a["w"], bias=a["bias"],
                                                    xs0=a["xs0"])[0] * du))
    for key, gk in (("x", "dx"), ("w", "dw"), ("bias", "dbias"), ("xs0", "dxs0")):
        fd = _fd(loss, args, key)
        np.testing.assert_allclose(g[gk], fd, rtol=1e-6, atol=1e-8, err_msg=key)


# ---------------------------------------------------------------------------
# Mamba-3 discretisation (dt, A, trap, raw angles) and BCNorm ahead of the scan
# ---------------------------------------------------------------------------
def _inv_softplus(v):
    return np.log(np.expm1(v))


def _disc_scan(x, dt, a, trap, omega, eps=0.0):
    """The oracle's discretisation followed by its scan, for one head with
    P = 1, N = 2 (one angle pair), raw B = C = (1, 0), D = 0, no gate."""
    L = x.shape[0]
    ones = np.ones((1, L, 1))
    d = oracle.m3_discretize(ones * _inv_softplus(dt), ones * _inv_softplus(-a), ones * trap,
                             np.full((1, L, 1), omega), np.tile([1.0, 0.0], (1, L, 1, 1)),
                             np.tile([1.0, 0.0], (1, L, 1, 1)), eps=eps)
    r = oracle.m3_fwd(x.reshape(1, L, 1, 1), d["B"], d["C"], d["alpha"], d["beta"], d["gamma"],
                      d["theta"])
    return r["out"][0, :, 0, 0]


def _exact_rotating(s, a, omega, Om):
    """w' = (a - i omega) w + x(s), x = sin(Om s), w(0) = 0, read out as
    2 Re w (B = C = sqrt(2) after the norm, a pair read as one complex number;
    the real state rotated by R(phi) is this complex state multiplied by
    e^{i phi})."""
    lam = a - 1j * omega
    w = (Om * np.exp(lam * s) - Om * np.cos(Om * s) - lam * np.sin(Om * s)) / (lam ** 2 + Om ** 2)
    return 2.0 * w.real


@pytest.mark.parametrize("omega", [0.0, 3.0])
def test_m3_discretisation_is_second_order(omega):
    """With trap = 0 (lam = 1/2) the discretised scan solves the continuous
    system to second order in dt (error / 4 when dt halves); the explicit end
    alone (lam -> 1) is first order.  A beta without its decay factor, a theta
    not scaled by dt or a wrong alpha breaks the order."""
    a, Om, T = -1.0, 2.0, 2.0

    def err(dt, trap):
        L = int(round(T / dt)) + 1
        s = dt * np.arange(L)
        y = _disc_scan(np.sin(Om * s), dt, a, trap, omega)
        return np.max(np.abs(y - _exact_rotating(s, a, omega, Om)))

    r2 = err(0.02, 0.0) / err(0.01, 0.0)
    assert 3.6 < r2 < 4.4, r2
    r1 = err(0.02, 40.0) / err(0.01, 40.0)
    assert 1.7 < r1 < 2.3, r1


def test_m3_discretisation_trapezoid_weights():
    """No decay (A -> 0), constant dt and unit input: S_t = dt (t + lam) per
    state entry, so y_t = 2 dt (t + lam); lam != 1/2 tells the two ends of
    the trapezoid apart."""
    L, dt, trap = 20, 0.1, 1.3
    lam = 1.0 / (1.0 + np.exp(-trap))
    ones = np.ones((1, L, 1))
    d = oracle.m3_discretize(ones * _inv_softplus(dt), ones * -60.0, ones * trap,
                             np.zeros((1, L, 1)), np.tile([1.0, 0.0], (1, L, 1, 1)),
                             np.tile([1.0, 0.0], (1, L, 1, 1)), eps=0.0)
    r = oracle.m3_fwd(np.ones((1, L, 1, 1)), d["B"], d["C"], d["alpha"], d["beta"], d["gamma"],
                      d["theta"])
    np.testing.assert_allclose(r["out"][0, :, 0, 0], 2 * dt * (np.arange(L) + lam), rtol=1e-12)


def test_m3_discretisation_floor_bias_and_norm():
    """A_floor bounds the decay rate from below; dt_bias is a per-head shift of
    dd_dt; BCNorm leaves unit mean square (eps = 0) and ignores the scale of
    each raw row, but not of another row."""
    Bsz, L, H, K, G, N = 2, 5, 3, 2, 2, 8
    dd_dt, dd_a, trap = _rand(Bsz, L, H), _rand(Bsz, L, H), _rand(Bsz, L, H)
    ang, Br, Cr = _rand(Bsz, L, K), _rand(Bsz, L, G, N), _rand(Bsz, L, G, N)
    dd_a[0, 0, 0] = -60.0  # softplus ~ 0: the floor holds
    d = oracle.m3_discretize(dd_dt, dd_a, trap, ang, Br, Cr, A_floor=0.25, eps=0.0)
    dt = np.log1p(np.exp(dd_dt))
    assert np.isclose(d["alpha"][0, 0, 0], np.exp(-0.25 * dt[0, 0, 0]), rtol=1e-14)
    assert np.all(d["alpha"] <= np.exp(-0.25 * dt) * (1 + 1e-15))
    bias = _rand(H)
    e = oracle.m3_discretize(dd_dt - bias, dd_a, trap, ang, Br, Cr, dt_bias=bias, A_floor=0.25,
                             eps=0.0)
    for k in ("alpha", "beta", "gamma", "theta"):
        np.testing.assert_allclose(e[k], d[k], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(np.mean(d["B"] ** 2, axis=-1), 1.0, rtol=1e-13)
    scale = np.exp(_rand(Bsz, L, G, 1))
    f = oracle.m3_discretize(dd_dt, dd_a, trap, ang, Br * scale, Cr * scale, eps=0.0)
    np.testing.assert_allclose(f["B"], d["B"], rtol=1e-12)
    np.testing.assert_allclose(f["C"], d["C"], rtol=1e-12)
    assert not np.allclose(f["B"][..., :1], (Br * scale)[..., :1] / np.sqrt(
        np.mean(Br ** 2, axis=(-1, -2), keepdims=True)))


def test_m3_discretisation_backward_finite_differences():
    """Central differences of a random linear functional of every output with
    respect to every input (with eps > 0 and a floor that clamps some
    entries)."""
    Bsz, L, H, K, G, N = 1, 4, 2, 2, 2, 4
    ins = dict(dd_dt=_rand(Bsz, L, H), dd_a=_rand(Bsz, L, H) * 2.0, trap=_rand(Bsz, L, H),
               angles=_rand(Bsz, L, K), B_raw=_rand(Bsz, L, G, N), C_raw=_rand(Bsz, L, G, N),
               dt_bias=_rand(H))
    ins["dd_a"][0, 0, 0] = -6.0  # clamped by the floor below
    kw = dict(A_floor=0.05, eps=1e-3)
    outs = oracle.m3_discretize(**ins, **kw)
    w = {k: _rand(*v.shape) for k, v in outs.items()}

    def loss(args):
        o = oracle.m3_discretize(**args, **kw)
        return sum(float(np.sum(w[k] * o[k])) for k in o)

    g = oracle.m3_discretize_bwd(**ins, dalpha=w["alpha"], dbeta=w["beta"], dgamma=w["gamma"],
                                 dtheta=w["theta"], dB=w["B"], dC=w["C"], **kw)
    names = dict(dd_dt="ddd_dt", dd_a="ddd_a", trap="dtrap", angles="dangles",
                 dt_bias="ddt_bias", B_raw="dB_raw", C_raw="dC_raw")
    h = 1e-6
    for name, gname in names.items():
        fd = np.zeros_like(ins[name])
        for i in np.ndindex(ins[name].shape):
            plus = {k: v.copy() for k, v in ins.items()}
            minus = {k: v.copy() for k, v in ins.items()}
            plus[name][i] += h
            minus[name][i] -= h
            fd[i] = (loss(plus) - loss(minus)) / (2 * h)
        np.testing.assert_allclose(g[gname], fd, rtol=1e-6, atol=1e-8, err_msg=name)
    assert g["ddd_a"][0, 0, 0] == 0.0
