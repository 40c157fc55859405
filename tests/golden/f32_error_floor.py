"""Writes f32_error_floor.json: how close a plain f32 evaluation of the
recurrences gets to the f64 oracle, per output tensor, under the parity
metrics of ``tests/_util.py``.

The f32 elementwise guard of the GPU parity tests is derived from this
record, not from any kernel: a kernel that accumulates in f32 (the rule of
the mamba-rs 0.7.0 README, "Features": every kernel accumulates in f32) is
held to a stated multiple of what the same recurrence evaluated step by step
in f32 reaches.  The evaluation below is the definition of each recurrence
(the Mamba-1 selective scan of the state-spaces/mamba README, "Selective
SSM"; the Mamba-3 SISO trapezoidal recurrence with cumulative RoPE angles
whose backward stages B3 BPTT and B4 RoPE mamba-rs 0.4.2
src/mamba3_siso/cpu/scratch.rs lays out), written with numpy float32
arithmetic throughout: sequential in time, each step's sums over the state
taken by numpy in f32.  It shares nothing with the CUDA path.  The inputs are
the seeded problems of the f32 GPU parity cases (``workloads.py``), and the
reference values come from ``oracle/`` alone.

    python tests/golden/f32_error_floor.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from selective_state_space_14_b200 import workloads as W  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "f32_error_floor.json")
f32 = np.float32

# the f32 parity cases of the GPU tests: Mamba-1 (B, D, N, L, G, bias, z, D, h0,
# softplus) and Mamba-3 (B, L, H, P, N, G, K, z, D, h0), with their seeds
M1_CASES = [
    ("m1_f32_b1_d64_n16_l256", None),
    ("B1D3N1L1", (1, 3, 1, 1, 1, False, True, True, False, True)),
    ("B2D5N3L7", (2, 5, 3, 7, 1, True, True, True, True, True)),
    ("B1D4N16L255", (1, 4, 16, 255, 1, True, False, False, True, True)),
    ("B1D4N16L257", (1, 4, 16, 257, 1, True, True, True, True, False)),
    ("B2D65N16L600", (2, 65, 16, 600, 1, True, True, True, True, True)),
    ("B1D8N64L300", (1, 8, 64, 300, 1, True, True, True, True, True)),
    ("B1D7N5L513", (1, 7, 5, 513, 1, False, True, True, False, True)),
    ("B2D256N8L130G2", (2, 256, 8, 130, 2, True, True, True, True, True)),
    ("B1D20N16L40", (1, 20, 16, 40, 1, True, True, True, True, True)),
    ("B1D8N128L300", (1, 8, 128, 300, 1, True, True, True, True, True)),
    ("B2D12N100L257", (2, 12, 100, 257, 1, False, True, True, True, True)),
]
# (B, L, H, P, N, G, K, z, D, h0): forward cases (seed 77 + L + H), backward
# cases (seed 91 + L + H)
M3_FWD_CASES = [
    (1, 1, 1, 16, 16, 1, 8, True, True, False),
    (2, 7, 2, 16, 16, 1, 4, True, True, True),
    (1, 64, 2, 32, 16, 1, 8, False, False, False),
    (1, 65, 3, 16, 32, 3, 16, True, True, True),
    (2, 200, 4, 64, 64, 2, 32, True, True, True),
    (1, 130, 2, 32, 64, 1, 0, True, False, True),
    (2, 70, 2, 32, 256, 2, 100, True, True, True),
]
M3_BWD_CASES = [
    (1, 1, 1, 16, 16, 1, 8, True, True, True),
    (2, 7, 2, 16, 16, 1, 4, True, True, True),
    (1, 64, 2, 32, 16, 1, 8, False, False, False),
    (1, 65, 3, 16, 32, 3, 16, True, True, True),
    (2, 200, 4, 64, 64, 2, 32, True, True, True),
    (1, 130, 2, 32, 64, 1, 0, True, False, True),
    (1, 70, 2, 32, 256, 1, 100, True, True, True),
]


# --------------------------------------------------------------------------
# parity metrics (as tests/_util.py states them)
# --------------------------------------------------------------------------
def norm_err(got, ref):
    ref = np.asarray(ref, np.float64)
    m = float(np.max(np.abs(ref))) if ref.size else 0.0
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref))) / (m if m > 0 else 1.0) \
        if ref.size else 0.0


def elem_err(got, ref):
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    floor = 1e-3 * float(np.max(np.abs(ref)))
    den = np.maximum(np.abs(ref), floor if floor > 0 else 1e-30)
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref) / den))


# --------------------------------------------------------------------------
# plain f32 evaluations
# --------------------------------------------------------------------------
def softplus(v):
    return np.maximum(v, f32(0)) + np.log1p(np.exp(-np.abs(v)))


def sigmoid(v):
    return f32(1) / (f32(1) + np.exp(-v))


def m1_f32(p):
    """Mamba-1 forward and BPTT backward in f32: h_t = exp(delta_t A) h_{t-1} +
    delta_t B_t x_t, y_t = C_t . h_t + D x_t, out_t = y_t silu(z_t); the
    backward walks the state adjoint lambda_t = g_t C_t + a_{t+1} lambda_{t+1}."""
    u, dr = p.u.as_f32(), p.delta.as_f32()
    Bsz, D, L = u.shape
    G, N = p.B.shape[1], p.A.shape[1]
    grp = np.arange(D) // (D // G)
    Bc, Cc = p.B.as_f32()[:, grp], p.C.as_f32()[:, grp]  # [B, D, N, L]
    A = p.A.astype(f32)
    bias = p.delta_bias.astype(f32) if p.delta_bias is not None else np.zeros(D, f32)
    Dp = p.D.astype(f32) if p.D is not None else np.zeros(D, f32)
    z = p.z.as_f32() if p.z is not None else None
    dout = p.dout.as_f32()
    h = p.h0.astype(f32).copy() if p.h0 is not None else np.zeros((Bsz, D, N), f32)
    hs = np.zeros((L + 1, Bsz, D, N), f32)
    hs[0] = h
    v = dr + bias[None, :, None]
    dl = softplus(v) if p.delta_softplus else v
    a_all = np.exp(dl[:, :, None, :] * A[None, :, :, None])  # [B, D, N, L]
    out = np.zeros_like(u)
    ys = np.zeros_like(u)
    for t in range(L):
        h = a_all[..., t] * h + (dl[:, :, t] * u[:, :, t])[..., None] * Bc[..., t]
        hs[t + 1] = h
        y = np.sum(Cc[..., t] * h, axis=2) + Dp * u[:, :, t]
        ys[:, :, t] = y
        out[:, :, t] = y * (z[:, :, t] * sigmoid(z[:, :, t])) if z is not None else y
    fwd = dict(out=out, final_state=h)
    # backward
    g = dout * (z * sigmoid(z)) if z is not None else dout
    res = dict(du=g * Dp[None, :, None], dA=np.zeros((D, N), f32),
               dB=np.zeros((Bsz, G, N, L), f32), dC=np.zeros((Bsz, G, N, L), f32),
               dD=np.sum(g * u, axis=(0, 2)), ddelta=np.zeros_like(u))
    if z is not None:
        s = sigmoid(z)
        res["dz"] = dout * ys * (s * (f32(1) + z * (f32(1) - s)))
    lam_next = np.zeros((Bsz, D, N), f32)
    a_next = np.zeros((Bsz, D, N), f32)
    dA = np.zeros((Bsz, D, N), f32)
    for t in range(L - 1, -1, -1):
        lam = g[:, :, t, None] * Cc[..., t] + a_next * lam_next
        a = a_all[..., t]
        hp = hs[t]
        dlt, ut = dl[:, :, t], u[:, :, t]
        for gg in range(G):
            sel = grp == gg
            res["dC"][:, gg, :, t] = np.sum(g[:, sel, t, None] * hs[t + 1][:, sel], axis=1)
            res["dB"][:, gg, :, t] = np.sum(lam[:, sel] * (dlt * ut)[:, sel, None], axis=1)
        res["du"][:, :, t] += dlt * np.sum(lam * Bc[..., t], axis=2)
        dd = np.sum(lam * (A[None] * a * hp + Bc[..., t] * ut[..., None]), axis=2)
        res["ddelta"][:, :, t] = dd * sigmoid(v[:, :, t]) if p.delta_softplus else dd
        dA += lam * dlt[..., None] * a * hp
        lam_next, a_next = lam, a
    res["dA"] = np.sum(dA, axis=0)
    res["ddelta_bias"] = np.sum(res["ddelta"], axis=(0, 2))
    res["dh0"] = a_next * lam_next
    return fwd, res


def rope(v, phi, K):
    """Rotate pairs (2k, 2k+1), k < K, of v [..., N] by phi [..., K]."""
    r = v.copy()
    if K == 0:
        return r
    c, s = np.cos(phi), np.sin(phi)
    v0, v1 = v[..., 0:2 * K:2], v[..., 1:2 * K:2]
    r[..., 0:2 * K:2] = c * v0 - s * v1
    r[..., 1:2 * K:2] = s * v0 + c * v1
    return r


def m3_f32(p):
    """Mamba-3 SISO forward and backward in f32: phi_t = phi_{t-1} + theta_t,
    Bt = R(phi) B, Ct = R(phi) C, K_t = x_t (outer) Bt_t,
    S_t = alpha_t S_{t-1} + beta_t K_{t-1} + gamma_t K_t, y_t = S_t Ct_t + D x_t;
    the backward carries the state adjoint and the beta term to the step
    before, then rotates dBt, dCt back and sums dphi in reverse for dtheta."""
    x = p.x.as_f32()
    Bsz, L, H, P = x.shape
    G, N, K = p.B.shape[2], p.B.shape[3], p.theta.shape[3]
    grp = np.arange(H) // (H // G)
    Bm, Cm = p.B.as_f32()[:, :, grp], p.C.as_f32()[:, :, grp]  # [B, L, H, N]
    al, be, ga = p.alpha.as_f32(), p.beta.as_f32(), p.gamma.as_f32()
    th = p.theta.as_f32()
    Dp = p.D.astype(f32) if p.D is not None else np.zeros(H, f32)
    z = p.z.as_f32() if p.z is not None else None
    dout = p.dout.as_f32()
    S = p.h0.astype(f32).copy() if p.h0 is not None else np.zeros((Bsz, H, P, N), f32)
    S0 = S.copy()
    phi = np.zeros((Bsz, H, K), f32)
    Kprev = np.zeros((Bsz, H, P, N), f32)
    Ss = np.zeros((L, Bsz, H, P, N), f32)
    Bts = np.zeros((L, Bsz, H, N), f32)
    Cts = np.zeros((L, Bsz, H, N), f32)
    phis = np.zeros((L, Bsz, H, K), f32)
    out = np.zeros_like(x)
    ys = np.zeros_like(x)
    for t in range(L):
        phi = phi + th[:, t]
        Bt, Ct = rope(Bm[:, t], phi, K), rope(Cm[:, t], phi, K)
        Kt = x[:, t][..., None] * Bt[:, :, None, :]
        S = al[:, t][..., None, None] * S + be[:, t][..., None, None] * Kprev \
            + ga[:, t][..., None, None] * Kt
        y = np.sum(S * Ct[:, :, None, :], axis=3) + Dp[None, :, None] * x[:, t]
        ys[:, t] = y
        out[:, t] = y * (z[:, t] * sigmoid(z[:, t])) if z is not None else y
        Kprev = Kt
        Ss[t], Bts[t], Cts[t], phis[t] = S, Bt, Ct, phi
    fwd = dict(out=out, final_state=S)
    g = dout * (z * sigmoid(z)) if z is not None else dout
    res = dict(dx=np.zeros_like(x), dB=np.zeros((Bsz, L, G, N), f32),
               dC=np.zeros((Bsz, L, G, N), f32), dalpha=np.zeros_like(al),
               dbeta=np.zeros_like(al), dgamma=np.zeros_like(al),
               dtheta=np.zeros((Bsz, L, H, K), f32), dD=np.sum(g * x, axis=(0, 1, 3)))
    if z is not None:
        s = sigmoid(z)
        res["dz"] = dout * ys * (s * (f32(1) + z * (f32(1) - s)))
    lam_next = np.zeros((Bsz, H, P, N), f32)
    al_n = np.zeros((Bsz, H), f32)
    be_n = np.zeros((Bsz, H), f32)
    acc = np.zeros((Bsz, H, K), f32)
    for t in range(L - 1, -1, -1):
        Bt, Ct = Bts[t], Cts[t]
        gt = g[:, t]
        lam = gt[..., None] * Ct[:, :, None, :] + al_n[..., None, None] * lam_next
        dK = ga[:, t][..., None, None] * lam + be_n[..., None, None] * lam_next
        Sprev = Ss[t - 1] if t > 0 else S0
        Kp = x[:, t - 1][..., None] * Bts[t - 1][:, :, None, :] if t > 0 else np.zeros_like(lam)
        Kt = x[:, t][..., None] * Bt[:, :, None, :]
        res["dalpha"][:, t] = np.sum(lam * Sprev, axis=(2, 3))
        res["dbeta"][:, t] = np.sum(lam * Kp, axis=(2, 3))
        res["dgamma"][:, t] = np.sum(lam * Kt, axis=(2, 3))
        dCt = np.sum(gt[..., None] * Ss[t], axis=2)
        dBt = np.sum(dK * x[:, t][..., None], axis=2)
        res["dx"][:, t] = np.sum(dK * Bt[:, :, None, :], axis=3) + Dp[None, :, None] * gt
        # RoPE backward: R^T per head, summed over the heads of a group
        phi = phis[t]
        dB_h = rope(dBt, -phi, K)
        dC_h = rope(dCt, -phi, K)
        for gg in range(G):
            sel = grp == gg
            res["dB"][:, t, gg] = np.sum(dB_h[:, sel], axis=1)
            res["dC"][:, t, gg] = np.sum(dC_h[:, sel], axis=1)
        if K:
            dphi = (dBt[..., 1:2 * K:2] * Bt[..., 0:2 * K:2] - dBt[..., 0:2 * K:2] * Bt[..., 1:2 * K:2]
                    + dCt[..., 1:2 * K:2] * Ct[..., 0:2 * K:2] - dCt[..., 0:2 * K:2] * Ct[..., 1:2 * K:2])
            acc = acc + dphi
            res["dtheta"][:, t] = acc
        lam_next, al_n, be_n = lam, al[:, t], be[:, t]
    res["dh0"] = al_n[..., None, None] * lam_next
    return fwd, res


# --------------------------------------------------------------------------
def m1_case(spec):
    if spec is None:
        return W.make("m1_f32_b1_d64_n16_l256")
    Bsz, D, N, L, G, bias, zz, Dd, h0, sp = spec
    p = W.m1_problem(Bsz, D, N, L, io="f32", seed=1000 + L + D, ngroups=G, bias=bias, with_z=zz,
                     with_D=Dd, with_h0=h0, delta_softplus=sp)
    if not sp:  # softplus off: delta kept positive and small, no bias (as the GPU case)
        p.delta = W.store(np.abs(p.delta.as_f32()) * 0.2, "f32")
        p.delta_bias = None
    return p


def main():
    record = {"metric": "elem: max |g - o| / max(|o|, 1e-3 max|o|); norm: max |g - o| / max |o|",
              "m1": {}, "m3": {}}
    for name, spec in M1_CASES:
        p = m1_case(spec)
        a = oracle.m1_problem_args(p)
        ref = dict(oracle.m1_fwd(**a))
        ref.update(oracle.m1_bwd(dout=p.dout.as_f64(), **a))
        fwd, bwd = m1_f32(p)
        got = dict(fwd, **bwd)
        record["m1"][name] = {k: {"elem": elem_err(got[k], ref[k]), "norm": norm_err(got[k], ref[k])}
                              for k in got if ref.get(k) is not None}
    for fam, cases, seed0, keys in (("fwd", M3_FWD_CASES, 77, ("out", "final_state")),
                                    ("bwd", M3_BWD_CASES, 91, None)):
        for c in cases:
            Bsz, L, H, P, N, G, K, zz, Dd, h0 = c
            p = W.m3_problem(Bsz, L, H, P, N, ngroups=G, nangles=K, io="f32", seed=seed0 + L + H,
                             with_z=zz, with_D=Dd, with_h0=h0)
            a = oracle.m3_problem_args(p)
            fwd, bwd = m3_f32(p)
            if fam == "fwd":
                ref, got = oracle.m3_fwd(**a), fwd
            else:
                ref, got = oracle.m3_bwd(dout=p.dout.as_f64(), **a), bwd
                got = {k: v for k, v in got.items()
                       if not (k == "dtheta" and K == 0) and not (k == "dz" and not zz)
                       and not (k == "dD" and not Dd)}
            name = f"{fam} B{Bsz}L{L}H{H}P{P}N{N}G{G}K{K}"
            record["m3"][name] = {k: {"elem": elem_err(got[k], ref[k]),
                                      "norm": norm_err(got[k], ref[k])}
                                  for k in (keys or got) if ref.get(k) is not None}
    worst = {fam: max((e["elem"], c, k) for c, ts in record[fam].items() for k, e in ts.items())
             for fam in ("m1", "m3")}
    record["max_elem"] = {fam: {"value": w[0], "case": w[1], "tensor": w[2]}
                          for fam, w in worst.items()}
    with open(OUT, "w") as f:
        json.dump(record, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps(record["max_elem"]))


if __name__ == "__main__":
    main()
