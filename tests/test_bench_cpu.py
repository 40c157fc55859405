"""Host-side pieces of bench.py: the algorithmic byte counts the roofline
divides by, the source-hash gate on the recorded ncu traffic, and the clock
sampler's behaviour without a GPU."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_m1_bytes_per_unit():
    # bwd: 7 io values per token-channel; B, C in and dB, dC (f32) out per
    # (b, t); A, D, bias in and dA, dD, dbias out
    B, D, N, L, io = 8, 1536, 16, 2048, 2
    fwd, bwd = bench.m1_bytes(B, D, N, L, io)
    tc, bt = B * D * L, B * L
    params = D * N * 4 + 2 * D * 4
    assert bwd == 7 * io * tc + 2 * N * io * bt + 2 * N * 4 * bt + params + D * N * 4 + 2 * D * 4
    assert fwd == 4 * io * tc + 2 * N * io * bt + params + B * D * N * 4
    assert bwd == 355688448  # the figure the bench line's roofline divides by


def test_m3_bytes_per_unit():
    B, L, H, P, N, G, K, io = 8, 2048, 24, 64, 64, 1, 32, 2
    fwd, bwd = bench.m3_bytes(B, L, H, P, N, G, K, io)
    assert fwd == 3 * io * B * L * H * P + (3 + K) * io * B * L * H + 2 * N * io * B * L * G \
        + B * H * P * N * 4
    assert round(fwd / 1e6, 1) == 185.9 and round(bwd / 1e6, 1) == 346.8


def test_decode_bytes():
    assert round(bench.su_bytes(256, 5120, 16, 2) / 1e6, 1) == 178.3


def test_m3_decode_bytes():
    B, H, P, N, G, K, io = 256, 24, 64, 64, 1, 32, 2
    # state, x_prev, bt_prev, phi read + written in f32; x, z, out, alpha,
    # beta, gamma, theta per head and B, C per group in io
    per_head = 2 * 4 * (P * N + P + N + K) + io * (3 * P + 3 + K)
    assert bench.m3su_bytes(B, H, P, N, G, K, io) == B * H * per_head + 2 * B * G * N * io
    assert round(bench.m3su_bytes(B, H, P, N, G, K, io) / 1e6, 1) == 212.0


def test_traffic_gated_by_source_hash(monkeypatch):
    assert bench.ncu_traffic("no_such_kernel.cu", "w") is None
    monkeypatch.setitem(bench.NCU_TRAFFIC, "m1_fwd.cu", ("0000000000000000", "w", 123))
    assert bench.ncu_traffic("m1_fwd.cu", "w") is None  # stale capture: not reported
    import hashlib
    path = os.path.join(ROOT, "selective_state_space_14_b200", "csrc", "m1_fwd.cu")
    h = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    monkeypatch.setitem(bench.NCU_TRAFFIC, "m1_fwd.cu", (h, "w", 123))
    assert bench.ncu_traffic("m1_fwd.cu", "w") == 123
    assert bench.ncu_traffic("m1_fwd.cu", "another workload") is None  # other sizes: not reported


def test_clock_sampler_without_gpu():
    s = bench.ClockSampler(0)
    s.start()
    r = s.stop()
    assert set(r) >= {"sm_mhz", "sm_max_mhz", "reasons"}


def test_conv_and_disc_bytes():
    # conv: x in, u out (forward); x, du in, dx out (backward), bf16
    fwd, bwd = bench.conv_bytes(8, 1536, 2048, 4, 2)
    assert fwd == 2 * 8 * 1536 * 2048 * 2 and bwd == 3 * 8 * 1536 * 2048 * 2
    # discretisation, per token: dd_dt, dd_a, trap (H each), angles (K), B_raw,
    # C_raw (G N each) in; alpha, beta, gamma (H each), theta (H K), B, C out
    tok, H, K, GN = 8 * 2048, 24, 32, 64
    fwd, bwd = bench.m3disc_bytes(8, 2048, 24, 64, 1, 32, 2)
    raw = tok * (3 * H + K + 2 * GN) * 2
    assert fwd == raw + tok * (3 * H + H * K + 2 * GN) * 2
    assert bwd == raw + tok * (3 * H + H * K + 2 * GN) * 4 + tok * (3 * H + K + 2 * GN) * 4
    assert round(fwd / 1e6, 1) == 39.3 and round(bwd / 1e6, 1) == 86.2


def test_oracle_beside_fills_every_workload():
    """The oracle timings beside the extra workloads run on the host alone and
    fill an entry for every workload that ran (none for one that failed)."""
    names = ["m3su_raw_bf16_b256_h24_p64_n64_k32_x1000", "m1_bf16_b8_d1536_n16_l2048",
             "su_bf16_b256_d5120_n16_x1000", "m3_bf16_b8_h24_p64_n64_k32_l2048",
             "m3su_bf16_b256_h24_p64_n64_k32_x1000", "m3disc_bf16_b8_h24_p64_n64_k32_l2048",
             "m1conv_bf16_b8_d1536_n16_l2048_w4"]
    res = {n: {"unit": "u"} for n in names}
    res[names[0]] = {"error": "x"}
    bench.oracle_beside(res, budget_s=0.0)
    assert "oracle" not in res[names[0]]
    for n in names[1:]:
        o = res[n]["oracle"]
        assert o["kind"] == "oracle" and o["value"] > 0 and o["unit"] == "u" and o["sample"]


def test_m3_decode_raw_bytes():
    B, H, P, N, G, K, io = 256, 24, 64, 64, 1, 32, 2
    plain = bench.m3su_bytes(B, H, P, N, G, K, io)
    raw = bench.m3su_raw_bytes(B, H, P, N, G, K, io)
    # theta [B, H, K] (and alpha .. gamma) out; dd_dt, dd_a, trap [B, H] and angles [B, K] in
    assert plain - raw == B * H * K * io - B * K * io


def test_reference_arm_prints_one_line():
    """`bench.py --impl reference` (the oracle on the host) prints one JSON line
    with the contract's keys, on the headline's metric and workload."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3
    assert d["metric"] == bench.METRIC and d["config"]["workload"] == bench.HEADLINE
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]


def test_m1_sfu_ops():
    """The compute ceiling's operation count: one 2^x per state element and step
    (its decay) plus the per-token transcendentals -- four in the forward
    (softplus: 2^x and a logarithm or reciprocal; the silu gate: 2^x and a
    reciprocal), six in the backward (softplus, and the sigmoids of the gate
    and of the delta pre-activation)."""
    B, D, N, L = 4, 5120, 16, 4096
    fwd, bwd = bench.m1_sfu_ops(B, D, N, L)
    tc = B * D * L
    assert fwd == tc * (N + 4) and bwd == tc * (N + 6)
    # at the 2.8B layer: 1.68e9 and 1.85e9 operations, the figures the bench
    # line's `compute` entries divide by the measured 2^x rate
    assert fwd == 1677721600 and bwd == 1845493760
