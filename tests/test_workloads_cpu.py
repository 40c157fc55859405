"""The seeded input generators: the same call gives the same bits (both sides
of every parity test draw from them), storage rounding is round-to-nearest-
even, and the raw-input generators have the shapes the entry points take.
CPU only."""
import numpy as np

from selective_state_space_14_b200 import workloads as W


def test_generators_are_deterministic():
    for make in (lambda: W.m1conv_problem(1, 8, 16, 40, seed=3),
                 lambda: W.m3disc_problem(1, 9, 2, 16, 16, nangles=4, io="bf16", seed=4)):
        a, b = make(), make()
        for k in ("w", "bias", "dt_bias"):
            if hasattr(a, k):
                assert np.array_equal(getattr(a, k), getattr(b, k)), k
        for k in ("dd_dt", "dd_a", "trap", "angles", "B_raw", "C_raw"):
            if hasattr(a, k):
                assert np.array_equal(getattr(a, k).data, getattr(b, k).data), k
    s1, d1 = W.m3su_raw_steps(2, 3, 16, nangles=4, n_pool=2)
    s2, d2 = W.m3su_raw_steps(2, 3, 16, nangles=4, n_pool=2)
    assert np.array_equal(d1, d2)
    for x, y in zip(s1, s2):
        for k in x:
            assert np.array_equal(x[k].data, y[k].data), k


def test_raw_input_shapes():
    q = W.m3disc_problem(2, 5, 3, 16, 32, ngroups=1, nangles=8, io="bf16")
    assert q.dd_dt.data.shape == (2, 5, 3) and q.angles.data.shape == (2, 5, 8)
    assert q.B_raw.data.shape == (2, 5, 1, 32) and q.dt_bias.shape == (3,)
    steps, dtb = W.m3su_raw_steps(4, 3, 32, ngroups=1, nangles=8, n_pool=3)
    assert len(steps) == 3 and dtb.shape == (3,)
    assert steps[0]["dd_dt"].data.shape == (4, 3) and steps[0]["angles"].data.shape == (4, 8)
    assert steps[0]["B_raw"].data.shape == (4, 1, 32)
    c = W.m1conv_problem(2, 6, 16, 10, width=3)
    assert c.w.shape == (6, 3) and c.bias.shape == (6,)
    assert np.all(np.abs(c.w) <= 1 / np.sqrt(3)) and np.all(np.abs(c.bias) <= 1 / np.sqrt(3))


def test_dt_bias_gives_the_mamba_dt_range():
    """softplus(dt_bias) is the dt the bias was drawn for: within [1e-3, 1e-1]."""
    q = W.m3disc_problem(1, 2, 64, 16, 16, nangles=4)
    dt0 = np.log1p(np.exp(q.dt_bias.astype(np.float64)))
    assert np.all(dt0 >= 1e-3 * 0.999) and np.all(dt0 <= 1e-1 * 1.001)


def test_bf16_storage_rounds_to_nearest_even():
    # 1 + 2^-8 lies halfway between two bf16 values: ties go to the even one (1.0);
    # 1 + 3 * 2^-8 lies halfway too, between 1 + 2^-7 and 1 + 2^-6: up, to the even one
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9], dtype=np.float32)
    t = W.store(x, "bf16").as_f64()
    assert t[0] == 1.0 and t[1] == 1.0 + 2.0 ** -6 and t[2] == 1.0
