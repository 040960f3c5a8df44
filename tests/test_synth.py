"""The seeded input generator: deterministic, and the distributions the
workload recipes ask for (CPU only)."""
import math

import numpy as np

import synth


def test_deterministic_and_name_keyed():
    a = synth.normal_bf16("x/a", (1000,), 1.0)
    b = synth.normal_bf16("x/a", (1000,), 1.0)
    c = synth.normal_bf16("x/b", (1000,), 1.0)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    assert not np.array_equal(a, synth.normal_bf16("x/a", (1000,), 1.0, seed=1))


def test_prefix_stability():
    """Element i depends only on (key, i): a longer draw extends a shorter one."""
    short = synth.normal_bf16("x/p", (100,), 1.0)
    long = synth.normal_bf16("x/p", (1000,), 1.0)
    assert np.array_equal(short, long[:100])


def test_uniform_moments():
    u = synth.uniform("x/u", 1_000_000)
    assert 0.0 <= u.min() and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 2e-3
    assert abs(u.var() - 1 / 12) < 1e-3


def test_normal_moments_and_outliers():
    n = 1_000_000
    z = synth.bf16_to_f32(synth.normal_bf16("x/n", (n,), 0.02)).astype(np.float64)
    assert abs(z.mean()) < 1e-4
    assert abs(z.std() / 0.02 - 1) < 5e-3
    o = synth.bf16_to_f32(synth.normal_bf16("x/n", (n,), 0.02, outlier_p=0.01, outlier_factor=50.0))
    changed = np.mean(o != z.astype(np.float32))
    assert abs(changed - 0.01) < 1.5e-3


def test_gelu_recipe():
    g = synth.bf16_to_f32(synth.gelu_normal_bf16("x/g", (1_000_000,))).astype(np.float64)
    # E[GELU(z)] = E[z Phi(z)] = 1 / (2 sqrt(pi)) for z ~ N(0, 1)
    assert abs(g.mean() - 1 / (2 * math.sqrt(math.pi))) < 3e-3
    assert g.min() > -0.2  # GELU's minimum is about -0.17


def test_workload_shapes():
    t = synth.tiny()
    assert t["A"].shape == (64, 256) and t["W"].shape == (512, 256) and t["bias"].shape == (512,)
    layout = synth.state_dict_layout()
    assert len(layout) == 192
    assert sum(int(np.prod(s)) for _, s in layout) == 1_610_612_736
