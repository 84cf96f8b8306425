"""The seeded generator: counter-based, reproducible, with the stated distributions."""
import numpy as np

from gen.workloads import WORKLOADS


def test_counter_based_prefix(gen_mod):
    wl = WORKLOADS["internimage_l_stage4_bf16_n64_12x12_c1280"]
    a = gen_mod.make_inputs(wl, n_images=3)
    b = gen_mod.make_inputs(wl, n_images=5)
    for k in a:
        assert np.array_equal(a[k], b[k][:3]), k


def test_reproducible_and_seed_sensitive(gen_mod):
    x1 = gen_mod.normal(7, 1, (1000,), 0.0, 1.0)
    x2 = gen_mod.normal(7, 1, (1000,), 0.0, 1.0)
    x3 = gen_mod.normal(8, 1, (1000,), 0.0, 1.0)
    x4 = gen_mod.normal(7, 2, (1000,), 0.0, 1.0)
    assert np.array_equal(x1, x2)
    assert not np.array_equal(x1, x3)
    assert not np.array_equal(x1, x4)


def test_splitmix64_reference_values(gen_mod):
    # SplitMix64 of state 0 (one increment, then the finaliser) is the
    # published first output of the generator seeded with 0.
    assert gen_mod.raw_hash(0, 0, 0) == 0xE220A8397B1DCDAF


def test_distributions(gen_mod):
    n = 1 << 20
    z = gen_mod.normal(1, 1, (n,), 0.0, 1.5)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.5) < 0.01
    u = gen_mod.uniform(1, 3, (n,), -2.0, 2.0)
    assert u.min() >= -2.0 and u.max() < 2.0
    assert abs(u.mean()) < 0.01 and abs(u.var() - 16.0 / 12.0) < 0.01


def test_far_offsets_fraction(gen_mod):
    wl = WORKLOADS["internimage_l_stage3_bf16_n64_24x24_c640"]
    d = gen_mod.make_inputs(wl, n_images=4)
    pairs = d["offset"].reshape(-1, 2)
    plain = gen_mod.make_inputs(WORKLOADS["internimage_l_stage3_bf16_n64_24x24_c640"].__class__(
        **{**wl.__dict__, "far": None}), n_images=4)["offset"].reshape(-1, 2)
    changed = np.any(pairs != plain, axis=1)
    assert abs(changed.mean() - 0.1) < 0.005
    assert np.all(np.abs(pairs[changed]) <= 8.0)
