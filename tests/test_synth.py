"""The seeded input generator: its SplitMix64 finalizer against the published SplitMix64
sequence (Steele, Lea & Flood, OOPSLA 2014: from state 0 the generator's first three outputs
are 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F), the transforms' moments, and
that any slice of a workload regenerates exactly (the generator is counter based)."""
import numpy as np

from fp4_block_scaled_nvfp4_b200 import synth


def test_splitmix64_finalizer_matches_the_published_sequence():
    g = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        got = [int(synth._mix(np.array([g * np.uint64(k)], dtype=np.uint64))[0]) for k in (1, 2, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_transform_moments():
    n = 1 << 20
    u = synth.uniform(5, 0, 0, n)
    assert 0.0 < u.min() and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 2e-3 and abs(u.var() - 1 / 12) < 2e-3
    z = synth.normal(5, 2, 0, n)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1.0) < 5e-3
    lap = synth.laplace(5, 4, 0, n)
    assert abs(lap.mean()) < 5e-3 and abs(lap.std() - 1.0) < 1e-2
    # Laplace: E|x| = b = 1/sqrt(2) for unit variance
    assert abs(np.abs(lap).mean() - 1 / np.sqrt(2)) < 5e-3


def test_counter_based_slices_regenerate_exactly():
    whole = synth.uniform(7, 3, 0, 4096)
    assert np.array_equal(whole[1000:1500], synth.uniform(7, 3, 1000, 500))
    a = synth.make("cfg3", rows=8, cols=256)
    b = synth.make("cfg3", rows=8, cols=256)
    assert np.array_equal(a["x"], b["x"])
