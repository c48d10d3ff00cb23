"""The seeded generators: deterministic, counter-based, and the C and numpy builds agree."""
import numpy as np

import synth


def test_c_and_numpy_generators_agree():
    for fn, args in [(synth.uniform_f32, (5, 2, 100_003)), (synth.int32_uniform, (5, 2, 100_003, -1000, 1000)),
                     (synth.uniform_f32, (1, 0, 1000, 0.0, 10.0))]:
        assert np.array_equal(fn(*args), fn(*args, native=False))
    x = synth.normal_f32(2, 1, 100_000, 1e-2)
    y = synth.normal_f32(2, 1, 100_000, 1e-2, native=False)
    assert np.max(np.abs(x.view(np.int32) - y.view(np.int32))) <= 1
    assert np.array_equal(synth.to_bf16_bits(x), synth.to_bf16_bits(x, native=False))


def test_counter_based_prefix_property_and_rank_independence():
    a = synth.uniform_f32(9, 3, 5000)
    b = synth.uniform_f32(9, 3, 1000)
    assert np.array_equal(a[:1000], b)
    assert not np.array_equal(a[:1000], synth.uniform_f32(9, 4, 1000))


def test_start_offset_selects_the_same_values():
    for native in (True, False):
        full = synth.normal_f32(3, 2, 5000, 1e-3, native=native)
        part = synth.normal_f32(3, 2, 1000, 1e-3, native=native, start=3000)
        assert np.array_equal(full[3000:4000], part)
        assert np.array_equal(synth.uniform_f32(1, 1, 900, native=native)[100:],
                              synth.uniform_f32(1, 1, 800, native=native, start=100))
        assert np.array_equal(synth.int32_uniform(1, 1, 900, -5, 5, native=native)[7:],
                              synth.int32_uniform(1, 1, 893, -5, 5, native=native, start=7))


def test_distributions():
    u = synth.uniform_f32(0, 0, 1_000_000)
    assert u.min() >= -1 and u.max() < 1 and abs(u.mean()) < 5e-3
    g = synth.normal_f32(0, 0, 1_000_000, 1e-3)
    assert abs(g.std() - 1e-3) < 2e-5 and abs(g.mean()) < 5e-6
    i = synth.int32_uniform(0, 0, 100_000, -1000, 1000)
    assert i.min() == -1000 and i.max() == 1000


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 1.0 + 2**-9], np.float32)
    h = synth.to_bf16_bits(x)
    assert synth.bf16_bits_to_f32(h).tolist() == [1.0, 1.0, 1.0 + 4 * 2**-8, -2.5, 1.0]
