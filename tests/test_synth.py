"""The seeded generator: C implementation equals its numpy statement, and the
draws have the requested distribution."""

import numpy as np

import synth


def test_c_generator_matches_numpy_statement():
    for seed, tid, seg, std, shape in [(0, 1, 0, 1.0, (300, 7)), (3, 2, 4, 1.5, (1000, 77)), (9, 5, 11, 0.5, (5,))]:
        assert np.array_equal(synth.bf16_normal(seed, tid, shape, std, seg),
                              synth.bf16_normal_numpy(seed, tid, shape, std, seg))


def test_draws_are_normal_with_the_requested_std():
    x = synth.bf16_bits_to_f32(synth.bf16_normal(1, 1, (400000,), 0.5)).astype(np.float64)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 0.5) < 5e-3
    assert abs(np.mean(x ** 4) / x.var() ** 2 - 3.0) < 0.05  # normal kurtosis


def test_streams_are_independent_of_draw_order():
    a = synth.bf16_normal(7, 3, (1000,), 1.0, 2)
    b = synth.bf16_normal(7, 3, (4000,), 1.0, 2)
    assert np.array_equal(a, b[:1000])
    assert not np.array_equal(a, synth.bf16_normal(7, 3, (1000,), 1.0, 3))
