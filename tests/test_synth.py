"""The seeded input generator: published SplitMix64 reference stream, the
Irwin-Hall(12) moments, bf16 rounding and slice consistency."""
import numpy as np

import synth
from exact import round_f32_to_bf16_bits


def test_splitmix64_reference_stream():
    # SplitMix64 with seed 1234567: the first five outputs of the published
    # reference implementation (Steele, Lea & Flood 2014 / Vigna's splitmix64.c).
    ref = [6457827717110365317, 3203168211198807973, 9817491932198370423,
           4593380528125082431, 16408922859458223821]
    assert [int(v) for v in synth.splitmix64_stream(1234567, 5)] == ref


def test_normal_moments_and_range():
    z = synth.normal_f32(99, synth.X, 1.0, (400000,))
    assert abs(float(z.mean())) < 0.01
    assert abs(float(z.var()) - 1.0) < 0.01
    assert float(np.abs(z).max()) < 6.0
    w = synth.normal_f32(99, synth.WGU, 0.02, (400000,))
    assert abs(float(w.std()) - 0.02) < 0.0005


def test_bf16_is_rne_of_f32_and_slices_agree():
    f = synth.normal_f32(5, synth.WD, 0.02, (10000,))
    b = synth.normal_bf16_bits(5, synth.WD, 0.02, (10000,))
    assert np.array_equal(b, round_f32_to_bf16_bits(f))
    part = synth.normal_bf16_bits(5, synth.WD, 0.02, (100,), start=4000)
    assert np.array_equal(part, b[4000:4100])


def test_streams_differ_by_tensor_and_seed():
    a = synth.normal_f32(1, synth.X, 1.0, (64,))
    b = synth.normal_f32(1, synth.WR, 1.0, (64,))
    c = synth.normal_f32(2, synth.X, 1.0, (64,))
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
