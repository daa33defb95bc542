"""The seeded input generator (shared by both sides; holds none of the method)."""
import numpy as np

import synth


def test_slices_are_independent_of_start():
    full = synth.normal_bf16_bits(7, synth.T_K, 0, 5000)
    part = synth.normal_bf16_bits(7, synth.T_K, 1234, 777)
    np.testing.assert_array_equal(full[1234:1234 + 777], part)


def test_streams_differ_and_look_normal():
    a = synth.normal_f32(1, synth.T_K, 0, 200000).astype(np.float64)
    b = synth.normal_f32(1, synth.T_V, 0, 200000).astype(np.float64)
    c = synth.normal_f32(2, synth.T_K, 0, 200000).astype(np.float64)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    for x in (a, b, c):
        assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
        assert np.abs(x).max() < 4.4
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.01


def test_table_is_bf16_exact_and_symmetric():
    t = synth.NORMAL_TABLE_F32
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(synth.NORMAL_TABLE_BITS), t)
    np.testing.assert_array_equal(t, -t[::-1])
    assert np.all(np.diff(t) >= 0)


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9], dtype=np.float32)
    got = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0 + 4 * 2 ** -8, -2.5, 1.0])


def test_ragged_lengths_rule():
    L = synth.ragged_lengths(3, 2000, 512, 16384)
    assert L.min() >= 512 and L.max() <= 16384
    assert np.all(L % 256 != 0)
    np.testing.assert_array_equal(L, synth.ragged_lengths(3, 2000, 512, 16384))


def test_planted_targets_distinct():
    t = synth.planted_targets(3, 4, 8192, 4)
    for row in t:
        assert len(set(row.tolist())) == 4


def test_workload_shapes():
    w = synth.WORKLOADS["decode_4m"]
    assert w.n_tokens == 1024 * 4096
    w5 = synth.WORKLOADS["bank_100m"]
    assert w5.n_tokens == 99_999_744


def test_gaussian_f32_streams():
    """The fp32 generator: deterministic, sliceable, N(0,1) moments, and values that
    use more than bf16's 8 significant bits."""
    x = synth.gaussian_f32(0, synth.T_K, 0, 200000)
    assert x.dtype == np.float32
    np.testing.assert_array_equal(x[1000:1500], synth.gaussian_f32(0, synth.T_K, 1000, 500))
    assert abs(float(x.mean())) < 0.02 and abs(float(x.std()) - 1.0) < 0.02
    assert np.mean((x.view(np.uint32) & 0xFFFF) == 0) < 1e-3
    assert not np.array_equal(x[:100], synth.gaussian_f32(1, synth.T_K, 0, 100))
