"""The seeded input generators (no method arithmetic): the torch version of
the normal stream used for the benchmark's large weight sets reproduces the
host stream, and the integer rows used by the exact-sum tests have the
stated range and peak."""
import numpy as np

import synthetic as syn


def test_normal_device_matches_host_stream_on_cpu():
    a = syn.normal_f32(987654321, 20001)
    b = syn.normal_device(987654321, 20001, "cpu", chunk=4096).numpy()
    np.testing.assert_array_equal(a, b)


def test_integer_rows_range_and_peak():
    x = syn.integer_rows(11, 7, 384)
    assert x.dtype == np.float32
    assert np.all(x == np.round(x)) and np.all(np.abs(x) <= 127)
    assert np.all(np.abs(x).max(axis=1) == 127)
