"""The seeded input generator: numpy definition == host C == (GPU test) CUDA."""
import numpy as np
import pytest

import qwen3_synth as synth


@pytest.fixture(scope="module")
def native():
    import __graft_entry__
    __graft_entry__.build()
    return synth.native()


def test_host_c_matches_numpy_definition(native):
    for tid, shape, mean, std in ((3, (1000, 37), 0.0, 1.0), (101, (4096,), 0.0, 0.02), (102, (513,), 1.0, 0.1)):
        a = synth.normal_bf16(1000, tid, shape, mean, std)
        b = synth.normal_bf16_fast(1000, tid, shape, mean, std)
        np.testing.assert_array_equal(a, b)


def test_index_base_slices(native):
    full = synth.normal_bf16(5, 9, (64, 100))
    part = synth.normal_bf16(5, 9, (10, 100), index_base=30 * 100)
    np.testing.assert_array_equal(full[30:40], part)
    partc = synth.normal_bf16_fast(5, 9, (10, 100), index_base=30 * 100)
    np.testing.assert_array_equal(full[30:40], partc)


def test_distribution_moments():
    x = synth.bf16_bits_to_f32(synth.normal_bf16(1, 2, (200000,), 0.0, 0.02)).astype(np.float64)
    assert abs(x.mean()) < 3 * 0.02 / np.sqrt(len(x)) * 2
    assert abs(x.std() - 0.02) < 0.02 * 0.01
    y = synth.bf16_bits_to_f32(synth.normal_bf16(1, 3, (200000,), 1.0, 0.1)).astype(np.float64)
    assert abs(y.mean() - 1.0) < 0.002 and abs(y.std() - 0.1) < 0.002


def test_uniform_int_range_and_spread():
    ids = synth.uniform_int(1001, synth.TID_IDS, (4, 2048), 151936)
    assert ids.min() >= 0 and ids.max() < 151936
    assert len(np.unique(ids)) > 7000


def test_uniform_int_host_c(native):
    import ctypes
    n = 10000
    out = np.empty(n, dtype=np.int32)
    assert native.qwen3synth_uniform_int_host(out.ctypes.data, n, 0, 77, 4, 151936) == 0
    np.testing.assert_array_equal(out, synth.uniform_int(77, 4, (n,), 151936))


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(f)
    back = synth.bf16_bits_to_f32(bits)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2 ** -6 and back[3] == -2.5
