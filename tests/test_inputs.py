"""Seeded input generator: known-answer vectors and value distribution (CPU)."""
import numpy as np

import seeded_inputs as si


def test_philox_known_answers():
    # Known-answer vectors of Philox4x32-10 (Salmon et al., SC'11, Random123 distribution)
    assert si.philox4x32_10((0, 0, 0, 0), (0, 0)) == (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)
    assert si.philox4x32_10((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2) == (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)
    assert si.philox4x32_10((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0)) == \
        (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)


def test_values_unit_variance_and_distinct_streams():
    a = si.bf16_bits_to_f64(si.frames(0, si.K, 0, 0, 4, 100000))
    assert abs(a.mean()) < 5e-3 and abs(a.std() - 1.0) < 5e-3 and np.abs(a).max() <= 6.0
    b = si.bf16_bits_to_f64(si.frames(0, si.V, 0, 0, 4, 100000))
    c = si.bf16_bits_to_f64(si.frames(1, si.K, 0, 0, 4, 100000))
    assert np.corrcoef(a.ravel(), b.ravel())[0, 1] < 0.01 and np.corrcoef(a.ravel(), c.ravel())[0, 1] < 0.01


def test_indexed_matches_dense_and_frame_offset():
    dense = si.frames(3, si.Q, 2, 10, 3, 5000)
    idx = np.array([0, 17, 4999, 123], dtype=np.uint32)
    np.testing.assert_array_equal(si.frame_elements(3, si.Q, 2, 11, idx), dense[1, idx])
    np.testing.assert_array_equal(si.frames(3, si.Q, 2, 11, 1, 5000)[0], dense[1])


def test_weight_scale_variance():
    w = si.bf16_bits_to_f64(si.conv_weights(0, 0, 2, 64))
    assert w.shape == (2, 2, 64, 64, 5)
    assert abs(w.var() * 5 * 64 - 1.0) < 0.02
