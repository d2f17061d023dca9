"""The exactness claims behind the seeded accumulators of the group-unit GEMMs
(no GPU): an int32 accumulator seeded with the bit pattern of 1.5 * 2^e and fed
integer increments reads, as an fp32 value, exactly 1.5 * 2^e + (increments
* ulp), and one fp32 subtraction recovers the integer.  Checked exhaustively
over the ranges the kernels rely on (IEEE binary32 round-to-nearest, as numpy
implements it)."""
import numpy as np


def _recover(seed_bits: int, seed_value: float, deltas: np.ndarray) -> np.ndarray:
    bits = (np.int64(seed_bits) + deltas.astype(np.int64)).astype(np.uint32)
    return bits.view(np.float32) - np.float32(seed_value)


def test_int4_seed_1p5_times_2_pow_19_with_weights_scaled_by_16():
    """Weights unpacked as 16 x the int4 code: the raw accumulator grows by
    16 * acc, the seed's ulp is 2^-4, so the value is 1.5 * 2^19 + acc for
    every |acc| <= 128 * 127 * 8 (a 128-wide group of int8 x int4 codes)."""
    acc = np.arange(-128 * 127 * 8, 128 * 127 * 8 + 1, dtype=np.int64)
    got = _recover(0x49400000, 786432.0, 16 * acc)
    np.testing.assert_array_equal(got.astype(np.int64), acc)
    assert np.float32(786432.0).view(np.uint32) == 0x49400000


def test_int8_seed_1p5_times_2_pow_23_covers_rotated_int4_groups():
    """Rotated int4 codes lie in [-112, 112]: a 128-wide group of products with
    int8 codes stays within 128 * 127 * 112 < 2^22, where the 1.5 * 2^23 seed
    (ulp 1) is exact; checked over the whole of |acc| < 2^22."""
    acc = np.arange(-(1 << 22) + 1, 1 << 22, dtype=np.int64)
    got = _recover(0x4B400000, 12582912.0, acc)
    np.testing.assert_array_equal(got.astype(np.int64), acc)
    assert 128 * 127 * 112 < (1 << 22)
    assert np.float32(12582912.0).view(np.uint32) == 0x4B400000


def test_seeds_are_exact_up_to_their_binade_edges_and_no_further():
    """Exact through |acc| = 2^18 (int4 seed) and 2^22 (int8 seed) -- the binade
    edges are themselves representable -- and wrong one step beyond."""
    for seed_bits, seed_value, scale, edge in ((0x49400000, 786432.0, 16, 1 << 18),
                                               (0x4B400000, 12582912.0, 1, 1 << 22)):
        for a in (edge, -edge):
            assert _recover(seed_bits, seed_value, np.array([scale * a]))[0] == a
        for a in (edge + 1, -edge - 1):
            assert _recover(seed_bits, seed_value, np.array([scale * a]))[0] != a
