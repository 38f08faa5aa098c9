"""The candidate test of the top-k compaction, checked on the CPU over every
first digit it is used for.

The GPU top-k keeps a row as a candidate when the first radix digit (top 12
bits) of its order-preserving key is at least the threshold digit d.  For
d > 0x800 (the digit of +0.0) the kernel instead compares the row's fp32 bits,
read as a signed integer, with the bits of the smallest value of bin d.  This
test restates both predicates in numpy and checks that they agree for every
such d on special values (signed zeros, subnormals, infinities, NaNs, the
values at and next to every bin edge) and on random floats."""
import numpy as np


def order_key(bits: np.ndarray) -> np.ndarray:
    """Order-preserving uint32 key of fp32 bit patterns; -0.0 maps like +0.0."""
    b = np.where(bits == np.uint32(0x80000000), np.uint32(0), bits).astype(np.uint32)
    neg = (b & np.uint32(0x80000000)) != 0
    return np.where(neg, ~b, b | np.uint32(0x80000000)).astype(np.uint32)


def by_digit(bits: np.ndarray, d: int) -> np.ndarray:
    return (order_key(bits) >> np.uint32(20)) >= np.uint32(d)


def by_signed_bits(bits: np.ndarray, d: int) -> np.ndarray:
    tbits = np.int32(((d << 20) & 0xFFFFFFFF) & 0x7FFFFFFF)
    return bits.view(np.int32) >= tbits


def _values() -> np.ndarray:
    rng = np.random.default_rng(0)
    special = np.array([0x00000000, 0x80000000, 0x00000001, 0x80000001, 0x007FFFFF, 0x807FFFFF,
                        0x7F800000, 0xFF800000, 0x7FC00000, 0xFFC00000, 0x7F800001, 0xFF800001,
                        0x3F800000, 0xBF800000, 0x7F7FFFFF, 0xFF7FFFFF], dtype=np.uint32)
    # every bin edge of the positive half (the smallest value of each bin and the
    # values on either side), and the same patterns with the sign bit set
    edges = (np.arange(0x800, 0x1000, dtype=np.uint64) << np.uint64(20)).astype(np.uint32) & np.uint32(0x7FFFFFFF)
    near = np.concatenate([edges, edges + np.uint32(1), edges - np.uint32(1)]).astype(np.uint32)
    near = np.concatenate([near, near | np.uint32(0x80000000)])
    rand = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    floats = rng.standard_normal(50_000).astype(np.float32).view(np.uint32)
    return np.concatenate([special, near, rand, floats])


def test_signed_bit_compare_matches_first_digit_above_zero_digit():
    bits = _values()
    for d in range(0x801, 0x1000):
        np.testing.assert_array_equal(by_signed_bits(bits, d), by_digit(bits, d), err_msg=f"digit {d:#x}")


def test_zero_digit_is_where_the_shortcut_stops():
    # at d = 0x800 the bin holds +0.0 and -0.0 (equal keys); -0.0's bits read as
    # a negative integer, so the integer test would drop it: the kernel keeps the
    # key comparison for d <= 0x800
    minus_zero = np.array([0x80000000], dtype=np.uint32)
    assert by_digit(minus_zero, 0x800)[0]
    assert not by_signed_bits(minus_zero, 0x800)[0]
