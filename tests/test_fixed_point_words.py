"""Host check of the fixed-point row sums' word arithmetic (the column-sorted SpMV of fp32
products): the scale makes the sum of a row's |terms| stay below 2^EB, EB = min(62, 2 lb +
30) (the segment's bound is its largest row sum of |a_ij| times max |v_j|), every term is
an integer split into a signed high word v >> 2lb and two lb-bit words, and a row of m
terms (m < 2^(32 - lb), lb chosen from the longest row) is summed word by word in 32-bit
arithmetic.  At the worst cases (the whole bound in one term, or spread over the longest
row, all of one sign) no word's sum leaves its 32 bits and the recombination is the exact
integer sum."""
import numpy as np
import pytest


def _lb_for(max_row_len: int) -> int:
    bits = int(max_row_len).bit_length()
    return max(1, min(20, 32 - bits))


def _sum_words(terms, lb):
    mask = (1 << lb) - 1
    hi = sum(int(v) >> (2 * lb) for v in terms)
    mid = sum((int(v) >> lb) & mask for v in terms)
    lo = sum(int(v) & mask for v in terms)
    return hi, mid, lo


@pytest.mark.parametrize("max_row_len", [1, 600, 4095, 4096, 65535, 200000])
@pytest.mark.parametrize("sign", [1, -1])
def test_words_do_not_overflow_and_recombine_exactly(max_row_len, sign):
    lb = _lb_for(max_row_len)
    eb = min(62, 2 * lb + 30)
    assert max_row_len * ((1 << lb) - 1) < 1 << 32          # the two lower words never carry out
    top = (1 << eb) - 1                                     # the row's sum of |terms| at most
    rng = np.random.default_rng(max_row_len)
    weights = [int(w) for w in rng.integers(1, 1 << 20, size=min(max_row_len, 4096))]
    total_w = sum(weights)
    cases = ([sign * top] + [0] * (max_row_len - 1),          # the bound in one term
             [sign * (top // max_row_len)] * max_row_len,    # spread over the longest row
             [sign * (top * w // total_w) for w in weights])  # a random split
    for terms in cases:
        assert sum(abs(t) for t in terms) <= top
        hi, mid, lo = _sum_words(terms, lb)
        assert -(1 << 31) <= hi < (1 << 31)                 # signed high word
        assert 0 <= mid < (1 << 32) and 0 <= lo < (1 << 32)  # unsigned lower words
        total = hi * (1 << (2 * lb)) + mid * (1 << lb) + lo
        assert total == sum(terms)
        assert abs(total) < (1 << 63)                        # exact in int64 before the fp64 rounding


def test_wrapping_high_word_is_read_back_signed():
    # the device adds the high words modulo 2^32 and reads the sum as int32
    lb = 20
    terms = [-(1 << 61)] * 3 + [5]
    hi = sum(int(v) >> (2 * lb) for v in terms)
    wrapped = hi & 0xFFFFFFFF
    assert (wrapped - (1 << 32) if wrapped >= (1 << 31) else wrapped) == hi
