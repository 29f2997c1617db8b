"""Pins for the nested reconstruction ("GRINQH" Section 3.3, bias correction):
exhaustive over all 256 codes and every width, against the bin-midpoint definition
and the error bound it implies."""
import math


def test_code_is_bin_midpoint(orc):
    for b in range(1, 8):
        width = 2 ** (8 - b)
        for q in range(256):
            lo = math.floor(q / width) * width       # start of q's b-bit bin
            mid = lo + width / 2.0                   # centre of [lo, lo + width)
            assert orc.code(q, b) == mid, (q, b)


def test_full_width_and_skip(orc):
    for q in range(256):
        assert orc.code(q, 8) == q
        assert orc.code(q, 0) == -1


def test_nesting_bound_and_mean(orc):
    prev_max, prev_mean = None, None
    for b in range(1, 9):
        err = [abs(orc.code(q, b) - q) for q in range(256)]
        bound = 0 if b == 8 else 2 ** (7 - b)
        assert max(err) == bound
        mean = sum(err) / 256.0
        # uniform codes in a bin of width w = 2^(8-b): mean |error| = w / 4
        assert mean == (0 if b == 8 else 2 ** (8 - b) / 4.0)
        if prev_max is not None:
            assert max(err) <= prev_max and mean <= prev_mean
        prev_max, prev_mean = max(err), mean
    # the bound is not pointwise monotone in b: q = 7 is 1 away at b = 4, 3 away at b = 5
    assert abs(orc.code(7, 4) - 7) == 1 and abs(orc.code(7, 5) - 7) == 3


def test_codes_are_bytes(orc):
    for b in range(1, 9):
        for q in range(256):
            assert 0 <= orc.code(q, b) <= 255
