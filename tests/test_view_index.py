"""The row-strided views' index arithmetic, checked with exact integers (no
GPU): the kernels get floor(e / cols) as the high 64 bits of
e * ceil(2^64 / cols), which is exact for e < 2^32 and 2 <= cols < 2^32
because the product's error is below e / 2^64 < 2^-32 < 1 / cols.  Checked
at the boundaries (e next to multiples of cols and to 2^32, powers of two,
cols near 2^31 and 2^32) and on random pairs."""
import random

import pytest

M64 = 1 << 64


def magic(cols):
    # the library's ceil(2^64 / cols), computed as floor((2^64 - 1) / cols) + 1
    return (M64 - 1) // cols + 1


def quotient(e, cols):
    return (e * magic(cols)) >> 64


@pytest.mark.parametrize("cols", [2, 3, 4, 7, 8, 64, 72, 1344, 4096, 4104, 11008, 14336,
                                  (1 << 31) - 1, 1 << 31, (1 << 32) - 1])
def test_quotient_exact_at_boundaries(cols):
    es = {0, 1, (1 << 32) - 1, (1 << 32) - 2}
    for q in (1, 2, 3, 1000, ((1 << 32) - 1) // cols):
        for d in (-2, -1, 0, 1, 2):
            e = q * cols + d
            if 0 <= e < (1 << 32):
                es.add(e)
    for e in es:
        assert quotient(e, cols) == e // cols, (e, cols)


def test_quotient_exact_random():
    rng = random.Random(7)
    for _ in range(200000):
        cols = rng.randrange(2, 1 << 32)
        e = rng.randrange(0, 1 << 32)
        assert quotient(e, cols) == e // cols, (e, cols)


def test_offset_of_view():
    """offset(e) = e + q * (ld - cols) addresses row q, column e - q cols."""
    cols, ld = 72, 96
    for e in range(0, 72 * 50):
        q = quotient(e, cols)
        assert e + q * (ld - cols) == (e // cols) * ld + e % cols
