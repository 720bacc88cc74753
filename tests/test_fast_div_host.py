"""The launch-time division the kernels use to find their (sequence, head,
tile) and k head from the block index: with l = ceil(log2 d) and
m = floor(2^32 (2^l - d) / d) + 1, floor(n / d) = (umulhi(n, m) + n) >> l for
0 <= n < 2^31 (Granlund and Montgomery, "Division by invariant integers using
multiplication", PLDI 1994, theorem 4.2 with N = 32).  The host computes m and
l in gdn_kernels.cuh (make_fast_div); this checks the identity itself in
exact integer arithmetic, over every divisor the library can meet (head
counts, GQA groups, tiles per head) and beyond, at the ends of the range and
at random points, with the 32-bit wrap of the sum checked too."""
import random

import pytest


def magic(d):
    l = 0
    while (1 << l) < d:
        l += 1
    m = ((1 << 32) * ((1 << l) - d)) // d + 1
    return m, l


def fdiv(n, d):
    m, l = magic(d)
    assert 0 < m < (1 << 32)
    t = ((n * m) >> 32) + n
    assert t < (1 << 32)  # the device adds in 32 bits
    return t >> l


DIVISORS = list(range(1, 300)) + [511, 512, 513, 1000, 4095, 4096, 4097, 65535, 65536, 1 << 20,
                                  (1 << 20) + 1, 12345677, (1 << 30) - 1, 1 << 30, (1 << 30) + 1,
                                  (1 << 31) - 1]


@pytest.mark.parametrize("d", DIVISORS)
def test_fast_division_matches_floor_division(d):
    rng = random.Random(d)
    top = (1 << 31) - 1
    ns = list(range(0, 3 * d + 3)) if d < 5000 else []
    ns += [top, top - 1, top - d, d * (top // d), d * (top // d) - 1]
    ns += [rng.randrange(0, top + 1) for _ in range(2000)]
    for n in ns:
        if 0 <= n <= top:
            assert fdiv(n, d) == n // d, (n, d)
