"""The multiply-shift division used by the copy kernels (Granlund and
Montgomery, 1994, section 4) agrees with integer division; checked here on
the formula, written out in Python the same way the host code computes it."""
import numpy as np


def _magic(d):
    l = 0
    while (1 << l) < d:
        l += 1
    m = ((((1 << l) - d) << 32) // d + 1) & 0xFFFFFFFF
    return m, l


def _div(n, m, l):
    t = (m * n) >> 32
    return (t + n) >> l


def test_fastdiv_formula():
    rng = np.random.default_rng(0)
    divs = list(range(1, 300)) + [384, 1536, 3072, 32760, 98280, 118800, 2 ** 20 + 7, 2 ** 30]
    for d in divs:
        m, l = _magic(d)
        ns = list(range(0, 2000)) + [int(x) for x in rng.integers(0, 2 ** 31, size=2000)] + [2 ** 31 - 1]
        ns += [d * q + r for q in (1, 2, 1000, (2 ** 31 - 1) // d) for r in (-1, 0, 1) if 0 <= d * q + r < 2 ** 31]
        for n in ns:
            assert _div(n, m, l) == n // d, (n, d)
