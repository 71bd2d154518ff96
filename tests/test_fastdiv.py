"""The kernels divide by launch constants with a multiply and a shift
(FastDiv in csrc/sm100.cuh): s = ceil(log2 d), m = ceil(2^(31+s) / d),
floor(n / d) = umulhi(n, m) >> (s - 1) for 0 <= n < 2^31.  This checks the
scheme against exact integer division over divisors and dividends that
stress it (powers of two and their neighbours, the top of the range)."""
import random


def make(d):
    if d <= 1:
        return d, 0, 0
    s = 0
    while (1 << s) < d:
        s += 1
    m = ((1 << (31 + s)) + d - 1) // d
    return d, m, s - 1


def fdiv(n, f):
    d, m, s1 = f
    return n if m == 0 else ((n * m) >> 32) >> s1


def test_multiplier_fits_32_bits_and_quotients_are_exact():
    rng = random.Random(7)
    divisors = list(range(1, 4097))
    divisors += [(1 << k) + o for k in range(1, 31) for o in (-1, 0, 1)]
    divisors += [rng.randrange(2, 1 << 31) for _ in range(2000)]
    for d in divisors:
        f = make(d)
        assert f[1] < (1 << 32)
        dividends = [0, 1, d - 1, d, d + 1, 2 * d - 1, (1 << 31) - 1, (1 << 31) - d]
        dividends += [rng.randrange(0, 1 << 31) for _ in range(64)]
        for n in dividends:
            if 0 <= n < (1 << 31):
                assert fdiv(n, f) == n // d, (n, d)
