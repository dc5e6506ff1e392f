"""Division by invariant integers (plan.h FastDiv): floor(n/d) == (n*m) >> p
for 0 <= n < 2^31, with l = ceil(log2 d), p = 31 + l, m = ceil(2^p / d).

The kernels of the prologue use this map for every index split; this checks the
multiplier bound (m < 2^32) and the quotient against integer division, over
every divisor up to 4096 and numerators at the edges of each quotient step.
"""
import random


def fastdiv_params(d):
    l = 0
    while (1 << l) < d:
        l += 1
    p = 31 + l
    m = ((1 << p) + d - 1) // d
    return m, p


def test_multiplier_fits_32_bits():
    for d in list(range(1, 4097)) + [65535, 65536, 65537, (1 << 31) - 1]:
        m, _ = fastdiv_params(d)
        assert m < (1 << 32), d


def test_quotients_match_integer_division():
    rng = random.Random(20261202)
    top = (1 << 31) - 1
    for d in range(1, 4097):
        m, p = fastdiv_params(d)
        ns = {0, 1, d - 1, d, d + 1, top, top - 1, top - (top % d), top - (top % d) - 1}
        ns.update(rng.randrange(0, top) for _ in range(20))
        ns.update(k * d - 1 for k in range(1, 40))
        for n in ns:
            if 0 <= n <= top:
                assert (n * m) >> p == n // d, (d, n)
