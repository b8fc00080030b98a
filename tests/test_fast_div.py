"""The multiply-shift division that the tcgen05 attention kernel decodes its
work units with (FastDiv in csrc/attend_tc.cuh): for a divisor d in
[1, 2^31) the host sets s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,
and the device computes n / d as (umulhi(m, n) + n) >> s for 0 <= n < 2^31
(Granlund and Montgomery, "Division by invariant integers using
multiplication", 1994).  The same 32-bit arithmetic is written out here and
compared with exact integer division; the kernel's own use is covered by the
attention parity tests, whose units span several partitions, head groups and
column chunks."""
import random


def make_fast_div(d):
    s = 0
    while (1 << s) < d:
        s += 1
    m = ((1 << 32) * ((1 << s) - d)) // d + 1
    assert 0 < m < (1 << 32) or (d == 1 and m == 1)
    return m, s


def fast_div(n, m, s):
    hi = (m * n) >> 32  # umulhi of two 32-bit operands
    return ((hi + n) & 0xFFFFFFFF) >> s


def test_small_divisors_exhaustive_numerators():
    for d in range(1, 300):
        m, s = make_fast_div(d)
        for n in range(0, 5 * d + 7):
            assert fast_div(n, m, s) == n // d, (n, d)


def test_edges_and_random_wide():
    rnd = random.Random(5)
    top = (1 << 31) - 1
    divisors = list(range(1, 70)) + [(1 << k) + e for k in range(1, 31) for e in (-1, 0, 1)] + [top, top - 1]
    divisors += [rnd.randrange(1, 1 << 31) for _ in range(300)]
    for d in divisors:
        if not 1 <= d <= top:
            continue
        m, s = make_fast_div(d)
        ns = [0, 1, d - 1, d, d + 1, top, top - 1, (top // d) * d, (top // d) * d - 1]
        ns += [rnd.randrange(0, 1 << 31) for _ in range(200)]
        for n in ns:
            if 0 <= n <= top:
                assert fast_div(n, m, s) == n // d, (n, d)
